"""The give-up path of the tensor-core kernels' bounded waits, exercised on
purpose without hanging or faulting anything.

Every wait of those kernels on another warp's or the copy engine's progress has
a limit (mhc_params.wait_ns, default 2 s).  A limit of 1 ns makes the first wait
that finds its phase incomplete give up: the kernel then records
MHC_ERR_TIMEOUT in the status word, waits (with its own fixed bound) for the
copies and MMAs it already issued, frees its tensor memory and returns.  The
test checks the status and then that an ordinary call on the same stream, same
buffers and same workspace gives oracle-matching results.
"""
import numpy as np
import pytest
import torch

from conftest import assert_close

pytestmark = pytest.mark.gpu

TIMEOUT = 5
TOL = 2e-2  # bf16 I/O (the tensor-core kernels run for bf16 with n = 4, 8 and 16)


@pytest.fixture(scope="module")
def mhc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from manifold_constrained_hyper_token_b200 import build
    build.build()
    import manifold_constrained_hyper_token_b200 as m
    return m


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _case(T, C, seed):
    from manifold_constrained_hyper_token_b200 import synth
    d = synth.layer_inputs(T, 4, C, seed=seed, dtype=torch.bfloat16, backward=True)
    return d, {k: v.cuda() for k, v in d.items()}


# (T, C): channel-split tiles (several CTAs per 128-token tile, combined through
# a counter) and one CTA per tile
SHAPES = [(300, 1024), (20000, 256)]


@pytest.mark.parametrize("T,C", SHAPES)
def test_pre_times_out_then_recovers(mhc, oracle_mod, T, C):
    d, dd = _case(T, C, seed=T + C)
    ws = torch.empty(max(1, mhc.mhc_pre_workspace_size(4, T, C, torch.bfloat16)),
                     dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"], wait_ns=1, workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == TIMEOUT
    st.zero_()
    h_in, Hpre, Hpost, Hres = mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"], workspace=ws,
                                          dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    idx = np.arange(0, T, max(1, T // 300))
    ref = oracle_mod.pre(d["x"][idx], d["phi"], d["b"], float(d["alpha"][0]))
    for k, got in (("h_in", h_in), ("H_pre", Hpre), ("H_post", Hpost), ("H_res", Hres)):
        assert_close(_np(got[torch.from_numpy(idx).cuda()]), ref[k], TOL, k)


@pytest.mark.parametrize("T,C", SHAPES)
@pytest.mark.parametrize("phase", ["map", "apply"])
def test_backward_times_out_then_recovers(mhc, oracle_mod, T, C, phase):
    """The mapping phase or the apply phase alone gives up; then the whole backward
    runs clean on the same workspace."""
    d, dd = _case(T, C, seed=2 * T + C)
    ws = torch.empty(mhc.mhc_backward_workspace_size(4, T, C, torch.bfloat16), dtype=torch.uint8,
                     device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    args = (dd["x"], dd["phi"], dd["b"], dd["alpha"], dd["f_out"], dd["grad_x_next"],
            dd["grad_h_in"], ws)
    mhc.mhc_backward_map(*args, wait_ns=1 if phase == "map" else 0, dev_status=st)
    mhc.mhc_backward_apply(dd["x"], dd["phi"], dd["grad_x_next"], dd["grad_h_in"], ws,
                           wait_ns=1 if phase == "apply" else 0, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == TIMEOUT
    st.zero_()
    gx, gphi, gb, ga, gf = mhc.mhc_backward(*args[:7], workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = oracle_mod.backward(d["x"], d["phi"], d["b"], float(d["alpha"][0]), d["f_out"],
                              d["grad_x_next"], d["grad_h_in"], chunk=4096)
    for k, got in (("grad_x", gx), ("grad_f_out", gf), ("grad_phi", gphi), ("grad_b", gb)):
        assert_close(_np(got), ref[k], TOL, k)


def test_fused_post_times_out_then_recovers(mhc, oracle_mod):
    T, C = 300, 1024
    d, dd = _case(T, C, seed=5)
    fwd = oracle_mod.pre(d["x"], d["phi"], d["b"], float(d["alpha"][0]))
    hp = torch.from_numpy(fwd["H_post"]).float().cuda()
    hr = torch.from_numpy(fwd["H_res"]).float().cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    mhc.mhc_post_fused(dd["x"], dd["f_out"], hp, hr, dd["phi"], dd["b"], dd["alpha"], wait_ns=1,
                       dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == TIMEOUT
    st.zero_()
    xn, hpre, hpost, hres = mhc.mhc_post_fused(dd["x"], dd["f_out"], hp, hr, dd["phi"], dd["b"],
                                               dd["alpha"], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref_xn = oracle_mod.post(d["x"], d["f_out"], fwd["H_post"], fwd["H_res"])
    assert_close(_np(xn), ref_xn, TOL, "x_next")


@pytest.mark.parametrize("n", [8, 16])
@pytest.mark.parametrize("phase", ["pre", "map", "apply"])
def test_wide_tensor_core_paths_time_out_then_recover(mhc, oracle_mod, n, phase):
    """The n = 8 and n = 16 tensor-core kernels (bf16) give up the same way: the
    mapping / projection in the forward and the backward, and the apply's phi u and
    grad_phi contractions."""
    from manifold_constrained_hyper_token_b200 import synth
    T, C = (300, 512) if n == 8 else (200, 256)
    d = synth.layer_inputs(T, n, C, seed=17 + n, dtype=torch.bfloat16, backward=True)
    dd = {k: v.cuda() for k, v in d.items()}
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if phase == "pre":
        mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"], wait_ns=1, dev_status=st)
    else:
        ws = torch.empty(mhc.mhc_backward_workspace_size(n, T, C, torch.bfloat16),
                         dtype=torch.uint8, device="cuda")
        mhc.mhc_backward_map(dd["x"], dd["phi"], dd["b"], dd["alpha"], dd["f_out"],
                             dd["grad_x_next"], dd["grad_h_in"], ws,
                             wait_ns=1 if phase == "map" else 0, dev_status=st)
        if phase == "apply":
            torch.cuda.synchronize()
            assert int(st.item()) == 0
            mhc.mhc_backward_apply(dd["x"], dd["phi"], dd["grad_x_next"], dd["grad_h_in"], ws,
                                   wait_ns=1, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == TIMEOUT
    st.zero_()
    h_in, Hpre, Hpost, Hres = mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"], dev_status=st)
    gx, gphi, gb, ga, gf = mhc.mhc_backward(dd["x"], dd["phi"], dd["b"], dd["alpha"], dd["f_out"],
                                            dd["grad_x_next"], dd["grad_h_in"], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    a = float(d["alpha"][0])
    ref = oracle_mod.pre(d["x"], d["phi"], d["b"], a)
    assert_close(_np(Hres), ref["H_res"], TOL, "H_res")
    assert_close(_np(h_in), ref["h_in"], TOL, "h_in")
    rb = oracle_mod.backward(d["x"], d["phi"], d["b"], a, d["f_out"], d["grad_x_next"],
                             d["grad_h_in"])
    assert_close(_np(gx), rb["grad_x"], TOL, "grad_x")
    assert_close(_np(gphi), rb["grad_phi"], TOL, "grad_phi")
