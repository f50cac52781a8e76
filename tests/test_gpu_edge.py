"""GPU edge cases against the fp64 oracle: residual logits far outside the
range where an unshifted float32 exp is finite, a permutation-dominant
residual bias, and non-finite inputs reported by the backward.

Sources: the Sinkhorn-Knopp projection of the residual mapping (chatgpz.de
explainer, section "Vielfaeltig eingeschraenkte Hyperverbindungen";
reportify.cn [16]); a permutation matrix is doubly stochastic, so a strongly
permutation-dominant logit matrix must come out close to that permutation.
The kernels subtract each row's maximum logit before exp (exact: the first
row pass divides any per-row factor out); the oracle takes exp in float64
without a shift, where e^100 is still finite.
"""
import numpy as np
import pytest
import torch

from conftest import assert_close

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-2}


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


def _perm_bias(n, big):
    """Residual logits `big` on the cyclic shift i -> (i + 1) mod n, 0 elsewhere;
    pre / post logits 0."""
    b = torch.zeros(n * n + 2 * n, dtype=torch.float32)
    for i in range(n):
        b[2 * n + i * n + (i + 1) % n] = big
    return b


def _inputs(T, n, C, dtype, seed, bias):
    from manifold_constrained_hyper_token_b200 import synth
    d = synth.layer_inputs(T, n, C, seed=seed, dtype=dtype, backward=True)
    d["b"] = bias
    return d


CASES = [(4, torch.bfloat16, 130, 256), (4, torch.float32, 65, 64), (8, torch.bfloat16, 65, 64),
         (2, torch.float32, 33, 24), (16, torch.bfloat16, 33, 64)]


@pytest.mark.parametrize("big", [30.0, 100.0], ids=["perm30", "exp_overflow100"])
@pytest.mark.parametrize("iters", [1, 20])
@pytest.mark.parametrize("n,dtype,T,C", CASES)
def test_large_residual_logits_pre(mhc, oracle_mod, big, iters, n, dtype, T, C):
    """A +30 bias makes H_res the permutation within e^-30 of each entry; a +100 bias
    puts the logits beyond float32 exp's range (e^88.7), which only the row-max shift
    survives."""
    d = _inputs(T, n, C, dtype, seed=7 * T + n, bias=_perm_bias(n, big))
    dd = {k: v.cuda() for k, v in d.items()}
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    h_in, Hpre, Hpost, Hres = mhc.mhc_pre(dd["x"], dd["phi"], dd["b"], dd["alpha"], t_max=iters,
                                          dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = oracle_mod.pre(d["x"], d["phi"], d["b"], float(d["alpha"][0]), iters=iters)
    tol = TOL[dtype]
    for k, got in (("H_pre", Hpre), ("H_post", Hpost), ("H_res", Hres), ("h_in", h_in)):
        assert_close(_np(got), ref[k], tol, k)
    P = np.zeros((n, n))
    for i in range(n):
        P[i, (i + 1) % n] = 1.0
    assert np.all(np.isfinite(_np(Hres)))
    assert float(np.max(np.abs(_np(Hres) - P))) < 1e-5


@pytest.mark.parametrize("big", [30.0, 100.0], ids=["perm30", "exp_overflow100"])
@pytest.mark.parametrize("n,dtype,T,C", CASES)
def test_large_residual_logits_backward(mhc, oracle_mod, big, n, dtype, T, C):
    d = _inputs(T, n, C, dtype, seed=11 * T + n, bias=_perm_bias(n, big))
    dd = {k: v.cuda() for k, v in d.items()}
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gx, gphi, gb, ga, gf = mhc.mhc_backward(dd["x"], dd["phi"], dd["b"], dd["alpha"], dd["f_out"],
                                            dd["grad_x_next"], dd["grad_h_in"], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = oracle_mod.backward(d["x"], d["phi"], d["b"], float(d["alpha"][0]), d["f_out"],
                              d["grad_x_next"], d["grad_h_in"])
    tol = TOL[dtype]
    for k, got in (("grad_x", gx), ("grad_f_out", gf), ("grad_phi", gphi), ("grad_b", gb)):
        assert_close(_np(got), ref[k], tol, k)


@pytest.mark.parametrize("n,dtype", [(4, torch.bfloat16), (4, torch.float32), (8, torch.bfloat16),
                                     (16, torch.bfloat16)])
@pytest.mark.parametrize("where", ["x", "phi"])
def test_backward_nonfinite_status(mhc, n, dtype, where):
    """A NaN in the stream buffer or in phi makes the recomputed RMS or a logit
    non-finite: the backward reports MHC_ERR_NONFINITE in the status word, and a
    following clean call on the same stream reports nothing."""
    from manifold_constrained_hyper_token_b200 import synth
    T, C = 150, 64
    d = {k: v.cuda() for k, v in synth.layer_inputs(T, n, C, seed=3, dtype=dtype).items()}
    bad = {k: v.clone() for k, v in d.items()}
    if where == "x":
        bad["x"][77, n - 1, 5] = float("nan")
    else:
        bad["phi"][3, 2] = float("nan")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    mhc.mhc_backward(bad["x"], bad["phi"], bad["b"], bad["alpha"], bad["f_out"], bad["grad_x_next"],
                     bad["grad_h_in"], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 4
    st.zero_()
    mhc.mhc_backward(d["x"], d["phi"], d["b"], d["alpha"], d["f_out"], d["grad_x_next"],
                     d["grad_h_in"], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
