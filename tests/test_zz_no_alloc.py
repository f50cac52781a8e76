"""mhc_backward_noalloc: the backward for callers that cannot allocate device
memory (a runtime that plans every buffer at start-up, a plugin handed only
its inputs and outputs, a process whose framework allocator holds the whole
device).  It runs on the library's fixed scratch array instead of a caller
workspace; its results must match mhc_backward's, call after call, whatever
the previous call left in that array.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import pytest
import torch

from conftest import assert_close, close_errs, rel_err

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


def _case(T, n, C, dtype, seed):
    from manifold_constrained_hyper_token_b200 import synth
    d = synth.layer_inputs(T, n, C, seed=seed, dtype=dtype, backward=True)
    return {k: v.cuda() for k, v in d.items()}


def _noalloc_via_abi(d, t_max=20, eps=1e-6, out=None):
    """Call the C entry point directly with caller-allocated outputs only."""
    from manifold_constrained_hyper_token_b200 import _lib, api
    T, n, C = d["x"].shape
    if out is None:
        out = (torch.empty_like(d["x"]), torch.empty_like(d["phi"]), torch.empty_like(d["b"]),
               torch.empty_like(d["alpha"]), torch.empty_like(d["f_out"]))
    p = api.params(n, T, C, d["x"].dtype, t_max, eps)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    st = _lib.load().mhc_backward_noalloc(
        ctypes.byref(p), ptr(d["x"]), ptr(d["phi"]), ptr(d["b"]), ptr(d["alpha"]), ptr(d["f_out"]),
        ptr(d["grad_x_next"]), ptr(d["grad_h_in"]), *[ptr(o) for o in out], None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out


# per stream count: two calls in a row with different sizes and inputs (the
# second must not see anything the first left in the shared scratch); n = 8
# with T = 6000 needs 3.9 MB of the 4 MiB array (656-byte records per token)
CASES = {4: ((1000, 4, 1024, 1), (333, 4, 512, 2)),
         8: ((6000, 8, 64, 3), (100, 8, 256, 4)),
         2: ((2000, 2, 512, 5), (77, 2, 64, 6))}


@pytest.mark.parametrize("n", [4, 8, 2])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_noalloc_matches_backward_on_consecutive_calls(mhc, dtype, n):
    for T, n, C, seed in CASES[n]:
        d = _case(T, n, C, dtype, seed)
        st, got = _noalloc_via_abi(d)
        assert st == 0, mhc.mhc_status_string(st)
        ref = mhc.mhc_backward(d["x"], d["phi"], d["b"], d["alpha"], d["f_out"],
                               d["grad_x_next"], d["grad_h_in"])
        torch.cuda.synchronize()
        for name, a, r in zip(("grad_x", "grad_phi", "grad_b", "grad_alpha", "grad_f_out"), got,
                              ref):
            e = rel_err(a.float().cpu().numpy(), r.float().cpu().numpy())
            assert e < TOL[dtype], (name, T, e)


def test_noalloc_rejects_sizes_beyond_scratch(mhc):
    from manifold_constrained_hyper_token_b200 import _lib, api
    T, n, C = 200000, 4, 64  # needs about 40 MB of scratch, above the 4 MiB array
    assert mhc.mhc_backward_workspace_size(n, T, C, torch.bfloat16) > 4 * 1024 * 1024
    p = api.params(n, T, C, torch.bfloat16)
    fake = ctypes.c_void_p(0x10000)
    st = _lib.load().mhc_backward_noalloc(ctypes.byref(p), *([fake] * 12), None, None)
    assert st == 6  # MHC_ERR_WORKSPACE, returned before any launch


def test_noalloc_allocates_nothing(mhc):
    """After a first call on the device (which looks up the array's address),
    further calls leave the device's free memory unchanged."""
    d = _case(1000, 4, 1024, torch.bfloat16, seed=7)
    st, out = _noalloc_via_abi(d)
    assert st == 0
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        st, _ = _noalloc_via_abi(d, out=out)  # the same caller-owned outputs
        assert st == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
