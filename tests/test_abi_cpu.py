"""Host-only checks of the C ABI: the library loads, exports every entry point
include/mhc.h declares, and rejects bad arguments before launching anything.
No test here launches a kernel."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from manifold_constrained_hyper_token_b200 import build, _lib
    build.build()
    return _lib.load()


def _declared():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"MHC_API\s+[\w\s\*]+?\b(mhc_\w+)\s*\(", src)
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    from manifold_constrained_hyper_token_b200 import _lib
    assert set(_lib.SYMBOLS) <= set(names)


def test_status_strings(lib):
    for s in range(0, 7):
        assert lib.mhc_status_string(s).decode().startswith("MHC_")
    assert b"unknown" in lib.mhc_status_string(99)


def test_version(lib):
    assert lib.mhc_version() >= 1


def test_params_struct_layout():
    """The ctypes mirror of mhc_params has the C layout: three int32/int64 pairs,
    eps, dtype, alpha_groups and the int64 wait limit (48 bytes)."""
    from manifold_constrained_hyper_token_b200 import _lib
    P = _lib.MhcParams
    assert ctypes.sizeof(P) == 48
    assert [P.T.offset, P.C.offset, P.eps.offset, P.wait_ns.offset] == [8, 16, 24, 40]


def _params(**kw):
    from manifold_constrained_hyper_token_b200 import _lib
    d = dict(n=4, t_max=20, T=16, C=64, eps=1e-6, dtype=1)
    d.update(kw)
    return _lib.MhcParams(**d)


def test_workspace_size_query(lib):
    p = _params(T=16384, C=7168)
    ws = lib.mhc_backward_workspace_size(ctypes.byref(p))
    assert ws >= 16384 * 52 * 4 and ws % 256 == 0
    assert lib.mhc_backward_workspace_size(ctypes.byref(_params(C=12))) == 0  # invalid -> 0
    assert lib.mhc_pre_workspace_size(ctypes.byref(p)) >= 0


@pytest.mark.parametrize("n", [8, 16])
def test_wide_tensor_core_workspaces(lib, n):
    """bf16 with n = 8 or 16 takes the tensor-core paths: mhc_pre needs the split phi^T
    copy (2M rows of nC bf16; at n = 16 also the per-token rows of projections, 580
    floats each).  At n = 16 the backward holds the apply's fp32 phi u scratch
    [T][n][C] on top of the per-token records; at n = 8 phi u stays in the apply
    kernel's tensor memory, so the backward holds the records (coefficients, U rows,
    C-reductions) and the phi copy only.  fp32 activations take the CUDA-core paths,
    whose forward needs no workspace."""
    T, C = 4096, 7168
    M = n * n + 2 * n
    bf = _params(n=n, T=T, C=C, dtype=1)
    pre = lib.mhc_pre_workspace_size(ctypes.byref(bf))
    assert pre >= 2 * M * n * C * 2 and pre % 256 == 0
    if n == 16:
        assert pre >= 2 * M * n * C * 2 + T * 580 * 4
    assert lib.mhc_post_fused_workspace_size(ctypes.byref(bf)) == pre
    bwd = lib.mhc_backward_workspace_size(ctypes.byref(bf))
    records = T * (M + M + 4) * 4   # coefficient records: H, u, kappa (padded)
    if n == 16:
        assert bwd >= T * n * C * 4 + 2 * M * n * C * 2 and bwd % 256 == 0
    else:
        u_rows, dots = T * 192 * 2, T * M * 4
        assert bwd >= records + u_rows + dots + 2 * M * n * C * 2 and bwd % 256 == 0
        assert bwd < T * n * C * 4   # no [T][n][C] fp32 scratch
    f32 = _params(n=n, T=T, C=C, dtype=0)
    assert lib.mhc_pre_workspace_size(ctypes.byref(f32)) == 0
    assert 0 < lib.mhc_backward_workspace_size(ctypes.byref(f32)) < bwd


@pytest.mark.parametrize("n,slot_floats", [(8, 128 * 80), (16, 128 * 288)])
def test_small_problem_workspace_holds_grad_phi_slots(lib, n, slot_floats):
    """The tensor-core apply at n = 8 and 16 splits grad_phi over up to 256
    persistent CTAs, each with two partial slots of 128 rows; the backward
    workspace holds them even when the problem itself is tiny."""
    bf = _params(n=n, T=1, C=8, dtype=1)
    bwd = lib.mhc_backward_workspace_size(ctypes.byref(bf))
    assert bwd >= 256 * 2 * slot_floats * 4


FAKE = ctypes.c_void_p(0x10000)   # 16-byte aligned, never dereferenced (validation fails first)
ODD = ctypes.c_void_p(0x10004)


@pytest.mark.parametrize("kw,code", [
    (dict(T=0), 1), (dict(T=2**31 - 256), 1), (dict(C=12), 1), (dict(C=0), 1), (dict(t_max=-1), 1),
    (dict(eps=-1.0), 1),
    (dict(eps=float("nan")), 1), (dict(n=3), 2), (dict(n=32), 2), (dict(dtype=7), 2),
    (dict(alpha_groups=2), 1), (dict(wait_ns=-1), 1),
    (dict(n=16, T=2**31 // 16), 1), (dict(n=8, T=2**31 // 8), 1),
])
def test_pre_rejects_bad_params(lib, kw, code):
    p = _params(**kw)
    st = lib.mhc_pre(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0, None,
                     None)
    assert st == code


def test_null_and_misaligned_pointers_rejected(lib):
    p = _params()
    assert lib.mhc_pre(ctypes.byref(p), None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0,
                       None, None) == 1
    assert lib.mhc_pre(ctypes.byref(p), ODD, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0,
                       None, None) == 1
    assert lib.mhc_post(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, None, None) == 1
    assert lib.mhc_post(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == 1  # aliasing
    assert lib.mhc_post(None, FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == 1
    assert lib.mhc_sinkhorn_knopp(4, 20, 0, FAKE, FAKE, None, None) == 1
    assert lib.mhc_sinkhorn_knopp(3, 20, 8, FAKE, FAKE, None, None) == 2
    assert lib.mhc_sinkhorn_knopp(4, -1, 8, FAKE, FAKE, None, None) == 1
    assert lib.mhc_depth_amax(4, 0, 8, FAKE, FAKE, FAKE, None, None) == 1
    assert lib.mhc_depth_amax(5, 8, 8, FAKE, FAKE, FAKE, None, None) == 2


def test_backward_workspace_checked(lib):
    p = _params()
    args = [FAKE] * 12
    st = lib.mhc_backward(ctypes.byref(p), *args, None, 0, None, None)
    assert st == 6
    need = lib.mhc_backward_workspace_size(ctypes.byref(p))
    st = lib.mhc_backward(ctypes.byref(p), *args, FAKE, need - 1, None, None)
    assert st == 6
    st = lib.mhc_backward(ctypes.byref(p), *args, ctypes.c_void_p(0x10010), need, None, None)
    assert st == 6  # not 256-byte aligned


def test_product_path_has_no_fallback():
    """The binding imports nothing from the oracle and refuses to run without the library."""
    import manifold_constrained_hyper_token_b200 as pkg
    pkg_dir = os.path.dirname(pkg.__file__)
    for f in os.listdir(pkg_dir):
        if f.endswith(".py"):
            src = open(os.path.join(pkg_dir, f)).read()
            assert not re.search(r"^\s*(import|from)\s+oracle", src, re.M), f
