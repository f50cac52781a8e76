"""fp64 CPU oracle for the mHC layer -- TEST INFRASTRUCTURE ONLY.

This package is the independent statement of what the CUDA path computes.  It
shares no code, headers, tables or helpers with the product library and must
never be imported by it: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` use it.

The arithmetic lives in ``mhc_oracle.c`` (plain C, double precision, OpenMP
over independent tokens only).  These wrappers only marshal numpy arrays.
Inputs are widened to float64 before the call; bf16 and fp32 values widen
exactly.

Pinned by ``tests/test_oracle_pins.py`` against closed forms, hand-worked
examples (``tests/golden/``), invariants of doubly stochastic matrices,
brute-force finite differences and textbook special cases.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mhc_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmhc_oracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile mhc_oracle.c into a shared library next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.orc_sinkhorn.argtypes = [i32, i32, i64, _D, _D]
        lib.orc_sinkhorn_backward.argtypes = [i32, i32, i64, _D, _D, _D]
        lib.orc_pre.argtypes = [i32, i64, i64, i32, dbl, _D, _D, _D, _D, _D, _D, _D, _D, _D, _D]
        lib.orc_post.argtypes = [i32, i64, i64, _D, _D, _D, _D, _D]
        lib.orc_backward.argtypes = [i32, i64, i64, i32, dbl, _D, _D, _D, _D, _D, _D, _D,
                                     _D, _D, _D, _D, _D]
        lib.orc_post_backward.argtypes = [i32, i64, i64, _D, _D, _D, _D, _D, _D]
        lib.orc_pre_backward.argtypes = [i32, i64, i64, i32, dbl, _D, _D, _D, _D, _D, _D, _D,
                                         _D, _D, _D, _D]
        lib.orc_depth_amax.argtypes = [i32, i64, i32, _D, _D, _D]
        lib.orc_num_threads.restype = i32
        lib.orc_set_num_threads.argtypes = [i32]
        for f in ("orc_sinkhorn", "orc_sinkhorn_backward", "orc_pre", "orc_post", "orc_backward",
                  "orc_post_backward", "orc_pre_backward", "orc_depth_amax",
                  "orc_set_num_threads"):
            getattr(lib, f).restype = None
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # a torch tensor: widen exactly through float32
        a = a.detach().cpu().float().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a: np.ndarray):
    return a.ctypes.data_as(_D)


def _alpha3(alpha):
    """alpha as [alpha_pre, alpha_post, alpha_res]; a single alpha is three equal
    entries.  Returns (array, whether alpha was a single value)."""
    a = np.asarray(_f64(alpha), dtype=np.float64).reshape(-1)
    if a.size == 1:
        return np.full(3, float(a[0])), True
    if a.size != 3:
        raise ValueError("alpha: one value or three (pre, post, res)")
    return np.ascontiguousarray(a), False


def num_threads() -> int:
    return int(_load().orc_num_threads())


def set_num_threads(k: int) -> None:
    _load().orc_set_num_threads(int(k))


def sinkhorn(logits, iters: int) -> np.ndarray:
    """Batched Sinkhorn-Knopp: logits [..., n, n] -> doubly stochastic estimate."""
    lg = _f64(logits)
    n = lg.shape[-1]
    B = lg.size // (n * n)
    out = np.empty_like(lg)
    _load().orc_sinkhorn(n, int(iters), B, _p(lg), _p(out))
    return out


def sinkhorn_backward(logits, dout, iters: int) -> np.ndarray:
    """Vector-Jacobian product of ``sinkhorn`` with respect to the logits."""
    lg, do = _f64(logits), _f64(dout)
    n = lg.shape[-1]
    B = lg.size // (n * n)
    dl = np.empty_like(lg)
    _load().orc_sinkhorn_backward(n, int(iters), B, _p(lg), _p(do), _p(dl))
    return dl


def pre(x, phi, b, alpha, iters: int = 20, eps: float = 1e-6):
    """x [T,n,C] -> dict(h_in [T,C], H_pre [T,n], H_post [T,n], H_res [T,n,n], z, r).
    alpha: one value, or three (pre, post, res) for per-group scales."""
    xd = _f64(x)
    T, n, C = xd.shape
    M = n * n + 2 * n
    ph, bd = _f64(phi).reshape(n * C, M), _f64(b).reshape(M)
    out = dict(h_in=np.empty((T, C)), H_pre=np.empty((T, n)), H_post=np.empty((T, n)),
               H_res=np.empty((T, n, n)), z=np.empty((T, M)), r=np.empty(T))
    a3, _ = _alpha3(alpha)
    _load().orc_pre(n, T, C, int(iters), float(eps), _p(xd), _p(ph), _p(bd), _p(a3),
                    _p(out["h_in"]), _p(out["H_pre"]), _p(out["H_post"]), _p(out["H_res"]),
                    _p(out["z"]), _p(out["r"]))
    return out


def post(x, f_out, H_post, H_res) -> np.ndarray:
    """x [T,n,C], f_out [T,C], H_post [T,n], H_res [T,n,n] -> x_next [T,n,C]."""
    xd = _f64(x)
    T, n, C = xd.shape
    fd, hp, hr = _f64(f_out), _f64(H_post), _f64(H_res)
    out = np.empty_like(xd)
    _load().orc_post(n, T, C, _p(xd), _p(fd), _p(hp), _p(hr), _p(out))
    return out


def backward(x, phi, b, alpha, f_out, grad_x_next, grad_h_in, iters: int = 20,
             eps: float = 1e-6, chunk: int | None = None):
    """Backward of pre+post with recompute.  Returns dict(grad_x, grad_phi, grad_b,
    grad_alpha, grad_f_out).  alpha is one value (grad_alpha a float) or three, the
    per-group scales of the pre, post and res logits (grad_alpha an array of
    three).  ``chunk`` runs T in consecutive token chunks (the parameter sums
    still accumulate in increasing token order)."""
    T = x.shape[0]
    n, C = x.shape[1], x.shape[2]
    M = n * n + 2 * n
    ph, bd = _f64(phi).reshape(n * C, M), _f64(b).reshape(M)
    a3, single = _alpha3(alpha)
    gphi = np.zeros((n * C, M))
    gb = np.zeros(M)
    ga = np.zeros(3)
    gx = np.empty((T, n, C))
    gf = np.empty((T, C))
    step = T if chunk is None else int(chunk)
    lib = _load()
    for t0 in range(0, T, step):
        t1 = min(T, t0 + step)
        xd, fd = _f64(x[t0:t1]), _f64(f_out[t0:t1])
        Gd, gd = _f64(grad_x_next[t0:t1]), _f64(grad_h_in[t0:t1])
        gxc = np.empty((t1 - t0, n, C))
        gfc = np.empty((t1 - t0, C))
        lib.orc_backward(n, t1 - t0, C, int(iters), float(eps), _p(xd), _p(ph), _p(bd),
                         _p(a3), _p(fd), _p(Gd), _p(gd), _p(gxc), _p(gphi), _p(gb),
                         _p(ga), _p(gfc))
        gx[t0:t1] = gxc
        gf[t0:t1] = gfc
    return dict(grad_x=gx, grad_phi=gphi, grad_b=gb, grad_f_out=gf,
                grad_alpha=float(ga[0] + ga[1] + ga[2]) if single else ga)


def post_backward(x, f_out, H_post, grad_x_next):
    """First half of the layer backward in training order: the reverse of the post
    merge with the forward's H_post.  Returns dict(grad_f_out [T,C],
    red [T, n*n + n] = (<G_i, x_j> row-major, then <G_i, f_out>))."""
    xd = _f64(x)
    T, n, C = xd.shape
    fd, hp, Gd = _f64(f_out), _f64(H_post), _f64(grad_x_next)
    gf = np.empty((T, C))
    red = np.empty((T, n * n + n))
    _load().orc_post_backward(n, T, C, _p(xd), _p(fd), _p(hp), _p(Gd), _p(gf), _p(red))
    return dict(grad_f_out=gf, red=red)


def pre_backward(x, phi, b, alpha, grad_x_next, grad_h_in, red, iters: int = 20,
                 eps: float = 1e-6, chunk: int | None = None):
    """Second half of the layer backward in training order: recompute the mapping and
    take grad_h_in and the post half's reductions.  Returns dict(grad_x, grad_phi,
    grad_b, grad_alpha)."""
    T = x.shape[0]
    n, C = x.shape[1], x.shape[2]
    M = n * n + 2 * n
    ph, bd = _f64(phi).reshape(n * C, M), _f64(b).reshape(M)
    rd = _f64(red).reshape(T, n * n + n)
    a3, single = _alpha3(alpha)
    gphi = np.zeros((n * C, M))
    gb = np.zeros(M)
    ga = np.zeros(3)
    gx = np.empty((T, n, C))
    step = T if chunk is None else int(chunk)
    lib = _load()
    for t0 in range(0, T, step):
        t1 = min(T, t0 + step)
        xd = _f64(x[t0:t1])
        Gd, gd = _f64(grad_x_next[t0:t1]), _f64(grad_h_in[t0:t1])
        rc = np.ascontiguousarray(rd[t0:t1])
        gxc = np.empty((t1 - t0, n, C))
        lib.orc_pre_backward(n, t1 - t0, C, int(iters), float(eps), _p(xd), _p(ph), _p(bd),
                             _p(a3), _p(Gd), _p(gd), _p(rc), _p(gxc), _p(gphi), _p(gb),
                             _p(ga))
        gx[t0:t1] = gxc
    return dict(grad_x=gx, grad_phi=gphi, grad_b=gb,
                grad_alpha=float(ga[0] + ga[1] + ga[2]) if single else ga)


def depth_amax(H) -> tuple[np.ndarray, np.ndarray]:
    """H [T, L, n, n] -> (gain_fwd [T], gain_bwd [T]) of P = H_L ... H_1."""
    Hd = _f64(H)
    T, L, n, _ = Hd.shape
    gf, gb = np.empty(T), np.empty(T)
    _load().orc_depth_amax(n, T, L, _p(Hd), _p(gf), _p(gb))
    return gf, gb
