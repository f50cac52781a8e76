"""Thin Python binding of libmhc.so (include/mhc.h).

Each function has the name of the C entry point it calls and only marshals
arguments: tensors become device pointers, shapes become an ``mhc_params``,
the stream is the current torch stream unless one is given.  Output tensors
are allocated with torch when the caller does not pass them.  Every step of
the computation runs in the library's CUDA kernels; a non-zero status raises
``MhcError``.  Tensors must be contiguous CUDA tensors on x's device.  Before
any launch every tensor is checked against the problem's sizes: the element
type the call reads or writes, and at least as many elements as it touches, so
that a mis-sized argument raises ValueError here instead of sending a kernel
past the end of an allocation.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib

DTYPE_CODE = {torch.float32: 0, torch.bfloat16: 1}
F32 = torch.float32


class MhcError(RuntimeError):
    """A libmhc entry point returned a non-zero mhc_status."""

    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {mhc_status_string(status)}")


def mhc_version() -> int:
    return int(_lib.load().mhc_version())


def mhc_status_string(status: int) -> str:
    return _lib.load().mhc_status_string(int(status)).decode()


def _check(st: int, where: str) -> None:
    if st != 0:
        raise MhcError(st, where)


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmhc takes CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("libmhc takes contiguous tensors only")
    return ctypes.c_void_p(t.data_ptr())


def _fits(t, numel, dtype, device, what):
    """Reject a tensor that the call would reinterpret (another element type),
    run past the end of (fewer elements than it reads or writes) or reach on
    another device.  None passes: the library rejects a missing required
    pointer itself."""
    if t is None:
        return
    if t.dtype != dtype:
        raise ValueError(f"{what}: dtype {t.dtype}, the call takes {dtype}")
    if t.numel() < numel:
        raise ValueError(f"{what}: {t.numel()} elements, the call touches {numel}")
    if t.device != device:
        raise ValueError(f"{what}: on {t.device}, the call runs on {device}")


def _on(t, device, what):
    """A workspace (any element type; the library checks its byte count) on the
    call's device."""
    if t is not None and t.device != device:
        raise ValueError(f"{what}: on {t.device}, the call runs on {device}")


def _maps_in(x, phi, b, alpha):
    """phi [nC, n^2+2n], b [n^2+2n], alpha [1] or [3]: fp32 on x's device."""
    T, n, C = x.shape
    M = n * n + 2 * n
    _fits(phi, n * C * M, F32, x.device, "phi")
    _fits(b, M, F32, x.device, "b")
    _fits(alpha, 1, F32, x.device, "alpha")


def _upstream(x, f_out, grad_x_next, grad_h_in):
    """The backward's activations: f_out and grad_h_in [T, C], grad_x_next
    [T, n, C], all of x's dtype (f_out may be None where the call takes none)."""
    T, n, C = x.shape
    _fits(f_out, T * C, x.dtype, x.device, "f_out")
    _fits(grad_x_next, T * n * C, x.dtype, x.device, "grad_x_next")
    _fits(grad_h_in, T * C, x.dtype, x.device, "grad_h_in")


def _grads_out(x, ag, gx, gphi, gb, ga, gf):
    """The backward's outputs: grad_x [T, n, C] and grad_f_out [T, C] of x's
    dtype; grad_phi, grad_b and grad_alpha (3 entries with per-group alpha)
    fp32."""
    T, n, C = x.shape
    M = n * n + 2 * n
    _fits(gx, T * n * C, x.dtype, x.device, "grad_x")
    _fits(gphi, n * C * M, F32, x.device, "grad_phi")
    _fits(gb, M, F32, x.device, "grad_b")
    _fits(ga, 3 if ag == 3 else 1, F32, x.device, "grad_alpha")
    _fits(gf, T * C, x.dtype, x.device, "grad_f_out")


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def params(n: int, T: int, C: int, dtype: torch.dtype, t_max: int = 20, eps: float = 1e-6,
           alpha_groups: int = 1, wait_ns: int = 0):
    """Build an ``mhc_params`` struct (alpha_groups 3: per-group alpha; wait_ns: limit of
    the tensor-core kernels' device-side waits, 0 = the library default)."""
    if dtype not in DTYPE_CODE:
        raise ValueError(f"unsupported activation dtype {dtype}")
    return _lib.MhcParams(n=int(n), t_max=int(t_max), T=int(T), C=int(C), eps=float(eps),
                          dtype=DTYPE_CODE[dtype], alpha_groups=int(alpha_groups),
                          wait_ns=int(wait_ns))


def _ag(alpha) -> int:
    """3 when alpha holds the pre, post and res scales, else 1 (one shared alpha)."""
    return 3 if alpha.numel() == 3 else 1


def mhc_pre_workspace_size(n: int, T: int, C: int, dtype: torch.dtype, t_max: int = 20,
                           eps: float = 1e-6) -> int:
    p = params(n, T, C, dtype, t_max, eps)
    return int(_lib.load().mhc_pre_workspace_size(ctypes.byref(p)))


def mhc_backward_workspace_size(n: int, T: int, C: int, dtype: torch.dtype, t_max: int = 20,
                                eps: float = 1e-6) -> int:
    p = params(n, T, C, dtype, t_max, eps)
    return int(_lib.load().mhc_backward_workspace_size(ctypes.byref(p)))


def _workspace(nbytes: int, device, ws):
    if nbytes == 0:
        return None, 0
    if ws is None:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return ws, ws.numel() * ws.element_size()


def mhc_pre(x, phi, b, alpha, *, t_max: int = 20, eps: float = 1e-6, wait_ns: int = 0,
            out=None, workspace=None, dev_status=None, stream=None):
    """x [T,n,C] -> (h_in [T,C], H_pre [T,n], H_post [T,n], H_res [T,n,n])."""
    T, n, C = x.shape
    p = params(n, T, C, x.dtype, t_max, eps, _ag(alpha), wait_ns)
    if out is None:
        out = (torch.empty(T, C, dtype=x.dtype, device=x.device),
               torch.empty(T, n, dtype=torch.float32, device=x.device),
               torch.empty(T, n, dtype=torch.float32, device=x.device),
               torch.empty(T, n, n, dtype=torch.float32, device=x.device))
    h_in, H_pre, H_post, H_res = out
    _maps_in(x, phi, b, alpha)
    _fits(h_in, T * C, x.dtype, x.device, "h_in")
    _fits(H_pre, T * n, F32, x.device, "H_pre")
    _fits(H_post, T * n, F32, x.device, "H_post")
    _fits(H_res, T * n * n, F32, x.device, "H_res")
    _fits(dev_status, 1, torch.int32, x.device, "dev_status")
    _on(workspace, x.device, "workspace")
    lib = _lib.load()
    ws, wsb = _workspace(int(lib.mhc_pre_workspace_size(ctypes.byref(p))), x.device, workspace)
    st = lib.mhc_pre(ctypes.byref(p), _p(x), _p(phi), _p(b), _p(alpha), _p(h_in), _p(H_pre),
                     _p(H_post), _p(H_res), _p(ws), wsb, _p(dev_status), _stream(stream))
    _check(st, "mhc_pre")
    return h_in, H_pre, H_post, H_res


def mhc_post(x, f_out, H_post, H_res, *, out=None, dev_status=None, stream=None):
    """x [T,n,C], f_out [T,C], H_post [T,n], H_res [T,n,n] -> x_next [T,n,C]."""
    T, n, C = x.shape
    p = params(n, T, C, x.dtype)
    x_next = torch.empty_like(x) if out is None else out
    _fits(f_out, T * C, x.dtype, x.device, "f_out")
    _fits(H_post, T * n, F32, x.device, "H_post")
    _fits(H_res, T * n * n, F32, x.device, "H_res")
    _fits(x_next, T * n * C, x.dtype, x.device, "x_next")
    _fits(dev_status, 1, torch.int32, x.device, "dev_status")
    st = _lib.load().mhc_post(ctypes.byref(p), _p(x), _p(f_out), _p(H_post), _p(H_res),
                              _p(x_next), _p(dev_status), _stream(stream))
    _check(st, "mhc_post")
    return x_next


def mhc_backward(x, phi, b, alpha, f_out, grad_x_next, grad_h_in, *, t_max: int = 20,
                 eps: float = 1e-6, wait_ns: int = 0, out=None, workspace=None, dev_status=None,
                 stream=None):
    """Gradients of pre+post with recompute.
    Returns (grad_x, grad_phi, grad_b, grad_alpha, grad_f_out)."""
    T, n, C = x.shape
    p = params(n, T, C, x.dtype, t_max, eps, _ag(alpha), wait_ns)
    if out is None:
        out = (torch.empty_like(x), torch.empty_like(phi), torch.empty_like(b),
               torch.empty_like(alpha), torch.empty_like(f_out))
    gx, gphi, gb, ga, gf = out
    _maps_in(x, phi, b, alpha)
    _upstream(x, f_out, grad_x_next, grad_h_in)
    _grads_out(x, _ag(alpha), gx, gphi, gb, ga, gf)
    _fits(dev_status, 1, torch.int32, x.device, "dev_status")
    _on(workspace, x.device, "workspace")
    lib = _lib.load()
    ws, wsb = _workspace(int(lib.mhc_backward_workspace_size(ctypes.byref(p))), x.device,
                         workspace)
    st = lib.mhc_backward(ctypes.byref(p), _p(x), _p(phi), _p(b), _p(alpha), _p(f_out),
                          _p(grad_x_next), _p(grad_h_in), _p(gx), _p(gphi), _p(gb), _p(ga),
                          _p(gf), _p(ws), wsb, _p(dev_status), _stream(stream))
    _check(st, "mhc_backward")
    return gx, gphi, gb, ga, gf


def mhc_backward_noalloc(x, phi, b, alpha, f_out, grad_x_next, grad_h_in, *, t_max: int = 20,
                         eps: float = 1e-6, wait_ns: int = 0, out=None, dev_status=None,
                         stream=None):
    """mhc_backward without a workspace: the library's fixed device scratch array is used
    (for callers that cannot allocate device memory).  Output tensors must be passed in
    ``out`` by callers that cannot allocate; they are created here only as a convenience.
    Returns (grad_x, grad_phi, grad_b, grad_alpha, grad_f_out)."""
    T, n, C = x.shape
    p = params(n, T, C, x.dtype, t_max, eps, _ag(alpha), wait_ns)
    if out is None:
        out = (torch.empty_like(x), torch.empty_like(phi), torch.empty_like(b),
               torch.empty_like(alpha), torch.empty_like(f_out))
    gx, gphi, gb, ga, gf = out
    _maps_in(x, phi, b, alpha)
    _upstream(x, f_out, grad_x_next, grad_h_in)
    _grads_out(x, _ag(alpha), gx, gphi, gb, ga, gf)
    _fits(dev_status, 1, torch.int32, x.device, "dev_status")
    st = _lib.load().mhc_backward_noalloc(ctypes.byref(p), _p(x), _p(phi), _p(b), _p(alpha),
                                          _p(f_out), _p(grad_x_next), _p(grad_h_in), _p(gx),
                                          _p(gphi), _p(gb), _p(ga), _p(gf), _p(dev_status),
                                          _stream(stream))
    _check(st, "mhc_backward_noalloc")
    return gx, gphi, gb, ga, gf


def mhc_post_fused(x, f_out, H_post, H_res, phi_next, b_next, alpha_next, *, t_max: int = 20,
                   eps: float = 1e-6, wait_ns: int = 0, out=None, workspace=None, dev_status=None,
                 stream=None):
    """Layer l's post merge fused with layer l+1's mapping.
    Returns (x_next [T,n,C], H_pre_next [T,n], H_post_next [T,n], H_res_next [T,n,n])."""
    T, n, C = x.shape
    p = params(n, T, C, x.dtype, t_max, eps, _ag(alpha_next), wait_ns)
    if out is None:
        out = (torch.empty_like(x), torch.empty(T, n, dtype=torch.float32, device=x.device),
               torch.empty(T, n, dtype=torch.float32, device=x.device),
               torch.empty(T, n, n, dtype=torch.float32, device=x.device))
    xn, hpre, hpost, hres = out
    _fits(f_out, T * C, x.dtype, x.device, "f_out")
    _fits(H_post, T * n, F32, x.device, "H_post")
    _fits(H_res, T * n * n, F32, x.device, "H_res")
    _maps_in(x, phi_next, b_next, alpha_next)
    _fits(xn, T * n * C, x.dtype, x.device, "x_next")
    _fits(hpre, T * n, F32, x.device, "H_pre_next")
    _fits(hpost, T * n, F32, x.device, "H_post_next")
    _fits(hres, T * n * n, F32, x.device, "H_res_next")
    _fits(dev_status, 1, torch.int32, x.device, "dev_status")
    _on(workspace, x.device, "workspace")
    lib = _lib.load()
    ws, wsb = _workspace(int(lib.mhc_post_fused_workspace_size(ctypes.byref(p))), x.device,
                         workspace)
    st = lib.mhc_post_fused(ctypes.byref(p), _p(x), _p(f_out), _p(H_post), _p(H_res),
                            _p(phi_next), _p(b_next), _p(alpha_next), _p(xn), _p(hpre),
                            _p(hpost), _p(hres), _p(ws), wsb, _p(dev_status), _stream(stream))
    _check(st, "mhc_post_fused")
    return xn, hpre, hpost, hres


def mhc_layer_input(x, H_pre, *, out=None, dev_status=None, stream=None):
    """h_in [T,C] = sum_i H_pre[i] x[i] (the second half of mhc_pre)."""
    T, n, C = x.shape
    p = params(n, T, C, x.dtype)
    h_in = torch.empty(T, C, dtype=x.dtype, device=x.device) if out is None else out
    _fits(H_pre, T * n, F32, x.device, "H_pre")
    _fits(h_in, T * C, x.dtype, x.device, "h_in")
    _fits(dev_status, 1, torch.int32, x.device, "dev_status")
    st = _lib.load().mhc_layer_input(ctypes.byref(p), _p(x), _p(H_pre), _p(h_in),
                                     _p(dev_status), _stream(stream))
    _check(st, "mhc_layer_input")
    return h_in


def mhc_post_backward(x, f_out, H_post, grad_x_next, *, out=None, dev_status=None, stream=None):
    """First half of the layer backward in training order (before F's backward).
    Returns (grad_f_out [T,C], red [T, n*n + n] float32)."""
    T, n, C = x.shape
    p = params(n, T, C, x.dtype)
    if out is None:
        out = (torch.empty_like(f_out),
               torch.empty(T, n * n + n, dtype=torch.float32, device=x.device))
    gf, red = out
    _fits(f_out, T * C, x.dtype, x.device, "f_out")
    _fits(H_post, T * n, F32, x.device, "H_post")
    _fits(grad_x_next, T * n * C, x.dtype, x.device, "grad_x_next")
    _fits(gf, T * C, x.dtype, x.device, "grad_f_out")
    _fits(red, T * (n * n + n), F32, x.device, "red")
    _fits(dev_status, 1, torch.int32, x.device, "dev_status")
    st = _lib.load().mhc_post_backward(ctypes.byref(p), _p(x), _p(f_out), _p(H_post),
                                       _p(grad_x_next), _p(gf), _p(red), _p(dev_status),
                                       _stream(stream))
    _check(st, "mhc_post_backward")
    return gf, red


def mhc_pre_backward(x, phi, b, alpha, grad_x_next, grad_h_in, red, *, t_max: int = 20,
                     eps: float = 1e-6, wait_ns: int = 0, out=None, workspace=None, dev_status=None,
                 stream=None):
    """Second half of the layer backward in training order (after F's backward).
    Returns (grad_x, grad_phi, grad_b, grad_alpha)."""
    T, n, C = x.shape
    p = params(n, T, C, x.dtype, t_max, eps, _ag(alpha), wait_ns)
    if out is None:
        out = (torch.empty_like(x), torch.empty_like(phi), torch.empty_like(b),
               torch.empty_like(alpha))
    gx, gphi, gb, ga = out
    _maps_in(x, phi, b, alpha)
    _upstream(x, None, grad_x_next, grad_h_in)
    _fits(red, T * (n * n + n), F32, x.device, "red")
    _grads_out(x, _ag(alpha), gx, gphi, gb, ga, None)
    _fits(dev_status, 1, torch.int32, x.device, "dev_status")
    _on(workspace, x.device, "workspace")
    lib = _lib.load()
    ws, wsb = _workspace(int(lib.mhc_pre_backward_workspace_size(ctypes.byref(p))), x.device,
                         workspace)
    st = lib.mhc_pre_backward(ctypes.byref(p), _p(x), _p(phi), _p(b), _p(alpha), _p(grad_x_next),
                              _p(grad_h_in), _p(red), _p(gx), _p(gphi), _p(gb), _p(ga), _p(ws),
                              wsb, _p(dev_status), _stream(stream))
    _check(st, "mhc_pre_backward")
    return gx, gphi, gb, ga


def mhc_backward_map(x, phi, b, alpha, f_out, grad_x_next, grad_h_in, workspace, *,
                     t_max: int = 20, eps: float = 1e-6, wait_ns: int = 0, dev_status=None,
                     stream=None):
    """Phase 1 of mhc_backward: per-token records into ``workspace`` (uint8 tensor of at
    least mhc_backward_workspace_size bytes)."""
    T, n, C = x.shape
    p = params(n, T, C, x.dtype, t_max, eps, _ag(alpha), wait_ns)
    _maps_in(x, phi, b, alpha)
    _upstream(x, f_out, grad_x_next, grad_h_in)
    _fits(dev_status, 1, torch.int32, x.device, "dev_status")
    _on(workspace, x.device, "workspace")
    st = _lib.load().mhc_backward_map(ctypes.byref(p), _p(x), _p(phi), _p(b), _p(alpha), _p(f_out),
                                      _p(grad_x_next), _p(grad_h_in), _p(workspace),
                                      workspace.numel(), _p(dev_status), _stream(stream))
    _check(st, "mhc_backward_map")


def mhc_backward_apply(x, phi, grad_x_next, grad_h_in, workspace, *, t_max: int = 20,
                       eps: float = 1e-6, wait_ns: int = 0, alpha_groups: int = 1, out=None,
                       dev_status=None, stream=None):
    """Phase 2 of mhc_backward (alpha_groups as in the map phase).
    Returns (grad_x, grad_phi, grad_b, grad_alpha, grad_f_out)."""
    T, n, C = x.shape
    p = params(n, T, C, x.dtype, t_max, eps, alpha_groups, wait_ns)
    M = n * n + 2 * n
    if out is None:
        out = (torch.empty_like(x), torch.empty_like(phi),
               torch.empty(M, dtype=torch.float32, device=x.device),
               torch.empty(3 if alpha_groups == 3 else 1, dtype=torch.float32, device=x.device),
               torch.empty(T, C, dtype=x.dtype, device=x.device))
    gx, gphi, gb, ga, gf = out
    _fits(phi, n * C * M, F32, x.device, "phi")
    _upstream(x, None, grad_x_next, grad_h_in)
    _grads_out(x, alpha_groups, gx, gphi, gb, ga, gf)
    _fits(dev_status, 1, torch.int32, x.device, "dev_status")
    _on(workspace, x.device, "workspace")
    st = _lib.load().mhc_backward_apply(ctypes.byref(p), _p(x), _p(phi), _p(grad_x_next),
                                        _p(grad_h_in), _p(gx), _p(gphi), _p(gb), _p(ga), _p(gf),
                                        _p(workspace), workspace.numel(), _p(dev_status),
                                        _stream(stream))
    _check(st, "mhc_backward_apply")
    return gx, gphi, gb, ga, gf


def mhc_sinkhorn_knopp(logits, iters: int = 20, *, out=None, dev_status=None, stream=None):
    """logits [..., n, n] fp32 -> Sinkhorn-Knopp estimate, same shape."""
    n = logits.shape[-1]
    B = logits.numel() // (n * n)
    res = torch.empty_like(logits) if out is None else out
    _fits(logits, B * n * n, F32, logits.device, "logits")
    _fits(res, B * n * n, F32, logits.device, "out")
    _fits(dev_status, 1, torch.int32, logits.device, "dev_status")
    st = _lib.load().mhc_sinkhorn_knopp(int(n), int(iters), int(B), _p(logits), _p(res),
                                        _p(dev_status), _stream(stream))
    _check(st, "mhc_sinkhorn_knopp")
    return res


def mhc_depth_amax(H, *, out=None, dev_status=None, stream=None):
    """H [T, L, n, n] fp32 -> (gain_fwd [T], gain_bwd [T]) of P = H[L-1] ... H[0]."""
    T, L, n, _ = H.shape
    if out is None:
        out = (torch.empty(T, dtype=torch.float32, device=H.device),
               torch.empty(T, dtype=torch.float32, device=H.device))
    gf, gb = out
    _fits(H, T * L * n * n, F32, H.device, "H")
    _fits(gf, T, F32, H.device, "gain_fwd")
    _fits(gb, T, F32, H.device, "gain_bwd")
    _fits(dev_status, 1, torch.int32, H.device, "dev_status")
    st = _lib.load().mhc_depth_amax(int(n), int(T), int(L), _p(H), _p(gf), _p(gb),
                                    _p(dev_status), _stream(stream))
    _check(st, "mhc_depth_amax")
    return gf, gb


def mhc_recompute_plan(n: int, L: int):
    """(block, resident): the recompute block size for an L-layer stack with n streams and
    the resident activations per token at the backward's peak, in units of C elements."""
    blk, res = ctypes.c_int32(0), ctypes.c_int64(0)
    st = _lib.load().mhc_recompute_plan(int(n), int(L), ctypes.byref(blk), ctypes.byref(res))
    _check(st, "mhc_recompute_plan")
    return int(blk.value), int(res.value)
