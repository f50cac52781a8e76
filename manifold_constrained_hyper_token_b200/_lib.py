"""ctypes loader for libmhc.so.  Raises if the library is missing: there is no
fallback implementation anywhere in this package."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmhc.so")

# mhc.h symbols this binding requires
SYMBOLS = ("mhc_version", "mhc_status_string", "mhc_pre_workspace_size", "mhc_pre", "mhc_post",
           "mhc_backward_workspace_size", "mhc_backward", "mhc_backward_map", "mhc_backward_apply",
           "mhc_backward_noalloc", "mhc_post_backward", "mhc_pre_backward_workspace_size",
           "mhc_pre_backward", "mhc_post_fused_workspace_size", "mhc_post_fused",
           "mhc_layer_input", "mhc_sinkhorn_knopp", "mhc_depth_amax", "mhc_recompute_plan")


class MhcParams(ctypes.Structure):
    """Mirror of ``mhc_params`` in include/mhc.h."""
    _fields_ = [("n", ctypes.c_int32), ("t_max", ctypes.c_int32), ("T", ctypes.c_int64),
                ("C", ctypes.c_int64), ("eps", ctypes.c_float), ("dtype", ctypes.c_int32),
                ("alpha_groups", ctypes.c_int32), ("wait_ns", ctypes.c_int64)]


_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libmhc.so not built ({LIB_PATH}); run "
                           "`python -m manifold_constrained_hyper_token_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    pp = ctypes.POINTER(MhcParams)
    lib.mhc_version.restype = i32
    lib.mhc_version.argtypes = []
    lib.mhc_status_string.restype = ctypes.c_char_p
    lib.mhc_status_string.argtypes = [i32]
    lib.mhc_pre_workspace_size.restype = sz
    lib.mhc_pre_workspace_size.argtypes = [pp]
    lib.mhc_pre.restype = i32
    lib.mhc_pre.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
    lib.mhc_post.restype = i32
    lib.mhc_post.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp]
    lib.mhc_backward_workspace_size.restype = sz
    lib.mhc_backward_workspace_size.argtypes = [pp]
    lib.mhc_backward.restype = i32
    lib.mhc_backward.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
    lib.mhc_backward_map.restype = i32
    lib.mhc_backward_map.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
    lib.mhc_backward_apply.restype = i32
    lib.mhc_backward_apply.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
    lib.mhc_backward_noalloc.restype = i32
    lib.mhc_backward_noalloc.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.mhc_post_backward.restype = i32
    lib.mhc_post_backward.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.mhc_pre_backward_workspace_size.restype = sz
    lib.mhc_pre_backward_workspace_size.argtypes = [pp]
    lib.mhc_pre_backward.restype = i32
    lib.mhc_pre_backward.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp,
                                     vp]
    lib.mhc_post_fused_workspace_size.restype = sz
    lib.mhc_post_fused_workspace_size.argtypes = [pp]
    lib.mhc_post_fused.restype = i32
    lib.mhc_post_fused.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
    lib.mhc_layer_input.restype = i32
    lib.mhc_layer_input.argtypes = [pp, vp, vp, vp, vp, vp]
    lib.mhc_sinkhorn_knopp.restype = i32
    lib.mhc_sinkhorn_knopp.argtypes = [i32, i32, i64, vp, vp, vp, vp]
    lib.mhc_depth_amax.restype = i32
    lib.mhc_depth_amax.argtypes = [i32, i64, i32, vp, vp, vp, vp, vp]
    lib.mhc_recompute_plan.restype = i32
    lib.mhc_recompute_plan.argtypes = [ctypes.c_int32, ctypes.c_int32,
                                       ctypes.POINTER(ctypes.c_int32),
                                       ctypes.POINTER(ctypes.c_int64)]
    _lib = lib
    return lib
