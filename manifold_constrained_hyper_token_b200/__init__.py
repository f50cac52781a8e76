"""mHC (manifold-constrained hyper-connections) layer hot path for NVIDIA B200.

The computation lives in ``libmhc.so`` (CUDA, sm_100a; C ABI in
``include/mhc.h``).  This package holds the build script, a ctypes binding
with the C entry points' names (``api``) and the seeded synthetic input
recipes (``synth``), and the depth-stack driver with block recompute (``depth``).
"""
from .api import (MhcError, mhc_backward, mhc_backward_apply, mhc_backward_map,
                  mhc_backward_noalloc, mhc_backward_workspace_size, mhc_depth_amax, mhc_post,
                  mhc_layer_input, mhc_post_backward, mhc_post_fused, mhc_pre,
                  mhc_pre_backward, mhc_pre_workspace_size, mhc_recompute_plan,
                  mhc_sinkhorn_knopp, mhc_status_string, mhc_version, params)

__all__ = ["MhcError", "mhc_backward", "mhc_backward_apply", "mhc_backward_map",
           "mhc_backward_noalloc", "mhc_backward_workspace_size", "mhc_depth_amax", "mhc_post",
           "mhc_layer_input", "mhc_post_backward", "mhc_post_fused", "mhc_pre",
           "mhc_pre_backward", "mhc_pre_workspace_size", "mhc_recompute_plan",
           "mhc_sinkhorn_knopp", "mhc_status_string", "mhc_version", "params"]
