"""ctypes view of libmoe.so (the C ABI declared in include/moe.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Loading fails loudly when the library has not been built;
there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

c_int, c_size_t, c_int64 = ctypes.c_int, ctypes.c_size_t, ctypes.c_int64
P = ctypes.c_void_p

MOE_OK = 0
MOE_DTYPE_BF16, MOE_DTYPE_MXFP8 = 0, 1
MOE_FLAG_RENORM = 1
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_CUDA",
                4: "MOE_ERR_WORKSPACE", 5: "MOE_ERR_DEVICE_CHECK", 6: "MOE_ERR_TIMEOUT"}


class MoeShape(ctypes.Structure):
    _fields_ = [("T", c_int), ("d_model", c_int), ("d_ff", c_int), ("n_experts", c_int),
                ("top_k", c_int), ("dtype", c_int), ("flags", c_int)]


SP = ctypes.POINTER(MoeShape)

# name -> argument types (restype is moe_status_t == int unless noted)
SIGNATURES = {
    "moe_create": [ctypes.POINTER(P), c_int],
    "moe_destroy": [P],
    "moe_workspace_size": [P, SP, ctypes.POINTER(c_size_t)],
    "moe_max_rows": [SP, ctypes.POINTER(c_int64)],
    "moe_router_topk": [P, SP, P, P, P, P, P, P, P, P, P, c_size_t, P],
    "moe_permute": [P, SP, P, P, P, P, P, P, P, c_size_t, P],
    "moe_permute_noalloc": [P, SP, P, P, P, P, P, P, P],
    "moe_route": [P, SP, P, P, P, P, P, P, c_size_t, P],
    "moe_permute_src": [P, SP, P, P, P, P, P, P, P, P, c_size_t, P],
    "moe_grouped_swiglu_fwd_combine": [P, SP, P, P, P, P, P, P, P, P, P, P, P, P, P, P],
    "moe_grouped_swiglu_fwd_gather": [P, SP, P, P, P, P, P, P, P, P, P],
    "moe_grouped_swiglu_recompute_gather": [P, SP, P, P, P, P, P, P, P],
    "moe_grouped_swiglu_bwd_gather": [P, SP, P, P, P, P, P, P, P, P, P, P, P, P, P],
    "moe_grouped_swiglu_fwd": [P, SP, P, P, P, P, P, P, P, P, c_size_t, P],
    "moe_grouped_swiglu_recompute": [P, SP, P, P, P, P, P, P, c_size_t, P],
    "moe_unpermute_combine": [P, SP, P, P, P, P, P, P],
    "moe_unpermute_combine_bwd": [P, SP, P, P, P, P, P, P, P, P, P],
    "moe_grouped_swiglu_bwd": [P, SP, P, P, P, P, P, P, P, P, P, P, P, P, c_size_t, P],
    "moe_permute_bwd": [P, SP, P, P, P, P, P, P],
    "moe_permute_router_bwd": [P, SP, P, P, P, P, P, P, P, P, P, P],
    "moe_shared_expert_fwd": [P, SP, P, P, P, P, P, P, P],
    "moe_shared_expert_bwd": [P, SP, P, P, P, P, P, P, P, P, P, P, P],
    "moe_router_topk_bwd": [P, SP, P, P, P, P, P, P, P, P, P, P, c_size_t, P],
    "moe_router_load_stats": [P, SP, P, P, c_int, P, P, c_size_t, P],
    "moe_router_aux_loss": [P, SP, P, c_int64, ctypes.c_float, P, P, P],
    "moe_mxfp8_quantize": [P, P, c_int64, c_int64, c_int, P, P, P],
    "moe_mxfp8_quantize_gemm": [P, P, c_int64, c_int64, c_int64, P, P, P, P, P],
    "moe_get_status": [P, ctypes.POINTER(c_int)],
    "moe_get_launch_count": [P, ctypes.POINTER(ctypes.c_uint64)],
    "moe_set_wait_limit": [P, ctypes.c_uint64],
    "moe_status_string": [c_int],
}

_lib = None


def load():
    """Loads libmoe.so once and declares every entry point."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m mixture_experts_layer_39_b200.build`"
            " (the MoE layer has no non-CUDA implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, args in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name == "moe_status_string" else c_int
    _lib = lib
    return lib
