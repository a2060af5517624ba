"""ctypes declarations of the C ABI in include/nanochat_b200.h.

Loading fails loudly when the in-tree CUDA library has not been built: there
is no CPU fallback for any entry point.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# NC_LIB_PATH selects another build of the same library (e.g. for A/B timing).
LIB_PATH = os.environ.get("NC_LIB_PATH") or os.path.join(HERE, "libnanochat_b200.so")

NC_OK = 0
NC_ERR_INVALID_ARG = -1
NC_ERR_UNSUPPORTED_SHAPE = -2
NC_ERR_WORKSPACE_TOO_SMALL = -3
NC_ERR_CUDA = -4
NC_ERR_BAD_TOKEN = -5
NC_ERR_DEVICE_TIMEOUT = -6
NC_ERR_NO_DEVICE = -7

NC_RECOMPUTE_NONE = 0
NC_RECOMPUTE_MLP = 1

NC_LM_HEAD_FUSED = 0
NC_LM_HEAD_MATERIALISED = 1

NC_PREC_BF16 = 0
NC_PREC_FP32_DEBUG = 1


class NcProfileRow(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_char_p), ("launches", ctypes.c_int64), ("ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


class NcAdamwGroup(ctypes.Structure):
    _fields_ = [("offset", ctypes.c_int64), ("count", ctypes.c_int64), ("lr", ctypes.c_float),
                ("beta1", ctypes.c_float), ("beta2", ctypes.c_float), ("eps", ctypes.c_float),
                ("weight_decay", ctypes.c_float)]


NC_ADAMW_MAX_GROUPS = 16


class NcConfig(ctypes.Structure):
    _fields_ = [("vocab", ctypes.c_int), ("d_model", ctypes.c_int), ("n_layer", ctypes.c_int),
                ("n_head", ctypes.c_int), ("n_kv_head", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("mlp_mult", ctypes.c_int), ("softcap", ctypes.c_float), ("rope_base", ctypes.c_float)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t

# name -> (restype, argtypes); every symbol include/nanochat_b200.h declares.
SIGNATURES = {
    "nc_model_create": (_I, [ctypes.POINTER(NcConfig), _I, ctypes.POINTER(_P)]),
    "nc_model_destroy": (None, [_P]),
    "nc_num_params": (ctypes.c_int64, [_P]),
    "nc_param_layout": (_I, [_P, _I, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_int64),
                             ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "nc_workspace_bytes": (_SZ, [_P, _I, _I]),
    "nc_forward_backward": (_I, [_P, _P, _P, _I, _I, _P, _P, _P, _P, _SZ, _P]),
    "nc_forward_backward_host": (_I, [_P, _P, _P, _I, _I, _P, _P, _P, _P, _SZ, _P]),
    "nc_forward_logits": (_I, [_P, _P, _I, _I, _P, _P, _P, _SZ, _P]),
    "nc_check": (_I, [_P, _P]),
    "nc_status_string": (ctypes.c_char_p, [_I]),
    "nc_profile_enable": (_I, [_P, _I]),
    "nc_profile_read": (_I, [_P, _P, ctypes.POINTER(NcProfileRow), _I]),
    "nc_launch_count": (ctypes.c_int64, []),
    "nc_grad_bucket_count": (_I, [_P]),
    "nc_grad_bucket": (_I, [_P, _I, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64)]),
    "nc_set_grad_events": (_I, [_P, ctypes.POINTER(ctypes.c_void_p), _I]),
    "nc_debug_expired_wait": (_I, [_P, _I, _P]),
    "nc_set_lm_head": (_I, [_P, _I, _I]),
    "nc_set_recompute": (_I, [_P, _I]),
    "nc_kv_cache_bytes": (_SZ, [_P, _I, _I]),
    "nc_inference_workspace_bytes": (_SZ, [_P, _I, _I]),
    "nc_prefill": (_I, [_P, _P, _I, _I, _P, _P, _I, _P, _P, _SZ, _P]),
    "nc_decode_step": (_I, [_P, _P, _I, _I, _P, _P, _I, _P, _P, _SZ, _P]),
    "nc_adamw_step": (_I, [ctypes.POINTER(NcAdamwGroup), _I, ctypes.c_int64, _I, _P, _P, _I, _P, _P, _P, _P]),
    "nc_gemm_wgrad_noalloc": (_I, [_I, _I, _I, _P, ctypes.c_int64, _P, ctypes.c_int64, _P, _I, _P, _P]),
    # include/nanochat_b200_testing.h
    "nc_test_gemm": (_I, [_I, _I, _I, _I, _P, ctypes.c_int64, _I, _P, ctypes.c_int64, _I, _I, _P,
                          ctypes.c_int64, _I, _P, ctypes.c_int64, _P, ctypes.c_int64, ctypes.c_float, _I, _P,
                          _SZ, _P, _P]),
    "nc_test_attention_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I]),
    "nc_test_attention": (_I, [_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _SZ, _I, _P, _P]),
}

_lib = None


def lib():
    """The loaded CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"bwd_step_b200: the CUDA library {LIB_PATH} is missing; build it with "
                "`python -m bwd_step_b200.build` (or __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib
