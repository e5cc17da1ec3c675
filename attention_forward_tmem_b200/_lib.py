"""ctypes declarations of the C ABI in ``include/wf_attn.h``.

Loads ``libwfattn.so`` from this package directory.  If the library is
missing the import fails with a message that says how to build it: there is
no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libwfattn.so")

# wf_status_t
WF_OK = 0
WF_ERR_INVALID_ARG = 1
WF_ERR_UNSUPPORTED = 2
WF_ERR_ORDER = 3
WF_ERR_CUDA = 4
WF_ERR_NO_MEMORY = 5
WF_ERR_TIMEOUT = 6
WF_ERR_NO_DEVICE = 7
STATUS_NAMES = {0: "WF_OK", 1: "WF_ERR_INVALID_ARG", 2: "WF_ERR_UNSUPPORTED", 3: "WF_ERR_ORDER",
                4: "WF_ERR_CUDA", 5: "WF_ERR_NO_MEMORY", 6: "WF_ERR_TIMEOUT", 7: "WF_ERR_NO_DEVICE"}

# wf_dtype_t
WF_F32, WF_BF16, WF_F16, WF_U8, WF_I32 = 0, 1, 2, 3, 4

# wf_mask_type_t
WF_MASK_NONE, WF_MASK_CAUSAL, WF_MASK_BOOL_KEEP, WF_MASK_ADDITIVE, WF_MASK_CAUSAL_TOP_LEFT = 0, 1, 2, 3, 4


class WfTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


_T = ctypes.POINTER(WfTensor)
_P = ctypes.c_void_p
_I32, _I64, _F32, _U32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_uint32

# name -> (restype, argtypes); every function the header declares
SIGNATURES = {
    "wf_attn_fwd": (_I32, [_T, _T, _T, _T, _T, _T, _T, _T, _I32, _I32, _F32, _I32, _T, _P]),
    "wf_attn_fwd_ex": (_I32, [_T, _T, _T, _T, _T, _T, _T, _T, _I32, _I32, _F32, _I32, _T, _T, _I32,
                              _P]),
    "wf_attn_merge": (_I32, [_T, _T, _T, _T, _P]),
    "wf_attn_dca": (_I32, [_T, _T, _T, _T, _T, _I64, _I32, _I32, _F32, _T, _T, _P]),
    "wf_attn_fwd_debug": (_I32, [_T, _T, _T, _T, _T, _T, _T, _T, _I32, _I32, _F32, _I32, _T, _P,
                                 _U32, _I64]),
    "wf_attn_fwd_varlen_noalloc": (_I32, [_T, _T, _T, _T, _T, _T, _T, _I32, _I32, _F32, _I32, _T,
                                          _P]),
    "wf_kvcache_create": (_I32, [_T, _T, _I32, _I64, _I64, _I64, ctypes.POINTER(_P)]),
    "wf_kvcache_before_update": (_I32, [_P, _I64]),
    "wf_kvcache_update": (_I32, [_P, _T, _T, _P]),
    "wf_kvcache_cached": (_I32, [_P, _T, _T, ctypes.POINTER(_I64)]),
    "wf_kvcache_update_attend": (_I32, [_P, _T, _T, _T, _I32, _F32, _T, _P]),
    "wf_kvcache_after_update": (_I32, [_P, _I64]),
    "wf_kvcache_get_state": (_I32, [_P, ctypes.POINTER(_I64), ctypes.POINTER(_I64),
                                    ctypes.POINTER(_I64), ctypes.POINTER(_I64),
                                    ctypes.POINTER(_I32)]),
    "wf_kvcache_set_state": (_I32, [_P, _I64]),
    "wf_kvcache_gather_logical": (_I32, [_P, _T, _T, _P]),
    "wf_kvcache_destroy": (None, [_P]),
    "wf_get_device_status": (_I32, [_P]),
    "wf_last_error_message": (ctypes.c_char_p, []),
    "wf_version": (_I32, []),
    "wf_shutdown": (None, []),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load the library once (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m attention_forward_tmem_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib
