"""ctypes view of libpisa.so (the C ABI declared in include/pisa.h).

Loading fails loudly when the library has not been built: there is no
fallback implementation of any step.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpisa.so")

PISA_OK = 0
PISA_ERR_INVALID_ARG = 1
PISA_ERR_UNSUPPORTED = 2
PISA_ERR_CUDA = 3
PISA_ERR_WORKSPACE = 4
PISA_ERR_TIMEOUT = 5
PISA_ERR_DEVICE = 6

PISA_MODE_HYD = 0
PISA_MODE_0TH = 1
PISA_MODE_1ST = 2
PISA_BF16 = 0
PISA_F32 = 1
PISA_SINK_NONE = -(2 ** 31)

# every exported symbol of include/pisa.h, with (restype, argtypes)
_P, _I, _Z, _D, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_double, ctypes.c_float


class PisaOptions(ctypes.Structure):
    _fields_ = [("scale", ctypes.c_float), ("cov_weight", ctypes.c_float),
                ("dtype", ctypes.c_int), ("workspace", ctypes.c_void_p),
                ("ws_bytes", ctypes.c_size_t), ("fuse_select", ctypes.c_int),
                ("idx_out", ctypes.c_void_p)]


SIGNATURES = {
    "pisa_num_blocks": (_I, [_I, _I]),
    "pisa_num_selected": (_I, [_I, _D]),
    "pisa_workspace_bytes": (_Z, [_I, _I, _I, _I, _I, _D, _I, _I]),
    "pisa_block_stats_workspace_bytes": (_Z, [_I, _I, _I, _I, _I]),
    "pisa_select_workspace_bytes": (_Z, [_I, _I, _I]),
    "pisa_sparse_attention_workspace_bytes": (_Z, [_I, _I, _I, _I, _I, _I]),
    "pisa_block_stats": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                              _P, _P, _P, _P, _P, _P, _Z, _P]),
    "pisa_select": (_I, [_P, _P, _P, _F, _F, _I, _I, _I, _I, _D, _I, _P, _P, _Z, _P]),
    "pisa_sparse_attention": (_I, [_P, _P, _P, _I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                   _F, _I, _P, _P, _Z, _P]),
    "pisa_sparse_attention_fwd": (_I, [_P, _P, _P, _I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                       _F, _I, _P, _P, _P, _P, _Z, _P]),
    "pisa_sparse_attention_bwd_workspace_bytes": (_Z, [_I, _I, _I, _I, _I, _I]),
    "pisa_sparse_attention_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I,
                                       _I, _F, _P, _P, _P, _P, _Z, _P]),
    "pisa_attention": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _D, _I, _I, _P]),
    "pisa_attention_ex": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _D, _I, _I,
                               ctypes.POINTER(PisaOptions), _P]),
    "pisa_dense_attention": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "pisa_dense_attention_workspace_bytes": (_Z, [_I, _I, _I, _I, _I]),
    "pisa_block_stats_noalloc": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                      _P, _P, _P, _P, _P, _P]),
    "pisa_selftest_timeout": (_I, [ctypes.c_uint64, _P]),
    "pisa_tail_score_histogram": (_I, [_P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _F, _F, _F, _I,
                                       _I, _P, _P, _P, _P]),
    "pisa_device_status": (_I, [_P]),
    "pisa_status_string": (ctypes.c_char_p, [_I]),
    "pisa_last_error": (ctypes.c_char_p, []),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libpisa.so once; raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m block_sparse_attention_stats_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
