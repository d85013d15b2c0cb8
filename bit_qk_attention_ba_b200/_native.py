"""ctypes binding of libba (include/ba.h): argument marshalling only.

Every compute step runs in the CUDA kernels of libba.so; this module turns
torch tensors into device pointers and sizes, passes the caller's current CUDA
stream, and raises on a non-OK status.  There is no fallback: if libba.so is
missing the import fails.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libba.so")

BA_OK, BA_ERR_INVALID_ARG, BA_ERR_UNSUPPORTED, BA_ERR_CUDA, BA_ERR_DEVICE_STATUS = 0, 1, 2, 3, 4
BA_F32, BA_BF16 = 0, 1
BA_BIAS_NONE, BA_BIAS_DENSE, BA_BIAS_RELPOS2D, BA_BIAS_RELPOS2D_CLS = 0, 1, 2, 3
BA_QK_AUTO, BA_QK_POPC, BA_QK_MMA_B1, BA_QK_TC_I8, BA_QK_TC_F8 = 0, 1, 2, 3, 4

# name -> (restype, argtypes); mirrors include/ba.h
_P, _I, _I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
SIGNATURES = {
    "ba_words": (_I, [_I]),
    "ba_vq_ld": (_I64, [_I]),
    "ba_pack_qk": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "ba_quant_v": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "ba_prepass_qkv": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "ba_attention_decode": (_I, [_P, _P, _I, _P, _P, _P, _P, _I, _P, _I64, _I, _I, _I, _P, _I64, _P, _I, _P]),
    "ba_attention_decode_workspace_bytes": (_I64, [_I, _I, _I, _I, _I]),
    "ba_prepass_launches": (_I, [_I, _I, _I]),
    "ba_attention_workspace_bytes": (_I64, [_I, _I, _I, _I, _I, _I, _I]),
    "ba_attention_fwd": (_I, [_P, _P, _P, _P, _P, _P, _I, _P, _I64, _I, _I, _I, _I, _I, _I, _P, _I64,
                              _P, _I, _P]),
    "ba_attention_fwd_variant": (_I, [_P, _P, _P, _P, _P, _P, _I, _P, _I64, _I, _I, _I, _I, _I, _I, _P, _I64,
                                      _P, _I, _I, _P]),
    "ba_attention_fwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _I, _P, _I64, _I, _I, _I, _I, _I, _I, _P, _I,
                                      _P]),
    "ba_fwd_graph_create": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _I, _P, _I64, _I, _I,
                                 _P, _I64, _P, _I, _I, ctypes.POINTER(_P)]),
    "ba_fwd_graph_launch": (_I, [_P, _P]),
    "ba_fwd_graph_kernels": (_I, [_P]),
    "ba_fwd_graph_destroy": (_I, [_P]),
    "ba_attention_bwd": (_I, [_P, _P, _I, _P, _P, _P, _P, _P, _P, _I, _P, _I64, _I, _I, _I, _I, _I, _I,
                              _P, _P, ctypes.c_float, _P, _I64, _P, _P, _P, _P, _P]),
    "ba_attention_bwd_workspace_bytes": (_I64, [_I, _I, _I]),
    "ba_scores_debug": (_I, [_P, _P, _I, _I, _I, _I, _P, _P]),
    "ba_check_device_status": (_I, [_P, ctypes.POINTER(ctypes.c_int)]),
    "ba_test_attention_fwd_starved": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _I64, _P, _I, _I, _I64,
                                           _P]),
    "ba_status_string": (ctypes.c_char_p, [_I]),
}


class BAError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__("%s failed: %s" % (fn, msg))
        self.status = status


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError("libba.so not built at %s (run python -m bit_qk_attention_ba_b200.build)" % path)
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = load()
    return _lib


def check(fn: str, status: int) -> None:
    if status != BA_OK:
        raise BAError(fn, status, lib().ba_status_string(status).decode())


def call(fn: str, *args) -> None:
    check(fn, getattr(lib(), fn)(*args))
