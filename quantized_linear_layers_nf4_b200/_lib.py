"""ctypes binding of ``lib/libnf4.so`` (the C ABI declared in ``include/nf4.h``).

Argument marshalling only.  Loading fails loudly when the library has not been
built: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libnf4.so")

NF4_OK = 0
NF4_ERR_DEVICE_TIMEOUT = -8
NF4_F32 = 0
NF4_BF16 = 1
NF4_BLOCKSIZE = 64
NF4_BLOCKSIZE2 = 256
NF4_WEIGHT_MAGIC = 0x4E463442
NF4_FP4_WEIGHT_MAGIC = 0x46503442
NF4_QUANT_NF4 = 0
NF4_QUANT_FP4 = 1
NF4_WEIGHT_VERSION = 1
NF4_ABI_VERSION = 1
NF4_DQ_NOALLOC_MAX_NB = 16777216
NF4_LINEAR_WEIGHTS_EARLY = 1
NF4_LINEAR_TEST_TIMEOUT = 0x80000000
NF4_LINEAR_GROUP_MAX = 4
NF4_DEQUANT_BATCH_MAX = 16

# Every function include/nf4.h declares, with (restype, argtypes).
_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32


class nf4_weight_t(ctypes.Structure):
    """Mirror of ``struct nf4_weight`` (host struct borrowing device pointers)."""
    _fields_ = [("magic", ctypes.c_uint32), ("version", ctypes.c_uint32), ("n", _i64), ("k", _i64),
                ("blocksize", _i32), ("blocksize2", _i32), ("wq", _p), ("absmax_q", _p),
                ("absmax_scale", _p), ("absmax_offset", _p)]


SIGNATURES = {
    "nf4_abi_version": (ctypes.c_int, []),
    "nf4_status_str": (ctypes.c_char_p, [ctypes.c_int]),
    "nf4_codebook": (ctypes.c_int, [_p]),
    "nf4_codebook_typed": (ctypes.c_int, [ctypes.c_int, _p]),
    "nf4_quantize_typed": (ctypes.c_int, [_p, ctypes.c_int, _i64, _i64, ctypes.c_int, _p, _p, _p]),
    "nf4_quantize": (ctypes.c_int, [_p, ctypes.c_int, _i64, _i64, _p, _p, _p]),
    "nf4_double_quant_workspace_bytes": (ctypes.c_size_t, [_i64]),
    "nf4_double_quant": (ctypes.c_int, [_p, _i64, _p, ctypes.c_size_t, _p, _p, _p, _p]),
    "nf4_double_quant_noalloc": (ctypes.c_int, [_p, _i64, _p, _p, _p, _p]),
    "nf4_dequantize": (ctypes.c_int, [ctypes.POINTER(nf4_weight_t), _p, ctypes.c_int, _p]),
    "nf4_linear": (ctypes.c_int, [_p, _i64, ctypes.POINTER(nf4_weight_t), _p, ctypes.c_int, _p, _p]),
    "nf4_linear_ex": (ctypes.c_int, [_p, _i64, ctypes.POINTER(nf4_weight_t), _p, ctypes.c_int, _p,
                                     ctypes.c_uint32, _p]),
    "nf4_linear_workspace_bytes": (ctypes.c_size_t, [_i64, _i64, _i64]),
    "nf4_linear_dx": (ctypes.c_int, [_p, _i64, ctypes.POINTER(nf4_weight_t), _p, ctypes.c_int, _p, _p]),
    "nf4_linear_lora_workspace_bytes": (ctypes.c_size_t, [_i64, _i64, _i64, ctypes.c_int32]),
    "nf4_linear_lora": (ctypes.c_int, [_p, _i64, ctypes.POINTER(nf4_weight_t), _p, _p, ctypes.c_int32,
                                       ctypes.c_float, _p, ctypes.c_int, _p, ctypes.c_uint32, _p, ctypes.c_size_t,
                                       _p]),
    "nf4_merge_lora": (ctypes.c_int, [ctypes.POINTER(nf4_weight_t), _p, _p, ctypes.c_int32, ctypes.c_float, _p,
                                      _p, _p, _p]),
    "nf4_linear_ws": (ctypes.c_int, [_p, _i64, ctypes.POINTER(nf4_weight_t), _p, ctypes.c_int, _p,
                                     ctypes.c_uint32, _p, ctypes.c_size_t, _p]),
    "nf4_linear_group": (ctypes.c_int, [_p, _i64, ctypes.POINTER(ctypes.POINTER(nf4_weight_t)), ctypes.c_int32,
                                        ctypes.POINTER(_p), ctypes.c_int, _p, ctypes.c_uint32, _p, ctypes.c_size_t,
                                        _p]),
    "nf4_linear_group_launches": (ctypes.c_int32, [_i64, ctypes.POINTER(_i64), ctypes.c_int32, _i64]),
    "nf4_dequantize_batch": (ctypes.c_int, [ctypes.POINTER(ctypes.POINTER(nf4_weight_t)), ctypes.c_int32,
                                            ctypes.POINTER(_p), ctypes.c_int, _p]),
}


class NF4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s failed: %s" % (where, lib().nf4_status_str(status).decode()))


_lib = None


def lib():
    """The loaded library; raises if it was never built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                "libnf4.so is missing (%s): build it with `python -m "
                "quantized_linear_layers_nf4_b200.build`; there is no CPU fallback" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        if L.nf4_abi_version() != NF4_ABI_VERSION:
            raise RuntimeError("libnf4.so ABI %d != binding ABI %d" % (L.nf4_abi_version(),
                                                                       NF4_ABI_VERSION))
        _lib = L
    return _lib


def check(status: int, where: str) -> None:
    if status != NF4_OK:
        raise NF4Error(status, where)
