"""ctypes wrapper over ``liboracle_nf4.so`` (test infrastructure only).

Each function takes and returns numpy arrays and forwards to the C function of
the same name in ``nf4_oracle.c``; the arithmetic lives there.
"""
import ctypes

import numpy as np

from .build_oracle import build

__all__ = [
    "norm_ppf", "codebook", "quantize", "dq_sum", "dq_mean", "double_quant", "absmax_hat",
    "dequantize", "dequantize_range", "f32_to_bf16", "bf16_to_f32", "linear_bf16", "linear_dx_bf16", "linear_lora_bf16", "lora_delta", "merge_lora", "unpack",
    "use_library",
]

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _bind(L):
    p = ctypes.c_void_p
    i64 = ctypes.c_int64
    L.orc_norm_ppf.argtypes = [ctypes.c_double]
    L.orc_norm_ppf.restype = ctypes.c_double
    L.orc_codebook.argtypes = [p]
    L.orc_codebook.restype = None
    L.orc_quantize_f32.argtypes = [p, i64, p, p]
    L.orc_quantize_f32.restype = ctypes.c_int
    L.orc_quantize_bf16.argtypes = [p, i64, p, p]
    L.orc_quantize_bf16.restype = ctypes.c_int
    L.orc_fp4_codebook.argtypes = [p]
    L.orc_fp4_codebook.restype = None
    L.orc_quantize_f32_qt.argtypes = [p, i64, ctypes.c_int, p, p]
    L.orc_quantize_f32_qt.restype = ctypes.c_int
    L.orc_quantize_bf16_qt.argtypes = [p, i64, ctypes.c_int, p, p]
    L.orc_quantize_bf16_qt.restype = ctypes.c_int
    L.orc_dequantize_range_qt.argtypes = [p, p, p, ctypes.c_float, i64, i64, ctypes.c_int, p]
    L.orc_dequantize_range_qt.restype = ctypes.c_int
    L.orc_dq_sum.argtypes = [p, i64]
    L.orc_dq_sum.restype = ctypes.c_double
    L.orc_dq_mean.argtypes = [p, i64]
    L.orc_dq_mean.restype = ctypes.c_float
    L.orc_double_quant.argtypes = [p, i64, p, p, p]
    L.orc_double_quant.restype = ctypes.c_int
    L.orc_absmax_hat.argtypes = [p, p, ctypes.c_float, i64]
    L.orc_absmax_hat.restype = ctypes.c_float
    L.orc_dequantize_range.argtypes = [p, p, p, ctypes.c_float, i64, i64, p]
    L.orc_dequantize_range.restype = ctypes.c_int
    L.orc_f32_to_bf16.argtypes = [p, i64, p]
    L.orc_f32_to_bf16.restype = None
    L.orc_linear_bf16.argtypes = [p, i64, p, i64, i64, p]
    L.orc_linear_bf16.restype = None
    L.orc_lora_delta.argtypes = [p, p, i64, i64, i64, p]
    L.orc_lora_delta.restype = None
    return L


def use_library(path):
    """Point the wrapper at another build of the oracle (used by the mutation
    test, which builds deliberately broken copies); ``None`` restores the
    default build."""
    global _lib
    _lib = None
    if path is not None:
        _lib = _bind(ctypes.CDLL(path))


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def norm_ppf(p: float) -> float:
    return lib().orc_norm_ppf(float(p))


QUANT_TYPES = {"nf4": 0, "fp4": 1}


def _qt(quant_type: str) -> int:
    if quant_type not in QUANT_TYPES:
        raise ValueError("quant_type must be 'nf4' or 'fp4'")
    return QUANT_TYPES[quant_type]


def codebook(quant_type: str = "nf4") -> np.ndarray:
    """The 16 levels: NF4 ascending, FP4 in code order."""
    c = np.zeros(16, dtype=np.float32)
    if _qt(quant_type) == 1:
        lib().orc_fp4_codebook(_ptr(c))
    else:
        lib().orc_codebook(_ptr(c))
    return c


def quantize(w: np.ndarray, quant_type: str = "nf4"):
    """w: float32 array, or uint16 array of bf16 bit patterns; any shape with
    size % 64 == 0.  Returns (wq uint8 [size/2], absmax float32 [size/64])."""
    qt = _qt(quant_type)
    w = np.ascontiguousarray(w)
    n = w.size
    wq = np.zeros(n // 2, dtype=np.uint8)
    absmax = np.zeros(n // 64, dtype=np.float32)
    if w.dtype == np.float32:
        rc = lib().orc_quantize_f32_qt(_ptr(w), n, qt, _ptr(wq), _ptr(absmax))
    elif w.dtype == np.uint16:
        rc = lib().orc_quantize_bf16_qt(_ptr(w), n, qt, _ptr(wq), _ptr(absmax))
    else:
        raise TypeError("oracle quantize takes float32 or bf16 bit patterns (uint16)")
    if rc != 0:
        raise ValueError("orc_quantize failed with %d" % rc)
    return wq, absmax


def dq_sum(absmax: np.ndarray) -> float:
    a = np.ascontiguousarray(absmax, dtype=np.float32)
    return lib().orc_dq_sum(_ptr(a), a.size)


def dq_mean(absmax: np.ndarray) -> np.float32:
    a = np.ascontiguousarray(absmax, dtype=np.float32)
    return np.float32(lib().orc_dq_mean(_ptr(a), a.size))


def double_quant(absmax: np.ndarray):
    """Returns (absmax_q int8 [nb], absmax_scale float32 [ceil(nb/256)], mu float32)."""
    a = np.ascontiguousarray(absmax, dtype=np.float32)
    nb = a.size
    q = np.zeros(nb, dtype=np.int8)
    s = np.zeros((nb + 255) // 256, dtype=np.float32)
    mu = np.zeros(1, dtype=np.float32)
    rc = lib().orc_double_quant(_ptr(a), nb, _ptr(q), _ptr(s), _ptr(mu))
    if rc != 0:
        raise ValueError("orc_double_quant failed with %d" % rc)
    return q, s, mu[0]


def absmax_hat(absmax_q: np.ndarray, absmax_scale: np.ndarray, mu) -> np.ndarray:
    q = np.ascontiguousarray(absmax_q, dtype=np.int8)
    s = np.ascontiguousarray(absmax_scale, dtype=np.float32)
    L = lib()
    return np.array([L.orc_absmax_hat(_ptr(q), _ptr(s), float(mu), b) for b in range(q.size)],
                    dtype=np.float32)


def dequantize_range(wq, absmax_q, absmax_scale, mu, begin: int, count: int,
                     quant_type: str = "nf4") -> np.ndarray:
    qt = _qt(quant_type)
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    q = np.ascontiguousarray(absmax_q, dtype=np.int8)
    s = np.ascontiguousarray(absmax_scale, dtype=np.float32)
    out = np.zeros(count, dtype=np.float32)
    rc = lib().orc_dequantize_range_qt(_ptr(wq), _ptr(q), _ptr(s), float(mu), int(begin), int(count), qt,
                                       _ptr(out))
    if rc != 0:
        raise ValueError("orc_dequantize_range failed with %d" % rc)
    return out


def dequantize(wq, absmax_q, absmax_scale, mu, quant_type: str = "nf4") -> np.ndarray:
    return dequantize_range(wq, absmax_q, absmax_scale, mu, 0, 2 * np.asarray(wq).size, quant_type)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.zeros(x.shape, dtype=np.uint16)
    lib().orc_f32_to_bf16(_ptr(x), x.size, _ptr(out))
    return out


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (no rounding involved)."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


def linear_bf16(x_bf16: np.ndarray, w_bf16: np.ndarray) -> np.ndarray:
    """x_bf16 [m,k], w_bf16 [n,k] as uint16 bit patterns -> y float64 [m,n]."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    m, k = x.shape
    n, k2 = w.shape
    assert k == k2
    y = np.zeros((m, n), dtype=np.float64)
    lib().orc_linear_bf16(_ptr(x), m, _ptr(w), n, k, _ptr(y))
    return y


def linear_dx_bf16(dy_bf16: np.ndarray, w_bf16: np.ndarray) -> np.ndarray:
    """Backward through the frozen quantized base: dX = dY * What.

    Page "Tim Dettmers 如何用 bitsandbytes 與 QLoRA 降低 LLM 訓練門檻？", section
    "QLoRA 把 frozen 4-bit base 與可訓練 adapter 分開": the 4-bit base is dequantized
    to the compute dtype in the backward pass as in the forward one, and never
    updated.  dy_bf16 [m, n] and w_bf16 [n, k] (the bf16 dequantized weight,
    row-major) as uint16 bit patterns -> dX float64 [m, k] with
    dX[i, c] = sum_r dY[i, r] * What[r, c], exact products and fp64 sums (the
    forward linear applied to the transposed weight)."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    return linear_bf16(dy_bf16, np.ascontiguousarray(w.T))


def linear_lora_bf16(x_bf16: np.ndarray, w_bf16: np.ndarray, down_bf16: np.ndarray, up_bf16: np.ndarray,
                     scale: float) -> np.ndarray:
    """The QLoRA layer: the frozen quantized base plus a low-rank update.

    Page "LLM 相關知識" (technicalnotes), section "2-2. LoRA（低秩適應）": the
    frozen W is used as W + dW with dW = A x B of rank r (A: out x r, B: r x in),
    trained in bf16; section 4: the base is frozen INT4, the LoRA matrices bf16.
    With W [n, k] (rows = outputs): dW = up [n, r] * down [r, k], and
        Y = X What^T + scale * (X down^T) up^T
    in fp64 with exact products (scale as given, e.g. lora_alpha / r).
    x_bf16 [m, k], w_bf16 [n, k], down_bf16 [r, k], up_bf16 [n, r] as uint16 bit
    patterns -> Y float64 [m, n]."""
    base = linear_bf16(x_bf16, w_bf16)
    x = bf16_to_f32(x_bf16).astype(np.float64)
    down = bf16_to_f32(down_bf16).astype(np.float64)
    up = bf16_to_f32(up_bf16).astype(np.float64)
    t = x @ down.T                       # [m, r]: the low-rank projection of X
    return base + float(scale) * (t @ up.T)


def lora_delta(up_bf16: np.ndarray, down_bf16: np.ndarray) -> np.ndarray:
    """delta = up * down as an fp32 fused-multiply-add chain in rank order (see
    orc_lora_delta).  up [n, r], down [r, k] bf16 bit patterns -> fp32 [n, k]."""
    up = np.ascontiguousarray(up_bf16, dtype=np.uint16)
    down = np.ascontiguousarray(down_bf16, dtype=np.uint16)
    n, r = up.shape
    r2, k = down.shape
    assert r == r2
    out = np.zeros((n, k), dtype=np.float32)
    lib().orc_lora_delta(_ptr(up), _ptr(down), n, r, k, _ptr(out))
    return out


def merge_lora(wq, absmax_q, absmax_scale, mu, n: int, k: int, down_bf16, up_bf16, scale: float,
               quant_type: str = "nf4"):
    """Merge a trained LoRA update into the quantized base and requantize it.

    Page "LLM 相關知識" (technicalnotes), section "8. LoRA 的合併（Merge）": INT4
    weights are dequantized to BF16, W_new = W + A x B is formed in BF16, and W_new
    is quantized again to INT4 for deployment.  Reading: What_bf16 is the bf16
    dequantized weight; delta = up * down (fp32, rank order, lora_delta);
    W_new = bf16_round(fp32(What_bf16 + fp32(scale * delta))); the new codes and
    fp32 absmax are the blockwise quantization of the bf16 W_new (quant_type's
    codebook, the same as the input's).
    Returns (w_new bf16 bits [n, k], wq_new uint8, absmax_new fp32)."""
    what = f32_to_bf16(dequantize_range(wq, absmax_q, absmax_scale, mu, 0, n * k, quant_type)).reshape(n, k)
    d = lora_delta(up_bf16, down_bf16)
    sd = (np.float32(scale) * d).astype(np.float32)                 # fp32 multiply
    s = (bf16_to_f32(what) + sd).astype(np.float32)                  # fp32 add
    w_new = f32_to_bf16(s)
    wq_new, absmax_new = quantize(w_new.reshape(-1), quant_type)
    return w_new, wq_new, absmax_new


def unpack(wq: np.ndarray) -> np.ndarray:
    """Packed bytes -> one index per element (high nibble first).  Pure layout."""
    wq = np.asarray(wq, dtype=np.uint8)
    out = np.empty(wq.size * 2, dtype=np.uint8)
    out[0::2] = wq >> 4
    out[1::2] = wq & 15
    return out
