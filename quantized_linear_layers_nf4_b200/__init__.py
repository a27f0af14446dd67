"""NF4 (4-bit NormalFloat) weight quantization with double quantization, and the
fused dequantize + bf16 linear, for NVIDIA B200 (sm_100a).

The work is done by ``lib/libnf4.so`` (C ABI in ``include/nf4.h``); this module
only marshals PyTorch device tensors and the current CUDA stream into those
calls.  Functions carry the C names:

* ``nf4_quantize(W)`` -> ``(wq, absmax)``
* ``nf4_double_quant(absmax)`` -> ``(absmax_q, absmax_scale, absmax_offset)``
* ``nf4_dequantize(weight, dtype)`` -> dense tensor
* ``nf4_linear(X, weight, dtype)`` -> ``Y = X @ W_hat^T`` (optionally with a
  split-k ``workspace`` from ``linear_workspace``)
* ``nf4_linear_group(X, weights, dtype)`` -> ``[X @ W_i^T]`` for weights that
  share X (q/k/v, gate/up), in one launch
* ``nf4_linear_dx(dY, weight, dtype)`` -> ``dX = dY @ W_hat`` (backward through
  the frozen base)
* ``nf4_linear_lora(X, weight, down, up, scale, workspace=...)`` -> the QLoRA
  layer ``X @ W_hat^T + scale * (X @ down^T) @ up^T``
* ``nf4_merge_lora(weight, down, up, scale)`` -> ``(wq, absmax, w_new)``: the
  trained update folded into the weight and quantized again (``merge_lora``
  adds the double quantization and returns an ``NF4Weight``)

``quantize_weight(W)`` runs the first two and returns an ``NF4Weight``.  Every
quantizing call takes ``quant_type="nf4"`` (the default) or ``"fp4"``; an
``NF4Weight`` remembers which codebook its codes index.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import NF4_BF16, NF4_F32, NF4Error, nf4_weight_t

__all__ = ["NF4Weight", "NF4Error", "nf4_quantize", "nf4_double_quant", "nf4_dequantize",
           "nf4_linear", "nf4_linear_ex", "nf4_linear_group", "nf4_linear_dx", "nf4_linear_lora", "lora_workspace",
           "nf4_merge_lora", "merge_lora", "nf4_dequantize_batch",
           "nf4_linear_workspace_bytes", "linear_workspace",
           "quantize_weight", "nf4_codebook", "library_path"]

_DTYPES = {torch.float32: NF4_F32, torch.bfloat16: NF4_BF16}
_QUANT_TYPES = {"nf4": _lib.NF4_QUANT_NF4, "fp4": _lib.NF4_QUANT_FP4}


def _quant_type(quant_type: str) -> int:
    if quant_type not in _QUANT_TYPES:
        raise ValueError("quant_type must be 'nf4' or 'fp4'")
    return _QUANT_TYPES[quant_type]


def library_path() -> str:
    return _lib.LIB_PATH


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _need_cuda(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def nf4_codebook(quant_type: str = "nf4") -> torch.Tensor:
    """The 16 levels the library uses (host copy): NF4 ascending, FP4 in code order."""
    out = torch.zeros(16, dtype=torch.float32)
    _lib.check(_lib.lib().nf4_codebook_typed(_quant_type(quant_type), _ptr(out)), "nf4_codebook")
    return out


def nf4_quantize(W: torch.Tensor, wq: torch.Tensor | None = None, absmax: torch.Tensor | None = None,
                 stream=None, quant_type: str = "nf4"):
    """Blockwise NF4 (or FP4) quantization of a 2-D fp32/bf16 CUDA tensor [n, k]."""
    qt = _quant_type(quant_type)
    _need_cuda(W, "W")
    if W.dim() != 2 or W.dtype not in _DTYPES:
        raise ValueError("W must be a 2-D float32 or bfloat16 tensor")
    n, k = W.shape
    numel = n * k
    if wq is None:
        wq = torch.empty(numel // 2, dtype=torch.uint8, device=W.device)
    if absmax is None:
        absmax = torch.empty(numel // 64, dtype=torch.float32, device=W.device)
    _lib.check(_lib.lib().nf4_quantize_typed(_ptr(W), _DTYPES[W.dtype], n, k, qt, _ptr(wq), _ptr(absmax),
                                             _stream(stream)), "nf4_quantize")
    return wq, absmax


def nf4_double_quant(absmax: torch.Tensor, absmax_q: torch.Tensor | None = None,
                     absmax_scale: torch.Tensor | None = None,
                     absmax_offset: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, stream=None):
    """Double quantization of the fp32 absmax vector."""
    _need_cuda(absmax, "absmax")
    nb = absmax.numel()
    L = _lib.lib()
    ws_bytes = L.nf4_double_quant_workspace_bytes(nb)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 8) // 8 + 1, dtype=torch.float64, device=absmax.device)
    if absmax_q is None:
        absmax_q = torch.empty(nb, dtype=torch.int8, device=absmax.device)
    if absmax_scale is None:
        absmax_scale = torch.empty((nb + 255) // 256, dtype=torch.float32, device=absmax.device)
    if absmax_offset is None:
        absmax_offset = torch.empty(1, dtype=torch.float32, device=absmax.device)
    _lib.check(L.nf4_double_quant(_ptr(absmax), nb, _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _ptr(absmax_q),
                                  _ptr(absmax_scale), _ptr(absmax_offset), _stream(stream)),
               "nf4_double_quant")
    return absmax_q, absmax_scale, absmax_offset


@dataclass
class NF4Weight:
    """A quantized [n, k] weight: device tensors plus the C struct that borrows them."""
    n: int
    k: int
    wq: torch.Tensor
    absmax_q: torch.Tensor
    absmax_scale: torch.Tensor
    absmax_offset: torch.Tensor
    quant_type: str = "nf4"

    def struct(self) -> nf4_weight_t:
        magic = _lib.NF4_FP4_WEIGHT_MAGIC if self.quant_type == "fp4" else _lib.NF4_WEIGHT_MAGIC
        return nf4_weight_t(magic, _lib.NF4_WEIGHT_VERSION, self.n, self.k,
                            _lib.NF4_BLOCKSIZE, _lib.NF4_BLOCKSIZE2, self.wq.data_ptr(),
                            self.absmax_q.data_ptr(), self.absmax_scale.data_ptr(),
                            self.absmax_offset.data_ptr())

    def nbytes(self) -> int:
        return (self.wq.numel() + self.absmax_q.numel() + 4 * self.absmax_scale.numel())


def quantize_weight(W: torch.Tensor, stream=None, quant_type: str = "nf4") -> NF4Weight:
    """nf4_quantize followed by nf4_double_quant; the fp32 absmax is dropped."""
    wq, absmax = nf4_quantize(W, stream=stream, quant_type=quant_type)
    q, s, mu = nf4_double_quant(absmax, stream=stream)
    return NF4Weight(W.shape[0], W.shape[1], wq, q, s, mu, quant_type)


def nf4_dequantize(weight: NF4Weight, dtype=torch.bfloat16, out: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    if dtype not in _DTYPES:
        raise ValueError("dtype must be float32 or bfloat16")
    if out is None:
        out = torch.empty((weight.n, weight.k), dtype=dtype, device=weight.wq.device)
    st = weight.struct()
    _lib.check(_lib.lib().nf4_dequantize(ctypes.byref(st), _ptr(out), _DTYPES[dtype],
                                         _stream(stream)), "nf4_dequantize")
    return out


def nf4_dequantize_batch(weights, dtype=torch.bfloat16, outs=None, stream=None):
    """[nf4_dequantize(w) for w in weights] in one launch (at most
    NF4_DEQUANT_BATCH_MAX weights; the same bits).  Returns the list of outputs."""
    if dtype not in _DTYPES:
        raise ValueError("dtype must be float32 or bfloat16")
    weights = list(weights)
    count = len(weights)
    if outs is None:
        outs = [torch.empty((w.n, w.k), dtype=dtype, device=w.wq.device) for w in weights]
    for o in outs:
        _need_cuda(o, "out")
    structs = [w.struct() for w in weights]
    wptrs = (ctypes.POINTER(nf4_weight_t) * max(count, 1))(*[ctypes.pointer(s) for s in structs])
    optrs = (ctypes.c_void_p * max(count, 1))(*[o.data_ptr() for o in outs])
    _lib.check(_lib.lib().nf4_dequantize_batch(wptrs, count, optrs, _DTYPES[dtype], _stream(stream)),
               "nf4_dequantize_batch")
    return outs


def nf4_linear_ex(X, weight, dtype=torch.bfloat16, out=None, dev_status=None, stream=None,
                  flags: int = 0, workspace=None):
    """Same as nf4_linear with the C flags word (NF4_LINEAR_WEIGHTS_EARLY,
    NF4_LINEAR_TEST_TIMEOUT)."""
    return nf4_linear(X, weight, dtype, out, dev_status, stream, workspace=workspace, flags=flags)


def nf4_linear_workspace_bytes(m: int, n: int, k: int) -> int:
    """Bytes of the optional split-k workspace of nf4_linear for these sizes on
    the current device (0: none needed)."""
    return int(_lib.lib().nf4_linear_workspace_bytes(m, n, k))


def linear_workspace(shapes, m: int = 16, device=None) -> torch.Tensor:
    """A zero-filled workspace large enough for nf4_linear at m tokens on every
    (n, k) in ``shapes`` (one buffer serves them all)."""
    nbytes = max([nf4_linear_workspace_bytes(m, n, k) for n, k in shapes] + [16])
    return torch.zeros((nbytes + 15) // 16 * 16, dtype=torch.uint8, device=device or "cuda")


def nf4_linear(X: torch.Tensor, weight: NF4Weight, dtype=torch.bfloat16,
               out: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
               stream=None, weights_early: bool = False,
               workspace: torch.Tensor | None = None, flags: int = 0) -> torch.Tensor:
    """Y = X @ W_hat^T for bf16 X [m, k]; Y [m, n] in ``dtype`` (bf16 or fp32).

    ``weights_early=True`` sets NF4_LINEAR_WEIGHTS_EARLY: the weight was not
    written by the work just before this call on the stream, so its loads may
    overlap that work (programmatic dependent launch).  ``workspace`` (from
    ``linear_workspace``) lets the decode path split the tiles of a weight over
    all SMs, with partial sums meeting in global memory; the results are the
    same bits as without it.  ``flags`` is OR'ed into the C flags word.  The
    call goes to ``nf4_linear_ws``."""
    _need_cuda(X, "X")
    if X.dtype != torch.bfloat16 or X.dim() != 2:
        raise ValueError("X must be a 2-D bfloat16 tensor")
    if dtype not in _DTYPES:
        raise ValueError("dtype must be float32 or bfloat16")
    m = X.shape[0]
    if out is None:
        out = torch.empty((m, weight.n), dtype=dtype, device=X.device)
    st = weight.struct()
    ds = ctypes.c_void_p(0) if dev_status is None else _ptr(dev_status)
    flags |= _lib.NF4_LINEAR_WEIGHTS_EARLY if weights_early else 0
    ws, ws_bytes = _ws(workspace)
    _lib.check(_lib.lib().nf4_linear_ws(_ptr(X), m, ctypes.byref(st), _ptr(out), _DTYPES[dtype], ds,
                                        flags, ws, ws_bytes, _stream(stream)), "nf4_linear_ws")
    return out


def _ws(workspace):
    if workspace is None:
        return ctypes.c_void_p(0), 0
    _need_cuda(workspace, "workspace")
    return _ptr(workspace), workspace.numel() * workspace.element_size()


def nf4_linear_group_launches(m: int, ns, k: int) -> int:
    """Kernel launches nf4_linear_group makes for weights of rows `ns` and width k
    at m tokens on the current device (1 when grouped into one launch)."""
    arr = (ctypes.c_int64 * len(ns))(*[int(n) for n in ns])
    r = _lib.lib().nf4_linear_group_launches(int(m), arr, len(ns), int(k))
    if r < 0:
        raise ValueError("invalid sizes or no usable device")
    return int(r)


def nf4_linear_group(X: torch.Tensor, weights, dtype=torch.bfloat16, outs=None,
                     dev_status: torch.Tensor | None = None, stream=None, weights_early: bool = False,
                     workspace: torch.Tensor | None = None, flags: int = 0):
    """[X @ W_i^T for W_i in weights] in one call for weights that share X and k
    (at most NF4_LINEAR_GROUP_MAX): one launch over all their row tiles when
    that is faster than one launch per weight.  Each output equals nf4_linear on
    that weight alone up to the fp32 summation order.  Returns the list of
    outputs."""
    _need_cuda(X, "X")
    if X.dtype != torch.bfloat16 or X.dim() != 2:
        raise ValueError("X must be a 2-D bfloat16 tensor")
    if dtype not in _DTYPES:
        raise ValueError("dtype must be float32 or bfloat16")
    weights = list(weights)
    count = len(weights)
    m = X.shape[0]
    if outs is None:
        outs = [torch.empty((m, w.n), dtype=dtype, device=X.device) for w in weights]
    structs = [w.struct() for w in weights]
    wptrs = (ctypes.POINTER(nf4_weight_t) * max(count, 1))(*[ctypes.pointer(s) for s in structs])
    yptrs = (ctypes.c_void_p * max(count, 1))(*[o.data_ptr() for o in outs])
    ds = ctypes.c_void_p(0) if dev_status is None else _ptr(dev_status)
    flags |= _lib.NF4_LINEAR_WEIGHTS_EARLY if weights_early else 0
    ws, ws_bytes = _ws(workspace)
    _lib.check(_lib.lib().nf4_linear_group(_ptr(X), m, wptrs, count, yptrs, _DTYPES[dtype], ds, flags, ws,
                                           ws_bytes, _stream(stream)), "nf4_linear_group")
    return outs


def nf4_linear_dx(dY: torch.Tensor, weight: NF4Weight, dtype=torch.bfloat16,
                  out: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                  stream=None) -> torch.Tensor:
    """dX = dY @ W_hat for bf16 dY [m, n] (n % 8 == 0); dX [m, k] in ``dtype``."""
    _need_cuda(dY, "dY")
    if dY.dtype != torch.bfloat16 or dY.dim() != 2 or dY.shape[1] != weight.n:
        raise ValueError("dY must be a 2-D bfloat16 tensor with n columns")
    if dtype not in _DTYPES:
        raise ValueError("dtype must be float32 or bfloat16")
    m = dY.shape[0]
    if out is None:
        out = torch.empty((m, weight.k), dtype=dtype, device=dY.device)
    st = weight.struct()
    ds = ctypes.c_void_p(0) if dev_status is None else _ptr(dev_status)
    _lib.check(_lib.lib().nf4_linear_dx(_ptr(dY), m, ctypes.byref(st), _ptr(out), _DTYPES[dtype], ds,
                                        _stream(stream)), "nf4_linear_dx")
    return out


def lora_workspace(m: int, shapes, r: int, device=None) -> torch.Tensor:
    """A zero-filled workspace for nf4_linear_lora at m tokens and rank r on every
    (n, k) in ``shapes``."""
    L = _lib.lib()
    nbytes = max([int(L.nf4_linear_lora_workspace_bytes(m, n, k, r)) for n, k in shapes] + [16])
    return torch.zeros((nbytes + 15) // 16 * 16, dtype=torch.uint8, device=device or "cuda")


def nf4_linear_lora(X: torch.Tensor, weight: NF4Weight, down: torch.Tensor, up: torch.Tensor, scale: float,
                    workspace: torch.Tensor, dtype=torch.bfloat16, out: torch.Tensor | None = None,
                    dev_status: torch.Tensor | None = None, stream=None,
                    weights_early: bool = False) -> torch.Tensor:
    """Y = X @ W_hat^T + scale * (X @ down^T) @ up^T with down bf16 [r, k] and up
    bf16 [n, r]; ``workspace`` from ``lora_workspace``."""
    for t, name in ((X, "X"), (down, "down"), (up, "up"), (workspace, "workspace")):
        _need_cuda(t, name)
    if X.dtype != torch.bfloat16 or down.dtype != torch.bfloat16 or up.dtype != torch.bfloat16:
        raise ValueError("X, down and up must be bfloat16")
    r = down.shape[0]
    if down.shape != (r, weight.k) or up.shape != (weight.n, r) or X.shape[1] != weight.k:
        raise ValueError("shapes: X [m, k], down [r, k], up [n, r]")
    if dtype not in _DTYPES:
        raise ValueError("dtype must be float32 or bfloat16")
    m = X.shape[0]
    if out is None:
        out = torch.empty((m, weight.n), dtype=dtype, device=X.device)
    st = weight.struct()
    ds = ctypes.c_void_p(0) if dev_status is None else _ptr(dev_status)
    flags = _lib.NF4_LINEAR_WEIGHTS_EARLY if weights_early else 0
    _lib.check(_lib.lib().nf4_linear_lora(_ptr(X), m, ctypes.byref(st), _ptr(down), _ptr(up), r, float(scale),
                                          _ptr(out), _DTYPES[dtype], ds, flags, _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream(stream)),
               "nf4_linear_lora")
    return out


def nf4_merge_lora(weight: NF4Weight, down: torch.Tensor, up: torch.Tensor, scale: float,
                   want_bf16: bool = False, wq: torch.Tensor | None = None,
                   absmax: torch.Tensor | None = None, stream=None):
    """Dequantize to bf16, add scale * up @ down in bf16 and quantize again.
    Returns (wq, absmax fp32, w_new bf16 [n, k] or None)."""
    for t, name in ((down, "down"), (up, "up")):
        _need_cuda(t, name)
    if down.dtype != torch.bfloat16 or up.dtype != torch.bfloat16:
        raise ValueError("down and up must be bfloat16")
    r = down.shape[0]
    if down.dim() != 2 or down.shape != (r, weight.k) or up.shape != (weight.n, r):
        raise ValueError("shapes: down [r, k], up [n, r]")
    numel = weight.n * weight.k
    dev = weight.wq.device
    if wq is None:
        wq = torch.empty(numel // 2, dtype=torch.uint8, device=dev)
    if absmax is None:
        absmax = torch.empty(numel // 64, dtype=torch.float32, device=dev)
    w_new = torch.empty((weight.n, weight.k), dtype=torch.bfloat16, device=dev) if want_bf16 else None
    st = weight.struct()
    _lib.check(_lib.lib().nf4_merge_lora(ctypes.byref(st), _ptr(down), _ptr(up), r, float(scale),
                                         ctypes.c_void_p(0) if w_new is None else _ptr(w_new), _ptr(wq),
                                         _ptr(absmax), _stream(stream)), "nf4_merge_lora")
    return wq, absmax, w_new


def merge_lora(weight: NF4Weight, down: torch.Tensor, up: torch.Tensor, scale: float, stream=None) -> NF4Weight:
    """nf4_merge_lora followed by nf4_double_quant: the merged, requantized weight."""
    wq, absmax, _ = nf4_merge_lora(weight, down, up, scale, stream=stream)
    q, s, mu = nf4_double_quant(absmax, stream=stream)
    return NF4Weight(weight.n, weight.k, wq, q, s, mu, weight.quant_type)
