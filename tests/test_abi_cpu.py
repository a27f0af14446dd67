"""C-ABI checks that need no GPU: the library loads, exports every function
include/nf4.h declares, its constants and struct layout match the header and
the Python binding, and host-side validation rejects bad arguments before any
launch.  Nothing here computes on a device."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
from quantized_linear_layers_nf4_b200 import _lib
from quantized_linear_layers_nf4_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nf4.h")


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nf4_[a-z0-9_]+)\s*\(", text)))


def test_header_functions_are_exported_and_bound(L):
    names = _declared_functions()
    assert "nf4_quantize" in names and "nf4_linear" in names
    for name in names:
        assert hasattr(L, name), "libnf4.so does not export %s" % name
        assert name in _lib.SIGNATURES, "binding has no signature for %s" % name
    assert set(_lib.SIGNATURES) == set(names)


def test_header_constants_match_binding():
    text = open(HEADER).read()

    def define(name):
        return int(re.search(r"#define\s+%s\s+(0x[0-9A-Fa-f]+|\d+)" % name, text).group(1), 0)

    assert define("NF4_BLOCKSIZE") == _lib.NF4_BLOCKSIZE == 64
    assert define("NF4_BLOCKSIZE2") == _lib.NF4_BLOCKSIZE2 == 256
    assert define("NF4_WEIGHT_MAGIC") == _lib.NF4_WEIGHT_MAGIC
    assert define("NF4_WEIGHT_VERSION") == _lib.NF4_WEIGHT_VERSION
    assert define("NF4_ABI_VERSION") == _lib.NF4_ABI_VERSION
    assert define("NF4_DEQUANT_BATCH_MAX") == _lib.NF4_DEQUANT_BATCH_MAX == 16
    assert ctypes.sizeof(_lib.nf4_weight_t) == 64


def test_status_strings(L):
    for code in range(-9, 1):
        s = L.nf4_status_str(code).decode()
        assert s.startswith("NF4_")
    assert L.nf4_status_str(-100).decode() == "unknown nf4 status"


def test_library_levels_equal_the_oracle_levels(L):
    """Two independent derivations of the 16 levels (the library's generated
    header and the oracle's Newton quantiles) agree bit for bit."""
    out = np.zeros(16, dtype=np.float32)
    assert L.nf4_codebook(out.ctypes.data_as(ctypes.c_void_p)) == 0
    assert np.array_equal(out.view(np.uint32), O.codebook().view(np.uint32))
    assert L.nf4_codebook(None) == -1


def test_library_fp4_values_equal_the_oracle_fp4_values(L):
    out = np.zeros(16, dtype=np.float32)
    assert L.nf4_codebook_typed(1, out.ctypes.data_as(ctypes.c_void_p)) == 0
    assert np.array_equal(out.view(np.uint32), O.codebook("fp4").view(np.uint32))
    assert L.nf4_codebook_typed(0, out.ctypes.data_as(ctypes.c_void_p)) == 0
    assert np.array_equal(out.view(np.uint32), O.codebook().view(np.uint32))
    assert L.nf4_codebook_typed(2, out.ctypes.data_as(ctypes.c_void_p)) == -4
    assert L.nf4_codebook_typed(1, None) == -1


def test_workspace_size(L):
    assert L.nf4_double_quant_workspace_bytes(0) == 0
    assert L.nf4_double_quant_workspace_bytes(1) == 8
    assert L.nf4_double_quant_workspace_bytes(256) == 8
    assert L.nf4_double_quant_workspace_bytes(257) == 16


FAKE = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced
ODD = ctypes.c_void_p(0x10004)       # 4-byte aligned only


def test_quantize_validation(L):
    q = L.nf4_quantize
    assert q(None, 0, 4, 64, FAKE, FAKE, None) == -1
    assert q(FAKE, 7, 4, 64, FAKE, FAKE, None) == -4
    assert q(FAKE, 0, 0, 64, FAKE, FAKE, None) == -2
    assert q(FAKE, 0, 3, 7, FAKE, FAKE, None) == -2          # 21 elements: not a multiple of 64
    assert q(FAKE, 0, -1, 64, FAKE, FAKE, None) == -2
    assert q(FAKE, 0, 2 ** 40, 2 ** 40, FAKE, FAKE, None) == -2  # overflow
    assert q(ODD, 0, 4, 64, FAKE, FAKE, None) == -3
    assert q(FAKE, 1, 4, 64, ODD, FAKE, None) == -3


def test_double_quant_validation(L):
    d = L.nf4_double_quant
    assert d(None, 10, FAKE, 8, FAKE, FAKE, FAKE, None) == -1
    assert d(FAKE, 0, FAKE, 8, FAKE, FAKE, FAKE, None) == -2
    assert d(FAKE, 2 ** 40, FAKE, 2 ** 40, FAKE, FAKE, FAKE, None) == -2
    assert d(FAKE, 300, FAKE, 8, FAKE, FAKE, FAKE, None) == -6     # needs 16 bytes
    assert d(FAKE, 300, None, 64, FAKE, FAKE, FAKE, None) == -6


def _weight(**kw):
    w = _lib.nf4_weight_t(_lib.NF4_WEIGHT_MAGIC, _lib.NF4_WEIGHT_VERSION, 128, 256, 64, 256,
                          FAKE.value, FAKE.value, FAKE.value, FAKE.value)
    for k, v in kw.items():
        setattr(w, k, v)
    return w


def test_weight_struct_validation(L):
    dq = L.nf4_dequantize
    lin = L.nf4_linear
    assert dq(ctypes.byref(_weight(magic=1)), FAKE, 1, None) == -5
    assert dq(ctypes.byref(_weight(version=2)), FAKE, 1, None) == -5
    assert dq(ctypes.byref(_weight(blocksize=32)), FAKE, 1, None) == -5
    assert dq(ctypes.byref(_weight(blocksize2=128)), FAKE, 1, None) == -5
    assert dq(ctypes.byref(_weight(wq=None)), FAKE, 1, None) == -1
    assert dq(ctypes.byref(_weight(n=3, k=7)), FAKE, 1, None) == -2
    assert dq(ctypes.byref(_weight(wq=FAKE.value + 8)), FAKE, 1, None) == -3
    assert dq(ctypes.byref(_weight()), None, 1, None) == -1
    assert dq(ctypes.byref(_weight()), FAKE, 5, None) == -4
    assert dq(ctypes.byref(_weight()), ODD, 1, None) == -3
    assert dq(None, FAKE, 1, None) == -1
    assert lin(FAKE, 0, ctypes.byref(_weight()), FAKE, 1, None, None) == -2
    assert lin(FAKE, 4, ctypes.byref(_weight(n=64, k=96)), FAKE, 1, None, None) == -2
    assert lin(FAKE, 4, ctypes.byref(_weight()), FAKE, 9, None, None) == -4
    assert lin(ODD, 4, ctypes.byref(_weight()), FAKE, 1, None, None) == -3
    assert lin(None, 4, ctypes.byref(_weight()), FAKE, 1, None, None) == -1
    lex = L.nf4_linear_ex
    assert lex(FAKE, 4, ctypes.byref(_weight()), FAKE, 1, None, 2, None) == -4   # unknown flag bit
    assert lex(FAKE, 4, ctypes.byref(_weight(magic=3)), FAKE, 1, None, 1, None) == -5
    assert lex(FAKE, 0, ctypes.byref(_weight()), FAKE, 1, None, 1, None) == -2


def test_dequantize_batch_validation(L):
    """Argument checks of nf4_dequantize_batch, all before any device query."""
    db = L.nf4_dequantize_batch
    W = ctypes.POINTER(_lib.nf4_weight_t)
    good = [_weight(), _weight(n=128, k=64)]
    wp = (W * 2)(*[ctypes.pointer(x) for x in good])
    op = (ctypes.c_void_p * 2)(FAKE.value, FAKE.value + 4096)
    assert db(None, 2, op, 1, None) == -1
    assert db(wp, 2, None, 1, None) == -1
    assert db(wp, 0, op, 1, None) == -2                         # count out of range
    assert db(wp, _lib.NF4_DEQUANT_BATCH_MAX + 1, op, 1, None) == -2
    assert db(wp, 2, op, 7, None) == -4                         # dtype
    bad = (W * 2)(ctypes.pointer(good[0]), ctypes.pointer(_weight(magic=1)))
    assert db(bad, 2, op, 1, None) == -5                        # second weight's state
    holes = (W * 2)(ctypes.pointer(good[0]), None)
    assert db(holes, 2, op, 1, None) == -1
    odd = (ctypes.c_void_p * 2)(FAKE.value, ODD.value)
    assert db(wp, 2, odd, 1, None) == -3
    nulls = (ctypes.c_void_p * 2)(FAKE.value, None)
    assert db(wp, 2, nulls, 1, None) == -1


def test_group_launch_plan_validation(L):
    """nf4_linear_group_launches rejects invalid sizes before any device query."""
    gl = L.nf4_linear_group_launches
    ns = (ctypes.c_int64 * 5)(4096, 4096, 4096, 4096, 4096)
    assert gl(16, None, 3, 4096) == -1
    assert gl(16, ns, 0, 4096) == -1
    assert gl(16, ns, 5, 4096) == -1          # more than NF4_LINEAR_GROUP_MAX
    assert gl(0, ns, 3, 4096) == -1
    assert gl(16, ns, 3, 100) == -1           # k % 64 != 0
    zero = (ctypes.c_int64 * 2)(4096, 0)
    assert gl(16, zero, 2, 4096) == -1


def test_linear_workspace_validation(L):
    lws = L.nf4_linear_ws
    w = ctypes.byref(_weight())
    # a misaligned workspace is rejected before any device query
    assert lws(FAKE, 4, w, FAKE, 1, None, 0, ODD, 1 << 20, None) == -3
    assert lws(FAKE, 4, w, FAKE, 1, None, 4, FAKE, 1 << 20, None) == -4    # unknown flag bit
    assert lws(FAKE, 0, w, FAKE, 1, None, 0, FAKE, 1 << 20, None) == -2
    assert lws(None, 4, w, FAKE, 1, None, 0, None, 0, None) == -1
    # sizes that are not a valid product need no workspace
    assert L.nf4_linear_workspace_bytes(0, 4096, 4096) == 0
    assert L.nf4_linear_workspace_bytes(16, 4096, 100) == 0


def test_linear_dx_validation(L):
    dx = L.nf4_linear_dx
    assert dx(None, 4, ctypes.byref(_weight()), FAKE, 1, None, None) == -1
    assert dx(FAKE, 0, ctypes.byref(_weight()), FAKE, 1, None, None) == -2
    assert dx(FAKE, 4, ctypes.byref(_weight(n=100, k=64)), FAKE, 1, None, None) == -2   # n % 8 != 0
    assert dx(FAKE, 4, ctypes.byref(_weight()), FAKE, 9, None, None) == -4
    assert dx(ODD, 4, ctypes.byref(_weight()), FAKE, 1, None, None) == -3
    assert dx(FAKE, 4, ctypes.byref(_weight(magic=7)), FAKE, 1, None, None) == -5


def test_linear_lora_validation(L):
    lo = L.nf4_linear_lora
    w = ctypes.byref(_weight())
    assert lo(FAKE, 4, w, None, FAKE, 16, 2.0, FAKE, 1, None, 0, FAKE, 1 << 20, None) == -1   # no down
    assert lo(FAKE, 4, w, FAKE, FAKE, 16, 2.0, FAKE, 1, None, 0, None, 0, None) == -1        # no workspace
    assert lo(FAKE, 4, w, FAKE, FAKE, 0, 2.0, FAKE, 1, None, 0, FAKE, 1 << 20, None) == -2   # rank 0
    assert lo(FAKE, 4, w, FAKE, FAKE, 300, 2.0, FAKE, 1, None, 0, FAKE, 1 << 20, None) == -2
    assert lo(FAKE, 4, w, FAKE, ODD, 16, 2.0, FAKE, 1, None, 0, FAKE, 1 << 20, None) == -3
    assert L.nf4_linear_lora_workspace_bytes(4, 4096, 4096, 0) == 0


def test_merge_lora_validation(L):
    mg = L.nf4_merge_lora
    w = ctypes.byref(_weight())
    assert mg(w, None, FAKE, 16, 2.0, None, FAKE, FAKE, None) == -1            # no down
    assert mg(w, FAKE, FAKE, 16, 2.0, None, None, FAKE, None) == -1            # no codes out
    assert mg(w, FAKE, FAKE, 16, 2.0, None, FAKE, None, None) == -1            # no absmax out
    assert mg(w, FAKE, FAKE, 0, 2.0, None, FAKE, FAKE, None) == -2             # rank 0
    assert mg(w, FAKE, FAKE, 257, 2.0, None, FAKE, FAKE, None) == -2
    assert mg(ctypes.byref(_weight(k=96)), FAKE, FAKE, 16, 2.0, None, FAKE, FAKE, None) == -2
    assert mg(w, FAKE, ODD, 16, 2.0, None, FAKE, FAKE, None) == -3
    assert mg(w, FAKE, FAKE, 16, 2.0, ODD, FAKE, FAKE, None) == -3             # w_new misaligned
    assert mg(ctypes.byref(_weight(magic=7)), FAKE, FAKE, 16, 2.0, None, FAKE, FAKE, None) == -5


def test_fp4_quantize_and_weight_validation(L):
    qt = L.nf4_quantize_typed
    assert qt(FAKE, 0, 4, 64, 2, FAKE, FAKE, None) == -4                      # unknown codebook
    assert qt(FAKE, 0, 4, 64, -1, FAKE, FAKE, None) == -4
    assert qt(None, 0, 4, 64, 1, FAKE, FAKE, None) == -1
    assert qt(FAKE, 0, 4, 65, 1, FAKE, FAKE, None) == -2
    assert L.nf4_dequantize(ctypes.byref(_weight(magic=_lib.NF4_FP4_WEIGHT_MAGIC + 1)), FAKE, 1, None) == -5
    # an FP4 weight passes the struct check and then needs a device (only asked
    # where there is none: these pointers are never valid device memory)
    import torch
    if not torch.cuda.is_available():
        assert L.nf4_dequantize(ctypes.byref(_weight(magic=_lib.NF4_FP4_WEIGHT_MAGIC)), FAKE, 1, None) in (-7, -9)


def test_valid_call_without_a_gpu_reports_instead_of_crashing(L):
    """On a host without a usable B200 a fully valid call must come back with a
    status (no device / unsupported device), never crash or launch."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; covered by the gpu tests")
    st = L.nf4_quantize(FAKE, 0, 4, 64, FAKE, FAKE, None)
    assert st in (-7, -9)
