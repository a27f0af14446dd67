"""nf4_double_quant_noalloc: double quantization for callers that cannot
allocate device memory (a plugin inside a framework that owns all device
memory, or a deployment with a memory plan fixed at start-up).  Its scratch is
a fixed device array inside the library instead of a caller workspace.

Checked through the C ABI against nf4_double_quant on the same inputs, on
consecutive calls that share the fixed scratch; outputs must be bit-identical
(the tolerance every double-quantization test uses)."""
import ctypes

import numpy as np
import pytest
import torch

from quantized_linear_layers_nf4_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nf4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_linear_layers_nf4_b200.build import build
    build()
    import quantized_linear_layers_nf4_b200 as m
    return m


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(nf4, absmax):
    L = nf4._lib.lib()
    nb = absmax.numel()
    q = torch.full((nb,), 99, dtype=torch.int8, device="cuda")
    s = torch.full(((nb + 255) // 256,), float("nan"), dtype=torch.float32, device="cuda")
    mu = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = L.nf4_double_quant_noalloc(_p(absmax), nb, _p(q), _p(s), _p(mu), stream)
    assert st == 0, L.nf4_status_str(st).decode()
    return q, s, mu


def _with_workspace(nf4, absmax):
    return nf4.nf4_double_quant(absmax)


def _same(a, b):
    torch.cuda.synchronize()
    return torch.equal(a.view(torch.int8) if a.dtype == torch.int8 else a.view(torch.int32),
                       b.view(torch.int8) if b.dtype == torch.int8 else b.view(torch.int32))


def test_noalloc_matches_the_workspace_entry_point_on_consecutive_calls(nf4):
    # call 1: the absmax of a 4096 x 4096 bf16 weight (1024 blocks of 256)
    W = synth.weight_normal(4096, 4096, seed=synth.seed_for(2, 64), dtype=torch.bfloat16, device="cuda")
    _, absmax1 = nf4.nf4_quantize(W)
    # call 2: a smaller, ragged vector (a partial last block) with other values,
    # so stale partial sums from call 1 would show up if they were ever read
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    absmax2 = torch.rand(1000, generator=g, device="cuda") * 0.05 + 0.01
    for absmax in (absmax1, absmax2):
        got = _noalloc(nf4, absmax)
        want = _with_workspace(nf4, absmax)
        for x, y, name in zip(got, want, ("absmax_q", "absmax_scale", "absmax_offset")):
            assert _same(x, y), name


def _header_limit() -> int:
    """NF4_DQ_NOALLOC_MAX_NB as the C header defines it."""
    import os
    import re
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "nf4.h")
    with open(path) as f:
        return int(re.search(r"#define\s+NF4_DQ_NOALLOC_MAX_NB\s+(\d+)", f.read()).group(1))


def test_noalloc_largest_size_and_the_limit(nf4):
    L = nf4._lib.lib()
    limit = _header_limit()
    assert limit == nf4._lib.NF4_DQ_NOALLOC_MAX_NB, "the binding's copy of the limit is stale"
    absmax = torch.rand(limit, device="cuda") * 0.1
    got = _noalloc(nf4, absmax)
    want = _with_workspace(nf4, absmax)
    for x, y in zip(got, want):
        assert _same(x, y)
    # one value past the fixed scratch: rejected on the host, nothing launched
    big = torch.empty(1, device="cuda")
    st = L.nf4_double_quant_noalloc(_p(big), limit + 1, _p(big), _p(big), _p(big), None)
    assert st == -6
    assert "workspace" in L.nf4_status_str(st).decode()
