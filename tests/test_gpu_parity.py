"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on the
same seeded inputs.

Bar: packed codes, absmax, double-quantized absmax codes and scales, the mean
and the dequantized weights (fp32 and bf16) bit-exact; the fused linear within
a relative Frobenius error of 2e-3 (fp32 output) against an fp64 GEMM on the
bf16-dequantized weight.  Full-size configurations are checked on whole arrays
for quantization / double quantization and on sampled rows for dequantization
and the linear."""
import numpy as np
import pytest
import torch

import oracle as O
from quantized_linear_layers_nf4_b200 import synth

pytestmark = pytest.mark.gpu

LINEAR_TOL = 2e-3
# Two fp32 results of the same products summed in different orders (k split
# across CTAs differently): each reordering of a k-term fp32 sum moves it by at
# most about k * 2^-24 * sum|x_i|, and the sums here partly cancel; at k = 11008
# the observed relative difference is about 1e-5.
FP32_ORDER_TOL = 1e-4


@pytest.fixture(scope="module")
def nf4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_linear_layers_nf4_b200.build import build
    build()
    import quantized_linear_layers_nf4_b200 as m
    return m


def _bits(t: torch.Tensor) -> np.ndarray:
    """Host copy of a tensor for the oracle: fp32 as float32, bf16 as uint16 bits."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16).reshape(-1)
    return t.numpy().reshape(-1)


def _gpu_chain(nf4, W, quant_type="nf4"):
    wq, absmax = nf4.nf4_quantize(W, quant_type=quant_type)
    q, s, mu = nf4.nf4_double_quant(absmax)
    weight = nf4.NF4Weight(W.shape[0], W.shape[1], wq, q, s, mu, quant_type)
    return weight, absmax


def _oracle_chain(Wh, quant_type="nf4"):
    wq, absmax = O.quantize(Wh, quant_type)
    q, s, mu = O.double_quant(absmax)
    return wq, absmax, q, s, mu


def _assert_equal(gpu: torch.Tensor, ref: np.ndarray, what: str):
    g = gpu.detach().cpu().numpy().reshape(-1)
    ref = np.asarray(ref).reshape(-1)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    if g.dtype == np.float32:
        g, ref = g.view(np.uint32), ref.astype(np.float32).view(np.uint32)
    bad = np.flatnonzero(g != ref)
    assert bad.size == 0, "%s: %d mismatches, first at %s: gpu %s oracle %s" % (
        what, bad.size, bad[:5], g[bad[:5]], ref[bad[:5]])


def _check_quant(nf4, W, full_dequant=True, rows=None, quant_type="nf4"):
    """Quantize + double-quant + dequant on the GPU and compare with the oracle.
    Returns (weight, oracle arrays) for further checks."""
    weight, absmax = _gpu_chain(nf4, W, quant_type)
    n, k = W.shape
    Wh = _bits(W)
    owq, oam, oq, os_, omu = _oracle_chain(Wh, quant_type)
    _assert_equal(absmax, oam, "absmax")
    _assert_equal(weight.wq, owq, "packed codes")
    _assert_equal(weight.absmax_q, oq, "absmax_q")
    _assert_equal(weight.absmax_scale, os_, "absmax_scale")
    _assert_equal(weight.absmax_offset, np.array([omu], np.float32), "absmax_offset (mean)")
    if full_dequant:
        d32 = nf4.nf4_dequantize(weight, torch.float32)
        d16 = nf4.nf4_dequantize(weight, torch.bfloat16)
        ref = O.dequantize(owq, oq, os_, omu, quant_type)
        _assert_equal(d32, ref, "dequant fp32")
        _assert_equal(d16.view(torch.int16).view(-1), O.f32_to_bf16(ref).view(np.int16), "dequant bf16")
    else:
        d32 = nf4.nf4_dequantize(weight, torch.float32)
        d16 = nf4.nf4_dequantize(weight, torch.bfloat16)
        for r in rows:
            ref = O.dequantize_range(owq, oq, os_, omu, r * k, k, quant_type)
            _assert_equal(d32[r], ref, "dequant fp32 row %d" % r)
            _assert_equal(d16[r].view(torch.int16), O.f32_to_bf16(ref).view(np.int16),
                          "dequant bf16 row %d" % r)
        del d32, d16
    return weight, (owq, oq, os_, omu)


def test_dequantize_batch(nf4):
    """nf4_dequantize_batch over weights of different shapes and codebooks (word
    counts that are and are not whole warp passes) gives, for each, the oracle's
    dequantization, fp32 and bf16."""
    shapes = [(64, 64, "nf4"), (96, 128, "fp4"), (1000, 320, "nf4"), (4096, 4096, "nf4"), (520, 640, "fp4")]
    weights, refs = [], []
    for i, (n, k, qt) in enumerate(shapes):
        W = synth.weight_normal(n, k, seed=2100 + i, dtype=torch.bfloat16, device="cuda")
        weight, orc = _check_quant(nf4, W, full_dequant=False, rows=[0], quant_type=qt)
        weights.append(weight)
        refs.append(orc)
    for dtype in (torch.float32, torch.bfloat16):
        outs = nf4.nf4_dequantize_batch(weights, dtype)
        torch.cuda.synchronize()
        for weight, (owq, oq, os_, omu), out in zip(weights, refs, outs):
            ref = O.dequantize(owq, oq, os_, omu, weight.quant_type)
            if dtype == torch.float32:
                _assert_equal(out, ref, "batch dequant fp32 %dx%d" % (weight.n, weight.k))
            else:
                _assert_equal(out.view(torch.int16).view(-1), O.f32_to_bf16(ref).view(np.int16),
                              "batch dequant bf16 %dx%d" % (weight.n, weight.k))
    # one weight alone, sixteen (the bound) of mixed sizes, and one more than the bound
    one = nf4.nf4_dequantize_batch(weights[2:3], torch.bfloat16)[0]
    assert torch.equal(one, nf4.nf4_dequantize(weights[2], torch.bfloat16))
    many = [weights[i % len(weights)] for i in range(16)]
    outs16 = nf4.nf4_dequantize_batch(many, torch.float32)
    for weight, out in zip(many, outs16):
        assert torch.equal(out, nf4.nf4_dequantize(weight, torch.float32))
    with pytest.raises(nf4.NF4Error):
        nf4.nf4_dequantize_batch([weights[0]] * 17, torch.bfloat16)


def _rel_fro(y: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(y.astype(np.float64) - ref) / max(np.linalg.norm(ref), 1e-300))


def _check_linear(nf4, X, weight, orc, token_rows=None, weight_rows=None, tol=LINEAR_TOL):
    """nf4_linear vs the oracle's fp64 GEMM on the bf16-dequantized weight, on
    the sampled token rows x weight rows.  Returns the fp32 relative error."""
    owq, oq, os_, omu = orc
    m, k = X.shape
    n = weight.n
    T = np.arange(m) if token_rows is None else np.asarray(token_rows)
    R = np.arange(n) if weight_rows is None else np.asarray(weight_rows)
    Y32 = nf4.nf4_linear(X, weight, torch.float32)
    Y16 = nf4.nf4_linear(X, weight, torch.bfloat16)
    torch.cuda.synchronize()
    wrows = np.stack([O.f32_to_bf16(O.dequantize_range(owq, oq, os_, omu, int(r) * k, k, weight.quant_type))
                      for r in R])
    xb = _bits(X).reshape(m, k)[T]
    ref = O.linear_bf16(np.ascontiguousarray(xb), np.ascontiguousarray(wrows))
    y32 = Y32.cpu().numpy()[np.ix_(T, R)]
    e32 = _rel_fro(y32, ref)
    assert e32 <= tol, "linear fp32 rel-Frobenius %.3g > %.3g" % (e32, tol)
    # the bf16 output is the fp32 result of the same kernel rounded once
    y16 = Y16.float().cpu().numpy()[np.ix_(T, R)]
    y32r = torch.from_numpy(np.ascontiguousarray(y32)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(y16, y32r), "bf16 output is not the rounded fp32 output"
    e16 = _rel_fro(y16, ref)
    assert e16 <= 2 * tol, "linear bf16 rel-Frobenius %.3g" % e16
    return e32


# ---------------------------------------------------------------------------
# Small cases: several tiles and ragged tails, both input dtypes.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n,k", [(1, 64), (3, 640), (5, 192), (64, 4096), (257, 320), (100, 6400),
                                 (2, 32)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_chain_small(nf4, n, k, dtype):
    W = synth.weight_normal(n, k, seed=n * 7 + k, std=0.02, dtype=dtype, device="cuda")
    _check_quant(nf4, W)


def test_edge_values(nf4):
    n, k = 8, 512
    W = synth.weight_normal(n, k, seed=77, std=0.02, dtype=torch.float32, device="cuda")
    W[0, 0:64] = 0.0                                 # zero block
    W[0, 64:128] = -0.0                              # negative-zero block
    W[1, 0:64] = 0.0
    W[1, 5] = -3.5                                   # single non-zero
    W[2, 0:64] = 0.25                                # constant block
    W[2, 64:128] = 1e-40                             # subnormals
    W[2, 130] = -1e-39
    W[3, 0:64] = torch.linspace(-1e30, 1e30, 64)     # huge values
    W[4, :] = 0.0                                    # a zero row (zero absmax, mean shifts)
    lv = torch.from_numpy(O.codebook()).cuda()
    W[5, 0:16] = lv                                  # exact levels, absmax 1
    W[5, 16:31] = (lv[:-1] + lv[1:]) / 2             # fp32-rounded midpoints
    W[6, 0:64] = torch.arange(64, dtype=torch.float32, device="cuda") - 31.5
    _check_quant(nf4, W)


@pytest.mark.parametrize("quant_type", ["nf4", "fp4"])
def test_quantize_near_thresholds(nf4, quant_type):
    """Codes of weights within a few ulps of every decision boundary (w / a at and
    around each midpoint between adjacent levels), for absmax values inside and
    outside the range where the quotient is formed without a division: bit-exact
    against the oracle's IEEE division and nearest-level search."""
    lv = O.codebook(quant_type).astype(np.float64)
    mids = (lv[:-1] + lv[1:]) / 2
    rows = []
    for a in (1.0, 0.37, 3.1e-5, 1234.5, 2.0 ** -59, 2.0 ** 59, 2.0 ** -61, 2.0 ** 61, 0.0123456):
        a32 = np.float32(a)
        vals = [a32]
        for c in mids:
            x = np.float32(c * float(a32))
            for d in range(-3, 4):
                y = x
                step = np.float32(np.inf) if d > 0 else np.float32(-np.inf)
                for _ in range(abs(d)):
                    y = np.nextafter(y, step)
                if abs(float(y)) <= float(a32):
                    vals.append(y)
        vals = np.array(vals, dtype=np.float32)
        vals = np.concatenate([vals, np.zeros((-len(vals)) % 64, np.float32)])
        for i in range(0, len(vals), 63):   # every block starts with a (its absmax)
            blk = np.concatenate([[a32], vals[i:i + 63]]).astype(np.float32)
            rows.append(np.concatenate([blk, np.zeros(64 - len(blk), np.float32)]))
    W = torch.from_numpy(np.concatenate(rows).reshape(-1, 256 if len(rows) % 4 == 0 else 64)).cuda()
    _check_quant(nf4, W, quant_type=quant_type)


def test_cfg1_full_chain_and_linear(nf4):
    """1024 x 1024 fp32 weight (seed 0), X 16 x 1024 bf16 (seed 1): everything
    checked on the whole output."""
    W = synth.weight_normal(1024, 1024, seed=0, std=0.02, dtype=torch.float32, device="cuda")
    X = synth.activations(16, 1024, seed=1, device="cuda")
    weight, orc = _check_quant(nf4, W)
    _check_linear(nf4, X, weight, orc)


@pytest.mark.parametrize("m", [1, 2, 4, 7, 8, 15, 16, 17, 33, 64])
def test_linear_token_counts(nf4, m):
    n, k = 200, 576
    W = synth.weight_normal(n, k, seed=300 + m, dtype=torch.bfloat16, device="cuda")
    X = synth.activations(m, k, seed=400 + m, device="cuda")
    weight, orc = _check_quant(nf4, W)
    _check_linear(nf4, X, weight, orc)


@pytest.mark.parametrize("m,n,k", [(17, 64, 64), (257, 300, 192), (300, 520, 640), (1024, 1024, 1024),
                                   (64, 8, 128), (513, 2048, 256)])
def test_gemm_path_ragged_tiles(nf4, m, n, k):
    """m > 16 runs the tcgen05 GEMM: tiles of 256 tokens x 256 weight rows with
    ragged edges in both, several k stages."""
    W = synth.weight_normal(n, k, seed=800 + m + n, dtype=torch.bfloat16, device="cuda")
    X = synth.activations(m, k, seed=900 + m, device="cuda")
    weight, orc = _check_quant(nf4, W, full_dequant=False, rows=[0, n - 1])
    _check_linear(nf4, X, weight, orc)


@pytest.mark.parametrize("n,k", [(8, 64), (1, 128), (9, 64), (24, 1088), (1000, 256)])
def test_linear_ragged_shapes(nf4, n, k):
    W = synth.weight_normal(n, k, seed=500 + n, dtype=torch.bfloat16, device="cuda")
    X = synth.activations(5, k, seed=600 + n, device="cuda")
    weight, orc = _check_quant(nf4, W)
    _check_linear(nf4, X, weight, orc)


@pytest.mark.parametrize("m", [3, 16])
def test_gemv_three_way_split_k(nf4, m):
    """11000 x 2304 makes the GEMV split k three ways (258 CTAs, rank row ranges
    of 42/43/43 rows, a partial last row tile): every output row is checked."""
    n, k = 11000, 2304
    W = synth.weight_normal(n, k, seed=700 + m, dtype=torch.bfloat16, device="cuda")
    X = synth.activations(m, k, seed=710 + m, device="cuda")
    weight, orc = _check_quant(nf4, W, full_dequant=False, rows=[0, 41, 42, 84, 85, 127, n - 1])
    _check_linear(nf4, X, weight, orc)


def _same_bits(a: torch.Tensor, b: torch.Tensor) -> bool:
    return torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                       b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32))


@pytest.mark.parametrize("n,k,m", [(4096, 4096, 16), (11008, 4096, 16), (11000, 2304, 3), (1000, 1024, 7),
                                   (4096, 11008, 1), (300, 576, 16), (64, 128, 5), (128, 64, 1),
                                   (2048, 640, 9), (19000, 4096, 16)])
def test_workspace_split_k_is_bit_identical(nf4, n, k, m):
    """nf4_linear_ws with a workspace (CTAs meet in global memory, the last one
    reduces) gives the same bits as the cluster path, for split-k factors 1 to
    8, leaves every counter at zero and matches the oracle on sampled rows."""
    W = synth.weight_normal(n, k, seed=1200 + n + k, dtype=torch.bfloat16, device="cuda")
    X = synth.activations(m, k, seed=1300 + m, device="cuda")
    weight, orc = _check_quant(nf4, W, full_dequant=False, rows=[0, n - 1])
    nb = nf4.nf4_linear_workspace_bytes(m, n, k)
    ws = nf4.linear_workspace([(n, k)], m=m)
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    for dtype in (torch.float32, torch.bfloat16):
        ref = nf4.nf4_linear(X, weight, dtype)
        for _ in range(2):   # twice: the counters must have been reset by the first call
            got = nf4.nf4_linear(X, weight, dtype, workspace=ws, dev_status=ds)
            torch.cuda.synchronize()
            assert _same_bits(got, ref)
    tiles = (n + 127) // 128
    if nb:
        assert int(ws[: 4 * tiles].view(torch.int32).abs().sum()) == 0, "split-k counters not reset"
    assert ds.item() == 0
    _check_linear(nf4, X, weight, orc, weight_rows=_sample_rows(n, 64, n + k))


def test_workspace_errors_and_graph_reuse(nf4):
    n, k, m = 4096, 4096, 16
    W = synth.weight_normal(n, k, seed=1400, dtype=torch.bfloat16, device="cuda")
    weight = nf4.quantize_weight(W)
    X = synth.activations(m, k, seed=1401, device="cuda")
    need = nf4.nf4_linear_workspace_bytes(m, n, k)
    assert need > 0
    small = torch.zeros(need // 2, dtype=torch.uint8, device="cuda")
    with pytest.raises(nf4.NF4Error) as e:
        nf4.nf4_linear(X, weight, torch.float32, workspace=small)
    assert "WORKSPACE" in str(e.value)
    # one workspace shared by a chain of launches inside a CUDA graph, with
    # programmatic dependent launch, gives the cluster path's bits every replay
    W2 = synth.weight_normal(11008, k, seed=1402, dtype=torch.bfloat16, device="cuda")
    w2 = nf4.quantize_weight(W2)
    ws = nf4.linear_workspace([(n, k), (11008, k)], m=m)
    y1 = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty(m, 11008, dtype=torch.bfloat16, device="cuda")
    r1 = nf4.nf4_linear(X, weight, torch.bfloat16)
    r2 = nf4.nf4_linear(X, w2, torch.bfloat16)

    def step():
        for _ in range(3):
            nf4.nf4_linear(X, weight, torch.bfloat16, out=y1, workspace=ws, weights_early=True)
            nf4.nf4_linear(X, w2, torch.bfloat16, out=y2, workspace=ws, weights_early=True)
    step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(3):
        y1.zero_(); y2.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y1.view(torch.int16), r1.view(torch.int16))
        assert torch.equal(y2.view(torch.int16), r2.view(torch.int16))


def _check_dx(nf4, dY, weight, orc, token_rows=None, tol=LINEAR_TOL):
    """nf4_linear_dx vs the oracle's fp64 dX = dY * What on the bf16-dequantized
    weight (every column, the sampled token rows)."""
    owq, oq, os_, omu = orc
    m, n = dY.shape
    k = weight.k
    T = np.arange(m) if token_rows is None else np.asarray(token_rows)
    D32 = nf4.nf4_linear_dx(dY, weight, torch.float32)
    D16 = nf4.nf4_linear_dx(dY, weight, torch.bfloat16)
    torch.cuda.synchronize()
    what = O.f32_to_bf16(O.dequantize_range(owq, oq, os_, omu, 0, n * k, weight.quant_type)).reshape(n, k)
    ref = O.linear_dx_bf16(np.ascontiguousarray(_bits(dY).reshape(m, n)[T]), what)
    d32 = D32.cpu().numpy()[T]
    e32 = _rel_fro(d32, ref)
    assert e32 <= tol, "dX fp32 rel-Frobenius %.3g > %.3g" % (e32, tol)
    d16 = D16.float().cpu().numpy()[T]
    d32r = torch.from_numpy(np.ascontiguousarray(d32)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(d16, d32r), "bf16 dX is not the rounded fp32 dX"
    return e32


@pytest.mark.parametrize("m,n,k", [(17, 64, 64), (257, 136, 320), (300, 520, 640), (64, 8, 128),
                                   (513, 2048, 256), (1, 200, 576)])
def test_linear_dx_ragged(nf4, m, n, k):
    """Backward through the frozen base, dX = dY * What: ragged token, row
    (contraction) and column tiles."""
    W = synth.weight_normal(n, k, seed=1500 + n + k, dtype=torch.bfloat16, device="cuda")
    dY = synth.activations(m, n, seed=1600 + m, device="cuda")
    weight, orc = _check_quant(nf4, W, full_dequant=False, rows=[0, n - 1])
    _check_dx(nf4, dY, weight, orc)


def test_linear_dx_prefill_shape(nf4):
    """dX for the MLP down/up shapes at 4096 tokens: W 11008 x 4096, dY 4096 x 11008."""
    m, n, k = 4096, 11008, 4096
    W = synth.weight_normal(n, k, seed=synth.seed_for(3, 0), dtype=torch.bfloat16, device="cuda")
    dY = synth.activations(m, n, seed=synth.seed_for(3, 7), device="cuda")
    weight, orc = _check_quant(nf4, W, full_dequant=False, rows=_sample_rows(n, 16, 3))
    _check_dx(nf4, dY, weight, orc, token_rows=_sample_rows(m, 12, 41))


def test_linear_dx_errors(nf4):
    W = synth.weight_normal(100, 64, seed=1700, dtype=torch.bfloat16, device="cuda")   # n % 8 != 0
    weight = nf4.quantize_weight(W)
    dY = synth.activations(4, 100, seed=1701, device="cuda")
    with pytest.raises(nf4.NF4Error):
        nf4.nf4_linear_dx(dY, weight, torch.float32)


@pytest.mark.parametrize("m,n,k,r,scale", [(16, 4096, 4096, 16, 2.0), (3, 11000, 2304, 64, 0.5),
                                           (16, 64, 128, 1, 2.0), (7, 1000, 1024, 8, 1.0),
                                           (16, 11008, 4096, 8, 2.0), (5, 19200, 320, 16, 1.5),
                                           (9, 1000, 320, 16, 0.5), (1, 4096, 11008, 16, 2.0),
                                           (300, 520, 640, 16, 2.0), (1024, 1024, 1024, 64, 0.25),
                                           (257, 136, 320, 5, 2.0), (512, 256, 512, 72, 1.0),
                                           (18944, 64, 64, 64, 1.0)])
def test_linear_lora(nf4, m, n, k, r, scale):
    """The QLoRA layer Y = X What^T + s (X down^T) up^T: decode path (k split 8, 3
    and 1; r = 8 and 16 with the down-projection formed inside the GEMV, over a
    ragged last k stage too, other ranks by a separate kernel) and prefill path
    (tensor-core term for r % 8 == 0 in one or two K tiles of 64 ranks, fp32
    epilogue otherwise; the tensor-core down-projection with k split and, at
    18944 tokens x 4 rank groups, unsplit), against the oracle; the bf16 output is
    the rounded fp32 output."""
    W = synth.weight_normal(n, k, seed=1800 + n + r, dtype=torch.bfloat16, device="cuda")
    X = synth.activations(m, k, seed=1810 + m, device="cuda")
    down = (synth.activations(r, k, seed=1820 + r, device="cuda").float() * 0.02).to(torch.bfloat16)
    up = (synth.activations(n, r, seed=1830 + r, device="cuda").float() * 0.02).to(torch.bfloat16)
    weight, orc = _check_quant(nf4, W, full_dequant=False, rows=[0, n - 1])
    owq, oq, os_, omu = orc
    ws = nf4.lora_workspace(m, [(n, k)], r)
    T = np.arange(m) if m <= 64 else _sample_rows(m, 24, m)
    R = np.arange(n) if n <= 4096 else _sample_rows(n, 256, n)
    Y32 = nf4.nf4_linear_lora(X, weight, down, up, scale, ws, dtype=torch.float32)
    Y16 = nf4.nf4_linear_lora(X, weight, down, up, scale, ws, dtype=torch.bfloat16)
    torch.cuda.synchronize()
    wrows = np.stack([O.f32_to_bf16(O.dequantize_range(owq, oq, os_, omu, int(rr) * k, k, weight.quant_type))
                      for rr in R])
    ref = O.linear_lora_bf16(np.ascontiguousarray(_bits(X).reshape(m, k)[T]), wrows, _bits(down).reshape(r, k),
                             np.ascontiguousarray(_bits(up).reshape(n, r)[R]), scale)
    y32 = Y32.cpu().numpy()[np.ix_(T, R)]
    e32 = _rel_fro(y32, ref)
    assert e32 <= LINEAR_TOL, "LoRA layer fp32 rel-Frobenius %.3g" % e32
    y16 = Y16.float().cpu().numpy()[np.ix_(T, R)]
    assert np.array_equal(y16, torch.from_numpy(np.ascontiguousarray(y32)).to(torch.bfloat16).float().numpy())
    # a zero scale leaves the base linear
    Y0 = nf4.nf4_linear_lora(X, weight, down, up, 0.0, ws, dtype=torch.float32)
    assert torch.equal(Y0, nf4.nf4_linear(X, weight, torch.float32))


@pytest.mark.parametrize("n,k,r,scale", [(128, 256, 16, 2.0), (100, 192, 5, 0.5), (1, 64, 1, 1.0),
                                         (300, 640, 256, 0.125), (4096, 4096, 64, 2.0), (11008, 4096, 16, 0.25)])
def test_merge_lora(nf4, n, k, r, scale):
    """Merge + requantize: the merged bf16 weight, its packed codes and fp32
    absmax bit-exact against the oracle (whole arrays), then the double
    quantization of the merged absmax; a zero scale requantizes the bf16
    dequantized weight."""
    W = synth.weight_normal(n, k, seed=1900 + n + r, dtype=torch.bfloat16, device="cuda")
    down = (synth.activations(r, k, seed=1910 + r, device="cuda").float() * 0.05).to(torch.bfloat16)
    up = (synth.activations(n, r, seed=1920 + r, device="cuda").float() * 0.05).to(torch.bfloat16)
    weight, orc = _check_quant(nf4, W, full_dequant=False, rows=[0, n - 1])
    owq, oq, os_, omu = orc
    wq, absmax, w_new = nf4.nf4_merge_lora(weight, down, up, scale, want_bf16=True)
    wq2, absmax2, none = nf4.nf4_merge_lora(weight, down, up, scale)
    torch.cuda.synchronize()
    assert none is None
    ow, owq_new, oam_new = O.merge_lora(owq, oq, os_, omu, n, k, _bits(down).reshape(r, k),
                                        _bits(up).reshape(n, r), scale)
    _assert_equal(w_new.view(torch.int16).view(-1), ow.view(np.int16), "merged bf16 weight")
    _assert_equal(wq, owq_new, "merged codes")
    _assert_equal(absmax, oam_new, "merged absmax")
    assert torch.equal(wq, wq2) and torch.equal(absmax, absmax2)
    merged = nf4.merge_lora(weight, down, up, scale)
    oq2, os2, omu2 = O.double_quant(oam_new)
    _assert_equal(merged.wq, owq_new, "merged weight codes")
    _assert_equal(merged.absmax_q, oq2, "merged absmax_q")
    _assert_equal(merged.absmax_scale, os2, "merged absmax_scale")
    _assert_equal(merged.absmax_offset, np.array([omu2], np.float32), "merged mean")
    # scale 0: the requantized bf16 dequantized weight, through the other kernels
    wq0, absmax0, w0 = nf4.nf4_merge_lora(weight, down, up, 0.0, want_bf16=True)
    d16 = nf4.nf4_dequantize(weight, torch.bfloat16)
    assert torch.equal(w0, d16)
    wq_ref, absmax_ref = nf4.nf4_quantize(d16)
    assert torch.equal(wq0, wq_ref) and torch.equal(absmax0, absmax_ref)


def test_merge_lora_errors(nf4):
    W = synth.weight_normal(64, 64, seed=1950, dtype=torch.bfloat16, device="cuda")
    weight = nf4.quantize_weight(W)
    down = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        nf4.nf4_merge_lora(weight, down, torch.zeros(64, 5, dtype=torch.bfloat16, device="cuda"), 1.0)
    with pytest.raises(nf4.NF4Error):   # rank above 256
        nf4.nf4_merge_lora(weight, torch.zeros(300, 64, dtype=torch.bfloat16, device="cuda"),
                           torch.zeros(64, 300, dtype=torch.bfloat16, device="cuda"), 1.0)


# ---------------------------------------------------------------------------
# FP4 codebook: the same kernels with the FP4 values in place of the NF4 levels.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n,k", [(1, 64), (5, 192), (257, 320), (100, 6400)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_fp4_quantize_chain(nf4, n, k, dtype):
    W = synth.weight_normal(n, k, seed=2000 + n * 7 + k, std=0.02, dtype=dtype, device="cuda")
    weight, _ = _check_quant(nf4, W, quant_type="fp4")
    assert weight.quant_type == "fp4"
    assert torch.equal(nf4.nf4_codebook("fp4"), torch.from_numpy(O.codebook("fp4")))


def test_fp4_edge_values(nf4):
    n, k = 4, 256
    W = synth.weight_normal(n, k, seed=2050, std=0.02, dtype=torch.float32, device="cuda")
    W[0, 0:64] = 0.0                                   # zero block -> code 0
    W[0, 64:128] = -0.0
    W[1, 0] = 1.0                                      # absmax 1
    c = torch.from_numpy(O.codebook("fp4")).cuda()
    W[1, 1:8] = c[1:8]                                 # exact values
    W[1, 9:16] = c[9:16]
    W[1, 16] = c[1] / 2                                # the exact tie between 0 and 1/12
    W[1, 17] = -c[1] / 2
    W[1, 18] = -1e-12                                  # tiny negative -> +0
    W[2, 0:64] = torch.arange(64, dtype=torch.float32, device="cuda") - 31.5
    weight, _ = _check_quant(nf4, W, quant_type="fp4")
    codes = O.unpack(weight.wq.cpu().numpy())
    assert np.all(codes[:128] == 0) and codes[k + 16] == 0 and codes[k + 17] == 0 and codes[k + 18] == 0
    assert not np.any(codes == 8)


@pytest.mark.parametrize("m,n,k", [(1, 200, 576), (16, 1000, 1024), (7, 11008, 512), (300, 520, 640),
                                   (1024, 1024, 1024)])
def test_fp4_linear(nf4, m, n, k):
    """Decode GEMV and tcgen05 GEMM on FP4 codes against the fp64 oracle."""
    W = synth.weight_normal(n, k, seed=2100 + n + m, dtype=torch.bfloat16, device="cuda")
    X = synth.activations(m, k, seed=2110 + m, device="cuda")
    weight, orc = _check_quant(nf4, W, full_dequant=False, rows=[0, n - 1], quant_type="fp4")
    R = np.arange(n) if n <= 2048 else _sample_rows(n, 256, n)
    _check_linear(nf4, X, weight, orc, weight_rows=R)
    ws = nf4.linear_workspace([(n, k)], m=m)
    a = nf4.nf4_linear(X, weight, torch.float32)
    b = nf4.nf4_linear(X, weight, torch.float32, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_fp4_dx_lora_and_merge(nf4):
    """Backward dX, the QLoRA layer (decode and prefill) and merge + requantize on
    an FP4 weight."""
    n, k, r = 520, 640, 16
    W = synth.weight_normal(n, k, seed=2200, dtype=torch.bfloat16, device="cuda")
    weight, orc = _check_quant(nf4, W, full_dequant=False, rows=[0, n - 1], quant_type="fp4")
    owq, oq, os_, omu = orc
    dY = synth.activations(300, n, seed=2201, device="cuda")
    _check_dx(nf4, dY, weight, orc)
    down = (synth.activations(r, k, seed=2202, device="cuda").float() * 0.02).to(torch.bfloat16)
    up = (synth.activations(n, r, seed=2203, device="cuda").float() * 0.02).to(torch.bfloat16)
    for m in (16, 300):
        X = synth.activations(m, k, seed=2204 + m, device="cuda")
        ws = nf4.lora_workspace(m, [(n, k)], r)
        Y = nf4.nf4_linear_lora(X, weight, down, up, 2.0, ws, dtype=torch.float32)
        torch.cuda.synchronize()
        wrows = O.f32_to_bf16(O.dequantize(owq, oq, os_, omu, "fp4")).reshape(n, k)
        ref = O.linear_lora_bf16(_bits(X).reshape(m, k), wrows, _bits(down).reshape(r, k), _bits(up).reshape(n, r),
                                 2.0)
        assert _rel_fro(Y.cpu().numpy(), ref) <= LINEAR_TOL
    wq, absmax, w_new = nf4.nf4_merge_lora(weight, down, up, 2.0, want_bf16=True)
    torch.cuda.synchronize()
    ow, owq_new, oam_new = O.merge_lora(owq, oq, os_, omu, n, k, _bits(down).reshape(r, k),
                                        _bits(up).reshape(n, r), 2.0, "fp4")
    _assert_equal(w_new.view(torch.int16).view(-1), ow.view(np.int16), "merged bf16 weight (fp4)")
    _assert_equal(wq, owq_new, "merged fp4 codes")
    _assert_equal(absmax, oam_new, "merged absmax (fp4)")
    assert nf4.merge_lora(weight, down, up, 2.0).quant_type == "fp4"


def test_deterministic_and_stream_aware(nf4):
    W = synth.weight_normal(512, 1024, seed=9, dtype=torch.bfloat16, device="cuda")
    X = synth.activations(16, 1024, seed=10, device="cuda")
    a, _ = _gpu_chain(nf4, W)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b, _ = _gpu_chain(nf4, W)
        yb = nf4.nf4_linear(X, b, torch.float32)
    s.synchronize()
    ya = nf4.nf4_linear(X, a, torch.float32)
    torch.cuda.synchronize()
    for name in ("wq", "absmax_q", "absmax_scale", "absmax_offset"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    assert torch.equal(ya, yb)


def test_weights_early_launch_gives_identical_results(nf4):
    """NF4_LINEAR_WEIGHTS_EARLY changes only when the weight loads may start;
    a chain of dependent linears (each reading the previous output) must give
    bit-identical results with and without it."""
    k = 1024
    ws = [nf4.quantize_weight(synth.weight_normal(k, k, seed=700 + j, dtype=torch.bfloat16, device="cuda"))
          for j in range(4)]
    X0 = synth.activations(7, k, seed=701, device="cuda")

    def chain(early):
        x = X0
        for w in ws:
            x = nf4.nf4_linear(x, w, torch.bfloat16, weights_early=early)
        return x
    a = chain(False)
    b = chain(True)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        c = chain(True)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(a, c)


@pytest.mark.parametrize("m", [1, 16])
def test_linear_group_matches_single_launches(nf4, m):
    """Weights that share X (q/k/v-like and gate/up-like) in one nf4_linear_group
    call: the same bits with and without a workspace; each output equal to
    nf4_linear on that weight alone up to the fp32 summation order (a grouped
    launch may split k differently from a single-weight one); the oracle matched
    on sampled rows."""
    k = 2048
    shapes = [(2048, k), (512, k), (512, k)]
    Ws = [synth.weight_normal(n, k, seed=2100 + i, dtype=torch.bfloat16, device="cuda") for i, (n, _) in enumerate(shapes)]
    X = synth.activations(m, k, seed=2110 + m, device="cuda")
    checked = [_check_quant(nf4, W, full_dequant=False, rows=[0, W.shape[0] - 1]) for W in Ws]
    weights = [wo[0] for wo in checked]
    ws = nf4.linear_workspace(shapes, m=m)
    for dtype in (torch.float32, torch.bfloat16):
        singles = [nf4.nf4_linear(X, w, dtype) for w in weights]
        with_ws = nf4.nf4_linear_group(X, weights, dtype, workspace=ws)
        without = nf4.nf4_linear_group(X, weights, dtype)
        torch.cuda.synchronize()
        tol = FP32_ORDER_TOL if dtype == torch.float32 else 1e-2
        for a, b, s1 in zip(with_ws, without, singles):
            assert _same_bits(a, b), "grouped launch: workspace and cluster paths differ"
            err = float((a.float() - s1.float()).norm() / s1.float().norm())
            assert err <= tol, "grouped vs single launch: %.3g" % err
    for (weight, orc), (n, _) in zip(checked, shapes):
        _check_linear(nf4, X, weight, orc, weight_rows=_sample_rows(n, 96, n))
    # the bench's layouts: q/k/v of a 4096-wide layer (one grouped launch) and
    # gate/up of an 11008-wide MLP
    for ns, kk in (([4096, 4096, 4096], 4096), ([11008, 11008], 4096)):
        ws2 = nf4.linear_workspace([(n, kk) for n in ns], m=m)
        Xg = synth.activations(m, kk, seed=2130 + m, device="cuda")
        grp = [nf4.quantize_weight(synth.weight_normal(n, kk, seed=2120 + i, dtype=torch.bfloat16, device="cuda"))
               for i, n in enumerate(ns)]
        outs = nf4.nf4_linear_group(Xg, grp, torch.float32, workspace=ws2, weights_early=True)
        outs_c = nf4.nf4_linear_group(Xg, grp, torch.float32)
        for a, b, w in zip(outs, outs_c, grp):
            assert _same_bits(a, b)
            s1 = nf4.nf4_linear(Xg, w, torch.float32)
            assert float((a - s1).norm() / s1.norm()) <= FP32_ORDER_TOL
        assert int(ws2[:4 * 1024].view(torch.int32).abs().sum()) == 0, "split-k counters not reset"
    # the launch plan on this device: q/k/v of a 4096-wide layer as one launch, gate/up
    # (each already a full wave) as one launch per weight, the GEMM path one per weight
    assert nf4.nf4_linear_group_launches(m, [4096, 4096, 4096], 4096) == 1
    assert nf4.nf4_linear_group_launches(m, [11008, 11008], 4096) == 2
    assert nf4.nf4_linear_group_launches(64, [4096, 4096, 4096], 4096) == 3
    with pytest.raises(ValueError):
        nf4.nf4_linear_group_launches(m, [4096] * 5, 4096)
    with pytest.raises(nf4.NF4Error):  # different k
        nf4.nf4_linear_group(X, [weights[0], nf4.quantize_weight(Ws[0][:, :1024].contiguous())])
    with pytest.raises(nf4.NF4Error):  # too many weights
        nf4.nf4_linear_group(X, weights + weights)


@pytest.mark.parametrize("m,n,k", [(16, 4096, 4096), (3, 300, 576), (64, 512, 1024)])
def test_bounded_wait_timeout_path(nf4, m, n, k):
    """NF4_LINEAR_TEST_TIMEOUT: the copy producers issue nothing and every device
    wait gives up after a few polls.  The call must end with NF4_ERR_DEVICE_TIMEOUT
    in dev_status, leave Y and the workspace untouched (the GEMM frees its tensor memory) and
    leave the stream usable: the next ordinary call is correct.  m = 64 runs the
    tcgen05 GEMM's timeout branches, m <= 16 the GEMV's."""
    W = synth.weight_normal(n, k, seed=2200 + n, dtype=torch.bfloat16, device="cuda")
    X = synth.activations(m, k, seed=2201 + m, device="cuda")
    weight = nf4.quantize_weight(W)
    ws = nf4.linear_workspace([(n, k)], m=m)
    for wsp in (ws, None):
        ref = nf4.nf4_linear(X, weight, torch.float32, workspace=wsp)
        ds = torch.zeros(1, dtype=torch.int32, device="cuda")
        y = torch.full((m, n), 7.0, dtype=torch.float32, device="cuda")
        before = ws.clone()
        nf4.nf4_linear(X, weight, torch.float32, out=y, dev_status=ds, workspace=wsp,
                       flags=nf4._lib.NF4_LINEAR_TEST_TIMEOUT)
        torch.cuda.synchronize()
        assert int(ds.item()) == nf4._lib.NF4_ERR_DEVICE_TIMEOUT
        assert bool((y == 7.0).all()), "a timed-out call wrote Y"
        assert torch.equal(ws, before), "a timed-out call touched the workspace"
        ds.zero_()
        again = nf4.nf4_linear(X, weight, torch.float32, dev_status=ds, workspace=wsp)
        torch.cuda.synchronize()
        assert int(ds.item()) == 0
        assert torch.equal(again, ref)


def test_dev_status_stays_clear(nf4):
    W = synth.weight_normal(256, 512, seed=11, dtype=torch.bfloat16, device="cuda")
    X = synth.activations(3, 512, seed=12, device="cuda")
    weight, _ = _gpu_chain(nf4, W)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nf4.nf4_linear(X, weight, torch.float32, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def test_errors_on_gpu(nf4):
    W = torch.zeros(3, 7, device="cuda")
    with pytest.raises(nf4.NF4Error):
        nf4.nf4_quantize(W)
    with pytest.raises(ValueError):
        nf4.nf4_quantize(torch.zeros(4, 64))          # host tensor
    W = synth.weight_normal(64, 96, seed=1, dtype=torch.bfloat16, device="cuda")
    weight, _ = _gpu_chain(nf4, W)                    # 64*96 is a multiple of 64
    X = synth.activations(2, 96, seed=2, device="cuda")
    with pytest.raises(nf4.NF4Error):                 # but k = 96 is not, for the linear
        nf4.nf4_linear(X, weight)


# ---------------------------------------------------------------------------
# Full-size configurations (the shapes the benchmark runs): whole arrays for
# quantization and double quantization, sampled rows for dequant and linear.
# ---------------------------------------------------------------------------

def _sample_rows(n, count, seed):
    rng = np.random.default_rng(seed)
    rows = set([0, n - 1, n // 2]) | set(rng.choice(n, size=min(count, n), replace=False).tolist())
    return np.array(sorted(rows))


@pytest.mark.parametrize("n,k", [(4096, 4096), (11008, 4096), (4096, 11008)])
def test_cfg2_decode_shapes(nf4, n, k):
    W = synth.weight_normal(n, k, seed=synth.seed_for(2, n // 64 + k // 64), dtype=torch.bfloat16,
                            device="cuda")
    rows = _sample_rows(n, 48, n + k)
    weight, orc = _check_quant(nf4, W, full_dequant=False, rows=rows)
    for m in (1, 4, 16):
        X = synth.activations(m, k, seed=synth.seed_for(2, 100 + m), device="cuda")
        _check_linear(nf4, X, weight, orc, weight_rows=_sample_rows(n, 192, m))


def test_cfg3_prefill_gemm(nf4):
    m, k, n = 4096, 4096, 11008
    W = synth.weight_normal(n, k, seed=synth.seed_for(3, 0), dtype=torch.bfloat16, device="cuda")
    X = synth.activations(m, k, seed=synth.seed_for(3, 1), device="cuda")
    weight, orc = _check_quant(nf4, W, full_dequant=False, rows=_sample_rows(n, 16, 3))
    _check_linear(nf4, X, weight, orc, token_rows=_sample_rows(m, 48, 31),
                  weight_rows=_sample_rows(n, 160, 32))
    # the token-count sweep that bench.py times on the same weight
    for mm in (128, 256, 512, 1024, 2048, 8192):
        Xs = synth.activations(mm, k, seed=synth.seed_for(3, 2) + mm, device="cuda")
        _check_linear(nf4, Xs, weight, orc, token_rows=_sample_rows(mm, 16, mm),
                      weight_rows=_sample_rows(n, 64, mm + 1))


def test_cfg4_layer_stack_sample(nf4):
    """Two decoder layers of the 7B-shaped stack (14 of the 224 tensors), each
    checked on whole arrays."""
    stack = synth.llama7b_stack()
    for idx in (0, 1, 2, 3, 4, 5, 6, 7 * 31 + 4, 7 * 31 + 6):
        _, name, n, k = stack[idx]
        W = synth.weight_normal(n, k, seed=synth.seed_for(4, idx), dtype=torch.bfloat16, device="cuda")
        _check_quant(nf4, W, full_dequant=False, rows=_sample_rows(n, 8, idx))


def test_cfg5_heavy_tailed_stress_layer(nf4):
    n, k = 28672, 8192
    W = synth.weight_student_t(n, k, seed=synth.seed_for(5, 0), device="cuda")
    rows = _sample_rows(n, 24, 5)
    weight, orc = _check_quant(nf4, W, full_dequant=False, rows=rows)
    del W
    for m in (1, 16, 512, 4096):
        X = synth.activations(m, k, seed=synth.seed_for(5, m), device="cuda")
        T = None if m <= 16 else _sample_rows(m, 24, m)
        _check_linear(nf4, X, weight, orc, token_rows=T, weight_rows=_sample_rows(n, 96, m + 1))
