"""Pins for the CPU oracle: each test ties an oracle function to something other
than the oracle itself -- scipy's normal quantile function, the equal-mass
property of the levels, exact rational argmin, the pages' printed figures,
closed forms, hand-derived sums and mathematical error bounds.

No GPU needed (not marked ``gpu``)."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O

f32 = np.float32


def _levels():
    return O.codebook()


# ---------------------------------------------------------------------------
# Levels: 16 normal quantiles, equal probability mass, normalised to [-1, 1],
# with an exact zero (xyzblog page, section 2.2, principle ①; yololab page,
# section on NF4 not being a generic FP4).
# ---------------------------------------------------------------------------

def test_codebook_invariants():
    c = _levels()
    assert c.dtype == np.float32 and c.shape == (16,)
    assert np.all(np.diff(c) > 0), "levels must be strictly increasing"
    assert c[0] == f32(-1.0) and c[15] == f32(1.0)
    assert c[7] == f32(0.0) and np.signbit(c[7]) == False  # noqa: E712
    assert int(np.sum(c < 0)) == 7 and int(np.sum(c > 0)) == 8
    assert int(np.sum(c == 0)) == 1


def test_norm_ppf_against_scipy():
    from scipy.stats import norm
    ps = np.concatenate([np.linspace(1e-6, 1 - 1e-6, 401), [1e-12, 1e-9, 0.5, 0.9677083333333333,
                                                           1 - 1e-9]])
    for p in ps:
        x = O.norm_ppf(p)
        ref = norm.ppf(p)
        assert abs(x - ref) <= 4e-15 * max(1.0, abs(ref)), (p, x, ref)


def test_levels_carry_equal_probability_mass():
    """Undo the normalisation (multiply by Phi^-1 of the outermost probability)
    and map back through the normal CDF: the positive levels must sit at
    probabilities evenly spaced from delta towards 1/2 in 8 steps, the negative
    ones in 7 steps (the equal-area construction)."""
    from scipy.stats import norm
    delta = 0.5 * ((1 - 1 / 30) + (1 - 1 / 32))
    top = norm.ppf(delta)
    c = _levels().astype(np.float64)
    pos = np.sort(c[c > 0])[::-1]
    neg = np.sort(-c[c < 0])[::-1]
    p_pos = norm.cdf(pos * top)
    p_neg = norm.cdf(neg * top)
    np.testing.assert_allclose(p_pos, delta - np.arange(8) * (delta - 0.5) / 8, atol=1e-7)
    np.testing.assert_allclose(p_neg, delta - np.arange(7) * (delta - 0.5) / 7, atol=1e-7)
    # equal spacing in probability = equal probability mass between neighbours
    assert np.allclose(np.diff(p_pos), -(delta - 0.5) / 8, atol=2e-7)


# ---------------------------------------------------------------------------
# Quantization: absmax per 64, x = w / absmax in fp32, nearest level (xyzblog
# page, section 2.2 worked example; Figure 2-2).
# ---------------------------------------------------------------------------

def _exact_argmin(x: np.float32, c: np.ndarray) -> int:
    """Index of the nearest level in exact rational arithmetic, ties to the
    lower index."""
    fx = Fraction(float(x))
    best, best_d = 0, None
    for i, ci in enumerate(c):
        d = abs(fx - Fraction(float(ci)))
        if best_d is None or d < best_d:
            best, best_d = i, d
    return best


def test_quantize_is_exact_argmin_on_random_blocks():
    rng = np.random.default_rng(11)
    c = _levels()
    w = (rng.standard_normal(64 * 12) * 0.02).astype(np.float32)
    w[64 * 3: 64 * 4] *= 1e-30          # a block of tiny values
    w[64 * 5: 64 * 6] = rng.integers(-3, 4, 64).astype(np.float32)  # integers, repeats
    wq, absmax = O.quantize(w)
    idx = O.unpack(wq)
    for b in range(12):
        blk = w[b * 64:(b + 1) * 64]
        am = np.max(np.abs(blk))
        assert absmax[b] == am
        for j in range(64):
            x = f32(blk[j]) / f32(am)       # IEEE fp32 division (numpy)
            assert idx[b * 64 + j] == _exact_argmin(x, c), (b, j, blk[j], am)


def test_quantize_at_and_around_every_midpoint():
    """Place x exactly at each midpoint between neighbouring levels (when the
    midpoint is an fp32 value), and one fp32 step either side of it."""
    c = _levels()
    vals = []
    for j in range(15):
        mid = (Fraction(float(c[j])) + Fraction(float(c[j + 1]))) / 2
        m32 = f32(float(mid))
        for v in (np.nextafter(m32, f32(-2)), m32, np.nextafter(m32, f32(2))):
            vals.append(v)
    vals = np.array(vals, dtype=np.float32)
    n = len(vals)
    pad = (-(n + 1)) % 64
    w = np.concatenate([[f32(1.0)], vals, np.zeros(pad, np.float32)]).astype(np.float32)
    wq, absmax = O.quantize(w)
    idx = O.unpack(wq)
    assert absmax[0] == 1.0
    for i, v in enumerate(w):
        assert idx[i] == _exact_argmin(v, c), (i, v)
    # ties really occur and go to the lower index
    ties = 0
    for j in range(15):
        mid = (Fraction(float(c[j])) + Fraction(float(c[j + 1]))) / 2
        if Fraction(float(f32(float(mid)))) == mid:
            ties += 1
            pos = 1 + 3 * j + 1
            assert idx[pos] == j
    assert ties > 0


def test_block_maximum_maps_to_an_end_level():
    rng = np.random.default_rng(5)
    w = (rng.standard_normal(64 * 50) * 0.02).astype(np.float32)
    wq, absmax = O.quantize(w)
    idx = O.unpack(wq)
    for b in range(50):
        blk = w[b * 64:(b + 1) * 64]
        j = int(np.argmax(np.abs(blk)))
        assert idx[b * 64 + j] == (15 if blk[j] > 0 else 0)


def test_zero_block_and_negative_zero():
    w = np.zeros(128, dtype=np.float32)
    w[64:] = (np.arange(64, dtype=np.float32) - 32) / 64
    w[70] = -0.0
    wq, absmax = O.quantize(w)
    idx = O.unpack(wq)
    assert absmax[0] == 0.0 and np.all(idx[:64] == 7)
    assert idx[70] == 7


def test_packing_puts_the_even_element_in_the_high_nibble(golden):
    ex = golden["block_layout_example"]
    w = np.zeros(64, dtype=np.float32)
    w[0], w[1] = 1.0, -1.0       # indices 15, 0
    w[2], w[3] = 0.0, 1.0        # indices 7, 15
    wq, _ = O.quantize(w)
    assert wq.size * ex["codes_per_byte"] == 64
    assert wq[0] == 0xF0 and wq[1] == 0x7F
    assert np.all(wq[2:] == 0x77)


def test_bf16_input_is_widened_exactly():
    rng = np.random.default_rng(3)
    wt = torch.from_numpy((rng.standard_normal(64 * 8) * 0.02).astype(np.float32)).to(torch.bfloat16)
    bits = wt.view(torch.int16).numpy().view(np.uint16)
    wq1, am1 = O.quantize(bits)
    wq2, am2 = O.quantize(wt.float().numpy())
    assert np.array_equal(wq1, wq2) and np.array_equal(am1, am2)


# ---------------------------------------------------------------------------
# bf16 rounding: the page's printed example and the IEEE tie rule.
# ---------------------------------------------------------------------------

def test_bf16_rounding_matches_the_page_example(golden):
    ex = golden["bf16_rounding_example"]
    x = np.array([f32(float(ex["input_decimal"]))], dtype=np.float32)
    assert abs(float(x[0]) - ex["fp32_stored"]) < 1e-15
    b = O.f32_to_bf16(x)
    assert float(O.bf16_to_f32(b)[0]) == ex["bf16_stored"]


def test_bf16_rounding_ties_to_even_and_matches_torch():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: goes to 1 (even);
    # 1 + 3 * 2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: goes to 1 + 2^-6.
    x = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8)], dtype=np.float32)
    y = O.bf16_to_f32(O.f32_to_bf16(x))
    assert y.tolist() == [1.0, 1 + 2 ** -6, -1.0]
    rng = np.random.default_rng(9)
    r = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    mine = O.f32_to_bf16(r)
    ref = torch.from_numpy(r).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)


# ---------------------------------------------------------------------------
# Double quantization: closed-form storage, fixed summation order, 8-bit error
# bound (xyzblog page, section 2.2 ②; zingnex page, paging and double-quant
# section; yololab page, double quantization section).
# ---------------------------------------------------------------------------

def test_storage_overhead_closed_form(golden):
    dq = golden["double_quant_overhead"]
    n, k = 256, 4096
    rng = np.random.default_rng(1)
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    wq, absmax = O.quantize(w)
    q, s, mu = O.double_quant(absmax)
    bits = (wq.nbytes + q.nbytes + s.nbytes) * 8 / (n * k)
    assert bits == 4 + 8 / 64 + 32 / (64 * 256) == 4.126953125
    assert dq["bits_per_param_absmax_fp32"] == 4 + absmax.nbytes * 8 / (n * k)
    saving = dq["bits_per_param_absmax_fp32"] - bits
    assert abs(saving - dq["saving_bits_per_param_approx"]) < 0.005
    assert abs(saving - golden["double_quant_saving_forum"]["saving_bits_per_param_approx"]) < 0.005
    assert abs(bits - dq["bits_per_param_after_dq_approx"]) < 0.005
    fp = golden["footprint_70b"]
    assert abs(fp["params"] * 16 / 8 / 1e9 - fp["fp16_gb_approx"]) < 1e-6
    gb = fp["params"] * bits / 8 / 1e9
    assert abs(gb - fp["nf4_gb_approx"]) / fp["nf4_gb_approx"] < 0.05


def test_page_example_layout(golden):
    ex = golden["block_layout_example"]
    out = 3
    w = (np.random.default_rng(2).standard_normal((out, ex["in_features"])) * 0.02).astype(np.float32)
    wq, absmax = O.quantize(w)
    assert absmax.size == out * ex["blocks_per_row"] == out * ex["in_features"] // ex["blocksize"]
    assert wq.nbytes == ex["packed_fraction_of_fp16"] * (out * ex["in_features"] * 2)


def test_dq_sum_follows_the_fixed_tree_order():
    # Halving tree over a zero-padded chunk of 256: 1 + 2^53 rounds to 2^53
    # (tie to even) at the h = 2 step, then 2^53 + 1 again rounds to 2^53.
    # Summed left to right the same values would give 2^53 + 2.
    a = np.array([1.0, 1.0, 2.0 ** 53, 0.0], dtype=np.float32)
    assert O.dq_sum(a) == 2.0 ** 53
    # with one more level (nb > 256) the chunk results are combined the same way
    b = np.zeros(512, dtype=np.float32)
    b[0], b[256] = 2.0 ** 53, 1.0
    b[1] = 1.0
    # chunk 0 -> 2^53 + 1 -> 2^53 (tie to even); chunk 1 -> 1; 2^53 + 1 -> 2^53
    assert O.dq_sum(b) == 2.0 ** 53


def test_dq_sum_is_the_exact_sum_when_representable():
    rng = np.random.default_rng(4)
    for nb in (1, 7, 256, 257, 1000, 70000):
        a = (rng.uniform(0.01, 0.08, nb)).astype(np.float32)
        exact = sum(Fraction(float(v)) for v in a)
        assert Fraction(O.dq_sum(a)) == exact
        mu = O.dq_mean(a)
        true_mu = exact / nb
        # one fp64 rounding then one fp32 rounding: within an fp32 ulp
        assert abs(Fraction(float(mu)) - true_mu) <= Fraction(float(np.spacing(mu)))


def test_double_quant_invariants_and_error_bound():
    rng = np.random.default_rng(6)
    nb = 1000  # 3 full blocks of 256 and a partial one
    absmax = (np.abs(rng.standard_normal(nb)) * 0.03 + 0.01).astype(np.float32)
    q, s, mu = O.double_quant(absmax)
    assert q.dtype == np.int8 and s.size == 4
    assert mu == O.dq_mean(absmax)
    ahat = O.absmax_hat(q, s, mu)
    for j in range(4):
        lo, hi = 256 * j, min(256 * (j + 1), nb)
        r = absmax[lo:hi].astype(np.float64) - float(mu)
        assert s[j] == np.max(np.abs(f32(absmax[lo:hi]) - mu))
        jm = int(np.argmax(np.abs(r)))
        assert abs(int(q[lo + jm])) == 127
        assert np.all(np.abs(q[lo:hi].astype(int)) <= 127)
        assert np.all(np.sign(q[lo:hi]) * np.sign(r) >= 0)
        order = np.argsort(absmax[lo:hi], kind="stable")
        assert np.all(np.diff(q[lo:hi][order].astype(int)) >= 0)   # monotone in absmax
        # 8-bit rounding error: at most half a step of s / 127, plus fp32 roundings
        err = np.abs(ahat[lo:hi].astype(np.float64) - absmax[lo:hi])
        assert np.all(err <= s[j] / 254 + 4 * np.spacing(np.float32(absmax[lo:hi].max())))


def test_double_quant_constant_absmax_gives_zero_scale():
    a = np.full(300, 0.037, dtype=np.float32)
    q, s, mu = O.double_quant(a)
    assert mu == f32(0.037) and np.all(s == 0) and np.all(q == 0)
    assert np.all(O.absmax_hat(q, s, mu) == mu)


# ---------------------------------------------------------------------------
# Dequantization (technicalnotes page, section 5 dynamic dequantization).
# ---------------------------------------------------------------------------

def test_dequantize_error_bound_and_end_levels():
    rng = np.random.default_rng(8)
    n, k = 16, 1024
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    wq, absmax = O.quantize(w)
    q, s, mu = O.double_quant(absmax)
    wh = O.dequantize(wq, q, s, mu).reshape(n, k)
    c = _levels().astype(np.float64)
    half_gap = np.max(np.diff(c)) / 2
    ahat = O.absmax_hat(q, s, mu).astype(np.float64)
    wb = w.reshape(-1, 64).astype(np.float64)
    whb = wh.reshape(-1, 64).astype(np.float64)
    for b in range(wb.shape[0]):
        bound = half_gap * absmax[b] + abs(ahat[b] - absmax[b]) + 1e-6 * absmax[b]
        assert np.all(np.abs(whb[b] - wb[b]) <= bound)
        j = int(np.argmax(np.abs(wb[b])))
        assert whb[b, j] == np.sign(wb[b, j]) * f32(ahat[b])


# ---------------------------------------------------------------------------
# fp64 linear (xyzblog page, section 2.2 code walk: matmul_4bit = dequant + matmul).
# ---------------------------------------------------------------------------

def test_linear_against_numpy_float64_and_exact_integers():
    rng = np.random.default_rng(10)
    x = torch.from_numpy(rng.standard_normal((5, 96)).astype(np.float32)).to(torch.bfloat16)
    w = torch.from_numpy((rng.standard_normal((7, 96)) * 0.02).astype(np.float32)).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    wb = w.view(torch.int16).numpy().view(np.uint16)
    y = O.linear_bf16(xb, wb)
    ref = x.double().numpy() @ w.double().numpy().T
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-15)
    xi = torch.tensor([[1, -2, 3], [0, 5, -1]], dtype=torch.bfloat16)
    wi = torch.tensor([[2, 2, 2], [-1, 0, 4]], dtype=torch.bfloat16)
    y = O.linear_bf16(xi.view(torch.int16).numpy().view(np.uint16),
                      wi.view(torch.int16).numpy().view(np.uint16))
    assert y.tolist() == [[4.0, 11.0], [8.0, -4.0]]


def test_normalisation_is_a_true_division():
    """x = w / absmax must be the correctly rounded quotient, not w * (1/absmax):
    find weights where the two differ across a decision midpoint and check the
    oracle follows the division."""
    c = _levels()
    found = 0
    for a in (f32(0.7), f32(0.0311), f32(0.123456), f32(1.9e-3), f32(0.0517)):
        recip = f32(1.0) / a
        cases = []
        for j in range(15):
            mid = (Fraction(float(c[j])) + Fraction(float(c[j + 1]))) / 2
            w0 = f32(float(mid * Fraction(float(a))))
            w = w0
            for _ in range(6):
                w = np.nextafter(w, f32(-2))
            for _ in range(13):
                x_div = f32(w) / a
                x_mul = f32(w) * recip
                if _exact_argmin(x_div, c) != _exact_argmin(x_mul, c):
                    cases.append(w)
                w = np.nextafter(w, f32(2))
        if not cases:
            continue
        blk = np.zeros(64, dtype=np.float32)
        blk[0] = a
        blk[1:1 + min(63, len(cases))] = cases[:63]
        wq, absmax = O.quantize(blk)
        idx = O.unpack(wq)
        assert absmax[0] == a
        for i in range(1, 1 + min(63, len(cases))):
            assert idx[i] == _exact_argmin(f32(blk[i]) / a, c)
        found += len(cases)
    assert found > 0, "no weight distinguishes division from reciprocal multiply"


# ---------------------------------------------------------------------------
# Backward through the frozen base: dX = dY * What (yololab page, section
# "QLoRA 把 frozen 4-bit base 與可訓練 adapter 分開": the base is dequantized in the
# backward pass too).  Pinned by the adjoint identity of the forward linear and
# by brute force on exact integer inputs.
# ---------------------------------------------------------------------------

def _bf16_bits(a):
    return (np.asarray(a, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_linear_dx_adjoint_identity():
    """<dY, X What^T> = <dY What, X> for every X, dY: the backward product is the
    adjoint of the forward one (a transposed or mis-indexed weight breaks it)."""
    rng = np.random.default_rng(21)
    for (m, n, k) in [(3, 5, 7), (4, 64, 64), (2, 96, 128)]:
        W = _bf16_bits(rng.standard_normal((n, k)).astype(np.float32))
        X = _bf16_bits(rng.standard_normal((m, k)).astype(np.float32))
        dY = _bf16_bits(rng.standard_normal((m, n)).astype(np.float32))
        y = O.linear_bf16(X, W)
        dx = O.linear_dx_bf16(dY, W)
        assert dx.shape == (m, k)
        lhs = float(np.sum(O.bf16_to_f32(dY).astype(np.float64) * y))
        rhs = float(np.sum(dx * O.bf16_to_f32(X).astype(np.float64)))
        assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs)), (lhs, rhs)


def test_linear_dx_exact_small_integers():
    """Small integers are exact in bf16 and their products and sums exact in
    fp64, so dX must equal the integer matrix product computed by loops."""
    rng = np.random.default_rng(22)
    m, n, k = 3, 5, 4
    Wi = rng.integers(-8, 9, size=(n, k))
    dYi = rng.integers(-8, 9, size=(m, n))
    dx = O.linear_dx_bf16(_bf16_bits(dYi), _bf16_bits(Wi))
    for i in range(m):
        for c in range(k):
            assert dx[i, c] == sum(int(dYi[i, r]) * int(Wi[r, c]) for r in range(n))


# ---------------------------------------------------------------------------
# LoRA layer: Y = X What^T + s (X down^T) up^T (technicalnotes page, sections
# "2-2. LoRA" and 4).  Pinned by the zero-scale case, by the merged-weight
# identity W' = What + s up down, and by integer brute force.
# ---------------------------------------------------------------------------

def test_linear_lora_zero_scale_is_the_base_linear():
    rng = np.random.default_rng(31)
    m, n, k, r = 3, 40, 64, 4
    X = _bf16_bits(rng.standard_normal((m, k)))
    W = _bf16_bits(rng.standard_normal((n, k)))
    D = _bf16_bits(rng.standard_normal((r, k)))
    U = _bf16_bits(rng.standard_normal((n, r)))
    assert np.array_equal(O.linear_lora_bf16(X, W, D, U, 0.0), O.linear_bf16(X, W))


def test_linear_lora_equals_the_merged_weight():
    """X (What + s up down)^T computed directly (merge first, then multiply)
    agrees with the layer's low-rank path to fp64 rounding."""
    rng = np.random.default_rng(32)
    for (m, n, k, r, s) in [(2, 24, 64, 3, 2.0), (4, 64, 128, 16, 0.5)]:
        X = _bf16_bits(rng.standard_normal((m, k)))
        W = _bf16_bits(rng.standard_normal((n, k)))
        D = _bf16_bits(rng.standard_normal((r, k)))
        U = _bf16_bits(rng.standard_normal((n, r)))
        y = O.linear_lora_bf16(X, W, D, U, s)
        wm = O.bf16_to_f32(W).astype(np.float64) + s * (O.bf16_to_f32(U).astype(np.float64)
                                                         @ O.bf16_to_f32(D).astype(np.float64))
        ym = O.bf16_to_f32(X).astype(np.float64) @ wm.T
        assert np.allclose(y, ym, rtol=1e-12, atol=1e-12)


def test_linear_lora_exact_small_integers():
    rng = np.random.default_rng(33)
    m, n, k, r = 2, 3, 5, 2
    Xi, Wi = rng.integers(-4, 5, size=(m, k)), rng.integers(-4, 5, size=(n, k))
    Di, Ui = rng.integers(-4, 5, size=(r, k)), rng.integers(-4, 5, size=(n, r))
    y = O.linear_lora_bf16(_bf16_bits(Xi), _bf16_bits(Wi), _bf16_bits(Di), _bf16_bits(Ui), 3.0)
    for i in range(m):
        for o in range(n):
            base = sum(int(Xi[i, c]) * int(Wi[o, c]) for c in range(k))
            low = sum(sum(int(Xi[i, c]) * int(Di[j, c]) for c in range(k)) * int(Ui[o, j]) for j in range(r))
            assert y[i, o] == base + 3 * low


# ---------------------------------------------------------------------------
# Merge + requantize (technicalnotes page, section "8. LoRA 的合併（Merge）").
# Pinned by integer brute force on the delta, by the zero-scale case (W_new is the
# bf16 dequant), and by the bound that links the merged weight to the LoRA layer.
# ---------------------------------------------------------------------------

def test_lora_delta_exact_small_integers():
    rng = np.random.default_rng(41)
    n, r, k = 3, 4, 5
    Ui, Di = rng.integers(-6, 7, size=(n, r)), rng.integers(-6, 7, size=(r, k))
    d = O.lora_delta(_bf16_bits(Ui), _bf16_bits(Di))
    for o in range(n):
        for c in range(k):
            assert d[o, c] == sum(int(Ui[o, j]) * int(Di[j, c]) for j in range(r))


def _quantized(rng, n, k):
    W = rng.standard_normal((n, k)).astype(np.float32) * 0.02
    wq, am = O.quantize(W)
    q, s, mu = O.double_quant(am)
    return wq, q, s, mu


def test_merge_zero_scale_is_the_bf16_dequant():
    rng = np.random.default_rng(42)
    n, k, r = 8, 128, 4
    wq, q, s, mu = _quantized(rng, n, k)
    D = _bf16_bits(rng.standard_normal((r, k)))
    U = _bf16_bits(rng.standard_normal((n, r)))
    w_new, wq2, am2 = O.merge_lora(wq, q, s, mu, n, k, D, U, 0.0)
    what = O.f32_to_bf16(O.dequantize(wq, q, s, mu)).reshape(n, k)
    assert np.array_equal(w_new, what)
    # and the requantized codes are the quantization of that bf16 weight
    wq3, am3 = O.quantize(what.reshape(-1))
    assert np.array_equal(wq2, wq3) and np.array_equal(am2.view(np.uint32), am3.view(np.uint32))


def test_merged_weight_matches_the_lora_layer_within_bf16_rounding():
    """X W_new^T differs from the fp64 LoRA layer only by W_new's rounding: each
    element of W_new is within 2^-8 relative of What + s up down (one fp32 add,
    one bf16 round), so |difference| <= 2^-8 * sum |x| |W_new| + fp32 slack."""
    rng = np.random.default_rng(43)
    n, k, r, m, sc = 16, 128, 8, 3, 2.0
    wq, q, s, mu = _quantized(rng, n, k)
    D = _bf16_bits(rng.standard_normal((r, k)) * 0.02)
    U = _bf16_bits(rng.standard_normal((n, r)) * 0.02)
    X = _bf16_bits(rng.standard_normal((m, k)))
    w_new, _, _ = O.merge_lora(wq, q, s, mu, n, k, D, U, sc)
    what = O.f32_to_bf16(O.dequantize(wq, q, s, mu)).reshape(n, k)
    y_merged = O.linear_bf16(X, w_new)
    y_layer = O.linear_lora_bf16(X, what, D, U, sc)
    xa = np.abs(O.bf16_to_f32(X).astype(np.float64))
    wa = np.abs(O.bf16_to_f32(w_new).astype(np.float64))
    bound = 2.0 ** -8 * (xa @ wa.T) + 1e-6
    assert np.all(np.abs(y_merged - y_layer) <= bound)


# ---------------------------------------------------------------------------
# FP4 codebook (xyzblog page, section 2.2 code walk: FP4 is the generic float
# format builder with a sign bit, 2 exponent bits and 1 mantissa bit; zingnex
# page, "4-bit 量化": FP4 is a conventional 4-bit float).  The same blockwise
# pipeline with that table in place of the NF4 levels.
# ---------------------------------------------------------------------------

def _e2m1_decoded() -> np.ndarray:
    """ml_dtypes' own decoding of the 16 bit patterns of its E2M1 type."""
    import ml_dtypes
    return np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)


def test_fp4_codebook_is_the_scaled_e2m1_format():
    v = _e2m1_decoded()
    ref = (v / np.max(np.abs(v))).astype(np.float32)
    c = O.codebook("fp4")
    assert np.array_equal(c.view(np.uint32), ref.view(np.uint32))   # -0 at code 8 included
    assert c[0] == 0 and not np.signbit(c[0]) and np.signbit(c[8])
    assert c[7] == f32(1.0) and c[15] == f32(-1.0)
    assert np.array_equal(c[8:], -c[:8])
    assert np.all(np.diff(c[:8]) > 0)
    # two values per binade after the subnormal pair, consecutive binades a factor 2 apart
    assert c[3] == 3 * c[1] and c[5] == 2 * c[3] and c[7] == 2 * c[5] and c[2] == 2 * c[1]


def test_fp4_quantize_is_exact_argmin_and_e2m1_rounding_off_ties():
    import ml_dtypes
    rng = np.random.default_rng(61)
    c = O.codebook("fp4")
    w = (rng.standard_normal(64 * 10) * 0.02).astype(np.float32)
    w[64 * 2: 64 * 3] *= 1e-30                                     # tiny values
    w[64 * 4: 64 * 5] = rng.integers(-6, 7, 64).astype(np.float32)   # exact grid points and ties
    w[64 * 6 + 3] = -1e-9                                          # tiny negative next to larger values
    # the one exact tie among the FP4 values: halfway between 0 and the smallest
    # subnormal (the other midpoints are not fp32 values)
    w[64 * 8: 64 * 9] = 0.0
    w[64 * 8] = 1.0
    w[64 * 8 + 1], w[64 * 8 + 2] = c[1] / 2, -c[1] / 2
    wq, absmax = O.quantize(w, "fp4")
    idx = O.unpack(wq)
    ties = 0
    for b in range(10):
        blk = w[b * 64:(b + 1) * 64]
        am = np.max(np.abs(blk))
        assert absmax[b] == am
        for j in range(64):
            x = f32(blk[j]) / f32(am)
            code = idx[b * 64 + j]
            assert code == _exact_argmin(x, c), (b, j, blk[j], am)
            assert code != 8, "the -0 code is never produced"
            # off a tie, the value is E2M1 round-to-nearest of 6x scaled back
            fx = Fraction(float(x))
            d = sorted(abs(fx - Fraction(float(ci))) for ci in set(c.tolist()))
            if d[0] == d[1]:
                ties += 1
                continue
            e = float(np.array([6.0 * float(x)]).astype(ml_dtypes.float4_e2m1fn).astype(np.float64)[0])
            assert c[code] == f32(e / 6.0), (x, code, e)
    assert ties > 0


def test_fp4_midpoints_tie_toward_zero_and_zero_blocks():
    c = O.codebook("fp4")
    mags = c[:8]
    vals = []
    for j in range(7):
        mid = (Fraction(float(mags[j])) + Fraction(float(mags[j + 1]))) / 2
        m32 = f32(float(mid))
        for v in (np.nextafter(m32, f32(-2)), m32, np.nextafter(m32, f32(2))):
            vals += [v, -v]
    vals = np.array(vals, dtype=np.float32)
    pad = (-(len(vals) + 1)) % 64
    w = np.concatenate([[f32(1.0)], vals, np.zeros(pad, np.float32)]).astype(np.float32)
    w = np.concatenate([w, np.zeros(64, np.float32)])              # a zero block
    w[-5] = -0.0
    wq, absmax = O.quantize(w, "fp4")
    idx = O.unpack(wq)
    for i, v in enumerate(w):
        assert idx[i] == _exact_argmin(v, c), (i, v)
    for j in range(7):
        mid = (Fraction(float(mags[j])) + Fraction(float(mags[j + 1]))) / 2
        if Fraction(float(f32(float(mid)))) == mid:                # an exact tie
            pos = 1 + 6 * j + 2
            assert idx[pos] == j and idx[pos + 1] == (8 + j if j > 0 else 0)
    assert absmax[-1] == 0.0 and np.all(idx[-64:] == 0)


def test_fp4_dequantize_error_bound_and_end_levels():
    rng = np.random.default_rng(62)
    n, k = 16, 1024
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    wq, absmax = O.quantize(w, "fp4")
    q, s, mu = O.double_quant(absmax)
    wh = O.dequantize(wq, q, s, mu, "fp4").reshape(n, k)
    c = O.codebook("fp4").astype(np.float64)
    half_gap = np.max(np.diff(np.sort(c))) / 2                     # (1 - 2/3) / 2
    assert abs(half_gap - 1.0 / 6.0) < 1e-7
    ahat = O.absmax_hat(q, s, mu).astype(np.float64)
    wb = w.reshape(-1, 64).astype(np.float64)
    whb = wh.reshape(-1, 64).astype(np.float64)
    idx = O.unpack(wq).reshape(-1, 64)
    for b in range(wb.shape[0]):
        bound = half_gap * absmax[b] + abs(ahat[b] - absmax[b]) + 1e-6 * absmax[b]
        assert np.all(np.abs(whb[b] - wb[b]) <= bound)
        j = int(np.argmax(np.abs(wb[b])))
        assert idx[b, j] == (7 if wb[b, j] > 0 else 15)
        assert whb[b, j] == np.sign(wb[b, j]) * f32(ahat[b])
    # the NF4 table gives a different (smaller) error on normal weights
    wq_n, am_n = O.quantize(w)
    qn, sn, mun = O.double_quant(am_n)
    err_n = np.mean((O.dequantize(wq_n, qn, sn, mun).reshape(n, k) - w) ** 2)
    err_f = np.mean((wh - w) ** 2)
    assert err_n < err_f


def test_fp4_merge_zero_scale_is_the_bf16_dequant():
    rng = np.random.default_rng(63)
    n, k, r = 8, 128, 4
    W = rng.standard_normal((n, k)).astype(np.float32) * 0.02
    wq, am = O.quantize(W, "fp4")
    q, s, mu = O.double_quant(am)
    D = _bf16_bits(rng.standard_normal((r, k)))
    U = _bf16_bits(rng.standard_normal((n, r)))
    w_new, wq2, am2 = O.merge_lora(wq, q, s, mu, n, k, D, U, 0.0, "fp4")
    what = O.f32_to_bf16(O.dequantize(wq, q, s, mu, "fp4")).reshape(n, k)
    assert np.array_equal(w_new, what)
    wq3, am3 = O.quantize(what.reshape(-1), "fp4")
    assert np.array_equal(wq2, wq3) and np.array_equal(am2.view(np.uint32), am3.view(np.uint32))


# ---------------------------------------------------------------------------
# The rounding sequences, bit for bit.  Each expected value is recomputed in
# exact rational arithmetic with an explicit round-to-nearest-even after every
# step the readings name (xyzblog page, section 2.2 ② and Figure 2-2 step 5 for
# the double quantization; technicalnotes page, section 5, for the dequantized
# weight): absmax dequant a = RN(RN(RN(q / 127) * s) + mu); code
# q = RNE(RN(RN(r / s) * 127)); mean mu = RN32(RN64(S / nb)); weight RN(c * a).
# ---------------------------------------------------------------------------

def _rn(x: Fraction, p: int, emin: int) -> Fraction:
    """x rounded to the nearest binary floating-point value with p significant
    bits and smallest normal exponent emin (gradual underflow), ties to even."""
    if x == 0:
        return Fraction(0)
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, emin)
    ulp = Fraction(2) ** (e - p + 1)
    n, rem = divmod(a, ulp)
    if 2 * rem > ulp or (2 * rem == ulp and n % 2 == 1):
        n += 1
    return n * ulp if x > 0 else -n * ulp


def _rn32(x: Fraction) -> Fraction:
    return _rn(x, 24, -126)


def _rn64(x: Fraction) -> Fraction:
    return _rn(x, 53, -1022)


def _rne_int(x: Fraction) -> int:
    n, rem = divmod(x, 1)
    if 2 * rem > 1 or (2 * rem == 1 and n % 2 == 1):
        n += 1
    return int(n)


def _F(v) -> Fraction:
    return Fraction(float(v))


def test_rounding_helper_against_ieee_hardware():
    """The exact-rational rounding used below agrees with numpy's IEEE fp32 and
    Python's fp64 arithmetic on random quotients, ties and subnormals."""
    rng = np.random.default_rng(40)
    for _ in range(2000):
        a, b = f32(rng.standard_normal()), f32(rng.uniform(0.01, 10))
        assert _rn32(_F(a) / _F(b)) == _F(a / b)
        assert _rn32(_F(a) * _F(b)) == _F(a * b)
        x, y = rng.standard_normal(), rng.uniform(0.1, 10)
        assert _rn64(Fraction(x) / Fraction(y)) == Fraction(x / y)
    assert _rn32(Fraction(1) + Fraction(1, 2 ** 24)) == 1                 # tie to even (down)
    assert _rn32(Fraction(1) + Fraction(3, 2 ** 24)) == 1 + Fraction(2, 2 ** 23)
    tiny = Fraction(3, 2 ** 150)                                           # half-way between subnormals
    assert _rn32(tiny) == _F(np.float32(float(tiny)))
    assert [_rne_int(Fraction(k, 2)) for k in (1, 3, 5, -1, -3)] == [0, 2, 2, 0, -2]


def test_absmax_dequant_is_three_roundings_in_order():
    """a = RN(RN(RN(q / 127) * s) + mu) for every int8 code: q / 127 a true
    quotient (not q * RN(1/127)), multiplied by s (not q * RN(s / 127)), then mu
    added.  s = 1, mu = 0 isolates the quotient."""
    rng = np.random.default_rng(41)
    q = np.arange(-127, 128, dtype=np.int8)
    cases = [(f32(1.0), f32(0.0))] + [(f32(rng.uniform(1e-3, 0.3)), f32(rng.uniform(0.0, 0.1)))
                                     for _ in range(6)] + [(f32(2.0 ** -20 * 3), f32(1e-6))]
    for s, mu in cases:
        got = O.absmax_hat(q, np.array([s], dtype=np.float32), mu)
        for qi, g in zip(q, got):
            want = _rn32(_rn32(_rn32(Fraction(int(qi), 127)) * _F(s)) + _F(mu))
            assert _F(g) == want, (int(qi), float(s), float(mu))


def _spec_mean(absmax: np.ndarray) -> np.float32:
    """mu = RN32(RN64(S / nb)) with S the oracle's fixed-tree fp64 sum (pinned
    on its own above)."""
    return np.float32(O.dq_sum(absmax) / float(absmax.size))


def test_dq_mean_divides_in_fp64_then_rounds_once_to_fp32():
    rng = np.random.default_rng(42)
    differ = 0
    for trial in range(60):
        nb = int(rng.integers(257, 3000)) | 1         # odd: the division is inexact
        absmax = (np.abs(rng.standard_normal(nb)) * 0.05 + 1e-3).astype(np.float32)
        S = O.dq_sum(absmax)
        want = _rn32(_rn64(Fraction(S) / nb))          # fp64 quotient, then fp32
        assert _F(O.dq_mean(absmax)) == want, (trial, nb)
        if _rn32(_rn32(Fraction(S)) / nb) != want:     # an fp32 division would differ here
            differ += 1
    assert differ > 0, "no sample separates fp64 from fp32 division"


def _spec_codes(absmax: np.ndarray):
    """The double-quantization codes and scales from the stated sequence."""
    mu = _F(_spec_mean(absmax))
    r = [_rn32(_F(a) - mu) for a in absmax]
    qs, ss = [], []
    for j in range(0, len(r), 256):
        blk = r[j:j + 256]
        s = max(abs(v) for v in blk)
        ss.append(s)
        for v in blk:
            qs.append(0 if s == 0 else _rne_int(_rn32(_rn32(v / s) * 127)))
    return qs, ss


def test_double_quant_code_is_the_stated_rounding_sequence():
    rng = np.random.default_rng(43)
    for nb in (1000, 256, 77):
        absmax = (np.abs(rng.standard_normal(nb)) * 0.04 + 2e-3).astype(np.float32)
        q, s, mu = O.double_quant(absmax)
        wq, ws = _spec_codes(absmax)
        assert [int(v) for v in q] == wq
        assert [_F(v) for v in s] == ws
        assert _F(mu) == _F(_spec_mean(absmax))


def _tie_block(n_target: int, seed: int):
    """An absmax vector in which one entry's RN(RN(r / s) * 127) is exactly
    n_target + 1/2, found by a short fixed-point search in fp32 arithmetic."""
    rng = np.random.default_rng(seed)
    nb = 2048
    absmax = (np.abs(rng.standard_normal(nb)) * 0.01 + 0.02).astype(np.float32)
    blk0 = 3 * 256                       # the tie entry sits in DQ block 3 ...
    absmax[blk0] = f32(0.2)              # ... whose largest |r| is set here
    j = blk0 + 17
    for _ in range(20):
        mu = _spec_mean(absmax)
        r = (absmax[blk0:blk0 + 256] - mu).astype(np.float32)
        s = f32(np.max(np.abs(r)))
        t = f32((n_target + 0.5) / 127.0)
        for _k in range(64):             # walk t until t * 127 rounds onto the half
            u = f32(t * f32(127.0))
            if u == f32(n_target + 0.5):
                break
            t = np.nextafter(t, f32(np.inf) if u < n_target + 0.5 else f32(-np.inf))
        rj = f32(t * s)
        x = f32(mu + rj)
        if absmax[j] == x:
            break
        absmax[j] = x
    return absmax, j


def test_double_quant_ties_round_half_to_even():
    """Entries whose scaled code RN(RN(r / s) * 127) is exactly k + 1/2 go to the
    even neighbour (both parities of k, both signs of r checked when found)."""
    found = 0
    for n_target, seed in ((40, 1), (41, 2), (70, 3), (9, 4), (100, 5)):
        absmax, j = _tie_block(n_target, seed)
        q, s, mu = O.double_quant(absmax)
        mu_e = _F(_spec_mean(absmax))
        r = _rn32(_F(absmax[j]) - mu_e)
        blk = 3 * 256
        smax = max(abs(_rn32(_F(a) - mu_e)) for a in absmax[blk:blk + 256])
        u = _rn32(_rn32(r / smax) * 127)
        if u.denominator != 2:
            continue                      # the search missed this target; others must hit
        found += 1
        assert int(q[j]) == _rne_int(u), (n_target, float(u))
        assert int(q[j]) % 2 == 0
    assert found >= 2, "too few exact ties constructed"


def test_weight_dequant_is_one_fp32_product():
    """w = RN(c[idx] * a): one fp32 rounding of the exact product, on random
    codes, scales and means (fp64-then-fp32 or any biased product differs on a
    few percent of these)."""
    rng = np.random.default_rng(44)
    c = O.codebook()
    nb = 300
    absmax = (np.abs(rng.standard_normal(nb)) * 0.03 + 1e-3).astype(np.float32)
    q, s, mu = O.double_quant(absmax)
    wq = rng.integers(0, 256, size=nb * 32, dtype=np.uint8)
    got = O.dequantize_range(wq, q, s, mu, 0, nb * 64)
    ahat = O.absmax_hat(q, s, mu)
    idx = O.unpack(wq)
    for e in range(0, nb * 64, 7):
        want = _rn32(_F(c[idx[e]]) * _F(ahat[e // 64]))
        assert _F(got[e]) == want, e
