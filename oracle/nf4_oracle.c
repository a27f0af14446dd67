/*
 * nf4_oracle.c -- CPU oracle for the NF4 + double-quantization weight path.
 *
 * TEST INFRASTRUCTURE ONLY (see nf4_oracle.h for the sources and the readings).
 * Plain loops, one thread, IEEE arithmetic with no contraction.  Nothing here is
 * blocked, fused or reordered beyond what each function's comment states.
 *
 * Pins (tests/test_oracle_*.py) tie every function to something other than
 * itself: scipy's normal quantile function, the equal-probability-mass property
 * of the levels, exact rational argmin on tiny tensors, the page's printed
 * rounding example (2.3 -> bf16 2.296875), the closed-form storage overhead, and
 * hand-derived sums for the fixed summation order.
 */
#define _GNU_SOURCE
#include "nf4_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------------------
 * Normal quantiles.
 * [P5] §2.2 principle ①: the levels are quantiles of N(0,1).  Phi^-1 is found
 * by Newton's method on a tail probability, so that the residual keeps its
 * relative precision far out in the tails:
 *   p <  1/2: solve  L(x) = p      with L(x) = erfc(-x / sqrt 2) / 2, x < 0;
 *   p >= 1/2: solve  U(x) = 1 - p  with U(x) = erfc( x / sqrt 2) / 2, x >= 0
 * (1 - p is exact for a double p >= 1/2).  Both tails are convex and monotone
 * on their side of 0, so Newton started at 0 approaches the root from the side
 * of 0 without overshooting.  Long double keeps the residual well below one
 * fp64 ulp of the result.
 * ------------------------------------------------------------------------- */
static long double phi_pdf(long double x) {
    const long double two_pi = 6.283185307179586476925286766559L;
    return expl(-0.5L * x * x) / sqrtl(two_pi);
}

double orc_norm_ppf(double p) {
    if (!(p > 0.0 && p < 1.0)) return NAN;
    const long double r2 = sqrtl(2.0L);
    const int upper = (p >= 0.5);
    const long double target = upper ? (1.0L - (long double)p) : (long double)p;
    long double x = 0.0L;
    for (int it = 0; it < 400; ++it) {
        long double step;
        if (upper) /* U' = -pdf: x <- x + (U(x) - target) / pdf(x) */
            step = -(0.5L * erfcl(x / r2) - target) / phi_pdf(x);
        else       /* L' = +pdf: x <- x - (L(x) - target) / pdf(x) */
            step = (0.5L * erfcl(-x / r2) - target) / phi_pdf(x);
        x -= step;
        if (fabsl(step) <= 1e-19L * (1.0L + fabsl(x))) break;
    }
    return (double)x;
}

/* ---------------------------------------------------------------------------
 * The 16 NF4 levels.
 * [P5] §2.2 ① and [P1] "NF4 不是一般四位元浮點格式": 16 levels taken from N(0,1)
 * quantiles so that each level carries equal probability mass, normalised to
 * [-1, 1].  The pages also require an exact zero, which 16 symmetric levels
 * cannot have, so the levels are built asymmetrically: 8 positive quantiles at
 * probabilities evenly spaced from delta down towards 1/2 (1/2 excluded), 7
 * negative ones likewise, and 0.  delta = ((1 - 1/30) + (1 - 1/32)) / 2 is the
 * outermost probability; the pages do not print it (external constant).
 * Computed in fp64, divided by the largest level so the ends are exactly +-1,
 * then rounded to fp32.
 * ------------------------------------------------------------------------- */
static int cmp_double(const void* a, const void* b) {
    double x = *(const double*)a, y = *(const double*)b;
    return (x > y) - (x < y);
}

void orc_codebook(float c[16]) {
    const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
    double v[16];
    int k = 0;
    for (int i = 0; i < 8; ++i) v[k++] = orc_norm_ppf(delta - i * (delta - 0.5) / 8.0);
    for (int i = 0; i < 7; ++i) v[k++] = -orc_norm_ppf(delta - i * (delta - 0.5) / 7.0);
    v[k++] = 0.0;
    qsort(v, 16, sizeof(double), cmp_double);
    const double top = v[15];
    for (int i = 0; i < 16; ++i) c[i] = (float)(v[i] / top);
}

static const float* codebook(void) {
    static float c[16];
    static int ready = 0;
    if (!ready) {
        orc_codebook(c);
        ready = 1;
    }
    return c;
}

/* ---------------------------------------------------------------------------
 * The FP4 codebook.  [P5] §2.2 code walk: bitsandbytes' FP4 is its generic
 * float-format builder instantiated with a sign bit, 2 exponent bits and 1
 * mantissa bit; [P3] "4-bit 量化": FP4 is a conventional 4-bit float; [P1] "NF4 不是
 * 一般四位元浮點格式": NF4 is not that IEEE-style FP4.  Reading: the code's bits
 * are s | e1 e0 | m with exponent bias 1; e = 0 is subnormal with magnitude m/2,
 * otherwise the magnitude is (1 + m/2) * 2^(e-1).  The 16 values are divided by
 * the largest magnitude in fp64 and rounded to fp32, so that, like the NF4
 * levels, they span [-1, 1].  The table is in code order (not sorted): codes
 * 0..7 are the non-negative values, 8..15 their negatives, code 8 is -0.
 * ------------------------------------------------------------------------- */
void orc_fp4_codebook(float c[16]) {
    double v[16];
    double top = 0.0;
    for (int code = 0; code < 16; ++code) {
        const int s = code >> 3, e = (code >> 1) & 3, m = code & 1;
        const double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
        v[code] = s ? -mag : mag;
        if (mag > top) top = mag;
    }
    for (int i = 0; i < 16; ++i) c[i] = (float)(v[i] / top);
}

static const float* fp4_codebook(void) {
    static float c[16];
    static int ready = 0;
    if (!ready) {
        orc_fp4_codebook(c);
        ready = 1;
    }
    return c;
}

static const float* table_of(int qt) { return qt == ORC_FP4 ? fp4_codebook() : codebook(); }

/* ---------------------------------------------------------------------------
 * Quantization ([P5] §2.2 example and Figure 2-2, steps 1-4):
 *   split the flattened weight into blocks of 64, absmax per block,
 *   x = w / absmax, map x to the nearest level, pack two 4-bit indices per byte.
 * ------------------------------------------------------------------------- */

/* Nearest level by exhaustive search over the 16 levels of table c, ties to the
 * lower index (for FP4, whose table is in code order, that sends a tie between
 * two magnitudes toward zero and every x of either sign nearest to zero to code
 * 0, +0).  Distances are taken in fp64: x and c_i are fp32 in [-1, 1], so every
 * comparison that is close enough to tie involves operands of similar magnitude
 * whose fp64 difference is exact. */
static int nearest_level(const float* c, float x) {
    int best = 0;
    double best_d = fabs((double)x - (double)c[0]);
    for (int i = 1; i < 16; ++i) {
        double d = fabs((double)x - (double)c[i]);
        if (d < best_d) {
            best_d = d;
            best = i;
        }
    }
    return best;
}

int orc_quantize_f32_qt(const float* w, int64_t n_elem, int qt, uint8_t* wq, float* absmax) {
    if (qt != ORC_NF4 && qt != ORC_FP4) return -4;
    if (n_elem <= 0 || n_elem % 64 != 0) return -2;
    const float* c = table_of(qt);
    const int64_t nb = n_elem / 64;
    for (int64_t b = 0; b < nb; ++b) {
        const float* blk = w + b * 64;
        float am = 0.0f;
        for (int j = 0; j < 64; ++j) {
            if (!isfinite(blk[j])) return -9;
            float a = fabsf(blk[j]);
            if (a > am) am = a;
        }
        absmax[b] = am;
        int idx[64];
        for (int j = 0; j < 64; ++j) {
            if (am == 0.0f) {
                /* zero block: every element is the exact-zero level (FP4: +0) */
                if (qt == ORC_FP4) idx[j] = 0;
                else idx[j] = 7;
            } else {
                float x = blk[j] / am;
                idx[j] = nearest_level(c, x);
            }
        }
        for (int i = 0; i < 32; ++i)
            wq[b * 32 + i] = (uint8_t)((idx[2 * i] << 4) | idx[2 * i + 1]);
    }
    return 0;
}

static float bf16_bits_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

int orc_quantize_bf16_qt(const uint16_t* w, int64_t n_elem, int qt, uint8_t* wq, float* absmax) {
    if (n_elem <= 0 || n_elem % 64 != 0) return -2;
    float tmp[64];
    for (int64_t b = 0; b < n_elem / 64; ++b) {
        for (int j = 0; j < 64; ++j) tmp[j] = bf16_bits_to_f32(w[b * 64 + j]);
        int rc = orc_quantize_f32_qt(tmp, 64, qt, wq + b * 32, absmax + b);
        if (rc) return rc;
    }
    return 0;
}

int orc_quantize_f32(const float* w, int64_t n_elem, uint8_t* wq, float* absmax) {
    return orc_quantize_f32_qt(w, n_elem, ORC_NF4, wq, absmax);
}

int orc_quantize_bf16(const uint16_t* w, int64_t n_elem, uint8_t* wq, float* absmax) {
    return orc_quantize_bf16_qt(w, n_elem, ORC_NF4, wq, absmax);
}

/* ---------------------------------------------------------------------------
 * Double quantization ([P5] §2.2 ② and Figure 2-2 step 5; [P1] "Double
 * quantization 連 scale 本身也壓縮"; [P3] "分页优化器与双量化").  The absmax values
 * are themselves quantized to 8 bits in blocks of 256 after subtracting their
 * mean.
 *
 * The mean's summation order is part of the definition, so that every
 * implementation rounds alike.  S is built in levels: the current list is cut
 * into chunks of 256 (the last chunk padded with zeros), each chunk is reduced
 * by the halving tree a[i] += a[i + h] for h = 128, 64, ..., 1, and the chunk
 * results form the next list, until one value remains.  The first level's
 * chunks are exactly the double-quantization blocks.
 * ------------------------------------------------------------------------- */
static double tree256(const double* v, int64_t count) {
    double a[256];
    for (int i = 0; i < 256; ++i) a[i] = (i < count) ? v[i] : 0.0;
    for (int h = 128; h >= 1; h >>= 1)
        for (int i = 0; i < h; ++i) a[i] = a[i] + a[i + h];
    return a[0];
}

double orc_dq_sum(const float* absmax, int64_t nb) {
    if (nb <= 0) return 0.0;
    double* cur = (double*)malloc(sizeof(double) * (size_t)nb);
    for (int64_t i = 0; i < nb; ++i) cur[i] = (double)absmax[i];
    int64_t n = nb;
    do {
        int64_t m = (n + 255) / 256;
        double* nxt = (double*)malloc(sizeof(double) * (size_t)m);
        for (int64_t j = 0; j < m; ++j) {
            int64_t cnt = n - j * 256;
            if (cnt > 256) cnt = 256;
            nxt[j] = tree256(cur + j * 256, cnt);
        }
        free(cur);
        cur = nxt;
        n = m;
    } while (n > 1);
    double s = cur[0];
    free(cur);
    return s;
}

float orc_dq_mean(const float* absmax, int64_t nb) {
    return (float)(orc_dq_sum(absmax, nb) / (double)nb);
}

int orc_double_quant(const float* absmax, int64_t nb, int8_t* absmax_q, float* absmax_scale,
                     float* mu_out) {
    if (nb <= 0) return -2;
    const float mu = orc_dq_mean(absmax, nb);
    const int64_t nb2 = (nb + 255) / 256;
    for (int64_t j = 0; j < nb2; ++j) {
        const int64_t lo = j * 256;
        const int64_t hi = (lo + 256 < nb) ? lo + 256 : nb;
        float s = 0.0f;
        for (int64_t b = lo; b < hi; ++b) {
            float r = absmax[b] - mu;
            float a = fabsf(r);
            if (a > s) s = a;
        }
        absmax_scale[j] = s;
        for (int64_t b = lo; b < hi; ++b) {
            float r = absmax[b] - mu;
            int q = 0;
            if (s != 0.0f) {
                float t = r / s;
                float u = t * 127.0f;
                q = (int)nearbyintf(u); /* default rounding mode: nearest, ties to even */
            }
            absmax_q[b] = (int8_t)q;
        }
    }
    *mu_out = mu;
    return 0;
}

/* Inverse of the double quantization, step by step in fp32. */
float orc_absmax_hat(const int8_t* absmax_q, const float* absmax_scale, float mu, int64_t b) {
    float t = (float)absmax_q[b] / 127.0f;
    float u = t * absmax_scale[b / 256];
    return u + mu;
}

/* ---------------------------------------------------------------------------
 * Dequantization ([P4] §5 "動態反量化": the 4-bit weights are turned back into the
 * compute dtype layer by layer; [P1] "QLoRA 把 frozen 4-bit base ...": the base
 * is dequantized in forward and backward):  w = fp32(c[idx] * a).
 * ------------------------------------------------------------------------- */
int orc_dequantize_range_qt(const uint8_t* wq, const int8_t* absmax_q, const float* absmax_scale,
                            float mu, int64_t begin, int64_t count, int qt, float* out_f32) {
    if (qt != ORC_NF4 && qt != ORC_FP4) return -4;
    if (begin < 0 || count < 0 || begin % 64 != 0 || count % 64 != 0) return -2;
    const float* c = table_of(qt);
    for (int64_t e = 0; e < count; ++e) {
        const int64_t g = begin + e;
        const uint8_t byte = wq[g / 2];
        const int idx = (g % 2 == 0) ? (byte >> 4) : (byte & 15);
        const float a = orc_absmax_hat(absmax_q, absmax_scale, mu, g / 64);
        out_f32[e] = c[idx] * a;
    }
    return 0;
}

int orc_dequantize_range(const uint8_t* wq, const int8_t* absmax_q, const float* absmax_scale,
                         float mu, int64_t begin, int64_t count, float* out_f32) {
    return orc_dequantize_range_qt(wq, absmax_q, absmax_scale, mu, begin, count, ORC_NF4, out_f32);
}

/* Round to nearest bf16, ties to even: keep the top 16 bits after adding half an
 * ulp of the kept part, biased by the kept part's lowest bit so that exact
 * halves go to the even neighbour.  Pinned by [P4] "精度 (Precision)": fp32(2.3)
 * becomes bf16 2.296875. */
void orc_f32_to_bf16(const float* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) {
        uint32_t u;
        memcpy(&u, &x[i], sizeof u);
        uint32_t lsb = (u >> 16) & 1u;
        u += 0x7FFFu + lsb;
        out[i] = (uint16_t)(u >> 16);
    }
}

/* The linear Y = X W^T ([P5] §2.2 code walk: matmul_4bit(x, weight, ...) is a
 * dequantize followed by a matmul) in fp64 on the bf16 values that the compute
 * dtype feeds the matmul ([P4] §5: weights are restored to BF16 before the
 * matrix multiply).  Every bf16 x bf16 product is exact in fp64; the sum runs
 * over k in order. */
void orc_lora_delta(const uint16_t* up, const uint16_t* down, int64_t n, int64_t r, int64_t k, float* delta) {
    for (int64_t o = 0; o < n; ++o)
        for (int64_t c = 0; c < k; ++c) {
            float acc = 0.0f;
            for (int64_t j = 0; j < r; ++j)
                acc = fmaf(bf16_bits_to_f32(up[o * r + j]), bf16_bits_to_f32(down[j * k + c]), acc);
            delta[o * k + c] = acc;
        }
}

void orc_linear_bf16(const uint16_t* x, int64_t m, const uint16_t* w, int64_t n, int64_t k,
                     double* y) {
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int64_t t = 0; t < k; ++t)
                acc += (double)bf16_bits_to_f32(x[i * k + t]) * (double)bf16_bits_to_f32(w[j * k + t]);
            y[i * n + j] = acc;
        }
}
