/*
 * nf4_oracle.h -- CPU oracle for the NF4 + double-quantization weight path.
 *
 * TEST INFRASTRUCTURE ONLY.  This library is a plain, slow, single-threaded
 * restatement of what the pages define; it exists so that the CUDA library can
 * be checked against something written independently of it.  Only the test
 * suite, the smoke check and the CPU-baseline leg of the benchmark may load it.
 * It shares no code, header, table or constant generator with the CUDA library.
 *
 * Sources (web pages, cited by title and section):
 *   [P1] "Tim Dettmers 如何用 bitsandbytes 與 QLoRA 降低 LLM 訓練門檻？" (yololab.net):
 *        sections "NF4 不是一般四位元浮點格式", "Double quantization 連 scale 本身也壓縮",
 *        "QLoRA 把 frozen 4-bit base 與可訓練 adapter 分開".
 *   [P3] "bitsandbytes：让大语言模型在消费级硬件上运行的量化神器" (zingnex.cn):
 *        sections "4-bit 量化（QLoRA 基础）", "分页优化器与双量化".
 *   [P4] "LLM 相關知識" (technicalnotes, tag qlora): section "精度 (Precision)" (the 2.3
 *        rounding table) and section "5. 動態反量化（Dynamic Dequantization）".
 *   [P5] "篇2-bitsandbytes-具体观-算法与实现剖析" (xyzblog): section 2.2 "QLoRA / NF4"
 *        (principle, code walk, worked example) and Figure 2-2 (NF4 + double
 *        quantization data pipeline).
 *
 * Conventions fixed here where the pages are silent (each one is a stated reading):
 *   - blocks of 64 consecutive elements of the flattened row-major weight; one fp32
 *     absmax per block ([P5] §2.2 example; fp32 because "4 bit + 0.5 bit absmax"
 *     means 32 bits per 64 weights);
 *   - x = w / absmax in IEEE fp32 (round to nearest even); a zero block maps to
 *     index 7 (the exact zero level);
 *   - index = argmin_i |x - c_i| evaluated exactly, ties to the lower index;
 *   - packing: element 2i in the high nibble of byte i, element 2i+1 in the low nibble;
 *   - double quantization: mu = fp32(S / nb) with S the fixed-order fp64 tree sum
 *     defined by orc_dq_sum; r = fp32(absmax - mu); per block of 256: s = max|r|,
 *     q = round_half_even(fp32(fp32(r / s) * 127)), q = 0 when s = 0;
 *   - absmax dequant: a = fp32(fp32(fp32(q / 127) * s) + mu), each step rounded;
 *   - weight dequant: w = fp32(c[idx] * a); the bf16 form rounds that to nearest even;
 *   - FP4 (the *_qt functions): the same pipeline with the 16 values of a sign,
 *     2-bit exponent (bias 1, subnormal at 0) and 1-bit mantissa float, in code
 *     order, scaled to [-1, 1]; a zero block maps to code 0 (+0).
 *
 * Every floating-point step is an IEEE binary32/binary64 operation with
 * round-to-nearest-even; the library is built with -ffp-contract=off and without
 * fast-math so that no step is fused or reordered.
 */
#ifndef NF4_ORACLE_H
#define NF4_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Inverse standard-normal CDF, Phi^-1(p), 0 < p < 1, by Newton's method on
 * Phi(x) = erfc(-x/sqrt(2))/2 carried out in long double. */
double orc_norm_ppf(double p);

/* The 16 NF4 levels, ascending, in fp32: c[0] = -1, c[7] = 0, c[15] = +1. */
void orc_codebook(float c[16]);

/* Codebook selector of the *_qt functions. */
#define ORC_NF4 0
#define ORC_FP4 1

/* The 16 FP4 values in code order (sign | 2 exponent bits, bias 1 | 1 mantissa
 * bit, subnormal at exponent 0), divided by the largest magnitude: codes 0..7 =
 * 0, 1/12, 1/6, 1/4, 1/3, 1/2, 2/3, 1 (fp32-rounded); codes 8..15 their
 * negatives (code 8 = -0). */
void orc_fp4_codebook(float c[16]);

/* Blockwise NF4 quantization of n_elem fp32 weights (n_elem % 64 == 0).
 * Writes wq[n_elem/2] packed codes and absmax[n_elem/64].  Returns 0, or -2 on a
 * bad size, -9 on a non-finite input. */
int orc_quantize_f32(const float* w, int64_t n_elem, uint8_t* wq, float* absmax);
/* Same, from bf16 bit patterns (widened exactly to fp32 first). */
int orc_quantize_bf16(const uint16_t* w, int64_t n_elem, uint8_t* wq, float* absmax);
/* The same with the codebook chosen by qt (ORC_NF4 or ORC_FP4; -4 otherwise).
 * A zero block is code 7 for NF4 and code 0 (+0) for FP4. */
int orc_quantize_f32_qt(const float* w, int64_t n_elem, int qt, uint8_t* wq, float* absmax);
int orc_quantize_bf16_qt(const uint16_t* w, int64_t n_elem, int qt, uint8_t* wq, float* absmax);

/* Fixed-order fp64 sum of the absmax values (the tree defined in the .c file). */
double orc_dq_sum(const float* absmax, int64_t nb);
/* mu = fp32(orc_dq_sum / nb). */
float orc_dq_mean(const float* absmax, int64_t nb);

/* Double quantization: absmax[nb] -> absmax_q[nb] (int8), absmax_scale[ceil(nb/256)],
 * *mu.  Returns 0 or -2 on nb <= 0. */
int orc_double_quant(const float* absmax, int64_t nb, int8_t* absmax_q,
                     float* absmax_scale, float* mu);

/* Reconstructed absmax of block b (global block index). */
float orc_absmax_hat(const int8_t* absmax_q, const float* absmax_scale, float mu, int64_t b);

/* Dequantize elements [begin, begin + count) of the flattened weight (begin and
 * count multiples of 64) into out_f32[count].  wq, absmax_q and absmax_scale are
 * the full arrays (global indexing). */
int orc_dequantize_range(const uint8_t* wq, const int8_t* absmax_q, const float* absmax_scale,
                         float mu, int64_t begin, int64_t count, float* out_f32);
/* The same with the codebook chosen by qt. */
int orc_dequantize_range_qt(const uint8_t* wq, const int8_t* absmax_q, const float* absmax_scale,
                            float mu, int64_t begin, int64_t count, int qt, float* out_f32);

/* fp32 -> bf16 bit pattern, round to nearest, ties to even (finite inputs). */
void orc_f32_to_bf16(const float* x, int64_t n, uint16_t* out);

/* y[m][n] = sum_k x[m][k] * w[n][k] in fp64, x and w given as bf16 bit patterns,
 * x [m,k] and w [n,k] row-major, y [m,n] row-major. */
/* LoRA merge delta ("LLM 相關知識", section "8. LoRA 的合併（Merge）": W_new = W + A x B
 * in BF16 after dequantizing): delta[o][c] = sum_j up[o][j] * down[j][c] as an fp32
 * fused multiply-add chain in j order starting from +0 (fmaf, one rounding per
 * step).  up bf16 [n, r], down bf16 [r, k] as bit patterns -> delta fp32 [n, k]. */
void orc_lora_delta(const uint16_t* up, const uint16_t* down, int64_t n, int64_t r, int64_t k, float* delta);

void orc_linear_bf16(const uint16_t* x, int64_t m, const uint16_t* w, int64_t n, int64_t k,
                     double* y);

#ifdef __cplusplus
}
#endif
#endif /* NF4_ORACLE_H */
