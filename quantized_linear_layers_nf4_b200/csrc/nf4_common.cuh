// nf4_common.cuh -- device-side constants and helpers shared by the NF4 kernels.
//
// Sources (web pages, cited by title and section):
//   [P1] "Tim Dettmers 如何用 bitsandbytes 與 QLoRA 降低 LLM 訓練門檻？" (yololab.net)
//   [P4] "LLM 相關知識" (technicalnotes, tag qlora)
//   [P5] "篇2-bitsandbytes-具体观-算法与实现剖析" (xyzblog)
//
// Every rounding step below is an explicit IEEE operation with round-to-nearest-
// even (__fdiv_rn, __fmul_rn, __fadd_rn, __fsub_rn) so that the compiler cannot
// contract or reorder it; the library is built without fast-math.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nf4_levels.h"

namespace nf4 {

constexpr int kBlock = 64;     // weights per absmax ([P5] §2.2 worked example)
constexpr int kBlock2 = 256;   // absmax values per double-quantization block
constexpr unsigned kFull = 0xffffffffu;

// The 16 levels and 15 decision thresholds ([P5] §2.2 principle ①).
static __constant__ float kLevels[16] = NF4_LEVELS_INIT;
static __constant__ float kThresh[15] = NF4_THRESHOLDS_INIT;

// Codebook ids: the weight's 4-bit codes index the NF4 levels or the FP4 values
// ([P5] §2.2 code walk: quant_type "nf4" or "fp4", the latter the generic float
// format with a sign, 2 exponent bits and 1 mantissa bit).  Same storage, same
// pipeline; only the table and the encoder differ.
constexpr int kCbNf4 = 0;
constexpr int kCbFp4 = 1;
static __constant__ float kCodebook[2][16] = {NF4_LEVELS_INIT, FP4_LEVELS_INIT};

// Thresholds as compile-time values, so that the encoder's comparisons use
// immediates and never index memory per element.
struct Thr {
    static constexpr float t[15] = NF4_THRESHOLDS_INIT;
};

// Nearest level of x in [-1, 1], ties to the lower index: idx = #{j : x > t_j},
// found by a four-step binary search over the sorted thresholds.
__device__ __forceinline__ int encode_nf4(float x) {
    constexpr float T0 = Thr::t[0], T1 = Thr::t[1], T2 = Thr::t[2], T3 = Thr::t[3];
    constexpr float T4 = Thr::t[4], T5 = Thr::t[5], T6 = Thr::t[6], T7 = Thr::t[7];
    constexpr float T8 = Thr::t[8], T9 = Thr::t[9], T10 = Thr::t[10], T11 = Thr::t[11];
    constexpr float T12 = Thr::t[12], T13 = Thr::t[13], T14 = Thr::t[14];
    const bool b3 = x > T7;
    const bool b2 = x > (b3 ? T11 : T3);
    const float t1 = b3 ? (b2 ? T13 : T9) : (b2 ? T5 : T1);
    const bool b1 = x > t1;
    float t0;
    if (b3) t0 = b2 ? (b1 ? T14 : T12) : (b1 ? T10 : T8);
    else    t0 = b2 ? (b1 ? T6 : T4) : (b1 ? T2 : T0);
    const bool b0 = x > t0;
    return (b3 ? 8 : 0) | (b2 ? 4 : 0) | (b1 ? 2 : 0) | (b0 ? 1 : 0);
}

// Level index of weight w in a block whose absmax is a ([P5] §2.2 example:
// W_norm = W / absmax, then the nearest level).  A zero block maps to the exact
// zero level.
__device__ __forceinline__ int quantize_one(float w, float a) {
    if (a == 0.0f) return 7;
    return encode_nf4(__fdiv_rn(w, a));
}

struct Fp4Thr {
    static constexpr float t[7] = FP4_THRESHOLDS_INIT;
};

// FP4 code of x in [-1, 1]: the magnitude index #{j : |x| > u_j} over the 7
// round-down midpoints of the magnitudes (three-step binary search), with the
// sign bit set for negative x, except that a zero magnitude is always code 0
// (+0).  This is the nearest FP4 value with ties going to the lower code (toward
// zero); code 8 (-0) is never produced.
__device__ __forceinline__ int encode_fp4(float x) {
    constexpr float U0 = Fp4Thr::t[0], U1 = Fp4Thr::t[1], U2 = Fp4Thr::t[2], U3 = Fp4Thr::t[3];
    constexpr float U4 = Fp4Thr::t[4], U5 = Fp4Thr::t[5], U6 = Fp4Thr::t[6];
    const float a = fabsf(x);
    const bool b2 = a > U3;
    const bool b1 = a > (b2 ? U5 : U1);
    const float u0 = b2 ? (b1 ? U6 : U4) : (b1 ? U2 : U0);
    const bool b0 = a > u0;
    const int mag = (b2 ? 4 : 0) | (b1 ? 2 : 0) | (b0 ? 1 : 0);
    return (mag != 0 && x < 0.0f) ? (8 | mag) : mag;
}

// Code of weight w in a block with absmax a under codebook CB; a zero block is
// the exact-zero code (NF4 7, FP4 0).
template <int CB>
__device__ __forceinline__ int quantize_code(float w, float a) {
    if (CB == kCbFp4) {
        if (a == 0.0f) return 0;
        return encode_fp4(__fdiv_rn(w, a));
    }
    return quantize_one(w, a);
}

// fp32(q / 127), the correctly rounded quotient, for an int8 code q, without a
// division: one multiply by the rounded reciprocal and one residual
// correction (Markstein's method, IBM J. Res. Dev. 34(1), 1990): with
// r = q * RN(1/127) and e = q - 127 r (exact by FMA), r + e * RN(1/127) rounds
// to the IEEE quotient.  Checked exhaustively for all 256 codes (exact rational
// arithmetic, tests/test_div127.py) and bit-for-bit by every dequant parity test.
__device__ __forceinline__ float div127(float q) {
    constexpr float kInv = 1.0f / 127.0f;  // RN(1/127)
    const float r = __fmul_rn(q, kInv);
    const float e = __fmaf_rn(-r, 127.0f, q);
    return __fmaf_rn(e, kInv, r);
}

// Reconstructed absmax from its double-quantized code:
// a = fp32(fp32(fp32(q / 127) * s) + mu).
__device__ __forceinline__ float absmax_hat(int q, float s, float mu) {
    return __fadd_rn(__fmul_rn(div127(static_cast<float>(q)), s), mu);
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h16) {
    return __uint_as_float(h16 << 16);
}

// Packs two fp32 values into one bf16x2 word, each rounded to nearest even;
// `lo` lands in bits 0..15 (the lower address / lower k index).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

}  // namespace nf4
