// nf4_encode.cuh -- the division-free code decision of the quantize kernel: the
// Markstein-corrected quotient, the NF4 bucket table and packed fp32 pairs.
//
// Sources: page "篇2-bitsandbytes-具体观-算法与实现剖析" (xyzblog), §2.2 (normalise
// by the block's absmax, nearest of the 16 levels); page "Tim Dettmers 如何用
// bitsandbytes 與 QLoRA 降低 LLM 訓練門檻？", section "NF4 不是一般四位元浮點格式".
#pragma once

#include <stdint.h>

#include "nf4_common.cuh"

namespace nf4 {

// The code of each element without a division and without a search.
//
// Quotient: q = RN(w / a) by Markstein's correction of a product with the
// correctly rounded reciprocal (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990): with r = RN(1 / a), q0 = RN(w r), e = w - a q0 (exact, one FMA) and
// q = RN(q0 + e r) is the IEEE quotient when nothing leaves the normal range.
// It is used for blocks whose absmax lies in [2^-60, 2^60]; for them every
// quotient that can reach a threshold (|q| >= 2^-8, far inside the band that
// maps to the zero level) keeps e exact.  Other blocks (zero, tiny, huge or
// non-finite absmax) divide.
//
// NF4 code of q in [-1, 1]: bucket b = round_half_even(128 q + 128) (one FMA
// onto the mantissa of 1.5 * 2^23) of a 257-entry table; at most one threshold
// falls in the closed q range of a bucket (NF4 thresholds are more than 1/128
// apart), so idx = base[b] + (q > thr[b]) with base[b] = #{j : t_j below the
// bucket}.  The table lives in shared memory, 16 copies so the 16 lanes of a
// half-warp never share a bank.
constexpr int kBuckets = 257;
constexpr int kTabCopies = 16;
constexpr float kBucketMagic = 12582912.0f + 128.0f;  // 1.5 * 2^23 + 128

__device__ __forceinline__ float quotient(float w, float a, float r) {
    const float q0 = __fmul_rn(w, r);
    const float e = __fmaf_rn(-q0, a, w);
    return __fmaf_rn(e, r, q0);
}

// Packed fp32 pairs: each half is rounded exactly as the scalar operation.
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ bool markstein_ok(float a) {
    return a >= 0x1p-60f && a <= 0x1p60f;  // false for 0, NaN and +inf too
}

// Fills tab[kBuckets * kTabCopies] for the NF4 codebook: each bucket's entry
// {threshold bits (+inf when none falls in the bucket), levels below} is formed
// once, into its first copy, then copied.  Called by every thread of the block;
// ends with a block barrier.
__device__ __forceinline__ void build_bucket_table(uint2* tab) {
    for (int b = threadIdx.x; b < kBuckets; b += blockDim.x) {
        const float lo = (static_cast<float>(b) - 0.5f) / 128.0f - 1.0f;
        const float hi = (static_cast<float>(b) + 0.5f) / 128.0f - 1.0f;
        uint32_t base = 0;
        float thr = __int_as_float(0x7f800000);
#pragma unroll
        for (int j = 0; j < 15; ++j) {
            const float t = kThresh[j];
            if (t < lo) ++base;
            else if (t <= hi) thr = t;
        }
        tab[b * kTabCopies] = make_uint2(__float_as_uint(thr), base);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kBuckets * kTabCopies; e += blockDim.x)
        if (e % kTabCopies != 0) tab[e] = tab[e - e % kTabCopies];
    __syncthreads();
}

// NF4 code of a quotient q in [-1, 1] from the bucket table (copy `cp` of 16).
__device__ __forceinline__ uint32_t bucket_code(float q, const uint2* tab, int cp) {
    const uint32_t b = __float_as_uint(__fmaf_rn(q, 128.0f, kBucketMagic)) & 0x1ffu;
    const uint2 ent = tab[b * kTabCopies + cp];
    return ent.y + (q > __uint_as_float(ent.x) ? 1u : 0u);
}

}  // namespace nf4
