// nf4_lora.cu -- the down-projection of a LoRA layer, t = scale * X down^T.
//
// Source: page "LLM 相關知識" (technicalnotes), section "2-2. LoRA（低秩適應）": the
// frozen W acts as W + dW with dW = A x B of low rank r, trained in bf16; with W
// stored [n, k] that is dW = up [n, r] * down [r, k], so
//   Y = X What^T + scale * (X down^T) up^T.
// This kernel computes t = scale * X down^T [m, r] in fp32; the linear kernels add
// t up^T in their epilogue.  One block per (token, 8 ranks), one warp per rank;
// each lane sums a fixed subset of k into four partial sums combined in a fixed
// order, and the warp adds the lanes in a fixed tree, so the result never
// depends on scheduling.
#include <cuda_bf16.h>

#include "nf4_common.cuh"
#include "nf4_internal.h"

namespace nf4 {
namespace lora {

__global__ void __launch_bounds__(256) k_lora_down(const __nv_bfloat16* __restrict__ X, int64_t k,
                                                   const __nv_bfloat16* __restrict__ down, int r, float scale,
                                                   float* __restrict__ t, __nv_bfloat16* __restrict__ t_hi,
                                                   __nv_bfloat16* __restrict__ t_lo) {
    // block (token, group of 8 ranks); warp w computes rank 8 * blockIdx.y + w
    const int64_t tok = blockIdx.x;
    const int j = static_cast<int>(blockIdx.y) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (j >= r) return;
    const __nv_bfloat16* x = X + tok * k;
    const __nv_bfloat16* d = down + static_cast<int64_t>(j) * k;
    // lane l sums the 8-element chunks l, l + 32, l + 64, ...; chunk i goes to
    // accumulator i mod 4 (four loads in flight), combined in a fixed order
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const int64_t nch = k / 8;
    for (int64_t base = lane; base < nch; base += 128) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t ch = base + 32 * q;
            if (ch < nch) {
                const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + ch * 8));
                const uint4 dv = __ldg(reinterpret_cast<const uint4*>(d + ch * 8));
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc[q] = __fmaf_rn(bf16_bits_to_float(xw[e] & 0xffffu), bf16_bits_to_float(dw[e] & 0xffffu), acc[q]);
                    acc[q] = __fmaf_rn(bf16_bits_to_float(xw[e] >> 16), bf16_bits_to_float(dw[e] >> 16), acc[q]);
                }
            }
        }
    }
    float v = __fadd_rn(__fadd_rn(acc[0], acc[1]), __fadd_rn(acc[2], acc[3]));
#pragma unroll
    for (int h = 16; h >= 1; h >>= 1) v = __fadd_rn(v, __shfl_xor_sync(kFull, v, h));
    if (lane == 0) {
        const float tv = __fmul_rn(v, scale);
        t[tok * r + j] = tv;
        if (t_hi) {
            const __nv_bfloat16 h = __float2bfloat16_rn(tv);
            t_hi[tok * r + j] = h;
            t_lo[tok * r + j] = __float2bfloat16_rn(__fsub_rn(tv, __bfloat162float(h)));
        }
    }
}

}  // namespace lora

cudaError_t launch_lora_down(const void* X, int64_t m, int64_t k, const void* down, int r, float scale, float* t,
                             __nv_bfloat16* t_hi, __nv_bfloat16* t_lo, cudaStream_t stream) {
    const dim3 grid(static_cast<unsigned>(m), static_cast<unsigned>((r + 7) / 8));
    lora::k_lora_down<<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(X), k,
                                                                      static_cast<const __nv_bfloat16*>(down), r,
                                                                      scale, t, t_hi, t_lo);
    return cudaGetLastError();
}

}  // namespace nf4
