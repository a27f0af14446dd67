// nf4_gemv.cu -- fused dequantize + linear for decode-sized batches (m <= 16), sm_100a.
//
// Sources: page "篇2-bitsandbytes-具体观-算法与实现剖析" (xyzblog), §2.2 code walk
// (matmul_4bit = dequantize + matmul); page "LLM 相關知識" (technicalnotes), §5
// "動態反量化" (weights restored to BF16 per layer for the matmul, then dropped);
// page "Tim Dettmers 如何用 bitsandbytes 與 QLoRA 降低 LLM 訓練門檻？", section "量化速度
// 取決於硬體與 kernel，不只位元數" (unfused 4-bit can lose to fp16; batch size moves the
// work between memory- and compute-bound).
//
// Y[t, r] = sum_c X[t, c] * What[r, c],  What[r, c] = bf16(fp32(level[idx] * a_block)).
//
// The multiply-adds run on the tensor cores (mma.sync m16n8k16, bf16 in, fp32
// accumulate) with the tokens as the MMA's M side (zero-padded to 16) and eight
// weight rows as its N side, so the CUDA cores only decode.  The k order inside
// each MMA is a permutation of the true k order (each lane takes 32 consecutive
// weights of one row), applied identically to X and the weights, so the dot
// products are unchanged.  Decode: one 256-entry table maps a packed byte to
// the two fp32 levels it encodes; each level is multiplied by the block's
// reconstructed absmax in fp32 and rounded to bf16, exactly as nf4_dequantize
// does.
#include "nf4_common.cuh"
#include "nf4_internal.h"

namespace nf4 {

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void load_x32(const __nv_bfloat16* __restrict__ row, int64_t c0, bool ok,
                                         uint32_t (&w)[16]) {
    if (ok) {
        const uint4* p = reinterpret_cast<const uint4*>(row + c0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 v = __ldg(p + q);
            w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int q = 0; q < 16; ++q) w[q] = 0u;
    }
}

// One warp computes an 8-row x 16-token tile of Y^T over all of k.
// Lane (g = lane / 4, i = lane % 4): weight row r0 + g, tokens g and g + 8,
// and within each 128-wide span of k the 32 columns [32 i, 32 i + 32).
template <bool kBf16Out>
__global__ void __launch_bounds__(128) k_nf4_gemv_simple(
    const __nv_bfloat16* __restrict__ X, int m, int64_t k, const uint8_t* __restrict__ wq,
    const int8_t* __restrict__ absmax_q, const float* __restrict__ absmax_scale,
    const float* __restrict__ mu_ptr, int64_t n, void* __restrict__ Y) {
    __shared__ float2 lut[256];  // byte -> (level of its high nibble, level of its low nibble)
    for (int e = threadIdx.x; e < 256; e += blockDim.x)
        lut[e] = make_float2(kLevels[e >> 4], kLevels[e & 15]);
    __syncthreads();

    const float mu = __ldg(mu_ptr);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int g = lane >> 2;
    const int i = lane & 3;
    const int64_t row0 = (static_cast<int64_t>(blockIdx.x) * 4 + warp) * 8;
    if (row0 >= n) return;
    const int64_t row = (row0 + g < n) ? row0 + g : n - 1;  // clamped; its outputs are not stored
    const uint8_t* wrow = wq + row * (k / 2);
    const int64_t blk_row = row * (k / 64);
    const bool tok_lo = g < m;
    const bool tok_hi = g + 8 < m;
    const __nv_bfloat16* x_lo = X + static_cast<int64_t>(tok_lo ? g : 0) * k;
    const __nv_bfloat16* x_hi = X + static_cast<int64_t>(tok_hi ? g + 8 : 0) * k;

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int64_t n_spans = (k + 127) / 128;
    for (int64_t sp = 0; sp < n_spans; ++sp) {
        const int64_t c0 = sp * 128 + 32 * i;  // first column of this lane's run
        const bool ok = c0 < k;                 // k % 64 == 0: a run is all in or all out
        uint4 raw = make_uint4(0u, 0u, 0u, 0u);
        float a = 0.0f;
        if (ok) {
            raw = __ldcs(reinterpret_cast<const uint4*>(wrow + c0 / 2));
            const int64_t b = blk_row + c0 / 64;
            a = absmax_hat(__ldg(absmax_q + b), __ldg(absmax_scale + (b >> 8)), mu);
        }
        uint32_t xl[16], xh[16];
        load_x32(x_lo, c0, ok && tok_lo, xl);
        load_x32(x_hi, c0, ok && tok_hi, xh);
        const uint32_t r[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const uint32_t word = r[s >> 1] >> (16 * (s & 1));
            const float2 p0 = lut[word & 0xffu];           // columns c0+4s, c0+4s+1
            const float2 p1 = lut[(word >> 8) & 0xffu];    // columns c0+4s+2, c0+4s+3
            const uint32_t b0 = pack_bf16x2(__fmul_rn(p0.x, a), __fmul_rn(p0.y, a));
            const uint32_t b1 = pack_bf16x2(__fmul_rn(p1.x, a), __fmul_rn(p1.y, a));
            mma_bf16_16816(acc, xl[2 * s], xh[2 * s], xl[2 * s + 1], xh[2 * s + 1], b0, b1);
        }
    }
    // acc[0..1] = Y[g][row0 + 2i + {0,1}], acc[2..3] = Y[g + 8][row0 + 2i + {0,1}]
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int t = g + 8 * h;
        if (t >= m) continue;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int64_t r = row0 + 2 * i + e;
            if (r >= n) continue;
            const float v = acc[2 * h + e];
            if (kBf16Out)
                reinterpret_cast<__nv_bfloat16*>(Y)[static_cast<int64_t>(t) * n + r] = __float2bfloat16_rn(v);
            else
                reinterpret_cast<float*>(Y)[static_cast<int64_t>(t) * n + r] = v;
        }
    }
}

cudaError_t launch_linear(const void* X, int64_t m, const uint8_t* wq, const int8_t* absmax_q,
                          const float* absmax_scale, const float* absmax_offset, int64_t n,
                          int64_t k, void* Y, bool y_bf16, int32_t* dev_status,
                          const DeviceInfo& dev, cudaStream_t stream) {
    (void)dev_status;
    (void)dev;
    const __nv_bfloat16* Xb = static_cast<const __nv_bfloat16*>(X);
    const unsigned blocks = static_cast<unsigned>((n + 31) / 32);
    const size_t ybytes = y_bf16 ? 2 : 4;
    for (int64_t t0 = 0; t0 < m; t0 += 16) {
        const int mt = static_cast<int>((m - t0) < 16 ? (m - t0) : 16);
        void* Yt = static_cast<char*>(Y) + static_cast<size_t>(t0) * n * ybytes;
        if (y_bf16)
            k_nf4_gemv_simple<true><<<blocks, 128, 0, stream>>>(Xb + t0 * k, mt, k, wq, absmax_q,
                                                                absmax_scale, absmax_offset, n, Yt);
        else
            k_nf4_gemv_simple<false><<<blocks, 128, 0, stream>>>(Xb + t0 * k, mt, k, wq, absmax_q,
                                                                 absmax_scale, absmax_offset, n, Yt);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace nf4
