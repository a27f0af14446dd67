// nf4_lora.cu -- the down-projection of a LoRA layer, t = scale * X down^T, and
// the merge of a trained update into the quantized weight (bottom of the file).
//
// Source: page "LLM 相關知識" (technicalnotes), section "2-2. LoRA（低秩適應）": the
// frozen W acts as W + dW with dW = A x B of low rank r, trained in bf16; with W
// stored [n, k] that is dW = up [n, r] * down [r, k], so
//   Y = X What^T + scale * (X down^T) up^T.
// The kernels here compute t = scale * X down^T [m, r] in fp32 ahead of the
// linear, which adds t up^T: k_lora_down for decode-sized m (used when the GEMV
// does not form t itself), k_lora_down_tc on the tensor cores for m > 16.  Both
// add in a fixed order, so the result never depends on scheduling.
#include <cuda_bf16.h>

#include "nf4_common.cuh"
#include "nf4_internal.h"
#include "nf4_ptx.cuh"

namespace nf4 {
namespace lora {

// t[tok, j] = scale * sum_c X[tok, c] * down[j, c] in fp32.  CTA (token, pair of
// ranks): warp w computes rank 2 * blockIdx.y + w / 4 over the k quarter w % 4;
// within a quarter lane l sums the 8-element chunks l, l + 32, ... into two
// accumulators (even and odd chunk rounds), and the quarters are added in
// order (q0 + q1) + (q2 + q3).  Under a programmatic dependent launch the next
// kernel (the dequant-GEMV, which prefetches its weights) may start at once;
// X may be the preceding kernel's output, so it is read after the wait.
__global__ void __launch_bounds__(256) k_lora_down(const __nv_bfloat16* __restrict__ X, int64_t k,
                                                   const __nv_bfloat16* __restrict__ down, int r, float scale,
                                                   float* __restrict__ t, __nv_bfloat16* __restrict__ t_hi,
                                                   __nv_bfloat16* __restrict__ t_lo) {
    __shared__ float part[2][4];
    grid_launch_dependents();
    grid_dependency_wait();
    const int64_t tok = blockIdx.x;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int j = static_cast<int>(blockIdx.y) * 2 + (warp >> 2);
    const int quarter = warp & 3;
    const int64_t nch = k / 8;
    const int64_t c0 = nch * quarter / 4, c1 = nch * (quarter + 1) / 4;
    float v = 0.0f;
    if (j < r) {
        const __nv_bfloat16* x = X + tok * k;
        const __nv_bfloat16* d = down + static_cast<int64_t>(j) * k;
        float acc[2] = {0.0f, 0.0f};
        for (int64_t base = c0 + lane; base < c1; base += 64) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int64_t ch = base + 32 * q;
                if (ch < c1) {
                    const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + ch * 8));
                    const uint4 dv = __ldg(reinterpret_cast<const uint4*>(d + ch * 8));
                    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc[q] = __fmaf_rn(bf16_bits_to_float(xw[e] & 0xffffu), bf16_bits_to_float(dw[e] & 0xffffu),
                                           acc[q]);
                        acc[q] = __fmaf_rn(bf16_bits_to_float(xw[e] >> 16), bf16_bits_to_float(dw[e] >> 16), acc[q]);
                    }
                }
            }
        }
        v = __fadd_rn(acc[0], acc[1]);
#pragma unroll
        for (int h = 16; h >= 1; h >>= 1) v = __fadd_rn(v, __shfl_xor_sync(kFull, v, h));
    }
    if (lane == 0) part[warp >> 2][quarter] = v;
    __syncthreads();
    if (threadIdx.x < 2) {
        const int jj = static_cast<int>(blockIdx.y) * 2 + threadIdx.x;
        if (jj < r) {
            const float* pq = part[threadIdx.x];
            const float tv = __fmul_rn(__fadd_rn(__fadd_rn(pq[0], pq[1]), __fadd_rn(pq[2], pq[3])), scale);
            t[tok * r + jj] = tv;
            if (t_hi) {
                const __nv_bfloat16 h = __float2bfloat16_rn(tv);
                t_hi[tok * r + jj] = h;
                t_lo[tok * r + jj] = __float2bfloat16_rn(__fsub_rn(tv, __bfloat162float(h)));
            }
        }
    }
}

// t for the prefill path (m > 16) on the tensor cores.  CTA (64-token block,
// k split, group of 16 ranks); warp w takes tokens 16w .. 16w + 15 of the block.
// Per 32 k a lane (g, i) loads 16 bytes of X rows g and g + 8 and of down rows g
// and g + 8 of the group, at k offset 8i: the first 8 bytes feed one
// m16n8k16 MMA and the second 8 bytes another, the MMA's k index 2i + e (e < 2)
// standing for k offset 8i + e and 2i + 8 + e for 8i + 2 + e (the same map for
// both operands, so the products are those of X down^T).  Rows past m or r are
// clamped: they only reach outputs that are not stored.  With nsplit > 1 every
// CTA stores its partial tile, and the last CTA of a (token block, rank group)
// to count in (one acquire-release add after a block barrier) adds the nsplit
// partials in split order and writes t = scale * sum, t_hi and t_lo.
constexpr int kTcTokens = 64;

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void put_t(int64_t idx, float v, float* __restrict__ t, __nv_bfloat16* __restrict__ t_hi,
                                      __nv_bfloat16* __restrict__ t_lo) {
    t[idx] = v;
    if (t_hi) {
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        t_hi[idx] = h;
        t_lo[idx] = __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(h)));
    }
}

__global__ void __launch_bounds__(128) k_lora_down_tc(const __nv_bfloat16* __restrict__ X, int64_t m, int64_t k,
                                                      const __nv_bfloat16* __restrict__ down, int r, int nsplit,
                                                      float scale, float* __restrict__ part, uint32_t* __restrict__ cnt,
                                                      float* __restrict__ t, __nv_bfloat16* __restrict__ t_hi,
                                                      __nv_bfloat16* __restrict__ t_lo) {
    __shared__ int s_last;
    grid_launch_dependents();
    grid_dependency_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, i = lane & 3;
    const int64_t tok0 = static_cast<int64_t>(blockIdx.x) * kTcTokens + 16 * warp;
    const int rank0 = 16 * static_cast<int>(blockIdx.z);
    const int split = static_cast<int>(blockIdx.y);
    const int64_t n32 = k / 32;
    const int64_t c0 = n32 * split / nsplit * 32, c1 = n32 * (split + 1) / nsplit * 32;
    auto clamp_row = [](int64_t v, int64_t hi) { return v < hi ? v : hi - 1; };
    const __nv_bfloat16* x0 = X + clamp_row(tok0 + g, m) * k + 8 * i;
    const __nv_bfloat16* x1 = X + clamp_row(tok0 + g + 8, m) * k + 8 * i;
    const __nv_bfloat16* d0 = down + clamp_row(rank0 + g, r) * k + 8 * i;
    const __nv_bfloat16* d1 = down + clamp_row(rank0 + 8 + g, r) * k + 8 * i;
    float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int64_t c = c0; c < c1; c += 32) {
        const uint4 xa = __ldg(reinterpret_cast<const uint4*>(x0 + c));
        const uint4 xb = __ldg(reinterpret_cast<const uint4*>(x1 + c));
        const uint4 da = __ldg(reinterpret_cast<const uint4*>(d0 + c));
        const uint4 db = __ldg(reinterpret_cast<const uint4*>(d1 + c));
        mma_bf16_16816(acc0, xa.x, xb.x, xa.y, xb.y, da.x, da.y);
        mma_bf16_16816(acc1, xa.x, xb.x, xa.y, xb.y, db.x, db.y);
        mma_bf16_16816(acc0, xa.z, xb.z, xa.w, xb.w, da.z, da.w);
        mma_bf16_16816(acc1, xa.z, xb.z, xa.w, xb.w, db.z, db.w);
    }
    // this lane's outputs: tokens tok0 + g (+ 8), ranks rank0 + 2i (+ 1) and rank0 + 8 + 2i (+ 1)
    const float* accs[2] = {acc0, acc1};
    if (nsplit == 1) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t tok = tok0 + g + 8 * (e >> 1);
                const int rank = rank0 + 8 * h + 2 * i + (e & 1);
                if (tok < m && rank < r) put_t(tok * r + rank, __fmul_rn(accs[h][e], scale), t, t_hi, t_lo);
            }
        return;
    }
    // partials [nsplit][m][16 x groups]
    const int rpad = 16 * static_cast<int>(gridDim.z);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
            const int64_t tok = tok0 + g + 8 * (e >> 1);
            if (tok < m)
                *reinterpret_cast<float2*>(part + (static_cast<int64_t>(split) * m + tok) * rpad + rank0 + 8 * h + 2 * i) =
                    make_float2(accs[h][e], accs[h][e + 1]);
        }
    __syncthreads();
    uint32_t* c = cnt + static_cast<int64_t>(blockIdx.z) * gridDim.x + blockIdx.x;
    if (threadIdx.x == 0) {
        uint32_t old;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(c) : "memory");
        s_last = old == static_cast<uint32_t>(nsplit - 1);
    }
    __syncthreads();
    if (!s_last) return;
    // four consecutive ranks of one token per step, every split's partial
    // requested before the first add
    for (int e = threadIdx.x; e < kTcTokens * 4; e += blockDim.x) {
        const int64_t tok = static_cast<int64_t>(blockIdx.x) * kTcTokens + e / 4;
        const int rq = rank0 + 4 * (e % 4);
        if (tok >= m || rq >= r) continue;
        float4 v[kLoraTcMaxSplit];
#pragma unroll
        for (int q = 0; q < kLoraTcMaxSplit; ++q)
            if (q < nsplit) v[q] = __ldcg(reinterpret_cast<const float4*>(part + (static_cast<int64_t>(q) * m + tok) * rpad + rq));
        float4 sum = v[0];
#pragma unroll
        for (int q = 1; q < kLoraTcMaxSplit; ++q)
            if (q < nsplit)
                sum = make_float4(__fadd_rn(sum.x, v[q].x), __fadd_rn(sum.y, v[q].y), __fadd_rn(sum.z, v[q].z),
                                  __fadd_rn(sum.w, v[q].w));
        const float o[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (rq + c < r) put_t(tok * r + rq + c, __fmul_rn(o[c], scale), t, t_hi, t_lo);
    }
    if (threadIdx.x == 0) *c = 0;  // ready for the next call
}

// ---------------------------------------------------------------------------
// Merge + requantize (page "LLM 相關知識" (technicalnotes), section "8. LoRA 的
// 合併（Merge）": the 4-bit weight is dequantized to bf16, the product of the two
// LoRA matrices is added in bf16, and the sum is quantized back to 4 bits for
// deployment).  Per element (o, c):
//   What  = bf16_rn(fp32(level * ahat))                 the bf16 dequantized weight
//   delta = fma chain over j = 0 .. r-1 of up[o][j] * down[j][c], from 0, in fp32
//   Wnew  = bf16_rn(fp32(What + fp32(scale * delta)))
// and Wnew is then quantized blockwise exactly as k_nf4_quantize does, with the
// weight's own codebook (NF4 or FP4).  Lane layout as in quantization: a lane
// owns 8 consecutive elements of one row (k % 64 == 0 keeps each 64-block
// inside a row), 8 lanes one block.  down is small ([r, k] bf16) and is re-read
// from L1/L2 by every row.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_nf4_merge_lora(const uint32_t* __restrict__ wq32,
                                                        const int8_t* __restrict__ absmax_q,
                                                        const float* __restrict__ absmax_scale,
                                                        const float* __restrict__ mu_ptr, int64_t k,
                                                        int64_t n_groups, const __nv_bfloat16* __restrict__ down,
                                                        const __nv_bfloat16* __restrict__ up, int r, float scale,
                                                        uint4* __restrict__ w_new, uint32_t* __restrict__ wq_out,
                                                        float* __restrict__ absmax_out, int codebook) {
    __shared__ float lv[16];
    if (threadIdx.x < 16) lv[threadIdx.x] = kCodebook[codebook][threadIdx.x];
    __syncthreads();
    const float mu = __ldg(mu_ptr);
    const uint16_t* up16 = reinterpret_cast<const uint16_t*>(up);
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t n_chunks = (n_groups + 31) >> 5;
    for (int64_t chunk = warp; chunk < n_chunks; chunk += n_warps) {
        const int64_t g = (chunk << 5) + lane;   // group of 8 elements
        const bool valid = g < n_groups;          // whole 8-lane blocks agree
        float w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = 0.0f;
        if (valid) {
            const uint32_t packed = __ldg(wq32 + g);
            const int64_t b = g >> 3;
            const float a = absmax_hat(__ldg(absmax_q + b), __ldg(absmax_scale + (b >> 8)), mu);
            const int64_t e0 = g * 8;
            const int64_t o = e0 / k;
            const int64_t c0 = e0 - o * k;
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
            const uint16_t* u_row = up16 + o * r;
            const __nv_bfloat16* d_col = down + c0;
#pragma unroll 4
            for (int j = 0; j < r; ++j) {
                const float u = bf16_bits_to_float(__ldg(u_row + j));
                const uint4 dv = __ldg(reinterpret_cast<const uint4*>(d_col + static_cast<int64_t>(j) * k));
                const uint32_t dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc[2 * i] = __fmaf_rn(u, bf16_bits_to_float(dw[i] & 0xffffu), acc[2 * i]);
                    acc[2 * i + 1] = __fmaf_rn(u, bf16_bits_to_float(dw[i] >> 16), acc[2 * i + 1]);
                }
            }
            uint32_t out[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t byte = (packed >> (8 * i)) & 0xffu;
                // element 2i sits in the high nibble
                const float what0 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(lv[byte >> 4], a)));
                const float what1 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(lv[byte & 15u], a)));
                const float s0 = __fadd_rn(what0, __fmul_rn(scale, acc[2 * i]));
                const float s1 = __fadd_rn(what1, __fmul_rn(scale, acc[2 * i + 1]));
                out[i] = pack_bf16x2(s0, s1);
                w[2 * i] = bf16_bits_to_float(out[i] & 0xffffu);
                w[2 * i + 1] = bf16_bits_to_float(out[i] >> 16);
            }
            if (w_new) __stcs(w_new + g, make_uint4(out[0], out[1], out[2], out[3]));
        }
        float a = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(w[e]));
        a = fmaxf(a, __shfl_xor_sync(kFull, a, 1));
        a = fmaxf(a, __shfl_xor_sync(kFull, a, 2));
        a = fmaxf(a, __shfl_xor_sync(kFull, a, 4));
        uint32_t packed = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float wh = w[2 * i], wl = w[2 * i + 1];
            const uint32_t hi = static_cast<uint32_t>(codebook == kCbFp4 ? quantize_code<kCbFp4>(wh, a)
                                                                          : quantize_code<kCbNf4>(wh, a));
            const uint32_t lo = static_cast<uint32_t>(codebook == kCbFp4 ? quantize_code<kCbFp4>(wl, a)
                                                                          : quantize_code<kCbNf4>(wl, a));
            packed |= ((hi << 4) | lo) << (8 * i);
        }
        if (valid) {
            wq_out[g] = packed;
            if ((lane & 7) == 0) absmax_out[g >> 3] = a;
        }
    }
}

}  // namespace lora

cudaError_t launch_lora_down(const void* X, int64_t m, int64_t k, const void* down, int r, float scale, float* t,
                             __nv_bfloat16* t_hi, __nv_bfloat16* t_lo, bool early, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(m), static_cast<unsigned>((r + 1) / 2), 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = early ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, lora::k_lora_down, static_cast<const __nv_bfloat16*>(X), k,
                              static_cast<const __nv_bfloat16*>(down), r, scale, t, t_hi, t_lo);
}

int lora_tc_splits(int64_t m, int64_t k, int r, int sm_count) {
    const int64_t blocks = ((m + lora::kTcTokens - 1) / lora::kTcTokens) * ((r + 15) / 16);
    int64_t s = (8 * static_cast<int64_t>(sm_count) + blocks - 1) / blocks;
    const int64_t cap_k = k / 32, cap_mem = (int64_t(1) << 22) / (m * 16 * ((r + 15) / 16));
    if (s > kLoraTcMaxSplit) s = kLoraTcMaxSplit;
    if (s > cap_k) s = cap_k;
    if (s > cap_mem) s = cap_mem;
    return s < 1 ? 1 : static_cast<int>(s);
}

size_t lora_tc_scratch_bytes(int64_t m, int64_t k, int r) {
    const int64_t blocks = ((m + lora::kTcTokens - 1) / lora::kTcTokens) * ((r + 15) / 16);
    const int64_t cap_mem = (int64_t(1) << 22) / (m * 16 * ((r + 15) / 16));
    int64_t s = kLoraTcMaxSplit;
    if (s > k / 32) s = k / 32;
    if (s > cap_mem) s = cap_mem;
    if (s <= 1) return 0;
    return static_cast<size_t>((blocks * 4 + 255) / 256 * 256) +
           static_cast<size_t>(s) * static_cast<size_t>(m) * 16 * static_cast<size_t>((r + 15) / 16) * sizeof(float);
}

cudaError_t launch_lora_down_tc(const void* X, int64_t m, int64_t k, const void* down, int r, float scale, float* t,
                                __nv_bfloat16* t_hi, __nv_bfloat16* t_lo, void* scratch, bool early,
                                const DeviceInfo& dev, cudaStream_t stream) {
    const int64_t tb = (m + lora::kTcTokens - 1) / lora::kTcTokens;
    const int groups = (r + 15) / 16;
    const int nsplit = lora_tc_splits(m, k, r, dev.sm_count);
    if (tb > 0x7fffffff) return cudaErrorInvalidValue;
    uint32_t* cnt = static_cast<uint32_t*>(scratch);
    float* part = scratch ? reinterpret_cast<float*>(static_cast<char*>(scratch) + (tb * groups * 4 + 255) / 256 * 256)
                          : nullptr;
    if (nsplit > 1 && scratch == nullptr) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tb), static_cast<unsigned>(nsplit), static_cast<unsigned>(groups));
    cfg.blockDim = dim3(128, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = early ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, lora::k_lora_down_tc, static_cast<const __nv_bfloat16*>(X), m, k,
                              static_cast<const __nv_bfloat16*>(down), r, nsplit, scale, part, cnt, t, t_hi, t_lo);
}

cudaError_t launch_merge_lora(const uint8_t* wq, const int8_t* absmax_q, const float* absmax_scale,
                              const float* absmax_offset, int64_t n, int64_t k, const void* down, const void* up,
                              int r, float scale, void* w_new, uint8_t* wq_out, float* absmax_out, int codebook,
                              const DeviceInfo& dev, cudaStream_t stream) {
    const int64_t n_groups = n * k / 8;
    const int64_t n_chunks = (n_groups + 31) / 32;
    int64_t blocks = (n_chunks + 7) / 8;
    const int64_t cap = static_cast<int64_t>(dev.sm_count) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    lora::k_nf4_merge_lora<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        reinterpret_cast<const uint32_t*>(wq), absmax_q, absmax_scale, absmax_offset, k, n_groups,
        static_cast<const __nv_bfloat16*>(down), static_cast<const __nv_bfloat16*>(up), r, scale,
        static_cast<uint4*>(w_new), reinterpret_cast<uint32_t*>(wq_out), absmax_out, codebook);
    return cudaGetLastError();
}

}  // namespace nf4
