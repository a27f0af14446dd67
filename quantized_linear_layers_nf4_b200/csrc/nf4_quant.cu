// nf4_quant.cu -- blockwise NF4 quantization and double quantization (sm_100a).
//
// Sources (web pages, cited by title and section):
//   [P1] "Tim Dettmers 如何用 bitsandbytes 與 QLoRA 降低 LLM 訓練門檻？" (yololab.net),
//        sections "NF4 不是一般四位元浮點格式" and "Double quantization 連 scale 本身也壓縮"
//   [P3] "bitsandbytes：让大语言模型在消费级硬件上运行的量化神器" (zingnex.cn),
//        section "分页优化器与双量化"
//   [P5] "篇2-bitsandbytes-具体观-算法与实现剖析" (xyzblog), §2.2 "QLoRA / NF4"
//        (principles ① ②, worked example) and Figure 2-2.
//
// Both kernels are HBM-bound streams.  Quantization reads the weight once
// (2 or 4 B/param) and writes 0.5 B/param of codes plus 4 B per 64 params of
// absmax: 128-bit loads, 8 lanes per 64-block, a 3-step xor-shuffle absmax and
// one packed 32-bit store per lane.  Double quantization is two small
// launches: per-256 fp64 partial sums, then the int8 encode, whose CTAs each
// finish the mean's fixed-order reduction from the partial sums first.
#include "nf4_common.cuh"
#include "nf4_encode.cuh"
#include "nf4_internal.h"
#include "nf4_ptx.cuh"

namespace nf4 {

// ---------------------------------------------------------------------------
// Quantization.  Lane layout: each lane owns 8 consecutive elements (one
// 32-bit word of packed codes); 8 consecutive lanes own one 64-element block,
// so a warp covers 4 blocks = 256 elements per iteration, loads coalesced.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void load8(const float* __restrict__ W, int64_t e, float (&w)[8]) {
    const float4 a = __ldcs(reinterpret_cast<const float4*>(W + e));
    const float4 b = __ldcs(reinterpret_cast<const float4*>(W + e + 4));
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
}

__device__ __forceinline__ void load8(const __nv_bfloat16* __restrict__ W, int64_t e, float (&w)[8]) {
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(W + e));
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        w[2 * i] = bf16_bits_to_float(u[i] & 0xffffu);   // lower address first
        w[2 * i + 1] = bf16_bits_to_float(u[i] >> 16);
    }
}

template <typename T, int CB>
__global__ void __launch_bounds__(256, 4) k_nf4_quantize(const T* __restrict__ W, int64_t n_groups,
                                                      uint32_t* __restrict__ wq32,
                                                      float* __restrict__ absmax) {
    __shared__ uint2 tab[CB == kCbNf4 ? kBuckets * kTabCopies : 1];
    if (CB == kCbNf4) build_bucket_table(tab);
    // the table above uses constants only; W and the outputs wait for the
    // preceding kernel (launched as its programmatic dependent)
    grid_dependency_wait();
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t n_chunks = (n_groups + 31) >> 5;
    // a warp takes kUnroll chunks per pass (chunk = 256 contiguous elements):
    // all their loads go out before any of them is encoded
    constexpr int kUnroll = 4;
    for (int64_t c0 = warp; c0 < n_chunks; c0 += n_warps * kUnroll) {
        float w[kUnroll][8];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t g = ((c0 + u * n_warps) << 5) + lane;  // group of 8 elements
            if (g < n_groups) {
                load8(W, g * 8, w[u]);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) w[u][j] = 0.0f;
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t g = ((c0 + u * n_warps) << 5) + lane;
            const bool valid = g < n_groups;                 // whole 8-lane blocks agree
            float a = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) a = fmaxf(a, fabsf(w[u][j]));
            a = fmaxf(a, __shfl_xor_sync(kFull, a, 1));
            a = fmaxf(a, __shfl_xor_sync(kFull, a, 2));
            a = fmaxf(a, __shfl_xor_sync(kFull, a, 4));
            uint32_t code[8];
            if (CB == kCbNf4 && __all_sync(kFull, markstein_ok(a))) {
                // the same quotient and bucket, two elements per packed instruction
                // (taken by whole warps; a warp with any other block uses the paths below)
                const float r = __frcp_rn(a);
                const uint64_t rr = f2(r, r), na = f2(-a, -a), k128 = f2(128.0f, 128.0f);
                const uint64_t mg = f2(kBucketMagic, kBucketMagic);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const uint64_t w2 = f2(w[u][2 * p], w[u][2 * p + 1]);
                    const uint64_t q0 = mul2(w2, rr);
                    const uint64_t e = fma2(q0, na, w2);
                    const uint64_t q2 = fma2(e, rr, q0);
                    const uint64_t b2 = fma2(q2, k128, mg);
                    float qv[2];
                    uint32_t bv[2];
                    asm("mov.b64 {%0, %1}, %2;" : "=f"(qv[0]), "=f"(qv[1]) : "l"(q2));
                    asm("mov.b64 {%0, %1}, %2;" : "=r"(bv[0]), "=r"(bv[1]) : "l"(b2));
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint2 ent = tab[(bv[h] & 0x1ffu) * kTabCopies + (threadIdx.x & 15)];
                        code[2 * p + h] = ent.y + (qv[h] > __uint_as_float(ent.x) ? 1u : 0u);
                    }
                }
            } else if (markstein_ok(a)) {
                const float r = __frcp_rn(a);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float q = quotient(w[u][j], a, r);
                    code[j] = CB == kCbNf4 ? bucket_code(q, tab, threadIdx.x & 15)
                                           : static_cast<uint32_t>(encode_fp4(q));
                }
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) code[j] = static_cast<uint32_t>(quantize_code<CB>(w[u][j], a));
            }
            uint32_t packed = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) packed |= ((code[2 * i] << 4) | code[2 * i + 1]) << (8 * i);  // element 2i high
            if (valid) {
                wq32[g] = packed;
                if ((lane & 7) == 0) absmax[g >> 3] = a;
            }
        }
    }
    grid_launch_dependents();
}

template <int CB>
static cudaError_t launch_quantize_cb(const void* W, bool w_bf16, int64_t n_groups, uint8_t* wq, float* absmax,
                               int64_t blocks, cudaStream_t stream) {
    if (w_bf16)
        return launch_pdl(k_nf4_quantize<__nv_bfloat16, CB>, dim3(static_cast<unsigned>(blocks)), dim3(256), stream,
                          static_cast<const __nv_bfloat16*>(W), n_groups, reinterpret_cast<uint32_t*>(wq), absmax);
    return launch_pdl(k_nf4_quantize<float, CB>, dim3(static_cast<unsigned>(blocks)), dim3(256), stream,
                      static_cast<const float*>(W), n_groups, reinterpret_cast<uint32_t*>(wq), absmax);
}

cudaError_t launch_quantize(const void* W, bool w_bf16, int64_t n_elem, uint8_t* wq, float* absmax, int codebook,
                            const DeviceInfo& dev, cudaStream_t stream) {
    const int64_t n_groups = n_elem / 8;
    const int64_t n_chunks = (n_groups + 31) / 32;
    int64_t blocks = (n_chunks + 7) / 8;
    // one wave of CTAs that stay resident (four per SM by their registers) and
    // walk the chunks with a grid stride
    const int64_t cap = static_cast<int64_t>(dev.sm_count) * 4;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (codebook == kCbFp4) return launch_quantize_cb<kCbFp4>(W, w_bf16, n_groups, wq, absmax, blocks, stream);
    return launch_quantize_cb<kCbNf4>(W, w_bf16, n_groups, wq, absmax, blocks, stream);
}

// ---------------------------------------------------------------------------
// Double quantization.
//
// The mean's summation order is fixed ([P5] §2.2 ② subtracts the mean of the
// absmax values; the order is this library's definition, shared with nothing):
// the list is cut into chunks of 256 (zero-padded), each chunk is reduced by
// a[i] += a[i + h] for h = 128, 64, ..., 1, and the chunk results form the next
// list until one value is left.
//
// One warp reduces one chunk: lane l holds elements l + 32 j (j = 0..7), so the
// h = 128, 64, 32 steps are in-register and h = 16..1 are shuffles; every add
// pairs the same two elements as the definition.
// ---------------------------------------------------------------------------
__device__ __forceinline__ double warp_tree256(double (&v)[8]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = v[j] + v[j + 4];    // h = 128
#pragma unroll
    for (int j = 0; j < 2; ++j) v[j] = v[j] + v[j + 2];    // h = 64
    v[0] = v[0] + v[1];                                     // h = 32
    double s = v[0];
#pragma unroll
    for (int h = 16; h >= 1; h >>= 1) s = s + __shfl_down_sync(kFull, s, h);
    return s;  // valid in lane 0
}

// Level 1: one fp64 partial per double-quantization block of 256 absmax.
__global__ void __launch_bounds__(256) k_dq_partials(const float* __restrict__ absmax, int64_t nb,
                                                     double* __restrict__ partials, int64_t nb2) {
    grid_dependency_wait();  // absmax comes from the preceding kernel
    grid_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t c = warp; c < nb2; c += n_warps) {
        double v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int64_t b = c * 256 + lane + 32 * j;
            v[j] = (b < nb) ? static_cast<double>(__ldg(absmax + b)) : 0.0;
        }
        const double s = warp_tree256(v);
        if (lane == 0) partials[c] = s;
    }
}

constexpr int kMeanLevel2 = 4096;  // max chunks after the first reduction (shared memory)

int64_t dq_max_nb() { return static_cast<int64_t>(256) * 256 * kMeanLevel2; }

size_t dq_workspace_bytes(int64_t nb) {
    if (nb <= 0) return 0;
    const int64_t nb2 = (nb + 255) / 256;
    return static_cast<size_t>(nb2) * sizeof(double);
}

// The remaining levels of the mean's tree over the nb2 chunk sums, by one CTA
// of `kEncodeThreads` threads: S, then mu = fp32(S / nb).  Every encode CTA
// does this for itself (the same adds in the same order, so every CTA gets the
// same bits), which saves a launch between the two passes.
constexpr int kEncodeThreads = 256;

__device__ float cta_mean(const double* __restrict__ partials, int64_t nb2, int64_t nb, double* buf_a,
                          double* buf_b) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int n_warps = kEncodeThreads / 32;
    const double* src = partials;
    double* dst = buf_a;
    int64_t n = nb2;
    while (n > 1) {
        const int64_t m = (n + 255) / 256;
        for (int64_t c = warp; c < m; c += n_warps) {
            double v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int64_t i = c * 256 + lane + 32 * j;
                v[j] = (i < n) ? src[i] : 0.0;
            }
            const double s = warp_tree256(v);
            if (lane == 0) dst[c] = s;
        }
        __syncthreads();
        src = dst;
        dst = (dst == buf_a) ? buf_b : buf_a;
        n = m;
    }
    return __double2float_rn(__ddiv_rn(src[0], static_cast<double>(nb)));
}

// Encode: the mean (above), then one warp per block of 256 absmax values.
// CTA 0 writes the mean.
__global__ void __launch_bounds__(kEncodeThreads) k_dq_encode(const float* __restrict__ absmax, int64_t nb,
                                                              int64_t nb2, const double* __restrict__ partials,
                                                              float* __restrict__ mu_out,
                                                              int8_t* __restrict__ absmax_q,
                                                              float* __restrict__ absmax_scale) {
    __shared__ double buf_a[kMeanLevel2];
    __shared__ double buf_b[kMeanLevel2 / 256 + 1];
    grid_dependency_wait();  // the partial sums come from the preceding kernel
    grid_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    // the warp's first block of absmax values is requested before the mean is
    // formed, so the two loads overlap
    float pre[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int64_t b = warp * 256 + lane + 32 * j;
        pre[j] = (warp < nb2 && b < nb) ? __ldg(absmax + b) : 0.0f;
    }
    const float mu = cta_mean(partials, nb2, nb, buf_a, buf_b);
    if (blockIdx.x == 0 && threadIdx.x == 0) *mu_out = mu;
    for (int64_t c = warp; c < nb2; c += n_warps) {
        float r[8];
        float s = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int64_t b = c * 256 + lane + 32 * j;
            const float v = (c == warp) ? pre[j] : ((b < nb) ? __ldg(absmax + b) : 0.0f);
            r[j] = (b < nb) ? __fsub_rn(v, mu) : 0.0f;
            s = fmaxf(s, fabsf(r[j]));
        }
#pragma unroll
        for (int h = 16; h >= 1; h >>= 1) s = fmaxf(s, __shfl_xor_sync(kFull, s, h));
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int64_t b = c * 256 + lane + 32 * j;
            if (b < nb) {
                int q = 0;
                if (s != 0.0f) q = __float2int_rn(__fmul_rn(__fdiv_rn(r[j], s), 127.0f));
                absmax_q[b] = static_cast<int8_t>(q);
            }
        }
        if (lane == 0) absmax_scale[c] = s;
    }
}

cudaError_t launch_double_quant(const float* absmax, int64_t nb, double* workspace, int8_t* absmax_q,
                                float* absmax_scale, float* absmax_offset, const DeviceInfo& dev,
                                cudaStream_t stream) {
    const int64_t nb2 = (nb + 255) / 256;
    int64_t blocks = (nb2 + 7) / 8;
    const int64_t cap = static_cast<int64_t>(dev.sm_count) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    // both as programmatic dependents: each launch overlaps the tail of the one before
    cudaError_t e = launch_pdl(k_dq_partials, dim3(static_cast<unsigned>(blocks)), dim3(256), stream, absmax, nb,
                               workspace, nb2);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_dq_encode, dim3(static_cast<unsigned>(blocks)), dim3(kEncodeThreads), stream, absmax, nb, nb2,
                      static_cast<const double*>(workspace), absmax_offset, absmax_q, absmax_scale);
}

}  // namespace nf4
