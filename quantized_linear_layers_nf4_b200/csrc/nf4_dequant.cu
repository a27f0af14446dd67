// nf4_dequant.cu -- NF4 + double-quantization state back to fp32 / bf16 (sm_100a).
//
// Source: page "LLM 相關知識" (technicalnotes, tag qlora), §5 "動態反量化": the 4-bit
// weights are restored to the compute dtype layer by layer; page "Tim Dettmers
// 如何用 bitsandbytes 與 QLoRA 降低 LLM 訓練門檻？", section on QLoRA: the frozen 4-bit
// base is dequantized in forward and backward.
//
// HBM-bound: reads 0.5 B/param of codes (+1 B per 64 of absmax codes) and
// writes 2 (bf16) or 4 (fp32) B/param.  Each lane decodes 32-bit words of codes
// (8 elements each), fetching each level from the lane that holds it, and writes 16 or
// 32 bytes per word with 128-bit stores; a warp takes four words per lane per
// pass (a warp's loads and stores stay contiguous) with all four loads issued
// before the first decode.  nf4_dequantize_batch runs several weights in one
// launch (a layer at load time), so the ramp and tail of a launch are paid once.
#include <cstring>

#include "nf4_common.cuh"
#include "nf4_internal.h"
#include "nf4_ptx.cuh"

namespace nf4 {

constexpr int kUnroll = 4;          // words per lane in one pass of a warp
constexpr int kPassWords = 32 * kUnroll;

// One pass of a warp: words base + 32 q + lane, q = 0 .. 3 (128 consecutive
// words, all loads issued before the first decode).  lvr holds level[lane % 16];
// a level is fetched from the lane that holds it (one shuffle, no shared-memory
// bank conflicts), so every lane takes part in every shuffle and lanes past the
// end decode a valid word and skip the store.
template <bool kBf16Out>
__device__ __forceinline__ void dequant_pass(const uint32_t* __restrict__ wq32, const int8_t* __restrict__ absmax_q,
                                             const float* __restrict__ absmax_scale, float mu, int64_t n_groups,
                                             void* __restrict__ out, int64_t base, float lvr, int lane) {
    uint32_t packed[kUnroll];
    float a[kUnroll];
#pragma unroll
    for (int q = 0; q < kUnroll; ++q) {
        const int64_t g = base + 32 * q + lane;
        const int64_t gg = g < n_groups ? g : base;      // a valid word (base always is)
        packed[q] = __ldcs(wq32 + gg);
        const int64_t b = gg >> 3;                       // 64-element block
        a[q] = absmax_hat(__ldg(absmax_q + b), __ldg(absmax_scale + (b >> 8)), mu);
    }
    uint64_t aa[kUnroll];  // {a, a}: the two levels of a byte scaled by one packed multiply
#pragma unroll
    for (int q = 0; q < kUnroll; ++q) asm("mov.b64 %0, {%1, %1};" : "=l"(aa[q]) : "f"(a[q]));
#pragma unroll
    for (int q = 0; q < kUnroll; ++q) {
        const int64_t g = base + 32 * q + lane;
        float v[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // a shuffle takes the low 5 bits of its source lane, and lanes l and
            // l + 16 hold the same level, so the shifted word needs no mask
            const int hi = static_cast<int>(packed[q] >> (8 * i + 4));  // element 2i: high nibble
            const int lo = static_cast<int>(packed[q] >> (8 * i));
            const float lh = __shfl_sync(kFull, lvr, hi), ll = __shfl_sync(kFull, lvr, lo);
            uint64_t p2;  // each half rounded as the scalar fp32 multiply
            asm("{\n\t.reg .b64 l;\n\tmov.b64 l, {%1, %2};\n\tmul.rn.f32x2 %0, l, %3;\n\t}"
                : "=l"(p2)
                : "f"(lh), "f"(ll), "l"(aa[q]));
            asm("mov.b64 {%0, %1}, %2;" : "=f"(v[2 * i]), "=f"(v[2 * i + 1]) : "l"(p2));
        }
        if (g >= n_groups) continue;
        if (kBf16Out) {
            uint4 o;
            o.x = pack_bf16x2(v[0], v[1]);
            o.y = pack_bf16x2(v[2], v[3]);
            o.z = pack_bf16x2(v[4], v[5]);
            o.w = pack_bf16x2(v[6], v[7]);
            __stcs(reinterpret_cast<uint4*>(out) + g, o);
        } else {
            float4* o = reinterpret_cast<float4*>(out) + 2 * g;
            __stcs(o, make_float4(v[0], v[1], v[2], v[3]));
            __stcs(o + 1, make_float4(v[4], v[5], v[6], v[7]));
        }
    }
}

template <bool kBf16Out>
__global__ void __launch_bounds__(256) k_nf4_dequantize(const uint32_t* __restrict__ wq32,
                                                        const int8_t* __restrict__ absmax_q,
                                                        const float* __restrict__ absmax_scale,
                                                        const float* __restrict__ mu_ptr,
                                                        int64_t n_groups, void* __restrict__ out,
                                                        int codebook) {
    const int lane = threadIdx.x & 31;
    const float lvr = kCodebook[codebook][lane & 15];
    grid_dependency_wait();  // launched as a programmatic dependent: inputs may come from the preceding kernel
    grid_launch_dependents();
    const float mu = __ldg(mu_ptr);
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t base = warp * kPassWords; base < n_groups; base += n_warps * kPassWords)
        dequant_pass<kBf16Out>(wq32, absmax_q, absmax_scale, mu, n_groups, out, base, lvr, lane);
}

// Several weights in one launch: the passes of weight i are pass0[i] ..
// pass0[i + 1] - 1 of one sequence that the warps stride through.
struct DequantBatch {
    const uint32_t* wq32[kMaxDequantBatch];
    const int8_t* absmax_q[kMaxDequantBatch];
    const float* absmax_scale[kMaxDequantBatch];
    const float* mu[kMaxDequantBatch];
    void* out[kMaxDequantBatch];
    int64_t n_groups[kMaxDequantBatch];
    int64_t pass0[kMaxDequantBatch + 1];
    int codebook[kMaxDequantBatch];
    int count;
};

template <bool kBf16Out>
__global__ void __launch_bounds__(256) k_nf4_dequantize_batch(const __grid_constant__ DequantBatch bt) {
    const int lane = threadIdx.x & 31;
    grid_dependency_wait();
    grid_launch_dependents();
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t p = warp; p < bt.pass0[bt.count]; p += n_warps) {
        int ti = 0;
        for (int i = 1; i < bt.count; ++i)
            if (p >= bt.pass0[i]) ti = i;
        const float lvr = kCodebook[bt.codebook[ti]][lane & 15];
        dequant_pass<kBf16Out>(bt.wq32[ti], bt.absmax_q[ti], bt.absmax_scale[ti], __ldg(bt.mu[ti]), bt.n_groups[ti],
                               bt.out[ti], (p - bt.pass0[ti]) * kPassWords, lvr, lane);
    }
}

cudaError_t launch_dequantize(const uint8_t* wq, const int8_t* absmax_q, const float* absmax_scale,
                              const float* absmax_offset, int64_t n_elem, void* out, bool out_bf16, int codebook,
                              const DeviceInfo& dev, cudaStream_t stream) {
    const int64_t n_groups = n_elem / 8;
    int64_t blocks = (n_groups + 1023) / 1024;
    const int64_t cap = static_cast<int64_t>(dev.sm_count) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    const uint32_t* wq32 = reinterpret_cast<const uint32_t*>(wq);
    if (out_bf16)
        return launch_pdl(k_nf4_dequantize<true>, dim3(static_cast<unsigned>(blocks)), dim3(256), stream, wq32,
                          absmax_q, absmax_scale, absmax_offset, n_groups, out, codebook);
    return launch_pdl(k_nf4_dequantize<false>, dim3(static_cast<unsigned>(blocks)), dim3(256), stream, wq32, absmax_q,
                      absmax_scale, absmax_offset, n_groups, out, codebook);
}

cudaError_t launch_dequantize_batch(const DequantItem* items, int count, bool out_bf16, const DeviceInfo& dev,
                                    cudaStream_t stream) {
    if (count < 1 || count > kMaxDequantBatch) return cudaErrorInvalidValue;
    DequantBatch bt;
    memset(&bt, 0, sizeof(bt));
    int64_t passes = 0;
    for (int i = 0; i < count; ++i) {
        bt.wq32[i] = reinterpret_cast<const uint32_t*>(items[i].wq);
        bt.absmax_q[i] = items[i].absmax_q;
        bt.absmax_scale[i] = items[i].absmax_scale;
        bt.mu[i] = items[i].absmax_offset;
        bt.out[i] = items[i].out;
        bt.n_groups[i] = items[i].n_elem / 8;
        bt.codebook[i] = items[i].codebook;
        bt.pass0[i] = passes;
        passes += (bt.n_groups[i] + kPassWords - 1) / kPassWords;
    }
    bt.pass0[count] = passes;
    bt.count = count;
    // eight 256-thread CTAs per SM, each warp striding over the passes
    int64_t blocks = (passes + 7) / 8;
    const int64_t cap = static_cast<int64_t>(dev.sm_count) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (out_bf16)
        return launch_pdl(k_nf4_dequantize_batch<true>, dim3(static_cast<unsigned>(blocks)), dim3(256), stream, bt);
    return launch_pdl(k_nf4_dequantize_batch<false>, dim3(static_cast<unsigned>(blocks)), dim3(256), stream, bt);
}

}  // namespace nf4
