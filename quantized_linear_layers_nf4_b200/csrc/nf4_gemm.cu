// nf4_gemm.cu -- fused dequantize + linear for large batches (prefill), sm_100a tcgen05.
//
// Sources: page "篇2-bitsandbytes-具体观-算法与实现剖析" (xyzblog), §2.2 code walk
// (matmul_4bit = dequantize + matmul) and §2.5 (per-architecture 4-bit GEMM
// files: prior art for older tensor cores); page "LLM 相關知識" (technicalnotes),
// §5 "動態反量化" (weights restored to BF16 per layer for the matmul); page "Tim
// Dettmers 如何用 bitsandbytes 與 QLoRA 降低 LLM 訓練門檻？", section "量化速度取決於硬體與
// kernel": with large batches the work is compute-bound.
//
//   Y[t, r] = sum_c X[t, c] * What[r, c],   What = bf16(fp32(level[idx] * a_block)).
//
// One CTA computes a 256 (tokens) x 256 (weight rows) tile of Y with the
// 5th-generation tensor cores: two 128 x 256 fp32 accumulators in tensor memory
// (all 512 columns), bf16 operands from shared memory in the canonical K-major
// 128-byte swizzled layout, 64 k per stage.
//
// * Warp 0 streams X tiles [256 x 64] with TMA; warp 2 streams the packed
//   4-bit tile [256 rows x 32 bytes] with TMA (no multicast anywhere).
// * Warps 4..11 (256 threads, one weight row each) dequantize on the CUDA
//   cores: per (row, 64-block) they reconstruct the absmax, multiply the 16
//   levels by it in fp32 and round to bf16 (the same values nf4_dequantize
//   produces), split that 16-entry table into byte planes and decode each
//   nibble with byte permutes -- no table lookups in shared memory, so the
//   tensor core keeps the shared-memory bandwidth for its operands.  Each
//   thread writes its 128-byte row of the swizzled B tile.
// * One thread of warp 1 issues tcgen05.mma (M = 128, N = 256, K = 16) for
//   both halves of the token tile, reusing the decoded weight tile, and
//   releases stages with tcgen05.commit.
// * After the k loop the dequant warps read the accumulators (tcgen05.ld) and
//   store Y.
// Every mbarrier wait is bounded; a wait that runs out records
// NF4_ERR_DEVICE_TIMEOUT, the CTA drains what it issued and frees its tensor
// memory before returning.
#include <mutex>

#include "nf4_common.cuh"
#include "nf4_decode.cuh"
#include "nf4_internal.h"
#include "nf4_ptx.cuh"
#include "nf4_tmap.h"

namespace nf4 {
namespace gemm {

constexpr int kBM = 256;  // tokens per CTA tile (two 128-row MMA halves)
constexpr int kBN = 256;  // weight rows per CTA tile (MMA N)
constexpr int kBK = 64;   // k per stage: one 128-byte swizzle row of bf16
constexpr int kStagesA = 3;
constexpr int kStagesB = 2;
constexpr int kStagesP = 4;
constexpr int kABytes = kBM * kBK * 2;  // 32768
constexpr int kBBytes = kBN * kBK * 2;  // 32768
constexpr int kPBytes = kBN * kBK / 2;  // 8192
constexpr int kDequantWarps = 8;
constexpr int kThreads = 32 * (4 + kDequantWarps);
constexpr uint32_t kTmemCols = 512;
constexpr int kOffB = kStagesA * kABytes;
constexpr int kOffP = kOffB + kStagesB * kBBytes;
constexpr int kOffBar = kOffP + kStagesP * kPBytes;
constexpr int kNumBars = 2 * kStagesA + 2 * kStagesB + 2 * kStagesP + 4;  // + low-rank tiles, MMA drain
constexpr int kSmemBytes = 1024 + kOffBar + kNumBars * 8 + 16;

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major,
// N = 256, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((kBN >> 3) << 17) | ((128 >> 4) << 24);

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

template <bool kBf16Out, bool kLora>
__global__ void __launch_bounds__(kThreads, 1)
k_nf4_gemm(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
           const int8_t* __restrict__ absmax_q, const float* __restrict__ absmax_scale,
           const float* __restrict__ mu_ptr, int64_t m, int64_t n, int64_t k, void* __restrict__ Y,
           int32_t* __restrict__ dev_status, const float* __restrict__ lora_t,
           const __nv_bfloat16* __restrict__ lora_up, int lora_r, int lora_tc,
           const __grid_constant__ CUtensorMap tm_thi, const __grid_constant__ CUtensorMap tm_tlo,
           const __grid_constant__ CUtensorMap tm_up, int codebook, uint32_t lim, int stall) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* full_a = bars;
    uint64_t* empty_a = full_a + kStagesA;
    uint64_t* full_b = empty_a + kStagesA;
    uint64_t* empty_b = full_b + kStagesB;
    uint64_t* full_p = empty_b + kStagesB;
    uint64_t* empty_p = full_p + kStagesP;
    uint64_t* acc_ready = empty_p + kStagesP;
    uint64_t* drained = acc_ready + 1;
    uint64_t* lora_full = drained + 1;   // low-rank tiles landed
    uint64_t* mma_done = lora_full + 1;   // every MMA issued so far has completed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kBN;
    const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kBM;
    const int nk = static_cast<int>(k / kBK);
    const uint32_t sbase = smem_u32(smem);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesA; ++s) {
            mbar_init(&full_a[s], 1);
            mbar_init(&empty_a[s], 1);
        }
        for (int s = 0; s < kStagesB; ++s) {
            mbar_init(&full_b[s], kDequantWarps);
            mbar_init(&empty_b[s], 1);
        }
        for (int s = 0; s < kStagesP; ++s) {
            mbar_init(&full_p[s], 1);
            mbar_init(&empty_p[s], kDequantWarps);
        }
        mbar_init(acc_ready, 1);
        mbar_init(drained, 1);
        mbar_init(lora_full, 1);
        mbar_init(mma_done, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool timed_out = false;
    if (warp == 0) {
        // ---------------------------- X producer ----------------------------
        if (lane == 0) {
            prefetch_tensormap(&tm_x);
            int issued = 0;
            for (int kt = 0; kt < (stall ? 0 : nk); ++kt) {
                const int s = kt % kStagesA;
                if (kt >= kStagesA && !mbar_wait_n(&empty_a[s], ((kt / kStagesA) - 1) & 1, lim)) {
                    timed_out = true;
                    break;
                }
                mbar_arrive_expect_tx(&full_a[s], kABytes);
                tma_load_2d(smem + s * kABytes, &tm_x, kt * kBK, static_cast<int32_t>(m0), &full_a[s]);
                issued = kt + 1;
            }
            if (timed_out)  // leave no copy in flight
                for (int kt = (issued > kStagesA ? issued - kStagesA : 0); kt < issued; ++kt)
                    mbar_wait_n(&full_a[kt % kStagesA], (kt / kStagesA) & 1, kWaitLimit);
        }
    } else if (warp == 2) {
        // ------------------------ packed-weight producer ----------------------
        if (lane == 0) {
            prefetch_tensormap(&tm_w);
            int issued = 0;
            for (int kt = 0; kt < (stall ? 0 : nk); ++kt) {
                const int s = kt % kStagesP;
                if (kt >= kStagesP && !mbar_wait_n(&empty_p[s], ((kt / kStagesP) - 1) & 1, lim)) {
                    timed_out = true;
                    break;
                }
                mbar_arrive_expect_tx(&full_p[s], kPBytes);
                tma_load_2d(smem + kOffP + s * kPBytes, &tm_w, kt * (kBK / 2), static_cast<int32_t>(n0),
                            &full_p[s]);
                issued = kt + 1;
            }
            if (timed_out)
                for (int kt = (issued > kStagesP ? issued - kStagesP : 0); kt < issued; ++kt)
                    mbar_wait_n(&full_p[kt % kStagesP], (kt / kStagesP) & 1, kWaitLimit);
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ----------------------------
        if (lane == 0) {
            for (int kt = 0; kt < nk; ++kt) {
                const int sa = kt % kStagesA;
                const int sb = kt % kStagesB;
                if (!mbar_wait_n(&full_a[sa], (kt / kStagesA) & 1, lim) || !mbar_wait_n(&full_b[sb], (kt / kStagesB) & 1, lim)) {
                    timed_out = true;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = sbase + sa * kABytes;
                const uint32_t b_addr = sbase + kOffB + sb * kBBytes;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int j = 0; j < kBK / 16; ++j)
                        tc_mma_bf16(tmem + h * 256, smem_desc_sw128(a_addr + h * (128 * 128) + 32 * j),
                                    smem_desc_sw128(b_addr + 32 * j), kIdesc, (kt > 0 || j > 0) ? 1u : 0u);
                tc_commit(&empty_a[sa]);
                tc_commit(&empty_b[sb]);
            }
            if (kLora && lora_tc && !timed_out) {
                // Low-rank term on the tensor cores: Y += t_hi up^T + t_lo up^T, with
                // t = t_hi + t_lo (two bf16 halves) and up as the B operand, in K
                // tiles of 64 ranks (zero-filled past r) loaded into the stage
                // buffers once every main-loop MMA has read them.
                const int nlt = (lora_r + 63) / 64;
                for (int lt = 0; lt < nlt && !timed_out; ++lt) {
                    tc_commit(mma_done);
                    if (!mbar_wait_n(mma_done, lt & 1, lim)) {
                        timed_out = true;
                        break;
                    }
                    mbar_arrive_expect_tx(lora_full, 3 * kABytes);
                    tma_load_2d(smem, &tm_thi, lt * 64, static_cast<int32_t>(m0), lora_full);
                    tma_load_2d(smem + kABytes, &tm_tlo, lt * 64, static_cast<int32_t>(m0), lora_full);
                    tma_load_2d(smem + 2 * kABytes, &tm_up, lt * 64, static_cast<int32_t>(n0), lora_full);
                    if (!mbar_wait_n(lora_full, lt & 1, lim)) {
                        timed_out = true;
                        break;
                    }
                    tc_fence_after();
                    const int ks = ((lora_r - lt * 64 < 64 ? lora_r - lt * 64 : 64) + 15) / 16;
                    for (int h = 0; h < 2; ++h)
                        for (int j = 0; j < ks; ++j) {
                            const uint64_t bd = smem_desc_sw128(sbase + 2 * kABytes + 32 * j);
                            tc_mma_bf16(tmem + h * 256, smem_desc_sw128(sbase + h * (128 * 128) + 32 * j), bd, kIdesc, 1u);
                            tc_mma_bf16(tmem + h * 256, smem_desc_sw128(sbase + kABytes + h * (128 * 128) + 32 * j), bd,
                                        kIdesc, 1u);
                        }
                }
            }
            tc_commit(timed_out ? drained : acc_ready);
            if (timed_out) mbar_wait_n(drained, 0, kWaitLimit);  // issued MMAs finish before TMEM is freed
        }
    } else if (warp >= 4) {
        // ------------------------ dequantize, then epilogue --------------------
        const int t = threadIdx.x - 128;  // weight row of the tile
        const int64_t row_c = (n0 + t < n) ? n0 + t : n - 1;  // rows past n: computed, never stored
        const int64_t kblocks = k / 64;
        const float mu = __ldg(mu_ptr);
        uint64_t cpair[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) cpair[j] = pack_f32x2(kCodebook[codebook][2 * j], kCodebook[codebook][2 * j + 1]);
        const uint32_t prow = sbase + kOffP + t * 32;
        const uint32_t brow = sbase + kOffB + t * 128;
        const uint32_t swz = static_cast<uint32_t>(t & 7);
        // Absmax inputs.  With k % 256 == 0 (and an aligned code array) the codes
        // of 4 consecutive stages are one aligned word and share one scale (a
        // group of 4 blocks never straddles a 256-block boundary); each group is
        // loaded one group ahead so the load latency hides behind 4 stages.
        const bool grouped = (kblocks & 3) == 0 && (reinterpret_cast<uintptr_t>(absmax_q) & 3) == 0;
        const int64_t rbase = row_c * kblocks;
        uint32_t qw_next = 0, qw_cur = 0;
        float s_next = 0.0f, s_cur = 0.0f;
        if (grouped) {
            qw_next = __ldg(reinterpret_cast<const uint32_t*>(absmax_q + rbase));
            s_next = __ldg(absmax_scale + (rbase >> 8));
        }
        for (int kt = 0; kt < nk; ++kt) {
            const int sp = kt % kStagesP;
            const int sb = kt % kStagesB;
            int q;
            float sc;
            if (grouped) {
                if ((kt & 3) == 0) {
                    qw_cur = qw_next;
                    s_cur = s_next;
                    const int64_t nb = rbase + ((kt + 4 < nk) ? kt + 4 : kt);
                    qw_next = __ldg(reinterpret_cast<const uint32_t*>(absmax_q + nb));
                    s_next = __ldg(absmax_scale + (nb >> 8));
                }
                q = static_cast<int8_t>((qw_cur >> (8 * (kt & 3))) & 0xffu);
                sc = s_cur;
            } else {
                const int64_t bidx = rbase + kt;
                q = __ldg(absmax_q + bidx);
                sc = __ldg(absmax_scale + (bidx >> 8));
            }
            if (!__all_sync(kFull, mbar_wait_n(&full_p[sp], (kt / kStagesP) & 1, lim))) {
                timed_out = true;
                break;
            }
            const uint4 r0 = lds128(prow + sp * kPBytes);
            const uint4 r1 = lds128(prow + sp * kPBytes + 16);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_p[sp]);
            Planes P;
            build_planes(cpair, absmax_hat(q, sc, mu), P);
            if (kt >= kStagesB && !__all_sync(kFull, mbar_wait_n(&empty_b[sb], ((kt / kStagesB) - 1) & 1, lim))) {
                timed_out = true;
                break;
            }
            const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
            const uint32_t bst = brow + sb * kBBytes;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t x = w[c] ^ 0x88888888u;
                uint32_t o0, o1, o2, o3;
                decode4(w[c], x, P, o0, o1);
                decode4(w[c] >> 16, x >> 16, P, o2, o3);
                sts128(bst + ((c ^ swz) << 4), o0, o1, o2, o3);
            }
            fence_proxy_async_shared();  // generic-proxy writes -> tensor-core reads
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_b[sb]);
        }
        // epilogue: accumulators -> Y
        const bool ok = !timed_out && __all_sync(kFull, mbar_wait_n(acc_ready, 0, lim));
        if (!ok) timed_out = true;
        tc_fence_after();
        const int wd = warp - 4;
        const int half = wd >> 2;
        const int quarter = warp & 3;  // tensor-memory lanes this warp may access
        const int64_t tok = m0 + half * 128 + quarter * 32 + lane;
        const bool vec = kBf16Out ? (n % 8 == 0) : (n % 4 == 0);
#pragma unroll 1
        for (int cc = 0; cc < kBN / 32; ++cc) {
            uint32_t r[32];
            if (ok) tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + half * 256 + cc * 32, r);
            const int64_t col0 = n0 + cc * 32;
            if (!ok || tok >= m || col0 >= n) continue;
            if (kLora && !lora_tc) {
                // low-rank term on the CUDA cores (rank not a multiple of 8):
                // + sum_j t[tok, j] * up[col, j], j ascending for every column
                const float* tr = lora_t + tok * lora_r;
                if ((lora_r & 7) == 0) {  // 16-byte aligned rows: 8 ranks per load
                    for (int j = 0; j < lora_r; j += 8) {
                        const float4 t0 = __ldg(reinterpret_cast<const float4*>(tr + j));
                        const float4 t1 = __ldg(reinterpret_cast<const float4*>(tr + j + 4));
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            if (col0 + e >= n) continue;
                            const uint4 u = __ldg(reinterpret_cast<const uint4*>(lora_up + (col0 + e) * lora_r + j));
                            float v = __uint_as_float(r[e]);
                            v = __fmaf_rn(t0.x, bf16_bits_to_float(u.x & 0xffffu), v);
                            v = __fmaf_rn(t0.y, bf16_bits_to_float(u.x >> 16), v);
                            v = __fmaf_rn(t0.z, bf16_bits_to_float(u.y & 0xffffu), v);
                            v = __fmaf_rn(t0.w, bf16_bits_to_float(u.y >> 16), v);
                            v = __fmaf_rn(t1.x, bf16_bits_to_float(u.z & 0xffffu), v);
                            v = __fmaf_rn(t1.y, bf16_bits_to_float(u.z >> 16), v);
                            v = __fmaf_rn(t1.z, bf16_bits_to_float(u.w & 0xffffu), v);
                            v = __fmaf_rn(t1.w, bf16_bits_to_float(u.w >> 16), v);
                            r[e] = __float_as_uint(v);
                        }
                    }
                } else {
                    for (int j = 0; j < lora_r; ++j) {
                        const float tv = __ldg(tr + j);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (col0 + e < n)
                                r[e] = __float_as_uint(__fmaf_rn(tv, __bfloat162float(lora_up[(col0 + e) * lora_r + j]),
                                                                 __uint_as_float(r[e])));
                    }
                }
            }
            if (kBf16Out) {
                __nv_bfloat16* yrow = reinterpret_cast<__nv_bfloat16*>(Y) + tok * n;
                if (vec && col0 + 32 <= n) {
                    uint32_t p[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        p[e] = pack_bf16x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
                    uint4* dst = reinterpret_cast<uint4*>(yrow + col0);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = make_uint4(p[4 * e], p[4 * e + 1], p[4 * e + 2], p[4 * e + 3]);
                } else {
                    for (int e = 0; e < 32 && col0 + e < n; ++e) yrow[col0 + e] = __float2bfloat16_rn(__uint_as_float(r[e]));
                }
            } else {
                float* yrow = reinterpret_cast<float*>(Y) + tok * n;
                if (vec && col0 + 32 <= n) {
                    uint4* dst = reinterpret_cast<uint4*>(yrow + col0);
#pragma unroll
                    for (int e = 0; e < 8; ++e) dst[e] = make_uint4(r[4 * e], r[4 * e + 1], r[4 * e + 2], r[4 * e + 3]);
                } else {
                    for (int e = 0; e < 32 && col0 + e < n; ++e) yrow[col0 + e] = __uint_as_float(r[e]);
                }
            }
        }
    }
    if (timed_out) record_timeout(dev_status);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Backward through the frozen base: dX[m, k] = dY[m, n] * What[n, k] (page "Tim
// Dettmers 如何用 bitsandbytes 與 QLoRA 降低 LLM 訓練門檻？", section "QLoRA 把 frozen
// 4-bit base 與可訓練 adapter 分開": the base is dequantized to the compute dtype in
// the backward pass as in the forward one).
//
// One CTA computes a 256 (tokens) x 256 (columns of W) tile of dX and loops over
// the rows of W, the contraction, 64 per stage.  The decoded tile is laid out
// like the forward's -- rows of 64 consecutive columns, 128-byte swizzled --
// which is the MN-major operand layout with N = columns (contiguous) and K =
// rows: four 64-column blocks of 64 rows, 8 KB each.  Warp 0 streams dY tiles
// [256 x 64] (K-major, like X in the forward), warp 2 the packed codes
// [64 rows x 128 B] (swizzled, so each dequant warp's reads hit distinct
// banks), warps 4..11 decode one (row, 64-column block) per thread per stage,
// warp 1 issues the MMAs with the weight as the MN-major B operand.
// ---------------------------------------------------------------------------
constexpr int kBKX = 64;                            // rows of W per stage (MMA K)
constexpr uint32_t kIdescDx = kIdesc | (1u << 16);  // B (the weight) MN-major

// MN-major, 128-byte swizzle: the leading byte offset is the stride between
// 64-column blocks (8 KB), the stride byte offset between 8-row groups (1 KB).
__device__ __forceinline__ uint64_t smem_desc_sw128_mn(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>(8192 >> 4) << 16;
    d |= static_cast<uint64_t>(1024 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

template <bool kBf16Out>
__global__ void __launch_bounds__(kThreads, 1)
k_nf4_gemm_dx(const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_w,
              const int8_t* __restrict__ absmax_q, const float* __restrict__ absmax_scale,
              const float* __restrict__ mu_ptr, int64_t m, int64_t n, int64_t k, void* __restrict__ dX,
              int32_t* __restrict__ dev_status, int codebook) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* full_a = bars;
    uint64_t* empty_a = full_a + kStagesA;
    uint64_t* full_b = empty_a + kStagesA;
    uint64_t* empty_b = full_b + kStagesB;
    uint64_t* full_p = empty_b + kStagesB;
    uint64_t* empty_p = full_p + kStagesP;
    uint64_t* acc_ready = empty_p + kStagesP;
    uint64_t* drained = acc_ready + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kBN;  // first column of W (and of dX)
    const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kBM;
    const int nr = static_cast<int>((n + kBKX - 1) / kBKX);
    const uint32_t sbase = smem_u32(smem);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesA; ++s) {
            mbar_init(&full_a[s], 1);
            mbar_init(&empty_a[s], 1);
        }
        for (int s = 0; s < kStagesB; ++s) {
            mbar_init(&full_b[s], kDequantWarps);
            mbar_init(&empty_b[s], 1);
        }
        for (int s = 0; s < kStagesP; ++s) {
            mbar_init(&full_p[s], 1);
            mbar_init(&empty_p[s], kDequantWarps);
        }
        mbar_init(acc_ready, 1);
        mbar_init(drained, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool timed_out = false;
    if (warp == 0) {
        // ---------------------------- dY producer ----------------------------
        if (lane == 0) {
            prefetch_tensormap(&tm_dy);
            int issued = 0;
            for (int rt = 0; rt < nr; ++rt) {
                const int s = rt % kStagesA;
                if (rt >= kStagesA && !mbar_wait(&empty_a[s], ((rt / kStagesA) - 1) & 1)) {
                    timed_out = true;
                    break;
                }
                mbar_arrive_expect_tx(&full_a[s], kABytes);
                tma_load_2d(smem + s * kABytes, &tm_dy, rt * kBKX, static_cast<int32_t>(m0), &full_a[s]);
                issued = rt + 1;
            }
            if (timed_out)  // leave no copy in flight
                for (int rt = (issued > kStagesA ? issued - kStagesA : 0); rt < issued; ++rt)
                    mbar_wait(&full_a[rt % kStagesA], (rt / kStagesA) & 1);
        }
    } else if (warp == 2) {
        // ------------------------ packed-weight producer ----------------------
        if (lane == 0) {
            prefetch_tensormap(&tm_w);
            int issued = 0;
            for (int rt = 0; rt < nr; ++rt) {
                const int s = rt % kStagesP;
                if (rt >= kStagesP && !mbar_wait(&empty_p[s], ((rt / kStagesP) - 1) & 1)) {
                    timed_out = true;
                    break;
                }
                mbar_arrive_expect_tx(&full_p[s], kPBytes);
                tma_load_2d(smem + kOffP + s * kPBytes, &tm_w, static_cast<int32_t>(c0 / 2), rt * kBKX, &full_p[s]);
                issued = rt + 1;
            }
            if (timed_out)
                for (int rt = (issued > kStagesP ? issued - kStagesP : 0); rt < issued; ++rt)
                    mbar_wait(&full_p[rt % kStagesP], (rt / kStagesP) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ----------------------------
        if (lane == 0) {
            for (int rt = 0; rt < nr; ++rt) {
                const int sa = rt % kStagesA;
                const int sb = rt % kStagesB;
                if (!mbar_wait(&full_a[sa], (rt / kStagesA) & 1) || !mbar_wait(&full_b[sb], (rt / kStagesB) & 1)) {
                    timed_out = true;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = sbase + sa * kABytes;
                const uint32_t b_addr = sbase + kOffB + sb * kBBytes;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int j = 0; j < kBKX / 16; ++j)
                        tc_mma_bf16(tmem + h * 256, smem_desc_sw128(a_addr + h * (128 * 128) + 32 * j),
                                    smem_desc_sw128_mn(b_addr + 2048 * j), kIdescDx, (rt > 0 || j > 0) ? 1u : 0u);
                tc_commit(&empty_a[sa]);
                tc_commit(&empty_b[sb]);
            }
            tc_commit(timed_out ? drained : acc_ready);
            if (timed_out) mbar_wait(drained, 0);  // issued MMAs finish before TMEM is freed
        }
    } else if (warp >= 4) {
        // ------------------------ dequantize, then epilogue --------------------
        const int t = threadIdx.x - 128;
        const int r = t & (kBKX - 1);  // row of the stage
        const int cb = t >> 6;         // 64-column block of the tile
        const int64_t kblocks = k / 64;
        int64_t colblk = c0 / 64 + cb;  // blocks past k: computed, never stored
        if (colblk > kblocks - 1) colblk = kblocks - 1;
        const float mu = __ldg(mu_ptr);
        uint64_t cpair[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) cpair[j] = pack_f32x2(kCodebook[codebook][2 * j], kCodebook[codebook][2 * j + 1]);
        const uint32_t swz = static_cast<uint32_t>(r & 7);
        const uint32_t prow = sbase + kOffP + r * 128;
        const uint32_t brow = sbase + kOffB + cb * (kBKX * 128) + r * 128;
        // absmax inputs of (row rt * 64 + r, colblk), one stage ahead; rows past
        // n are clamped (their codes and dY are zero-filled, so they add nothing)
        auto row_of = [&](int rt) {
            const int64_t row = static_cast<int64_t>(rt) * kBKX + r;
            return row < n ? row : n - 1;
        };
        int64_t bidx = row_of(0) * kblocks + colblk;
        int q_next = __ldg(absmax_q + bidx);
        float s_next = __ldg(absmax_scale + (bidx >> 8));
        for (int rt = 0; rt < nr; ++rt) {
            const int sp = rt % kStagesP;
            const int sb = rt % kStagesB;
            const int q = q_next;
            const float sc = s_next;
            bidx = row_of(rt + 1 < nr ? rt + 1 : rt) * kblocks + colblk;
            q_next = __ldg(absmax_q + bidx);
            s_next = __ldg(absmax_scale + (bidx >> 8));
            if (!__all_sync(kFull, mbar_wait(&full_p[sp], (rt / kStagesP) & 1))) {
                timed_out = true;
                break;
            }
            const uint4 r0 = lds128(prow + sp * kPBytes + ((((2 * cb) ^ static_cast<int>(swz))) << 4));
            const uint4 r1 = lds128(prow + sp * kPBytes + ((((2 * cb + 1) ^ static_cast<int>(swz))) << 4));
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_p[sp]);
            Planes P;
            build_planes(cpair, absmax_hat(q, sc, mu), P);
            if (rt >= kStagesB && !__all_sync(kFull, mbar_wait(&empty_b[sb], ((rt / kStagesB) - 1) & 1))) {
                timed_out = true;
                break;
            }
            const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
            const uint32_t bst = brow + sb * kBBytes;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t x = w[c] ^ 0x88888888u;
                uint32_t o0, o1, o2, o3;
                decode4(w[c], x, P, o0, o1);
                decode4(w[c] >> 16, x >> 16, P, o2, o3);
                sts128(bst + ((c ^ swz) << 4), o0, o1, o2, o3);
            }
            fence_proxy_async_shared();  // generic-proxy writes -> tensor-core reads
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_b[sb]);
        }
        // epilogue: accumulators -> dX
        const bool ok = !timed_out && __all_sync(kFull, mbar_wait(acc_ready, 0));
        if (!ok) timed_out = true;
        tc_fence_after();
        const int wd = warp - 4;
        const int half = wd >> 2;
        const int quarter = warp & 3;  // tensor-memory lanes this warp may access
        const int64_t tok = m0 + half * 128 + quarter * 32 + lane;
        const bool vec = kBf16Out ? (k % 8 == 0) : (k % 4 == 0);
#pragma unroll 1
        for (int cc = 0; cc < kBN / 32; ++cc) {
            uint32_t rr[32];
            if (ok) tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + half * 256 + cc * 32, rr);
            const int64_t col0 = c0 + cc * 32;
            if (!ok || tok >= m || col0 >= k) continue;
            if (kBf16Out) {
                __nv_bfloat16* drow = reinterpret_cast<__nv_bfloat16*>(dX) + tok * k;
                if (vec && col0 + 32 <= k) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = pack_bf16x2(__uint_as_float(rr[2 * e]), __uint_as_float(rr[2 * e + 1]));
                    uint4* dst = reinterpret_cast<uint4*>(drow + col0);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                } else {
                    for (int e = 0; e < 32 && col0 + e < k; ++e) drow[col0 + e] = __float2bfloat16_rn(__uint_as_float(rr[e]));
                }
            } else {
                float* drow = reinterpret_cast<float*>(dX) + tok * k;
                if (vec && col0 + 32 <= k) {
                    uint4* dst = reinterpret_cast<uint4*>(drow + col0);
#pragma unroll
                    for (int e = 0; e < 8; ++e) dst[e] = make_uint4(rr[4 * e], rr[4 * e + 1], rr[4 * e + 2], rr[4 * e + 3]);
                } else {
                    for (int e = 0; e < 32 && col0 + e < k; ++e) drow[col0 + e] = __uint_as_float(rr[e]);
                }
            }
        }
    }
    if (timed_out) record_timeout(dev_status);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace gemm

cudaError_t launch_gemm(const void* X, int64_t m, const uint8_t* wq, const int8_t* absmax_q,
                        const float* absmax_scale, const float* absmax_offset, int64_t n, int64_t k, void* Y,
                        bool y_bf16, int32_t* dev_status, const LoraArgs& lora, int codebook,
                        uint32_t test_flags, const DeviceInfo& dev, cudaStream_t stream) {
    static bool attr_set[64][4] = {};
    if (dev.device < 0 || dev.device >= 64) return cudaErrorInvalidDevice;
    const bool lo = lora.t != nullptr;
    const void* fn = y_bf16 ? (lo ? reinterpret_cast<const void*>(&gemm::k_nf4_gemm<true, true>)
                                  : reinterpret_cast<const void*>(&gemm::k_nf4_gemm<true, false>))
                            : (lo ? reinterpret_cast<const void*>(&gemm::k_nf4_gemm<false, true>)
                                  : reinterpret_cast<const void*>(&gemm::k_nf4_gemm<false, false>));
    const int vi = (y_bf16 ? 1 : 0) + (lo ? 2 : 0);
    {
        static std::mutex mu;
        std::lock_guard<std::mutex> lock(mu);
        if (!attr_set[dev.device][vi]) {
            const cudaError_t e =
                cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm::kSmemBytes);
            if (e != cudaSuccess) return e;
            attr_set[dev.device][vi] = true;
        }
    }
    CUtensorMap tm_x, tm_w;
    cudaError_t e = tmap_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, static_cast<uint64_t>(k),
                            static_cast<uint64_t>(m), static_cast<uint64_t>(k * 2), gemm::kBK, gemm::kBM,
                            CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    e = tmap_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, wq, static_cast<uint64_t>(k / 2), static_cast<uint64_t>(n),
                static_cast<uint64_t>(k / 2), gemm::kBK / 2, gemm::kBN, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>((n + gemm::kBN - 1) / gemm::kBN),
                    static_cast<unsigned>((m + gemm::kBM - 1) / gemm::kBM));
    // the low-rank term on the tensor cores needs 16-byte rows of t_hi / t_lo / up (r % 8 == 0)
    int lora_tc = 0;
    CUtensorMap tm_thi = tm_x, tm_tlo = tm_x, tm_up = tm_x;  // unused unless lora_tc
    if (lo && lora.t_hi && lora.t_lo && lora.r % 8 == 0) {
        const uint64_t rr = static_cast<uint64_t>(lora.r);
        e = tmap_2d(&tm_thi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora.t_hi, rr, static_cast<uint64_t>(m), rr * 2,
                    64, gemm::kBM, CU_TENSOR_MAP_SWIZZLE_128B);
        if (e != cudaSuccess) return e;
        e = tmap_2d(&tm_tlo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora.t_lo, rr, static_cast<uint64_t>(m), rr * 2,
                    64, gemm::kBM, CU_TENSOR_MAP_SWIZZLE_128B);
        if (e != cudaSuccess) return e;
        e = tmap_2d(&tm_up, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora.up, rr, static_cast<uint64_t>(n), rr * 2,
                    64, gemm::kBN, CU_TENSOR_MAP_SWIZZLE_128B);
        if (e != cudaSuccess) return e;
        lora_tc = 1;
    }
#define NF4_GEMM_LAUNCH(B, L)                                                                               \
    gemm::k_nf4_gemm<B, L><<<grid, gemm::kThreads, gemm::kSmemBytes, stream>>>(                              \
        tm_x, tm_w, absmax_q, absmax_scale, absmax_offset, m, n, k, Y, dev_status, lora.t, lora.up, lora.r,  \
        lora_tc, tm_thi, tm_tlo, tm_up, codebook, (test_flags & kTestStall) ? 64u : kWaitLimit,            \
        (test_flags & kTestStall) ? 1 : 0)
    if (y_bf16) {
        if (lo) NF4_GEMM_LAUNCH(true, true); else NF4_GEMM_LAUNCH(true, false);
    } else {
        if (lo) NF4_GEMM_LAUNCH(false, true); else NF4_GEMM_LAUNCH(false, false);
    }
#undef NF4_GEMM_LAUNCH
    return cudaGetLastError();
}

cudaError_t launch_gemm_dx(const void* dY, int64_t m, const uint8_t* wq, const int8_t* absmax_q,
                           const float* absmax_scale, const float* absmax_offset, int64_t n, int64_t k, void* dX,
                           bool dx_bf16, int32_t* dev_status, int codebook, const DeviceInfo& dev,
                           cudaStream_t stream) {
    static bool attr_set[64][2] = {};
    if (dev.device < 0 || dev.device >= 64) return cudaErrorInvalidDevice;
    const void* fn = dx_bf16 ? reinterpret_cast<const void*>(&gemm::k_nf4_gemm_dx<true>)
                             : reinterpret_cast<const void*>(&gemm::k_nf4_gemm_dx<false>);
    {
        static std::mutex mu;
        std::lock_guard<std::mutex> lock(mu);
        if (!attr_set[dev.device][dx_bf16]) {
            const cudaError_t e =
                cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm::kSmemBytes);
            if (e != cudaSuccess) return e;
            attr_set[dev.device][dx_bf16] = true;
        }
    }
    CUtensorMap tm_dy, tm_w;
    // dY [m, n] bf16, K-major boxes [256 tokens x 64 rows of W]
    cudaError_t e = tmap_2d(&tm_dy, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY, static_cast<uint64_t>(n),
                            static_cast<uint64_t>(m), static_cast<uint64_t>(n * 2), gemm::kBKX, gemm::kBM,
                            CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    // codes [n, k/2] bytes, boxes [64 rows x 128 B] (256 columns), 128-byte swizzled
    e = tmap_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, wq, static_cast<uint64_t>(k / 2), static_cast<uint64_t>(n),
                static_cast<uint64_t>(k / 2), gemm::kBN / 2, gemm::kBKX, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>((k + gemm::kBN - 1) / gemm::kBN),
                    static_cast<unsigned>((m + gemm::kBM - 1) / gemm::kBM));
    if (dx_bf16)
        gemm::k_nf4_gemm_dx<true><<<grid, gemm::kThreads, gemm::kSmemBytes, stream>>>(
            tm_dy, tm_w, absmax_q, absmax_scale, absmax_offset, m, n, k, dX, dev_status, codebook);
    else
        gemm::k_nf4_gemm_dx<false><<<grid, gemm::kThreads, gemm::kSmemBytes, stream>>>(
            tm_dy, tm_w, absmax_q, absmax_scale, absmax_offset, m, n, k, dX, dev_status, codebook);
    return cudaGetLastError();
}

}  // namespace nf4
