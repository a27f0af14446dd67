// nf4_gemv.cu -- fused dequantize + linear for decode-sized batches (m <= 16), sm_100a.
//
// Sources: page "篇2-bitsandbytes-具体观-算法与实现剖析" (xyzblog), §2.2 code walk
// (matmul_4bit = dequantize + matmul); page "LLM 相關知識" (technicalnotes), §5
// "動態反量化" (weights restored to BF16 per layer for the matmul, then dropped);
// page "Tim Dettmers 如何用 bitsandbytes 與 QLoRA 降低 LLM 訓練門檻？", section "量化速度
// 取決於硬體與 kernel，不只位元數" (unfused 4-bit can lose to fp16; batch size moves the
// work between memory- and compute-bound).
//
//   Y[t, r] = sum_c X[t, c] * What[r, c],   What[r, c] = bf16(fp32(level[idx] * a_block)).
//
// The operation is HBM-bound: per weight 0.5 B of codes plus 1/64 B of absmax
// code must stream from HBM.  Design (one CTA = 128 weight rows x a slice of k,
// eight warps, two CTAs per SM):
//
// * Rings in shared memory, filled by TMA (no multicast): 3 slots of packed
//   codes [128 rows x 128 B] and 3 slots of X [16 tokens x 256], both 128-byte
//   swizzled so that the fragment reads are bank-conflict free.  A warp copies
//   its codes of a stage into registers first and then leaves the codes slot;
//   the last warp out refills it at once, so the next load overlaps the decode.
//   X slots are refilled the same way after the stage is done.  mbarriers carry
//   the TMA byte counts; every wait is bounded.
// * Reconstructed absmax a = fp32(fp32(fp32(q / 127) * s) + mu): every thread
//   computes two of the stage's 512 values one stage ahead (its inputs are
//   loaded three stages ahead) into a 4-deep table ring.
// * Warp w owns rows 32 (w mod 4) .. + 31 and 64-blocks 2 (w div 4) + {0, 1} of
//   every stage.  The multiply-adds run on the tensor cores (mma.sync m16n8k16,
//   bf16 in, fp32 accumulate) with the 16 token slots as the MMA's M side
//   (zero-filled beyond m) and 8 weight rows as its N side.  Each lane owns 16
//   consecutive weights of a block row; the MMA k order is a permutation of the
//   true k order applied identically to X and the weights.
// * Decode: a 256-entry table maps a packed byte to the two fp32 levels it
//   encodes (replicated 16x so a half-warp's lookups never share a bank); each
//   level is multiplied by the block's reconstructed absmax in fp32 and rounded
//   to bf16 -- the same values nf4_dequantize produces.
// * Split-k: the CTAs of a thread-block cluster share a row tile and split k.
//   Each rank pushes the partial sums of the rows another rank owns into that
//   rank's shared memory; the owner adds them in rank order, so results are
//   deterministic and no global scratch is needed.
#include "nf4_common.cuh"
#include "nf4_internal.h"
#include "nf4_ptx.cuh"
#include "nf4_tmap.h"

namespace nf4 {
namespace gemv {

constexpr int kRows = 128;                       // weight rows per CTA
constexpr int kStageK = 256;                     // k per pipeline stage
constexpr int kRing = 3;                         // stages in flight per CTA
constexpr int kConsumers = 8;                    // consumer warps
constexpr int kTiles = 4;                        // 8-row MMA tiles per warp (32 rows) and block
constexpr int kThreads = 32 * kConsumers;        // no dedicated producer warp
constexpr int kWBytes = kRows * kStageK / 2;     // 16384: packed codes of a stage
constexpr int kXBox = 16 * 64 * 2;               // 2048: X box of 16 tokens x 64 k (bf16)
constexpr int kXBytes = 4 * kXBox;               // 8192
constexpr int kAring = 4;                        // reconstructed-absmax tables in flight
constexpr int kAhatBytes = 4 * kRows * 4;        // 2048: one stage's table, [row][block]
constexpr int kLutBytes = 16 * 256 * 8;          // 32768
constexpr int kXRingOff = kRing * kWBytes;       // codes ring first, then the X ring
constexpr int kRingBytes = kRing * (kWBytes + kXBytes);
constexpr int kAhatOff = kRingBytes;
constexpr int kLutOff = kAhatOff + kAring * kAhatBytes;
constexpr int kBarOff = kLutOff + kLutBytes;
// two CTAs per SM: (113 KiB + 1 KiB reserved) x 2 within the SM's 228 KiB
constexpr int kSmemBytes = kBarOff + (2 * kRing + kAring + 1) * 8 + 4 * kRing * 4;
static_assert(kWBytes % 1024 == 0 && kXBytes % 1024 == 0, "slots keep the 1 KiB alignment the 128-byte swizzle needs");
static_assert(kSmemBytes + 1024 <= 228 * 1024 / 2, "two CTAs fit on an SM");
// Per-block partial sums are stored [token][row] with a padded token pitch so
// that the 8 row groups of a warp write distinct banks.
constexpr int kRedPitch = kRows + 8;
// Epilogue buffers, all inside the (then idle) ring: the two per-block-pair
// partials, the CTA's folded partial [token][row], and the split-k receive
// area [sender][token][rows of this rank].
constexpr int kPartOff = 2 * 16 * kRedPitch * 4;
constexpr int kRecvOff = kPartOff + 16 * kRows * 4;
static_assert(kRecvOff + 16 * kRows * 4 <= kRingBytes, "reduction fits in the ring");

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte `b` (0..3) of `word` in the low 8 bits, zeros above (one byte permute).
__device__ __forceinline__ uint32_t byte_of(uint32_t word, uint32_t b) {
    uint32_t d;
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(d) : "r"(word), "r"(0x4440u | b));
    return d;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint64_t lds_b64(uint32_t addr) {
    uint64_t v;
    asm volatile("ld.shared.b64 %0, [%1];" : "=l"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint64_t dup_f32x2(float a) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(a));
    return r;
}

// Two levels (one packed byte) times the block's absmax, each product rounded
// to fp32 (one packed f32x2 multiply), then both rounded to bf16: the high
// nibble (lower k) lands in the low half.
__device__ __forceinline__ uint32_t scale_pack(uint64_t levels, uint64_t aa) {
    uint32_t out;
    asm("{\n\t.reg .b64 r;\n\t.reg .f32 lo, hi;\n\t"
        "mul.rn.f32x2 r, %1, %2;\n\t"
        "mov.b64 {lo, hi}, r;\n\t"
        "cvt.rn.bf16x2.f32 %0, hi, lo;\n\t}"
        : "=r"(out)
        : "l"(levels), "l"(aa));
    return out;
}

// Reconstructed-absmax inputs of one stage for one thread.  Thread t owns row
// (t mod 128) of the tile and blocks 2 (t div 128) + {0, 1} of the stage: the
// row's 4 int8 codes of the stage packed in one word, and the
// double-quantization scales of the thread's two blocks.
struct AbsmaxIn {
    uint32_t q;
    float s0, s1;
};

__device__ __forceinline__ void load_absmax_in(AbsmaxIn& a, const int8_t* __restrict__ absmax_q,
                                               const float* __restrict__ absmax_scale, int64_t grow, int half,
                                               int st, int64_t n, int64_t kblocks, bool aligned4) {
    const int64_t kb = static_cast<int64_t>(st) * 4;
    if (aligned4) {
        // k % 256 == 0 and an aligned code array: a row's 4 codes of a stage are
        // one aligned word.  Every load is unconditional (rows past n are
        // clamped; their results are never stored), so nothing waits for it
        // until the stage is used.
        const int64_t r = grow < n ? grow : n - 1;
        const int64_t b0 = r * kblocks + kb + 2 * half;
        a.q = __ldg(reinterpret_cast<const uint32_t*>(absmax_q + (b0 - 2 * half)));
        a.s0 = __ldg(absmax_scale + (b0 >> 8));
        a.s1 = __ldg(absmax_scale + ((b0 + 1) >> 8));
        return;
    }
    // general shapes: gather the codes byte by byte; blocks past k get q = 0
    uint32_t q = 0;
    float s0 = 0.0f, s1 = 0.0f;
    if (grow < n) {
        const int64_t b0 = grow * kblocks + kb;
        const int64_t nvalid = kblocks - kb;  // >= 1
#pragma unroll
        for (int b = 0; b < 4; ++b)
            if (b < nvalid) q |= static_cast<uint32_t>(static_cast<uint8_t>(__ldg(absmax_q + b0 + b))) << (8 * b);
        const int64_t last = b0 + (nvalid < 4 ? nvalid : 4) - 1;
        const int64_t ba = b0 + 2 * half, bb = ba + 1;
        s0 = __ldg(absmax_scale + ((ba < last ? ba : last) >> 8));
        s1 = __ldg(absmax_scale + ((bb < last ? bb : last) >> 8));
    }
    a.q = q;
    a.s0 = s0;
    a.s1 = s1;
}

// Keeps the compiler from hoisting work that uses `a` above the point where
// this is called (the values pass through an opaque asm).
__device__ __forceinline__ void pin(AbsmaxIn& a) {
    asm volatile("" : "+r"(a.q), "+f"(a.s0), "+f"(a.s1));
}

// a = fp32(fp32(fp32(q / 127) * s) + mu) for the thread's two blocks, stored
// to the stage's [row][block] table.
__device__ __forceinline__ void store_ahat(uint32_t ahat_row, int half, const AbsmaxIn& a, float mu) {
    const uint32_t qq = a.q >> (16 * half);
    const float q0 = static_cast<float>(static_cast<int8_t>(qq & 0xffu));
    const float q1 = static_cast<float>(static_cast<int8_t>((qq >> 8) & 0xffu));
    const float a0 = __fadd_rn(__fmul_rn(div127(q0), a.s0), mu);
    const float a1 = __fadd_rn(__fmul_rn(div127(q1), a.s1), mu);
    asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(ahat_row + 8u * half), "f"(a0), "f"(a1) : "memory");
}

constexpr int kPrefetch = 3;  // stages of absmax inputs in flight per thread

// Codes [128 rows x 128 B] of stage `st` into a codes slot.
__device__ __forceinline__ void issue_w(uint8_t* dst, const CUtensorMap* tm_w, uint64_t* bar, int st, int64_t row0) {
    mbar_arrive_expect_tx(bar, kWBytes);
    tma_load_2d(dst, tm_w, st * (kStageK / 2), static_cast<int32_t>(row0), bar);
}

// X [16 tokens x 256] of stage `st` (4 boxes of 64 columns) into an X slot.
__device__ __forceinline__ void issue_x(uint8_t* dst, const CUtensorMap* tm_x, uint64_t* bar, int st) {
    mbar_arrive_expect_tx(bar, kXBytes);
#pragma unroll
    for (int b = 0; b < 4; ++b) tma_load_2d(dst + b * kXBox, tm_x, st * kStageK + 64 * b, 0, bar);
}

// Counts a warp out of a ring slot; acquire-release so that the warp's reads
// of the slot are ordered before the refill that the last warp issues.
__device__ __forceinline__ uint32_t slot_leave(uint32_t* counter) {
    uint32_t old;
    asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;" : "=r"(old) : "r"(smem_u32(counter)) : "memory");
    return old;
}

template <bool kBf16Out, bool kM16>
__global__ void __launch_bounds__(kThreads, 2)
k_nf4_gemv(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
           const int8_t* __restrict__ absmax_q, const float* __restrict__ absmax_scale,
           const float* __restrict__ mu_ptr, int m, int64_t n, int64_t k, int cluster, int weights_early,
           void* __restrict__ Y, int32_t* __restrict__ dev_status) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // The 128-byte swizzle needs 1 KiB-aligned stages.  The dynamic window is
    // declared so aligned; should a platform place it otherwise, every CTA
    // sees the same base and returns here, before any barrier, with an error.
    if (smem_u32(smem_raw) & 1023u) {
        if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0 && dev_status)
            atomicExch(dev_status, -9 /* NF4_ERR_UNSUPPORTED_DEVICE */);
        return;
    }
    uint8_t* ring = smem_raw;                 // codes slots, then X slots
    uint8_t* xring = smem_raw + kXRingOff;
    float2* lut = reinterpret_cast<float2*>(smem_raw + kLutOff);
    uint64_t* wfull = reinterpret_cast<uint64_t*>(smem_raw + kBarOff);  // codes of a stage landed
    uint64_t* xfull = wfull + kRing;                                     // X of a stage landed
    uint64_t* afull = xfull + kRing;                                     // absmax table of a stage written
    uint64_t* rfull = afull + kAring;                                    // split-k partials received
    uint32_t* wdone = reinterpret_cast<uint32_t*>(rfull + 1);            // warps out of a codes slot
    uint32_t* xdone = wdone + kRing;                                     // warps out of an X slot
    int* wissued = reinterpret_cast<int*>(xdone + kRing);                // last use issued per codes slot
    int* xissued = wissued + kRing;                                      // last use issued per X slot

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kRows;
    const int64_t kblocks = k / 64;
    const int n_stages = static_cast<int>((k + kStageK - 1) / kStageK);
    const int rank = static_cast<int>(blockIdx.y);
    const int s0 = static_cast<int>((static_cast<int64_t>(n_stages) * rank) / cluster);
    const int s1 = static_cast<int>((static_cast<int64_t>(n_stages) * (rank + 1)) / cluster);
    const int nst = s1 - s0;  // >= 1
    const int n_pre = nst < kRing ? nst : kRing;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRing; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&xfull[s], 1);
            wdone[s] = xdone[s] = 0;
            wissued[s] = xissued[s] = -1;
        }
        for (int s = 0; s < kAring; ++s) mbar_init(&afull[s], kConsumers);
        mbar_init(rfull, cluster > 1 ? cluster - 1 : 1);
        fence_mbar_init();
        prefetch_tensormap(&tm_w);
        prefetch_tensormap(&tm_x);
        if (!weights_early) grid_dependency_wait();
        // the weights of the first stages start streaming before anything else
        for (int j = 0; j < n_pre; ++j) {
            issue_w(ring + j * kWBytes, &tm_w, &wfull[j], s0 + j, row0);
            wissued[j] = 0;
            if (!weights_early) {
                issue_x(xring + j * kXBytes, &tm_x, &xfull[j], s0 + j);
                xissued[j] = 0;
            }
        }
    }

    // absmax inputs of the first kPrefetch + 1 stages (rows past n clamped)
    const int arow = threadIdx.x & (kRows - 1);
    const int half = threadIdx.x >> 7;
    const bool aligned4 = (kblocks & 3) == 0 && (reinterpret_cast<uintptr_t>(absmax_q) & 3) == 0;
    const int64_t agrow = row0 + arow;
    AbsmaxIn first;
    AbsmaxIn pre[kPrefetch];
    load_absmax_in(first, absmax_q, absmax_scale, agrow, half, s0, n, kblocks, aligned4);
#pragma unroll
    for (int d = 0; d < kPrefetch; ++d)
        load_absmax_in(pre[d], absmax_q, absmax_scale, agrow, half, min(s0 + 1 + d, n_stages - 1), n, kblocks,
                       aligned4);
    const float mu = __ldg(mu_ptr);

    // byte -> (level of high nibble, level of low nibble), 16 copies so that
    // the 16 lanes of a half-warp always read distinct banks.  Thread t writes
    // 16-byte chunks c = t + 256 it (two copies of byte c / 8): its low nibble
    // (t / 8) mod 16 is fixed and its high nibble is 2 it + t / 128, so every
    // level comes from an immediate and the build touches no memory but the table.
    static_assert(kLutBytes / 16 == 8 * kThreads, "eight chunks per thread");
    {
        constexpr float kLv[16] = NF4_LEVELS_INIT;
        const int lo_idx = (threadIdx.x >> 3) & 15;
        float lo = kLv[0];
#pragma unroll
        for (int v = 1; v < 16; ++v) lo = (lo_idx == v) ? kLv[v] : lo;
        const bool odd = (threadIdx.x >> 7) != 0;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const float hi = odd ? kLv[2 * it + 1] : kLv[2 * it];
            sts128(smem_u32(lut) + 16u * (threadIdx.x + kThreads * it),
                   make_uint4(__float_as_uint(hi), __float_as_uint(lo), __float_as_uint(hi), __float_as_uint(lo)));
        }
    }
    __syncthreads();  // barriers initialised, LUT written

    if (threadIdx.x == 0 && weights_early) {
        // weights are in flight; X (the preceding kernel's output) only after it finished
        grid_dependency_wait();
        for (int j = 0; j < n_pre; ++j) {
            issue_x(xring + j * kXBytes, &tm_x, &xfull[j], s0 + j);
            xissued[j] = 0;
        }
    }
    // the absmax table of the first stage
    const uint32_t ahat_base = smem_u32(smem_raw + kAhatOff);
    const uint32_t ahat_mine = ahat_base + arow * 16u;
    pin(first);
    store_ahat(ahat_mine, half, first, mu);
    __syncwarp();
    if (lane == 0) mbar_arrive(&afull[0]);
    // Under a programmatic dependent launch, sleep here (rather than poll the
    // ring) until the preceding kernel has finished; otherwise a no-op.
    grid_dependency_wait();

    const int g = lane >> 2;
    const int i = lane & 3;
    const int bpair = warp >> 2;         // the warp's two 64-blocks of the stage: 2 bpair, 2 bpair + 1
    const int rbase = (warp & 3) * 32;   // first of this warp's 32 rows
    const uint32_t lut_lane = smem_u32(lut) + (lane & 15) * 8u;
    float acc[kTiles][4];
#pragma unroll
    for (int t = 0; t < kTiles; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

    bool timed_out = false;
    for (int j0 = 0; j0 < nst && !timed_out; j0 += kPrefetch) {
#pragma unroll
        for (int d = 0; d < kPrefetch; ++d) {
            const int j = j0 + d;
            if (j >= nst) break;
            const int slot = j % kRing;
            // absmax table of the next stage.  Its table slot held stage j - 3:
            // this warp saw stage j - 1's table complete, so every warp has begun
            // stage j - 2 and is done with stage j - 3.
            if (j + 1 < nst) {
                const int nslot = (j + 1) % kAring;
                pin(pre[d]);
                store_ahat(ahat_mine + nslot * kAhatBytes, half, pre[d], mu);
                __syncwarp();
                if (lane == 0) mbar_arrive(&afull[nslot]);
                // (unconditional, clamped to a valid stage, so no select waits on the loads)
                load_absmax_in(pre[d], absmax_q, absmax_scale, agrow, half,
                               min(s0 + j + 1 + kPrefetch, n_stages - 1), n, kblocks, aligned4);
            }
            // every lane polls; the warp proceeds only if all of them saw the stage
            const int aslot = j % kAring;
            const uint32_t par = (j / kRing) & 1;
            if (!__all_sync(kFull, mbar_wait(&wfull[slot], par) && mbar_wait(&afull[aslot], (j / kAring) & 1))) {
                timed_out = true;
                break;
            }
            // This warp's codes of the stage into registers (rows rbase + 8 t + g,
            // 8 bytes per lane = 16 consecutive weights of a block), then leave the
            // codes slot: the last warp out refills it while the decode runs.
            const uint32_t wstage = smem_u32(ring + slot * kWBytes);
            uint2 raw[2][kTiles];
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
                const uint32_t wb = wstage + (rbase + g) * 128 +
                                    ((((2 * (2 * bpair + bb) + (i >> 1)) ^ g) << 4) + ((i & 1) << 3));
#pragma unroll
                for (int t = 0; t < kTiles; ++t) raw[bb][t] = lds64(wb + t * 8 * 128);
            }
            __syncwarp();
            if (lane == 0 && slot_leave(&wdone[slot]) == static_cast<uint32_t>(kConsumers * (j / kRing + 1) - 1) &&
                j + kRing < nst) {
                issue_w(ring + slot * kWBytes, &tm_w, &wfull[slot], s0 + j + kRing, row0);
                wissued[slot] = j / kRing + 1;
            }
            if (!__all_sync(kFull, mbar_wait(&xfull[slot], par))) {
                timed_out = true;
                break;
            }
            const uint32_t xstage = smem_u32(xring + slot * kXBytes);
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
                const int blk = 2 * bpair + bb;
                // X fragments: tokens g and g + 8, k = 16 i .. 16 i + 15 of block blk
                const uint32_t xb = xstage + blk * kXBox;
                const uint4 xa0 = lds128(xb + g * 128 + (((2 * i) ^ g) << 4));
                const uint4 xa1 = lds128(xb + g * 128 + (((2 * i + 1) ^ g) << 4));
                uint4 xc0 = make_uint4(0u, 0u, 0u, 0u), xc1 = xc0;
                if (kM16) {
                    xc0 = lds128(xb + (g + 8) * 128 + (((2 * i) ^ g) << 4));
                    xc1 = lds128(xb + (g + 8) * 128 + (((2 * i + 1) ^ g) << 4));
                }
                const uint32_t xa[8] = {xa0.x, xa0.y, xa0.z, xa0.w, xa1.x, xa1.y, xa1.z, xa1.w};
                const uint32_t xc[8] = {xc0.x, xc0.y, xc0.z, xc0.w, xc1.x, xc1.y, xc1.z, xc1.w};
                const uint32_t ab = ahat_base + aslot * kAhatBytes + ((rbase + g) * 4 + blk) * 4;
#pragma unroll
                for (int t = 0; t < kTiles; ++t) {
                    const uint64_t aa = dup_f32x2(lds_f32(ab + 128 * t));
                    uint32_t bw[8];
#pragma unroll
                    for (int b = 0; b < 8; ++b) {
                        const uint32_t word = (b < 4) ? raw[bb][t].x : raw[bb][t].y;
                        bw[b] = scale_pack(lds_b64(lut_lane + (byte_of(word, b & 3) << 7)), aa);
                    }
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_16816(acc[t], xa[2 * s], xc[2 * s], xa[2 * s + 1], xc[2 * s + 1], bw[2 * s],
                                  bw[2 * s + 1]);
                }
            }
            // the last warp out of the X slot refills it
            __syncwarp();
            if (lane == 0 && slot_leave(&xdone[slot]) == static_cast<uint32_t>(kConsumers * (j / kRing + 1) - 1) &&
                j + kRing < nst) {
                issue_x(xring + slot * kXBytes, &tm_x, &xfull[slot], s0 + j + kRing);
                xissued[slot] = j / kRing + 1;
            }
        }
    }
    // the next kernel on the stream may start its prologue (its weight
    // prefetch overlaps our epilogue)
    grid_launch_dependents();

    // fold the warps: red[bpair][token][row] (the four row groups of a block
    // pair land in disjoint rows of the same buffer)
    timed_out = __syncthreads_or(timed_out);  // every warp is done with the ring
    if (timed_out) {
        // leave no copy in flight: wait (bounded) for every stage issued
        if (threadIdx.x == 0) {
            record_timeout(dev_status);
            for (int s = 0; s < kRing; ++s) {
                if (wissued[s] >= 0) mbar_wait(&wfull[s], wissued[s] & 1);
                if (xissued[s] >= 0) mbar_wait(&xfull[s], xissued[s] & 1);
            }
        }
        __syncthreads();
    }
    float* red = reinterpret_cast<float*>(ring) + bpair * 16 * kRedPitch;
#pragma unroll
    for (int t = 0; t < kTiles; ++t) {
        const int r = rbase + 8 * t + 2 * i;
        *reinterpret_cast<float2*>(&red[g * kRedPitch + r]) = make_float2(acc[t][0], acc[t][1]);
        *reinterpret_cast<float2*>(&red[(g + 8) * kRedPitch + r]) = make_float2(acc[t][2], acc[t][3]);
    }
    __syncthreads();
    const float* redf = reinterpret_cast<const float*>(ring);
    float4* part4 = reinterpret_cast<float4*>(ring + kPartOff);
    constexpr int kQ = 16 * kRows / 4;  // float4s of partial sums per CTA
    constexpr int kB = 16 * kRedPitch;  // floats per block buffer
    for (int e = threadIdx.x; e < kQ; e += kThreads) {
        const int off = (e / (kRows / 4)) * kRedPitch + 4 * (e % (kRows / 4));
        const float4 a = *reinterpret_cast<const float4*>(redf + off);
        const float4 b = *reinterpret_cast<const float4*>(redf + kB + off);
        part4[e] = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
    }

    // Cluster split-k: rank q owns rows [q * 128 / C, (q + 1) * 128 / C).  Every
    // rank sends the partials of q's rows into q's receive area and arrives on
    // q's barrier; q adds the C partials in rank order and writes Y.  Nothing
    // reads another CTA's memory, so no rank waits for the others to finish.
    const int rows_per_rank = kRows / cluster;
    const int quads = rows_per_rank / 4;
    const int r_lo = rank * rows_per_rank;
    const uint32_t recv_addr = smem_u32(ring + kRecvOff);
    if (cluster > 1) {
        cluster_sync();  // every rank is done with its ring: receive areas are free
        for (int e = threadIdx.x; e < m * (kRows / 4); e += kThreads) {
            const int tok = e / (kRows / 4);
            const int r = 4 * (e % (kRows / 4));
            const int q = r / rows_per_rank;
            if (q == rank) continue;
            const uint32_t off =
                static_cast<uint32_t>(((rank * 16 + tok) * rows_per_rank + (r - q * rows_per_rank)) * 4);
            st_shared_cluster_f32x4(map_shared_rank(recv_addr + off, q), part4[tok * (kRows / 4) + r / 4]);
        }
        fence_acq_rel_cluster();
        __syncthreads();
        if (threadIdx.x < cluster && threadIdx.x != rank)
            mbar_arrive_remote(map_shared_rank(smem_u32(rfull), threadIdx.x));
        if (!mbar_wait_cluster(rfull, 0)) {
            record_timeout(dev_status);
            return;
        }
    }
    for (int e = threadIdx.x; e < m * quads; e += kThreads) {
        const int tok = e / quads;
        const int rr = 4 * (e % quads);
        const float4 own = part4[tok * (kRows / 4) + (r_lo + rr) / 4];
        float4 sum = own;
        for (int q = 0; q < cluster; ++q) {
            const float4 v = (q == rank) ? own
                                         : *reinterpret_cast<const float4*>(
                                               ring + kRecvOff + ((q * 16 + tok) * rows_per_rank + rr) * 4);
            sum = (q == 0) ? v : make_float4(sum.x + v.x, sum.y + v.y, sum.z + v.z, sum.w + v.w);
        }
        const float o[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int64_t grow = row0 + r_lo + rr + c;
            if (grow >= n) break;
            if (kBf16Out)
                reinterpret_cast<__nv_bfloat16*>(Y)[static_cast<int64_t>(tok) * n + grow] = __float2bfloat16_rn(o[c]);
            else
                reinterpret_cast<float*>(Y)[static_cast<int64_t>(tok) * n + grow] = o[c];
        }
    }
}

}  // namespace gemv

// Cluster size (k split) for a weight of n rows and k columns: the smallest of
// 1, 2, 4, 8 that gives at least one CTA per SM, without giving any CTA an
// empty k range.
static int gemv_cluster(int64_t n, int64_t k, int sm_count) {
    const int64_t tiles = (n + gemv::kRows - 1) / gemv::kRows;
    const int64_t stages = (k + gemv::kStageK - 1) / gemv::kStageK;
    int c = 1;
    while (c < 8 && tiles * c < sm_count && 2 * c <= stages) c *= 2;
    return c;
}

template <bool kBf16Out, bool kM16>
static cudaError_t launch_gemv(const CUtensorMap& tm_w, const CUtensorMap& tm_x, const int8_t* absmax_q,
                               const float* absmax_scale, const float* absmax_offset, int mt, int64_t n,
                               int64_t k, int cluster, bool weights_early, void* Yt, int32_t* dev_status,
                               int device, cudaStream_t stream) {
    static bool attr_set[64] = {};
    if (!attr_set[device]) {
        const cudaError_t e = cudaFuncSetAttribute(gemv::k_nf4_gemv<kBf16Out, kM16>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, gemv::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set[device] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((n + gemv::kRows - 1) / gemv::kRows), cluster, 1);
    cfg.blockDim = dim3(gemv::kThreads, 1, 1);
    cfg.dynamicSmemBytes = gemv::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = cluster;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = weights_early ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, gemv::k_nf4_gemv<kBf16Out, kM16>, tm_w, tm_x, absmax_q, absmax_scale,
                              absmax_offset, mt, n, k, cluster, weights_early ? 1 : 0, Yt, dev_status);
}

cudaError_t launch_linear(const void* X, int64_t m, const uint8_t* wq, const int8_t* absmax_q,
                          const float* absmax_scale, const float* absmax_offset, int64_t n,
                          int64_t k, void* Y, bool y_bf16, int32_t* dev_status, bool weights_early,
                          const DeviceInfo& dev, cudaStream_t stream) {
    if (dev.device < 0 || dev.device >= 64) return cudaErrorInvalidDevice;
    if (m > kGemvMaxTokens)
        return launch_gemm(X, m, wq, absmax_q, absmax_scale, absmax_offset, n, k, Y, y_bf16, dev_status, dev,
                           stream);
    CUtensorMap tm_w;
    cudaError_t e = tmap_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, wq, static_cast<uint64_t>(k / 2),
                            static_cast<uint64_t>(n), static_cast<uint64_t>(k / 2), 128, gemv::kRows,
                            CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    const int cluster = gemv_cluster(n, k, dev.sm_count);
    const size_t ybytes = y_bf16 ? 2 : 4;
    const __nv_bfloat16* Xb = static_cast<const __nv_bfloat16*>(X);
    for (int64_t t0 = 0; t0 < m; t0 += 16) {
        const int mt = static_cast<int>((m - t0) < 16 ? (m - t0) : 16);
        CUtensorMap tm_x;
        e = tmap_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Xb + t0 * k, static_cast<uint64_t>(k),
                    static_cast<uint64_t>(mt), static_cast<uint64_t>(k * 2), 64, 16, CU_TENSOR_MAP_SWIZZLE_128B);
        if (e != cudaSuccess) return e;
        void* Yt = static_cast<char*>(Y) + static_cast<size_t>(t0) * n * ybytes;
        if (y_bf16)
            e = (mt > 8) ? launch_gemv<true, true>(tm_w, tm_x, absmax_q, absmax_scale, absmax_offset, mt, n, k,
                                                   cluster, weights_early, Yt, dev_status, dev.device, stream)
                         : launch_gemv<true, false>(tm_w, tm_x, absmax_q, absmax_scale, absmax_offset, mt, n, k,
                                                    cluster, weights_early, Yt, dev_status, dev.device, stream);
        else
            e = (mt > 8) ? launch_gemv<false, true>(tm_w, tm_x, absmax_q, absmax_scale, absmax_offset, mt, n, k,
                                                    cluster, weights_early, Yt, dev_status, dev.device, stream)
                         : launch_gemv<false, false>(tm_w, tm_x, absmax_q, absmax_scale, absmax_offset, mt, n,
                                                     k, cluster, weights_early, Yt, dev_status, dev.device, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace nf4
