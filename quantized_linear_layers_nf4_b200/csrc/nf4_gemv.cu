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
// code must stream from HBM.  Design (one CTA = 128 weight rows x a slice of k):
//
// * A producer warp streams 256-wide k stages through a 3-deep shared-memory
//   ring with TMA (no multicast): a [128 rows x 128 B] tile of packed codes and
//   the matching [16 tokens x 256] tile of X, both 128-byte swizzled so the
//   consumers' reads are bank-conflict free.  Its 32 lanes also reconstruct the
//   stage's absmax values (loaded one stage ahead, so their latency hides behind
//   the ring).  mbarriers carry full/empty state; every wait is bounded.
// * Eight consumer warps: warp w owns 64-block (w % 4) of every stage for 64
//   of the 128 rows, so one X fragment serves 8 MMAs.  The multiply-adds run on the tensor
//   cores (mma.sync m16n8k16, bf16 in, fp32 accumulate) with the 16 token slots
//   as the MMA's M side (zero-filled beyond m) and 8 weight rows as its N side.
//   X fragments come from ldmatrix in the MMA's own layout; for k chunk s of a
//   block, lane (g, i) decodes bytes 8s + i and 8s + 4 + i of row g (weights
//   16s + 2i, +1 and 16s + 8 + 2i, +1), so the k order is the true one.
// * Decode: a 256-entry table maps a packed byte to the two fp32 levels it
//   encodes (replicated 16x so a half-warp's lookups never share a bank); each
//   level is multiplied by the block's reconstructed absmax in fp32 and rounded
//   to bf16 -- the same values nf4_dequantize produces.
// * Split-k: the C CTAs of a row tile split k.  Without a workspace they form a
//   thread-block cluster and add their fp32 partials through distributed shared
//   memory; with a caller's workspace they store them there and the last to
//   count in adds them.  Both add in rank order, so the bits are the same and
//   deterministic.
// * One launch may cover the row tiles of several weights that share X (a
//   grid-constant group struct; each CTA picks its weight by its tile).
// * LoRA layers (r = 8 or 16): the CTAs also form their share of
//   t = scale * X down^T from the same X fragments and exchange it with the
//   partial sums; the epilogue adds t up^T before rounding.
#include <cstring>
#include <mutex>

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
constexpr int kTiles = 8;                        // 8-row MMA tiles per consumer warp (64 rows)
constexpr int kThreads = 32 * (kConsumers + 1);  // + one producer warp
constexpr int kWBytes = kRows * kStageK / 2;     // 16384: packed codes of a stage
constexpr int kXBox = 16 * 64 * 2;               // 2048: X box of 16 tokens x 64 k (bf16)
constexpr int kXBytes = 4 * kXBox;               // 8192
constexpr int kTmaBytes = kWBytes + kXBytes;     // bytes a stage receives by TMA
constexpr int kAhatBytes = 4 * kRows * 4;        // 2048: reconstructed absmax, [row][block]
constexpr int kStageBytes = kTmaBytes + kAhatBytes;  // 26624 = 26 KiB (keeps 1 KiB alignment)
constexpr int kLutBytes = 16 * 256 * 8;          // 32768
constexpr int kRingBytes = kRing * kStageBytes;
constexpr int kSmemBytes = 1024 /*alignment slack*/ + kRingBytes + kLutBytes + 2 * kRing * 8;
static_assert(kStageBytes % 1024 == 0, "stages keep the 1 KiB alignment the 128-byte swizzle needs");
// Per-block partial sums are stored [token][row] with a padded token pitch so
// that the 8 row groups of a warp write distinct banks.
constexpr int kRedPitch = kRows + 8;
static_assert(4 * 16 * kRedPitch * 4 + 16 * kRows * 4 <= kRingBytes, "reduction fits in the ring");
// After the block partials (red) and the CTA's partial tile (part4): the four
// blocks' down-projection sums [4][16 tokens][16 ranks] and the CTA's t (the
// fused LoRA down-projection), in floats from the start of the ring.
constexpr int kTredOff = 4 * 16 * kRedPitch + 16 * kRows;
constexpr int kTOff = kTredOff + 4 * 256;
// Then the tile's up rows, transposed: [16 ranks][128 rows] fp32.
static_assert((kTOff + 256 + 16 * kRows) * 4 <= kRingBytes, "down-projection sums fit in the ring");

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// v + sum_j t[tok * r + j] * up[row * r + j], in j order (the low-rank term of
// a LoRA layer, added to the fp32 result before it is stored).
__device__ __forceinline__ float lora_term(float v, const float* __restrict__ lt, const __nv_bfloat16* __restrict__ up,
                                           int r, int tok, int64_t row) {
    const float* tr = lt + static_cast<int64_t>(tok) * r;
    const __nv_bfloat16* ur = up + row * r;
    int j = 0;
    if ((r & 7) == 0) {  // rows of up and t are 16-byte aligned: 8 ranks per load pair
        for (; j < r; j += 8) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(ur + j));
            const float4 t0 = __ldg(reinterpret_cast<const float4*>(tr + j));
            const float4 t1 = __ldg(reinterpret_cast<const float4*>(tr + j + 4));
            v = __fmaf_rn(t0.x, bf16_bits_to_float(u.x & 0xffffu), v);
            v = __fmaf_rn(t0.y, bf16_bits_to_float(u.x >> 16), v);
            v = __fmaf_rn(t0.z, bf16_bits_to_float(u.y & 0xffffu), v);
            v = __fmaf_rn(t0.w, bf16_bits_to_float(u.y >> 16), v);
            v = __fmaf_rn(t1.x, bf16_bits_to_float(u.z & 0xffffu), v);
            v = __fmaf_rn(t1.y, bf16_bits_to_float(u.z >> 16), v);
            v = __fmaf_rn(t1.z, bf16_bits_to_float(u.w & 0xffffu), v);
            v = __fmaf_rn(t1.w, bf16_bits_to_float(u.w >> 16), v);
        }
    }
    for (; j < r; ++j) v = __fmaf_rn(__ldg(tr + j), __bfloat162float(ur[j]), v);
    return v;
}

// The same sums for four consecutive rows with t and up in shared memory (the
// fused down-projection): ts [token][16], ut [rank][128 rows] (up as fp32), rl
// the first row's index in the tile.
__device__ __forceinline__ void lora_quad_shared(float (&o)[4], const float* ts, const float* ut, int r, int tok,
                                                 int rl) {
    for (int j = 0; j < r; ++j) {
        const float tj = ts[tok * 16 + j];
        const float4 u = *reinterpret_cast<const float4*>(ut + j * 128 + rl);
        o[0] = __fmaf_rn(tj, u.x, o[0]);
        o[1] = __fmaf_rn(tj, u.y, o[1]);
        o[2] = __fmaf_rn(tj, u.z, o[2]);
        o[3] = __fmaf_rn(tj, u.w, o[3]);
    }
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// Four 8x8 bf16 matrices, one 16-byte row address per lane: the registers come
// back in the layout of an m16n8k16 A fragment.
__device__ __forceinline__ uint4 ldsm_x4(uint32_t addr) {
    uint4 v;
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
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

// B fragments of down for k stage `st`, block blk: the k pairs 8q + 2i of the
// block (q = 2s + half), zero past k or for a rank past r.
__device__ __forceinline__ void load_down(uint32_t (&b)[8], const __nv_bfloat16* __restrict__ drow, int st, int blk,
                                          int i, int64_t k, bool rank_ok) {
    const int64_t kb = static_cast<int64_t>(st) * kStageK;
#pragma unroll
    for (int q = 0; q < 8; ++q)
        b[q] = (rank_ok && kb + 64 * blk + 8 * q + 2 * i < k) ? __ldg(reinterpret_cast<const uint32_t*>(drow + kb + 8 * q))
                                                              : 0u;
}

// Thread 2 row + h holds up[row0 + row][8h .. 8h + 7] (zeros past n or r);
// ut[j][row] = fp32(up[row0 + row][j]).
__device__ __forceinline__ void stage_up(float* ut, uint4 v, int row, int h, int r) {
    if (threadIdx.x >= 256 || 8 * h >= r) return;
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        ut[(8 * h + 2 * q) * 128 + row] = bf16_bits_to_float(w[q] & 0xffffu);
        ut[(8 * h + 2 * q + 1) * 128 + row] = bf16_bits_to_float(w[q] >> 16);
    }
}

// Rows grow0 .. grow0 + 3 of token `tok` (rows past n are dropped), the
// low-rank term added first when there is one (t and up from shared memory, ts
// and ut, when ts is set, else from lt and up): one vector store when all four
// rows are in range and the address is aligned, else one store per row.
template <bool kBf16Out, bool kLora>
__device__ __forceinline__ void store_quad(void* __restrict__ Y, int64_t n, int tok, int64_t grow0, float (&o)[4],
                                           const float* __restrict__ lt, const __nv_bfloat16* __restrict__ up, int r,
                                           const float* ts, const float* ut, int rl) {
    if (kLora) {
        if (ts) {
            lora_quad_shared(o, ts, ut, r, tok, rl);
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (grow0 + c < n) o[c] = lora_term(o[c], lt, up, r, tok, grow0 + c);
        }
    }
    const int64_t idx = static_cast<int64_t>(tok) * n + grow0;
    if (kBf16Out) {
        __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(Y) + idx;
        if (grow0 + 3 < n && (reinterpret_cast<uintptr_t>(y) & 7) == 0) {
            const __nv_bfloat162 p0 = __floats2bfloat162_rn(o[0], o[1]);
            const __nv_bfloat162 p1 = __floats2bfloat162_rn(o[2], o[3]);
            *reinterpret_cast<uint2*>(y) =
                make_uint2(*reinterpret_cast<const uint32_t*>(&p0), *reinterpret_cast<const uint32_t*>(&p1));
            return;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (grow0 + c < n) y[c] = __float2bfloat16_rn(o[c]);
    } else {
        float* y = reinterpret_cast<float*>(Y) + idx;
        if (grow0 + 3 < n && (reinterpret_cast<uintptr_t>(y) & 15) == 0) {
            *reinterpret_cast<float4*>(y) = make_float4(o[0], o[1], o[2], o[3]);
            return;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (grow0 + c < n) y[c] = o[c];
    }
}

// The producer's per-stage absmax inputs.  Lane l owns rows l + 32 u (u = 0..3)
// and the stage's 4 blocks of each: the 4 int8 codes of a row packed in one
// word, and the (at most two) double-quantization scales its 4 blocks use.
struct AbsmaxIn {
    uint32_t q[4];
    float s_lo[4], s_hi[4];
};

__device__ __forceinline__ void load_absmax_in(AbsmaxIn& a, const int8_t* __restrict__ absmax_q,
                                               const float* __restrict__ absmax_scale, int64_t row0,
                                               int lane, int st, int64_t n, int64_t kblocks,
                                               bool aligned4) {
    const int64_t kb0 = static_cast<int64_t>(st) * 4;
    if (aligned4) {
        // k % 256 == 0 and an aligned code array: a row's 4 codes of a stage are
        // one aligned word.  Every load is unconditional (rows past n are
        // clamped; their results are never stored) and lands directly in its
        // field, so nothing waits for it until the stage is used.
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            int64_t grow = row0 + lane + 32 * u;
            grow = grow < n ? grow : n - 1;
            const int64_t b0 = grow * kblocks + kb0;
            a.q[u] = __ldg(reinterpret_cast<const uint32_t*>(absmax_q + b0));
            a.s_lo[u] = __ldg(absmax_scale + (b0 >> 8));
            a.s_hi[u] = __ldg(absmax_scale + ((b0 + 3) >> 8));
        }
        return;
    }
    // general shapes: gather the codes byte by byte (stalls, but correct)
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int64_t grow = row0 + lane + 32 * u;
        uint32_t q = 0;
        float lo = 0.0f, hi = 0.0f;
        if (grow < n) {
            const int64_t b0 = grow * kblocks + kb0;
            const int64_t nvalid = kblocks - kb0;  // >= 1
#pragma unroll
            for (int b = 0; b < 4; ++b)
                if (b < nvalid)
                    q |= static_cast<uint32_t>(static_cast<uint8_t>(__ldg(absmax_q + b0 + b))) << (8 * b);
            const int64_t blast = b0 + (nvalid < 4 ? nvalid : 4) - 1;
            lo = __ldg(absmax_scale + (b0 >> 8));
            hi = __ldg(absmax_scale + (blast >> 8));
        }
        a.q[u] = q;
        a.s_lo[u] = lo;
        a.s_hi[u] = hi;
    }
}

// Keeps the compiler from hoisting work that uses `a` above the point where
// this is called (the values pass through an opaque asm).
__device__ __forceinline__ void pin(AbsmaxIn& a) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
        asm volatile("" : "+r"(a.q[u]), "+f"(a.s_lo[u]), "+f"(a.s_hi[u]));
}

constexpr int kPrefetch = 3;  // stages of absmax inputs in flight per producer lane

// The weights of one launch (1 .. kMaxGroup, same k, same X): row tiles
// tile0[i] .. tile0[i+1]-1 of the grid belong to weight i.
struct GemvGroup {
    CUtensorMap tm_w[kMaxGroup];  // codes [n x k/2 bytes], boxes [128 rows x 128 B], 128-byte swizzle
    const int8_t* absmax_q[kMaxGroup];
    const float* absmax_scale[kMaxGroup];
    const float* mu[kMaxGroup];
    void* y[kMaxGroup];
    int64_t n[kMaxGroup];
    int tile0[kMaxGroup];
    int count;
};

template <bool kBf16Out, bool kM16, bool kLora>
__global__ void __launch_bounds__(kThreads, 2)
k_nf4_gemv(const __grid_constant__ GemvGroup grp, const __grid_constant__ CUtensorMap tm_x,
           int m, int64_t k, int cluster, int weights_early,
           int32_t* __restrict__ dev_status, uint32_t* __restrict__ ws_cnt,
           float4* __restrict__ ws_part, const float* __restrict__ lora_t, const __nv_bfloat16* __restrict__ lora_up,
           int lora_r, const __nv_bfloat16* __restrict__ lora_down, float lora_scale, int codebook, uint32_t lim,
           int stall) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    float2* lut = reinterpret_cast<float2*>(smem + kRingBytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRingBytes + kLutBytes);
    uint64_t* empty = full + kRing;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // this CTA's weight: the last one whose tiles start at or before blockIdx.x
    int wi = 0;
#pragma unroll
    for (int i = 1; i < kMaxGroup; ++i)
        if (i < grp.count && static_cast<int>(blockIdx.x) >= grp.tile0[i]) wi = i;
    const CUtensorMap* tm_w = &grp.tm_w[wi];
    const int8_t* __restrict__ absmax_q = grp.absmax_q[wi];
    const float* __restrict__ absmax_scale = grp.absmax_scale[wi];
    const float* __restrict__ mu_ptr = grp.mu[wi];
    void* __restrict__ Y = grp.y[wi];
    const int64_t n = grp.n[wi];
    const int64_t row0 = static_cast<int64_t>(static_cast<int>(blockIdx.x) - grp.tile0[wi]) * kRows;
    const int64_t kblocks = k / 64;
    const int n_stages = static_cast<int>((k + kStageK - 1) / kStageK);
    const int rank = static_cast<int>(blockIdx.y);
    const int s0 = static_cast<int>((static_cast<int64_t>(n_stages) * rank) / cluster);
    const int s1 = static_cast<int>((static_cast<int64_t>(n_stages) * (rank + 1)) / cluster);

    __shared__ int s_bad;   // some warp of this CTA gave up a wait
    __shared__ int s_last;  // this CTA is the last of its tile to finish (workspace split-k)
    if (threadIdx.x == 0) {
        s_bad = 0;
        for (int s = 0; s < kRing; ++s) {
            mbar_init(&full[s], 2);   // the TMA bytes' arrive + the absmax-ready arrive
            mbar_init(&empty[s], kConsumers);
        }
        fence_mbar_init();
    }
    __syncthreads();

    bool timed_out = false;
    if (warp == kConsumers) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            prefetch_tensormap(tm_w);
            prefetch_tensormap(&tm_x);
        }
        if (!weights_early) grid_dependency_wait();
        const float mu = __ldg(mu_ptr);
        int last_use[kRing];
#pragma unroll
        for (int s = 0; s < kRing; ++s) last_use[s] = -1;
        bool x_ready = !weights_early;  // X (the previous kernel's output) may be read
        const int n_pre = (s1 - s0) < kRing ? (s1 - s0) : kRing;
        const bool aligned4 = (kblocks & 3) == 0 && (reinterpret_cast<uintptr_t>(absmax_q) & 3) == 0;
        AbsmaxIn pre[kPrefetch];
#pragma unroll
        for (int d = 0; d < kPrefetch; ++d)
            load_absmax_in(pre[d], absmax_q, absmax_scale, row0, lane, min(s0 + d, n_stages - 1), n, kblocks, aligned4);
        for (int st0 = s0; st0 < s1 && !timed_out && !stall; st0 += kPrefetch) {
#pragma unroll
            for (int d = 0; d < kPrefetch; ++d) {
                const int st = st0 + d;
                if (st >= s1) break;
                const int j = st - s0;
                const int slot = j % kRing;
                const int use = j / kRing;
                if (j >= kRing && !__all_sync(kFull, mbar_wait_n(&empty[slot], (use - 1) & 1, lim))) {
                    timed_out = true;
                    break;
                }
                uint8_t* stage = ring + slot * kStageBytes;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[slot], kTmaBytes);
                    tma_load_2d(stage, tm_w, st * (kStageK / 2), static_cast<int32_t>(row0), &full[slot]);
                    if (x_ready) {
#pragma unroll
                        for (int b = 0; b < 4; ++b)
                            tma_load_2d(stage + kWBytes + b * kXBox, &tm_x, st * kStageK + 64 * b, 0, &full[slot]);
                    }
                    last_use[slot] = use;
                }
                pin(pre[d]);  // the copies above are issued before the absmax work below
                // reconstructed absmax a = fp32(fp32(fp32(q / 127) * s) + mu) of this stage.
                // Blocks past k or rows past n get q = s = 0 (a = mu, finite): X is
                // zero-filled there, so their products vanish.
                const uint32_t ahat = smem_u32(stage + kTmaBytes);  // [row][block] floats
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int row = lane + 32 * u;
                    const int64_t b0 = (row0 + row) * kblocks + static_cast<int64_t>(st) * 4;
                    float a4[4];
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        const float sc = (((b0 + b) >> 8) == (b0 >> 8)) ? pre[d].s_lo[u] : pre[d].s_hi[u];
                        const float qf = static_cast<float>(static_cast<int8_t>((pre[d].q[u] >> (8 * b)) & 0xffu));
                        a4[b] = __fadd_rn(__fmul_rn(div127(qf), sc), mu);
                    }
                    sts128(ahat + row * 16u, make_uint4(__float_as_uint(a4[0]), __float_as_uint(a4[1]),
                                                        __float_as_uint(a4[2]), __float_as_uint(a4[3])));
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[slot]);
                // (unconditional, clamped to a valid stage, so no select waits on the loads)
                load_absmax_in(pre[d], absmax_q, absmax_scale, row0, lane, min(st + kPrefetch, n_stages - 1), n,
                               kblocks, aligned4);
                if (!x_ready && j + 1 == n_pre) {
                    // weights of the first stages are in flight; now wait for the
                    // preceding kernel before touching X
                    grid_dependency_wait();
                    x_ready = true;
                    if (lane == 0)
                        for (int jj = 0; jj <= j; ++jj) {
                            uint8_t* stg = ring + (jj % kRing) * kStageBytes;
#pragma unroll
                            for (int b = 0; b < 4; ++b)
                                tma_load_2d(stg + kWBytes + b * kXBox, &tm_x, (s0 + jj) * kStageK + 64 * b, 0,
                                            &full[jj % kRing]);
                        }
                }
            }
        }
        if (!x_ready) grid_dependency_wait();
        // every copy of this CTA is issued: the next kernel on the stream may
        // start its prologue (its weight prefetch overlaps our last stages)
        grid_launch_dependents();
        // on a timeout leave no copy in flight: wait (bounded) for every stage issued
        if (timed_out && lane == 0)
            for (int s = 0; s < kRing; ++s)
                if (last_use[s] >= 0) mbar_wait(&full[s], last_use[s] & 1);
    } else {
        // ------------------------------ consumers -----------------------------
        // byte -> (level of high nibble, level of low nibble), 16 copies so that
        // the 16 lanes of a half-warp always read distinct banks.  Consumer
        // thread t writes 16-byte chunks c = t + 256 it (two copies of byte
        // c / 8): its low nibble (t / 8) mod 16 is fixed and its high nibble is
        // 2 it + t / 128, so every level is an immediate and the build touches
        // no memory but the table.  The FP4 codebook reads its values from
        // constant memory instead.
        static_assert(kLutBytes / 16 == 8 * 32 * kConsumers, "eight chunks per consumer thread");
        {
            const int lo_idx = (threadIdx.x >> 3) & 15;
            const bool odd = (threadIdx.x >> 7) != 0;
            if (codebook == kCbNf4) {
                constexpr float kLv[16] = NF4_LEVELS_INIT;
                float lo = kLv[0];
#pragma unroll
                for (int v = 1; v < 16; ++v) lo = (lo_idx == v) ? kLv[v] : lo;
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const float hi = odd ? kLv[2 * it + 1] : kLv[2 * it];
                    sts128(smem_u32(lut) + 16u * (threadIdx.x + 32 * kConsumers * it),
                           make_uint4(__float_as_uint(hi), __float_as_uint(lo), __float_as_uint(hi),
                                      __float_as_uint(lo)));
                }
            } else {
                const float lo = kCodebook[kCbFp4][lo_idx];
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const float hi = kCodebook[kCbFp4][2 * it + (odd ? 1 : 0)];
                    sts128(smem_u32(lut) + 16u * (threadIdx.x + 32 * kConsumers * it),
                           make_uint4(__float_as_uint(hi), __float_as_uint(lo), __float_as_uint(hi),
                                      __float_as_uint(lo)));
                }
            }
        }
        named_bar_sync(1, 32 * kConsumers);
        // Under a programmatic dependent launch, sleep here (rather than poll
        // the ring) until the preceding kernel has finished; otherwise a no-op.
        grid_dependency_wait();

        const int g = lane >> 2;
        const int i = lane & 3;
        const int blk = warp & 3;          // 64-block of the stage
        const int rbase = (warp >> 2) * 64;  // first of this warp's 64 rows
        const uint32_t lut_lane = smem_u32(lut) + (lane & 15) * 8u;
        // the X row this lane addresses for ldmatrix: token (lane & 7) + 8 ((lane >> 3) & 1)
        const uint32_t x_lane = ((lane & 7) + 8 * ((lane >> 3) & 1)) * 128;
        // the two 16-byte chunks of a block row (128-byte swizzle, row & 7 == g);
        // lane i decodes byte i of each of their 8 words
        const uint32_t wc0 = ((2 * blk) ^ g) << 4, wc1 = ((2 * blk + 1) ^ g) << 4;
        const uint32_t sel_i = 0x4440u | static_cast<uint32_t>(i);
        // Fused down-projection of a LoRA layer (r = 8 or 16): warp (blk, h) adds
        // X[:, block] down[8h .. 8h + 7, block]^T into tacc with the same X
        // fragments; lane (g, i) reads rank 8h + g of down at the MMA's k pairs.
        const bool t_on = kLora && lora_down != nullptr && 8 * (warp >> 2) < lora_r;
        const int t_rank = 8 * (warp >> 2) + g;
        const __nv_bfloat16* __restrict__ drow =
            kLora && lora_down != nullptr
                ? lora_down + static_cast<int64_t>(t_rank < lora_r ? t_rank : 0) * k + 64 * blk + 2 * i
                : nullptr;
        float tacc[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t bA[8];  // the current stage's down fragments
        if (kLora && t_on) load_down(bA, drow, s0, blk, i, k, t_rank < lora_r);
        float acc[kTiles][4];
#pragma unroll
        for (int t = 0; t < kTiles; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

        for (int st = s0; st < s1; ++st) {
            const int j = st - s0;
            const int slot = j % kRing;
            // every lane polls; the warp proceeds only if all of them saw the stage
            if (!__all_sync(kFull, mbar_wait_n(&full[slot], (j / kRing) & 1, lim))) {
                timed_out = true;
                break;
            }
            const uint32_t stage = smem_u32(ring + slot * kStageBytes);
            // X fragments: tokens g and g + 8, k = 16 i .. 16 i + 15 of this warp's block
            // A fragments of the block's four k16 chunks: tokens 0-7 / 8-15 x the
            // chunk's two 16-byte halves (128-byte swizzle, row & 7 == lane & 7)
            const uint32_t xb = stage + kWBytes + blk * kXBox;
            uint4 xf[4];
#pragma unroll
            for (int s = 0; s < 4; ++s) xf[s] = ldsm_x4(xb + x_lane + (((2 * s + (lane >> 4)) ^ (lane & 7)) << 4));
            const uint32_t wrow = stage + (rbase + g) * 128;
            const uint32_t ab = stage + kTmaBytes + ((rbase + g) * 4 + blk) * 4;
            // each tile's codes and reconstructed absmax are read one tile ahead
            uint4 c0 = lds128(wrow + wc0), c1 = lds128(wrow + wc1);
            float av = lds_f32(ab);
#pragma unroll
            for (int t = 0; t < kTiles; ++t) {
                uint4 n0 = c0, n1 = c1;
                float an = av;
                if (t + 1 < kTiles) {
                    n0 = lds128(wrow + (t + 1) * 8 * 128 + wc0);
                    n1 = lds128(wrow + (t + 1) * 8 * 128 + wc1);
                    an = lds_f32(ab + 128 * (t + 1));
                }
                const uint32_t wv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                const uint64_t aa = dup_f32x2(av);
                uint32_t bw[8];
#pragma unroll
                for (int b = 0; b < 8; ++b) {
                    uint32_t byte;
                    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(byte) : "r"(wv[b]), "r"(sel_i));
                    bw[b] = scale_pack(lds_b64(lut_lane + (byte << 7)), aa);
                }
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_16816(acc[t], xf[s].x, xf[s].y, xf[s].z, xf[s].w, bw[2 * s], bw[2 * s + 1]);
                c0 = n0;
                c1 = n1;
                av = an;
            }
            if (kLora && t_on) {
#pragma unroll
                for (int s = 0; s < 4; ++s) mma_16816(tacc, xf[s].x, xf[s].y, xf[s].z, xf[s].w, bA[2 * s], bA[2 * s + 1]);
                if (st + 1 < s1) load_down(bA, drow, st + 1, blk, i, k, t_rank < lora_r);  // next stage's, in flight
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }

        // fold the consumer warps: red[blk][token][row] (the two row halves of a
        // block land in disjoint rows of the same buffer)
        __syncwarp();
        named_bar_sync(1, 32 * kConsumers);  // every consumer is done with the ring
        if (kLora && t_on) {
            // tred[blk][token][rank]
            float* tr = reinterpret_cast<float*>(ring) + kTredOff + blk * 256;
            const int j = 8 * (warp >> 2) + 2 * i;
            tr[g * 16 + j] = tacc[0];
            tr[g * 16 + j + 1] = tacc[1];
            tr[(g + 8) * 16 + j] = tacc[2];
            tr[(g + 8) * 16 + j + 1] = tacc[3];
        }
        float* red = reinterpret_cast<float*>(ring) + blk * 16 * kRedPitch;
#pragma unroll
        for (int t = 0; t < kTiles; ++t) {
            const int r = rbase + 8 * t + 2 * i;
            *reinterpret_cast<float2*>(&red[g * kRedPitch + r]) = make_float2(acc[t][0], acc[t][1]);
            *reinterpret_cast<float2*>(&red[(g + 8) * kRedPitch + r]) = make_float2(acc[t][2], acc[t][3]);
        }
        grid_dependency_wait();  // Y may still be in use by the preceding kernel
    }
    if (timed_out) {
        record_timeout(dev_status);
        s_bad = 1;
    }
    __syncthreads();
    // after a timeout the CTA writes neither Y nor the workspace (its sums are incomplete)
    const bool bad = s_bad != 0;
    const float* redf = reinterpret_cast<const float*>(ring);
    float4* part4 = reinterpret_cast<float4*>(ring) + 4 * 16 * kRedPitch / 4;
    constexpr int kQ = 16 * kRows / 4;  // float4s of partial sums per CTA
    constexpr int kQS = kQ + 64;         // a workspace slot: the partial tile, then the CTA's t [16][16]
    constexpr int kB = 16 * kRedPitch;  // floats per block buffer
    for (int e = threadIdx.x; e < kQ; e += kThreads) {
        const int off = (e / (kRows / 4)) * kRedPitch + 4 * (e % (kRows / 4));
        const float4 a = *reinterpret_cast<const float4*>(redf + off);
        const float4 b = *reinterpret_cast<const float4*>(redf + kB + off);
        const float4 c = *reinterpret_cast<const float4*>(redf + 2 * kB + off);
        const float4 d = *reinterpret_cast<const float4*>(redf + 3 * kB + off);
        part4[e] = make_float4(((a.x + b.x) + c.x) + d.x, ((a.y + b.y) + c.y) + d.y,
                               ((a.z + b.z) + c.z) + d.z, ((a.w + b.w) + c.w) + d.w);
    }
    // The CTA's share of the fused down-projection: thread e < 256 holds
    // t[e / 16][e % 16], the four blocks added in order (ranks >= r unused).
    // Its up rows are fetched now and staged (transposed, [rank][row]) once the
    // tile's t is known.
    const bool t_fused = kLora && lora_down != nullptr;
    float* tful = reinterpret_cast<float*>(ring) + kTOff;
    float* utile = reinterpret_cast<float*>(ring) + kTOff + 256;
    float tv = 0.f;
    uint4 upv = make_uint4(0u, 0u, 0u, 0u);
    const int up_row = static_cast<int>(threadIdx.x) / 2, up_h = static_cast<int>(threadIdx.x) & 1;  // r = 16
    if (t_fused && threadIdx.x < 256) {
        const float* tr = redf + kTredOff + threadIdx.x;
        tv = ((tr[0] + tr[256]) + tr[512]) + tr[768];
        if (8 * up_h < lora_r && row0 + up_row < n)
            upv = __ldg(reinterpret_cast<const uint4*>(lora_up + (row0 + up_row) * lora_r + 8 * up_h));
    }

    if (ws_part != nullptr) {
        // Split-k through the caller's workspace: each CTA stores its partial
        // sums and counts itself in; the last of the tile's C CTAs adds the
        // partials in rank order (the order the cluster path uses) and writes Y.
        if (bad) return;
        const int tile = static_cast<int>(blockIdx.x);
        float4* part_g = ws_part + static_cast<int64_t>(tile) * cluster * kQS;
        for (int e = threadIdx.x; e < m * (kRows / 4); e += kThreads) part_g[rank * kQS + e] = part4[e];
        if (t_fused && threadIdx.x < m * 16) reinterpret_cast<float*>(part_g + rank * kQS + kQ)[threadIdx.x] = tv;
        __syncthreads();
        // One acquire-release add at GPU scope publishes the whole CTA's stores
        // (ordered before it by the barrier) and, for the last CTA, makes every
        // other CTA's partials visible to the loads below.
        if (threadIdx.x == 0) {
            uint32_t old;
            asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(ws_cnt + tile) : "memory");
            s_last = old == static_cast<uint32_t>(cluster - 1);
        }
        __syncthreads();
        if (!s_last) return;
        // Each thread owns at most two float4s of the tile; every load of both
        // (all C parts) goes out before the first add, so the reduction costs one
        // L2 round trip.  The adds keep rank order.
        static_assert(2 * kThreads >= kQ, "two float4s per thread cover the tile");
        const int ne = m * (kRows / 4);
        float4 v[2][8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = static_cast<int>(threadIdx.x) + h * kThreads;
            if (e < ne) {
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (q < cluster) v[h][q] = (q == rank) ? part4[e] : __ldcg(part_g + q * kQS + e);
            }
        }
        if (t_fused) {
            // t = scale * (the parts' shares added in rank order)
            float pv[8];
            if (threadIdx.x < m * 16) {
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (q < cluster)
                        pv[q] = (q == rank) ? tv
                                            : __ldcg(reinterpret_cast<const float*>(part_g + q * kQS + kQ) + threadIdx.x);
            }
            stage_up(utile, upv, up_row, up_h, lora_r);
            if (threadIdx.x < m * 16) {
                float ts = pv[0];
#pragma unroll
                for (int q = 1; q < 8; ++q)
                    if (q < cluster) ts += pv[q];
                tful[threadIdx.x] = ts * lora_scale;
            }
            __syncthreads();
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = static_cast<int>(threadIdx.x) + h * kThreads;
            if (e >= ne) break;
            float4 sum = v[h][0];
#pragma unroll
            for (int q = 1; q < 8; ++q)
                if (q < cluster)
                    sum = make_float4(sum.x + v[h][q].x, sum.y + v[h][q].y, sum.z + v[h][q].z, sum.w + v[h][q].w);
            float o[4] = {sum.x, sum.y, sum.z, sum.w};
            store_quad<kBf16Out, kLora>(Y, n, e / (kRows / 4), row0 + 4 * (e % (kRows / 4)), o, lora_t, lora_up,
                                        lora_r, t_fused ? tful : nullptr, utile, 4 * (e % (kRows / 4)));
        }
        if (threadIdx.x == 0) ws_cnt[tile] = 0;  // ready for the next call
        return;
    }

    // cluster split-k: rank r adds rows [r * 128 / C, (r + 1) * 128 / C) over all ranks in rank order
    // (a fused down-projection runs here only with C = 1: the CTA's t is the whole t)
    if (t_fused) {
        if (threadIdx.x < 256) tful[threadIdx.x] = tv * lora_scale;
        stage_up(utile, upv, up_row, up_h, lora_r);
    }
    cluster_sync();
    const int r_lo = (rank * kRows) / cluster;
    const int rows_per_rank = ((rank + 1) * kRows) / cluster - r_lo;
    const int quads = rows_per_rank / 4;
    const uint32_t part_addr = smem_u32(part4);
    if (!bad && kRows % (4 * cluster) != 0) {
        // C = 3, 5, 6, 7: row ranges of uneven length, one float per load
        for (int e = threadIdx.x; e < m * rows_per_rank; e += kThreads) {
            const int tok = e / rows_per_rank;
            const int r = r_lo + e % rows_per_rank;
            const uint32_t off = static_cast<uint32_t>((tok * kRows + r) * 4);
            float v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (q < cluster) v[q] = ld_shared_cluster_f32(map_shared_rank(part_addr + off, q));
            float sum = v[0];
#pragma unroll
            for (int q = 1; q < 8; ++q)
                if (q < cluster) sum = sum + v[q];
            const int64_t grow = row0 + r;
            if (grow < n) {
                if (kLora) sum = lora_term(sum, lora_t, lora_up, lora_r, tok, grow);
                if (kBf16Out)
                    reinterpret_cast<__nv_bfloat16*>(Y)[static_cast<int64_t>(tok) * n + grow] = __float2bfloat16_rn(sum);
                else
                    reinterpret_cast<float*>(Y)[static_cast<int64_t>(tok) * n + grow] = sum;
            }
        }
    }
    for (int e = threadIdx.x; e < (!bad && kRows % (4 * cluster) == 0 ? m * quads : 0); e += kThreads) {
        const int tok = e / quads;
        const int r = r_lo + 4 * (e % quads);
        const uint32_t off = static_cast<uint32_t>((tok * kRows + r) * 4);
        float4 v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (q < cluster) v[q] = ld_shared_cluster_f32x4(map_shared_rank(part_addr + off, q));
        float4 sum = v[0];
#pragma unroll
        for (int q = 1; q < 8; ++q)
            if (q < cluster) sum = make_float4(sum.x + v[q].x, sum.y + v[q].y, sum.z + v[q].z, sum.w + v[q].w);
        float o[4] = {sum.x, sum.y, sum.z, sum.w};
        store_quad<kBf16Out, kLora>(Y, n, tok, row0 + r, o, lora_t, lora_up, lora_r, t_fused ? tful : nullptr, utile,
                                    r);
    }
    cluster_sync();  // keep this CTA's partials alive until every rank has read them
}

}  // namespace gemv

// Cluster size (k split) for `tiles` row tiles of `stages` k stages.  The
// default is the smallest of 1, 2, 4, 8 that gives at least one CTA per SM
// without giving any CTA fewer than two stages.  Two CTAs fit on an SM, so the
// busiest SM's work is (CTAs on it) x (stages per CTA); another size of 1 .. 8
// that stays in one wave replaces the default when it cuts that work by at least
// a fifth (11008 rows: 258 CTAs of 6 stages instead of 172 of 8, i.e. 12 instead
// of 16).  Any size above 1 keeps tiles x size within two CTAs per SM.
static int64_t gemv_busiest(int64_t tiles, int64_t stages, int c, int sm_count) {
    const int64_t per_sm = (tiles * c + sm_count - 1) / sm_count;
    return per_sm * ((stages + c - 1) / c);
}

static int gemv_cluster_tiles(int64_t tiles, int64_t stages, int sm_count) {
    int c = 1;
    while (c < 8 && tiles * c < sm_count && 2 * c <= stages) c *= 2;
    const int64_t base = gemv_busiest(tiles, stages, c, sm_count);
    int best = c;
    int64_t best_cost = base;
    for (int cc = 2; cc <= 8; ++cc) {
        if (2 * cc > stages || tiles * cc > 2 * static_cast<int64_t>(sm_count)) break;
        const int64_t cost = gemv_busiest(tiles, stages, cc, sm_count);
        if (5 * cost <= 4 * base && cost < best_cost) {
            best = cc;
            best_cost = cost;
        }
    }
    return best;
}

static int64_t gemv_tiles(int64_t n) { return (n + gemv::kRows - 1) / gemv::kRows; }
static int64_t gemv_stages(int64_t k) { return (k + gemv::kStageK - 1) / gemv::kStageK; }

static int gemv_cluster(int64_t n, int64_t k, int sm_count) {
    return gemv_cluster_tiles(gemv_tiles(n), gemv_stages(k), sm_count);
}

// Workspace layout, the same for every shape so that one buffer can serve a
// sequence of different linears and groups: kWsCounters 32-bit counters (one per
// 128-row tile of a launch), then C slots per row tile, each an fp32 partial tile
// [16 tokens x 128 rows] followed by the CTA's share of a fused LoRA
// down-projection [16 tokens x 16 ranks].  A split k keeps tiles x C within two
// CTAs per SM, so the slots never number more than 2 x SMs.
constexpr int64_t kWsCounters = 1024;
constexpr size_t kWsCounterBytes = kWsCounters * 4;
constexpr size_t kWsPartBytes = (16 * gemv::kRows + 16 * 16) * sizeof(float);

static bool gemv_ws_usable(int64_t tiles, int cluster) { return cluster > 1 && tiles <= kWsCounters; }

bool gemv_fuses_lora(int64_t m, int64_t n, int64_t k, int r, bool has_ws, const DeviceInfo& dev) {
    if (m > kGemvMaxTokens || (r != 8 && r != 16)) return false;
    const int cluster = gemv_cluster(n, k, dev.sm_count);
    return cluster == 1 || (has_ws && gemv_ws_usable(gemv_tiles(n), cluster));
}

size_t linear_workspace_bytes(int64_t m, int64_t n, int64_t k, const DeviceInfo& dev) {
    if (m > kGemvMaxTokens) return 0;
    if (!gemv_ws_usable(gemv_tiles(n), gemv_cluster(n, k, dev.sm_count))) return 0;
    return kWsCounterBytes + 2 * static_cast<size_t>(dev.sm_count) * kWsPartBytes;
}

template <bool kBf16Out, bool kM16, bool kLora>
static cudaError_t launch_gemv(const gemv::GemvGroup& grp, int64_t tiles, const CUtensorMap& tm_x, int mt,
                               int64_t k, int cluster, bool weights_early, int32_t* dev_status, void* ws,
                               const LoraArgs& lora, int codebook, uint32_t test_flags, int device,
                               cudaStream_t stream) {
    static std::mutex mu;
    static bool attr_set[64] = {};
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!attr_set[device]) {
            const cudaError_t e = cudaFuncSetAttribute(gemv::k_nf4_gemv<kBf16Out, kM16, kLora>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize, gemv::kSmemBytes);
            if (e != cudaSuccess) return e;
            attr_set[device] = true;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles), cluster, 1);
    cfg.blockDim = dim3(gemv::kThreads, 1, 1);
    cfg.dynamicSmemBytes = gemv::kSmemBytes;
    cfg.stream = stream;
    // With a workspace (and a split k) the CTAs of a tile need not be co-scheduled: no cluster.
    const bool use_ws = ws != nullptr && gemv_ws_usable(tiles, cluster);
    uint32_t* ws_cnt = use_ws ? static_cast<uint32_t*>(ws) : nullptr;
    float4* ws_part = use_ws ? reinterpret_cast<float4*>(static_cast<char*>(ws) + kWsCounterBytes) : nullptr;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (!use_ws) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 1;
        attr[na].val.clusterDim.y = cluster;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (weights_early) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, gemv::k_nf4_gemv<kBf16Out, kM16, kLora>, grp, tm_x, mt, k, cluster,
                              weights_early ? 1 : 0, dev_status, ws_cnt, ws_part, lora.t, lora.up, lora.r, lora.down,
                              lora.scale, codebook, (test_flags & kTestStall) ? 64u : kWaitLimit,
                              (test_flags & kTestStall) ? 1 : 0);
}

// One of the eight instantiations: output type, more than 8 tokens, LoRA term.
static cudaError_t dispatch_gemv(bool bf16, bool m16, bool lora_on, const gemv::GemvGroup& grp, int64_t tiles,
                                 const CUtensorMap& tm_x, int mt, int64_t k, int cluster, bool early, int32_t* ds,
                                 void* ws, const LoraArgs& lora, int codebook, uint32_t test_flags, int device,
                                 cudaStream_t stream) {
#define NF4_GEMV_CASE(B, M, L)                                                                                   \
    if (bf16 == B && m16 == M && lora_on == L)                                                                  \
        return launch_gemv<B, M, L>(grp, tiles, tm_x, mt, k, cluster, early, ds, ws, lora, codebook, test_flags, \
                                    device, stream);
    NF4_GEMV_CASE(true, true, false)
    NF4_GEMV_CASE(true, false, false)
    NF4_GEMV_CASE(false, true, false)
    NF4_GEMV_CASE(false, false, false)
    NF4_GEMV_CASE(true, true, true)
    NF4_GEMV_CASE(true, false, true)
    NF4_GEMV_CASE(false, true, true)
    NF4_GEMV_CASE(false, false, true)
#undef NF4_GEMV_CASE
    return cudaErrorInvalidValue;
}

// One dequant-GEMV launch over the row tiles of `count` weights (m <= 16).
static cudaError_t gemv_launch_group(const void* X, int64_t m, int64_t k, const LinearWeight* w, int count,
                                     bool y_bf16, int32_t* dev_status, bool weights_early, void* ws,
                                     const LoraArgs& lora, int codebook, uint32_t test_flags, const DeviceInfo& dev,
                                     cudaStream_t stream) {
    gemv::GemvGroup grp;
    memset(&grp, 0, sizeof(grp));
    int64_t tiles = 0;
    for (int i = 0; i < count; ++i) {
        const cudaError_t e = tmap_2d(&grp.tm_w[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, w[i].wq, static_cast<uint64_t>(k / 2),
                                      static_cast<uint64_t>(w[i].n), static_cast<uint64_t>(k / 2), 128, gemv::kRows,
                                      CU_TENSOR_MAP_SWIZZLE_128B);
        if (e != cudaSuccess) return e;
        grp.absmax_q[i] = w[i].absmax_q;
        grp.absmax_scale[i] = w[i].absmax_scale;
        grp.mu[i] = w[i].absmax_offset;
        grp.y[i] = w[i].y;
        grp.n[i] = w[i].n;
        grp.tile0[i] = static_cast<int>(tiles);
        tiles += gemv_tiles(w[i].n);
    }
    grp.count = count;
    if (tiles > 0x7fffffff) return cudaErrorInvalidValue;
    const int cluster = gemv_cluster_tiles(tiles, gemv_stages(k), dev.sm_count);
    // portable cluster sizes only (the split-k epilogue handles any of 1 .. 8)
    if (cluster < 1 || cluster > 8) return cudaErrorInvalidConfiguration;
    CUtensorMap tm_x;
    const cudaError_t e = tmap_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, static_cast<uint64_t>(k),
                                  static_cast<uint64_t>(m), static_cast<uint64_t>(k * 2), 64, 16,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    if (lora.down != nullptr && cluster > 1 && !(ws != nullptr && gemv_ws_usable(tiles, cluster)))
        return cudaErrorInvalidValue;  // a fused down-projection needs C = 1 or the workspace split-k
    return dispatch_gemv(y_bf16, m > 8, lora.t != nullptr || lora.down != nullptr, grp, tiles, tm_x,
                         static_cast<int>(m), k, cluster,
                         weights_early, dev_status, ws, lora, codebook, test_flags, dev.device, stream);
}

static cudaError_t linear_one(const void* X, int64_t m, const LinearWeight& w, int64_t k, bool y_bf16,
                              int32_t* dev_status, bool weights_early, void* ws, const LoraArgs& lora, int codebook,
                              uint32_t test_flags, const DeviceInfo& dev, cudaStream_t stream) {
    if (m > kGemvMaxTokens)
        return launch_gemm(X, m, w.wq, w.absmax_q, w.absmax_scale, w.absmax_offset, w.n, k, w.y, y_bf16, dev_status,
                           lora, codebook, test_flags, dev, stream);
    return gemv_launch_group(X, m, k, &w, 1, y_bf16, dev_status, weights_early, ws, lora, codebook, test_flags, dev,
                             stream);
}

cudaError_t launch_linear(const void* X, int64_t m, const uint8_t* wq, const int8_t* absmax_q,
                          const float* absmax_scale, const float* absmax_offset, int64_t n,
                          int64_t k, void* Y, bool y_bf16, int32_t* dev_status, bool weights_early,
                          void* ws, const LoraArgs& lora, int codebook, const DeviceInfo& dev,
                          cudaStream_t stream) {
    if (dev.device < 0 || dev.device >= 64) return cudaErrorInvalidDevice;
    LinearWeight w;
    w.wq = wq;
    w.absmax_q = absmax_q;
    w.absmax_scale = absmax_scale;
    w.absmax_offset = absmax_offset;
    w.n = n;
    w.y = Y;
    return linear_one(X, m, w, k, y_bf16, dev_status, weights_early, ws, lora, codebook, 0u, dev, stream);
}

// Fixed cost of one launch, in units of one k stage of the busiest SM (a stage
// of two CTAs streams 32 KB of codes, about a microsecond): what a launch costs
// beyond its streaming (start-up, ring fill, split-k exchange).
constexpr int64_t kLaunchCostStages = 4;

// The weights of a group share X and k.  For m <= 16 they run as one launch over
// all their row tiles when the model of the busiest SM's work (stages, plus a
// fixed cost per launch) says it beats one launch per weight; q / k / v of a
// 4096-wide layer (3 x 32 tiles) do, gate / up of an 11008-wide MLP (2 x 86
// tiles, already one wave each) do not.  Larger m runs the GEMM once per weight.
bool group_in_one_launch(int64_t m, const int64_t* n, int count, int64_t k, bool lora, const DeviceInfo& dev) {
    if (m > kGemvMaxTokens || count < 2 || lora) return false;
    const int64_t stages = gemv_stages(k);
    int64_t separate = 0, tiles = 0;
    for (int i = 0; i < count; ++i) {
        const int64_t ti = gemv_tiles(n[i]);
        separate += gemv_busiest(ti, stages, gemv_cluster_tiles(ti, stages, dev.sm_count), dev.sm_count) +
                    kLaunchCostStages;
        tiles += ti;
    }
    const int64_t grouped =
        gemv_busiest(tiles, stages, gemv_cluster_tiles(tiles, stages, dev.sm_count), dev.sm_count) +
        kLaunchCostStages;
    return grouped < separate && tiles <= kWsCounters;
}

cudaError_t launch_linear_group(const void* X, int64_t m, int64_t k, const LinearWeight* w, int count,
                                bool y_bf16, int32_t* dev_status, bool weights_early, void* ws, const LoraArgs& lora,
                                int codebook, uint32_t test_flags, const DeviceInfo& dev, cudaStream_t stream) {
    if (dev.device < 0 || dev.device >= 64) return cudaErrorInvalidDevice;
    if (count < 1 || count > kMaxGroup) return cudaErrorInvalidValue;
    int64_t ns[kMaxGroup];
    for (int i = 0; i < count; ++i) ns[i] = w[i].n;
    if (group_in_one_launch(m, ns, count, k, lora.t != nullptr, dev))
        return gemv_launch_group(X, m, k, w, count, y_bf16, dev_status, weights_early, ws, lora, codebook,
                                 test_flags, dev, stream);
    for (int i = 0; i < count; ++i) {
        const cudaError_t e = linear_one(X, m, w[i], k, y_bf16, dev_status, weights_early, ws, lora, codebook,
                                         test_flags, dev, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace nf4
