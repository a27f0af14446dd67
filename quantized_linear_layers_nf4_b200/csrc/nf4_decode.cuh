// nf4_decode.cuh -- decoding packed 4-bit codes into the bf16 dequantized weight
// on the CUDA cores, shared by the fused linears.
//
// Sources: page "篇2-bitsandbytes-具体观-算法与实现剖析" (xyzblog), §2.2 code walk
// (dequantize: level[idx] * absmax, then the matmul in the compute dtype); page
// "LLM 相關知識" (technicalnotes), §5 "動態反量化" (4-bit weights restored to BF16 per
// layer for the matrix multiply).
//
// The decoder here produces What = bf16_rn(fp32_rn(level[idx] * a)) -- the same
// bits nf4_dequantize writes -- as bf16x2 words in k order (lower k in the low
// half): per (row, 64-block) the 16 products are formed once and split into
// byte planes; each nibble is then decoded with byte permutes (integer pipe, no
// shared-memory traffic).
#pragma once

#include <stdint.h>

#include "nf4_common.cuh"

namespace nf4 {

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// (a & ~c) | (b & c)
__device__ __forceinline__ uint32_t select_bytes(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xD8;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ uint64_t dup_f32x2(float a) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(a));
    return r;
}

// Two levels (one packed byte, high nibble in the low 32 bits) times a, each
// product rounded to fp32 by one packed f32x2 multiply, both rounded to bf16:
// the high nibble (lower k) lands in the low half.
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

// bf16 table of one (row, block), as byte planes: plane h[q] holds the high
// bytes of entries 4q..4q+3, plane l[q] their low bytes.
struct Planes {
    uint32_t h[4], l[4];
};

// T[i] = bf16(fp32(c_i * a)) for the 16 levels (pairs of levels multiplied by
// one packed f32x2 multiply), split into byte planes.
__device__ __forceinline__ void build_planes(const uint64_t (&cpair)[8], float a, Planes& P) {
    const uint64_t aa = dup_f32x2(a);
    uint32_t t[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) t[j] = scale_pack(cpair[j], aa);
    // scale_pack puts the first level of a pair in the low half, so t[j] =
    // {T[2j] low half, T[2j+1] high half}
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        P.h[q] = prmt(t[2 * q], t[2 * q + 1], 0x7531);
        P.l[q] = prmt(t[2 * q], t[2 * q + 1], 0x6420);
    }
}

// Four nibbles (the low 16 bits of s; s ^ 0x8888 in sx) -> two bf16x2 words in
// k order.  For a nibble n < 8 the first permute picks T[n]'s byte and the
// second yields a sign fill; for n >= 8 the other way round; a byte mask built
// from each nibble's top bit selects the right one.  Nibble order in a packed
// byte is (element 2i high, element 2i+1 low), so the final permutes swap
// each pair back into k order.
__device__ __forceinline__ void decode4(uint32_t s, uint32_t sx, const Planes& P, uint32_t& o0, uint32_t& o1) {
    const uint32_t hA = prmt(P.h[0], P.h[1], s);
    const uint32_t hB = prmt(P.h[2], P.h[3], sx);
    const uint32_t lA = prmt(P.l[0], P.l[1], s);
    const uint32_t lB = prmt(P.l[2], P.l[3], sx);
    const uint32_t m = prmt(s * 16u, s, 0xD9C8);  // byte k = 0xff iff nibble k >= 8
    const uint32_t h = select_bytes(hA, hB, m);
    const uint32_t l = select_bytes(lA, lB, m);
    o0 = prmt(l, h, 0x4051);
    o1 = prmt(l, h, 0x6273);
}

}  // namespace nf4
