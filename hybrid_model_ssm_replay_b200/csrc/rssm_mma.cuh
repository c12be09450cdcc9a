// rssm_mma.cuh -- warp-level tensor-core dot products for the replay kernels.
//
// The verify of K+1 tokens reads one state tile [P][N] and forms, for every
// row p and token j, h[p] . C_j -- a [P x N] x [N x (K+1)] product -- plus
// the replay terms sum_s coef[j][s] x_s[p] ([P x T] x [T x (K+1)]). Done on
// the CUDA cores every (row, token) sum needs a reduction across the lanes
// that hold the row's columns; with mma.sync the sums land in the
// accumulator fragment, one (row, token) per register, and the FMAs and
// shuffles of the reduction disappear. The decode of an FP4 copy uses the
// same route with the 8 columns of the product as the 8 scale blocks of a
// row (the block scales are applied afterwards, once per block).
//
// Operand precision (every product is formed exactly; sums are fp32):
//  * fp32 state: tf32 m16n8k8 with the state split into hi + lo tf32 parts
//    (hi keeps the top 11 significant bits; lo = h - hi is exact in fp32
//    and keeps 11 more), so h . C carries ~22 bits; C (bf16) is exact in tf32;
//  * bf16 state: bf16 m16n8k16, exact operands;
//  * e4m3 / FP4 state: f16 m16n8k16; e4m3 and e2m1 values, and e2m1 times
//    an e4m3 block scale, are exact in f16; C (bf16) is converted to f16,
//    exact for |C| >= 2^-17 (below that the f16 spacing is 2^-24);
//  * replay terms: x (bf16) is exact in tf32, coef is split hi + lo.
//
// Fragment layouts are those of the PTX ISA for mma.m16n8k8 (.tf32) and
// mma.m16n8k16 (.bf16/.f16), lane = 4 g + t:
//   A: a0 (row g, k lo), a1 (row g+8, k lo), a2 (row g, k hi), a3 (row g+8, k hi)
//      k lo / hi = {t} / {t+4} for k8, {2t, 2t+1} / {2t+8, 2t+9} for k16;
//   B: b0 (k lo, col g), b1 (k hi, col g);
//   D: d0 (row g, col 2t), d1 (row g, col 2t+1), d2 (row g+8, col 2t), d3 (row g+8, col 2t+1).
// Which physical column of the state a lane's "k" stands for is free, as
// long as the A and B operands of that lane agree; the kernels give lane t
// the 32 columns 32t..32t+31 (d_state 128), read in 8-column chunks, and
// rotate the chunk order by t where that spreads shared-memory banks.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace rssm {

// D += A B, A 16x8 tf32 (row-major), B 8x8 tf32 (column-major), D fp32.
__device__ __forceinline__ void mma_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D += A B, A 16x16 bf16, B 16x8 bf16 (pairs packed low element first).
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D += A B, A 16x16 f16, B 16x8 f16.
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// fp32 v = hi + lo with hi exact in tf32 (low 13 mantissa bits cleared) and
// lo = v - hi exact in fp32. Both returned as bit patterns.
__device__ __forceinline__ void tf32_split(float v, uint32_t& hi, uint32_t& lo) {
    const uint32_t h = __float_as_uint(v) & 0xFFFFE000u;
    hi = h;
    lo = __float_as_uint(v - __uint_as_float(h));
}

// The two bf16 of a 32-bit word as fp32 bit patterns (exact).
__device__ __forceinline__ uint32_t bf16lo_bits(uint32_t w) { return w << 16; }
__device__ __forceinline__ uint32_t bf16hi_bits(uint32_t w) { return w & 0xFFFF0000u; }

// Two bf16 (one word, low element first) as an f16 pair, rounded to nearest.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
    uint32_t h;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(__uint_as_float(w & 0xFFFF0000u)), "f"(__uint_as_float(w << 16)));
    return h;
}

// Eight e2m1 codes (one word, element 0 in the low nibble of byte 0) as
// four f16 pairs, h[k] = elements 2k (low half) and 2k+1 (exact).
__device__ __forceinline__ void e2m1x8_h2(uint32_t w, uint32_t (&h)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
}

// Four e4m3 codes (one word, element 0 in the low byte) as two f16 pairs (exact).
__device__ __forceinline__ void e4m3x4_h2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 l, h;\n\t"
        "mov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

// Packed f16 pair product (exact when the products fit f16, as e2m1 x e4m3 do).
__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Four 8x8 b16 matrices from shared memory, transposed: lane 8j + r gives
// the address of row r of matrix j; register j receives matrix j with lane
// (g, t) holding its elements (2t, g) and (2t + 1, g) -- the A fragment of a
// row-major operand stored k-major, or the B fragment of an operand stored
// [k][n].
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// Two fp32 values as a bf16 pair, rounded to nearest (lo in the low half).
__device__ __forceinline__ uint32_t f32x2_to_bf16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// An f16 pair (h, h) from the low or high half of x.
__device__ __forceinline__ uint32_t h2_dup_lo(uint32_t x) { return (x & 0xFFFFu) | (x << 16); }
__device__ __forceinline__ uint32_t h2_dup_hi(uint32_t x) { return (x >> 16) | (x & 0xFFFF0000u); }

}  // namespace rssm
