// rssm_device.cuh -- device-side building blocks of librssm (sm_100a).
//
//  * shared-memory bulk copies (cp.async.bulk, completion on an mbarrier),
//    and waits bounded by %globaltimer, so no kernel can spin forever;
//  * Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers:
//    As Easy as 1, 2, 3", SC'11);
//  * the number formats of the precision split (ReplaySSM article,
//    devotd.net "nvidia-replayssm-hybrid-model-ssm-decoding-state-buffer",
//    s4 "Prevent low-precision errors from accumulating again"):
//    stochastic rounding to bf16 / e4m3 in integer arithmetic on the fp32
//    bits, nearest rounding to e4m3 (scales) and e2m1 (FP4 codes) with the
//    hardware cvt instructions, and their decoders.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace rssm {

constexpr int kThreads = 256;               // threads per CTA of the one-CTA-per-tile kernels
constexpr int kWarps = kThreads / 32;
constexpr int kMaxCap = 32;                 // buffer slots per request (interval + drafts)
constexpr int kMaxHeadDim = 256;           // largest head_dim (rssm_check_desc)
constexpr int kMaxTok = 8;                  // tokens per verify call (K + 1)
constexpr int kMidTok = 5;                  // verify kernels specialised for K <= 4
constexpr int kPipeStagesMax = 24;          // shared-memory stages of the pipelined kernels
constexpr unsigned long long kWaitNs = 2000000000ull;  // bound of every wait (mbarrier, stage tag)

// ------------------------------------------------------------------ errors

__device__ __forceinline__ void set_error(int32_t* err, int32_t code) {
    if (err) atomicCAS(err, 0, code);
}

// ------------------------------------------------ mbarrier + bulk copies

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// Global -> shared bulk copy; bytes and both addresses multiples of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// One bounded try: the thread may sleep until the phase completes or about
// `hint_ns` pass. True once phase `parity` has completed.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits for phase `parity` of the barrier, at most about limit_ns. True on completion.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity, 100000u)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity, 100000u)) {
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// Waits until the shared-memory word *p equals v, at most about limit_ns.
__device__ __forceinline__ bool smem_wait_eq_bounded(const volatile int* p, int v, uint64_t limit_ns) {
    if (*p == v) return true;
    const uint64_t t0 = globaltimer_ns();
    while (*p != v) {
        if (globaltimer_ns() - t0 > limit_ns) return false;
        __nanosleep(64);
    }
    return true;
}

// ------------------------------------------------------------- loads

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// Four consecutive input elements as float4 (16-byte / 8-byte vector loads).
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                       __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
}

__device__ __forceinline__ float dot4(float4 a, float4 b) {
    return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

// d = a * b + c on two fp32 lanes at once: the packed fp32 FMA of sm_100
// (each lane an IEEE fma, rounded to nearest, exactly as fmaf).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// The rank-T update of an 8-row x 4-column register block with packed FMAs:
// acc2[p][c] holds rows 2p, 2p+1 of column c; per slot, w2[p] = the slot's
// weighted x of rows 2p, 2p+1 and b the slot's 4 B values. Each element sees
// acc = fma(w, b, acc) in slot order, as with scalar FMAs.
__device__ __forceinline__ void rank1_8x4(float2 (&acc2)[4][4], const float2 (&w2)[4], float4 b) {
    const float2 bd[4] = {make_float2(b.x, b.x), make_float2(b.y, b.y), make_float2(b.z, b.z), make_float2(b.w, b.w)};
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc2[p][c] = fma2(w2[p], bd[c], acc2[p][c]);
}

__device__ __forceinline__ float4 acc2_row(const float2 (&acc2)[4][4], int k) {
    const int p = k >> 1;
    return (k & 1) ? make_float4(acc2[p][0].y, acc2[p][1].y, acc2[p][2].y, acc2[p][3].y)
                   : make_float4(acc2[p][0].x, acc2[p][1].x, acc2[p][2].x, acc2[p][3].x);
}

__device__ __forceinline__ void acc2_set_row(float2 (&acc2)[4][4], int k, float4 v) {
    const int p = k >> 1;
    if (k & 1) {
        acc2[p][0].y = v.x; acc2[p][1].y = v.y; acc2[p][2].y = v.z; acc2[p][3].y = v.w;
    } else {
        acc2[p][0].x = v.x; acc2[p][1].x = v.y; acc2[p][2].x = v.z; acc2[p][3].x = v.w;
    }
}

// Sum over aligned groups of `width` lanes (width a power of two <= 32).
__device__ __forceinline__ float group_sum(float v, int width) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
        if (off < width) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// ------------------------------------------------------------------ Philox

// Philox4x32-10: ten rounds; round i uses key + i * (0x9E3779B9, 0xBB67AE85).
// The round keys depend only on the seed, so a kernel forms them once
// (PhiloxKeys) and every draw spends per round two 32 x 32 -> 64-bit
// multiplies (high and low halves at once) and two three-input XORs.
struct PhiloxKeys {
    uint32_t x[10], y[10];
};

__host__ __device__ __forceinline__ PhiloxKeys philox_keys(uint64_t seed) {
    PhiloxKeys K;
    uint32_t kx = static_cast<uint32_t>(seed), ky = static_cast<uint32_t>(seed >> 32);
#pragma unroll
    for (int i = 0; i < 10; ++i) {
        K.x[i] = kx;
        K.y[i] = ky;
        kx += 0x9E3779B9u;
        ky += 0xBB67AE85u;
    }
    return K;
}

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, const PhiloxKeys& K) {
#pragma unroll
    for (int i = 0; i < 10; ++i) {
        const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c.x;
        const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c.z;
        c = make_uint4(static_cast<uint32_t>(p1 >> 32) ^ c.y ^ K.x[i], static_cast<uint32_t>(p1),
                       static_cast<uint32_t>(p0 >> 32) ^ c.w ^ K.y[i], static_cast<uint32_t>(p0));
    }
    return c;
}

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
    return philox4x32_10(c, philox_keys(static_cast<uint64_t>(k.x) | (static_cast<uint64_t>(k.y) << 32)));
}

// Draws whose counters (c0, c1, c2, c3) share c1, c2, c3 (one head of one
// request at one flush): the parts of the first two rounds that do not
// depend on c0 -- the second word's multiply in round one and the first
// word's in round two -- are formed once (PhiloxFixed); each draw then runs
// the same ten rounds with two multiplies fewer.
struct PhiloxFixed {
    uint32_t f1k;  // round-one output y, xored with round two's x key
    uint32_t g, h;  // round two's multiply of round-one output x: high half ^ y key, low half
    uint32_t c3k;  // c3 ^ round one's y key
};

__device__ __forceinline__ PhiloxFixed philox_fixed(uint32_t c1, uint32_t c2, uint32_t c3, const PhiloxKeys& K) {
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c2;
    const uint32_t x1 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ K.x[0];
    const uint64_t q0 = static_cast<uint64_t>(0xD2511F53u) * x1;
    PhiloxFixed F;
    F.f1k = static_cast<uint32_t>(p1) ^ K.x[1];
    F.g = static_cast<uint32_t>(q0 >> 32) ^ K.y[1];
    F.h = static_cast<uint32_t>(q0);
    F.c3k = c3 ^ K.y[0];
    return F;
}

__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, const PhiloxFixed& F, const PhiloxKeys& K) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c0;  // round one: (x1, y1, z1, w1)
    const uint32_t z1 = static_cast<uint32_t>(p0 >> 32) ^ F.c3k, w1 = static_cast<uint32_t>(p0);
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * z1;  // round two
    uint4 c = make_uint4(static_cast<uint32_t>(p1 >> 32) ^ F.f1k, static_cast<uint32_t>(p1), F.g ^ w1, F.h);
#pragma unroll
    for (int i = 2; i < 10; ++i) {
        const uint64_t q0 = static_cast<uint64_t>(0xD2511F53u) * c.x;
        const uint64_t q1 = static_cast<uint64_t>(0xCD9E8D57u) * c.z;
        c = make_uint4(static_cast<uint32_t>(q1 >> 32) ^ c.y ^ K.x[i], static_cast<uint32_t>(q1),
                       static_cast<uint32_t>(q0 >> 32) ^ c.w ^ K.y[i], static_cast<uint32_t>(q0));
    }
    return c;
}

// ------------------------------------------------------ stochastic rounding
// |v| = q (m + f) with q the target spacing at |v|; the magnitude rounds up
// iff r < floor(f * 2^32). Worked on the fp32 bit pattern.

// bf16 keeps the top 16 bits of fp32, so f * 2^16 is the low 16 bits L and
// the result is (u >> 16) + [(r >> 16) < L]. One add forms it: L + 0xFFFF -
// (r >> 16) reaches 2^16 exactly when (r >> 16) < L, so the carry into the
// high half is the rounding increment. Two values packed into one word
// (v0 in the low half); a NaN stays a NaN (quiet bit set).
__device__ __forceinline__ uint32_t sr_bf16x2(float v0, float v1, uint32_t r0, uint32_t r1) {
    const uint32_t u0 = __float_as_uint(v0), u1 = __float_as_uint(v1);
    const uint32_t t0 = (v0 != v0) ? (u0 | 0x00400000u) : u0 + (0xFFFFu - (r0 >> 16));
    const uint32_t t1 = (v1 != v1) ? (u1 | 0x00400000u) : u1 + (0xFFFFu - (r1 >> 16));
    return __byte_perm(t0, t1, 0x7632);  // the high halves of t0, t1
}



// OCP e4m3 ("fn"): bias 7, spacing 2^(E-3) for |v| >= 2^-6, 2^-9 below;
// |v| >= 448 (and inf) saturates to 448, NaN -> 0x7F.
__device__ __forceinline__ uint32_t sr_e4m3(float v, uint32_t r) {
    const uint32_t u = __float_as_uint(v);
    const uint32_t sign = (u >> 24) & 0x80u;
    const uint32_t a = u & 0x7FFFFFFFu;
    if (a > 0x7F800000u) return 0x7Fu;
    if (a >= 0x43E00000u) return sign | 0x7Eu;
    uint32_t code, F;
    if (a >= 0x3C800000u) {
        // normal: the exponent and top 3 mantissa bits re-biased (127 -> 7);
        // the 20 bits below them are the fraction
        code = (a >> 20) - (120u << 3);
        F = a << 12;
    } else {
        // below 2^-6: t = |v| 2^9 < 8 is exact, code = floor(t), and the
        // fraction scaled by 2^32 is exact too (at most 24 significant bits).
        // Float arithmetic on purpose: an integer-only form (a 32.32
        // fixed-point shift) costs more ALU issue, the refresh's bound.
        const float t = __uint_as_float(a) * 512.0f;
        const float m = truncf(t);
        code = static_cast<uint32_t>(m);
        F = __float2uint_rz((t - m) * 4294967296.0f);
    }
    return sign | (code + (r < F ? 1u : 0u));
}

// sr_e4m3 for |v| < 448 (not NaN, no saturation).
__device__ __forceinline__ uint32_t sr_e4m3_in_range(float v, uint32_t r) {
    const uint32_t u = __float_as_uint(v);
    const uint32_t sign = (u >> 24) & 0x80u;
    const uint32_t a = u & 0x7FFFFFFFu;
    uint32_t code, F;
    if (a >= 0x3C800000u) {
        code = (a >> 20) - (120u << 3);
        F = a << 12;
    } else {
        const float t = __uint_as_float(a) * 512.0f;
        const float m = truncf(t);
        code = static_cast<uint32_t>(m);
        F = __float2uint_rz((t - m) * 4294967296.0f);
    }
    return sign | (code + (r < F ? 1u : 0u));
}

// --------------------------------------------------------- nearest rounding

// e4m3, round to nearest even, saturating (hardware conversion).
__device__ __forceinline__ uint32_t e4m3_rn(float v) {
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(v));
    return out & 0xFFu;
}

// Two e2m1 codes (nearest even, saturating to +-6): lo in bits 0..3, hi in 4..7.
__device__ __forceinline__ uint32_t e2m1x2_rn(float lo, float hi) {
    uint32_t out;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "mov.b32 %0, {t, t, t, t};\n\t}"
        : "=r"(out)
        : "f"(hi), "f"(lo));
    return out & 0xFFu;
}

// Two e4m3 codes (16 bits, element 0 in the low byte) as an fp16 pair
// (hardware conversion; every e4m3 value is exact in fp16).
__device__ __forceinline__ uint32_t e4m3x2_h2(uint32_t codes16) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<unsigned short>(codes16)));
    return h;
}

__device__ __forceinline__ float2 h2_f2(uint32_t h) { return __half22float2(*reinterpret_cast<const __half2*>(&h)); }

__device__ __forceinline__ float e4m3_val(uint32_t c) { return h2_f2(e4m3x2_h2(c & 0xFFu)).x; }

__device__ __forceinline__ float bf16_val(uint32_t bits) { return __uint_as_float(bits << 16); }

// Four e2m1 codes (16 bits, element 0 in the low nibble) as floats, exactly
// (hardware conversion of each byte to an fp16 pair, low nibble first).
__device__ __forceinline__ float4 e2m1x4_val(uint32_t codes16) {
    uint32_t h01, h23;
    asm("{\n\t.reg .b8 b0, b1;\n\t"
        "mov.b16 {b0, b1}, %2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t}"
        : "=r"(h01), "=r"(h23)
        : "h"(static_cast<unsigned short>(codes16)));
    const float2 a = h2_f2(h01), b = h2_f2(h23);
    return make_float4(a.x, a.y, b.x, b.y);
}

// Eight e2m1 codes (32 bits, element 0 in the low nibble) as floats times
// scale (exact: hardware conversion of each byte to an fp16 pair). The word
// is split into its four bytes inside one asm block.
__device__ __forceinline__ void e2m1x8_val(uint32_t w, float scale, float* v) {
    uint32_t h0, h1, h2, h3;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
        : "r"(w));
    const uint32_t h[4] = {h0, h1, h2, h3};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = h2_f2(h[i]);
        v[2 * i] = f.x * scale;
        v[2 * i + 1] = f.y * scale;
    }
}

// Dot product of eight e2m1 codes (32 bits, element 0 in the low nibble)
// with c[0..7], unscaled, added to acc in element order.
__device__ __forceinline__ float e2m1x8_dot(uint32_t w, const float* c, float acc) {
    uint32_t h0, h1, h2, h3;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
        : "r"(w));
    float2 f = h2_f2(h0);
    acc = fmaf(f.x, c[0], acc);
    acc = fmaf(f.y, c[1], acc);
    f = h2_f2(h1);
    acc = fmaf(f.x, c[2], acc);
    acc = fmaf(f.y, c[3], acc);
    f = h2_f2(h2);
    acc = fmaf(f.x, c[4], acc);
    acc = fmaf(f.y, c[5], acc);
    f = h2_f2(h3);
    acc = fmaf(f.x, c[6], acc);
    acc = fmaf(f.y, c[7], acc);
    return acc;
}

// Four FP4 values: codes times their block scale (products are exact).
__device__ __forceinline__ float4 fp4x4_val(uint32_t codes16, float scale) {
    const float4 v = e2m1x4_val(codes16);
    return make_float4(v.x * scale, v.y * scale, v.z * scale, v.w * scale);
}

// Four e4m3 codes (32 bits, element 0 in the low byte) to floats.
__device__ __forceinline__ float4 e4m3x4_val(uint32_t w) {
    const float2 a = h2_f2(e4m3x2_h2(w & 0xFFFFu)), b = h2_f2(e4m3x2_h2(w >> 16));
    return make_float4(a.x, a.y, b.x, b.y);
}

// Four bf16 (two 32-bit words, element 0 in the low half) to floats.
__device__ __forceinline__ float4 bf16x4_val(uint2 w) {
    return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u),
                       __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xFFFF0000u));
}

// FP4 copy of 16 contiguous values held as one float4 by each of 4
// consecutive lanes: scale = e4m3_rn(amax / 6), codes = e2m1_rn(v / scale)
// with both quotients the correctly rounded fp32 ones, all codes 0 when the
// scale is 0. All 32 lanes must call it. Returns this lane's 16 code bits
// and sets *scale_code.
//
// The quotients are bracketed instead of divided: for x >= 0 and c_lo <=
// 1/d <= c_hi, x c_lo <= x / d <= x c_hi, and fp32 rounding and both
// nearest-even conversions are monotone, so when the two ends convert to the
// same code, that is the code of the rounded quotient. 1/6 lies between two
// adjacent floats; 1/scale comes from rcp.approx (within 2^-23 relative) and
// is widened by 2^-19 either way. Only a lane whose ends differ (a quotient
// within about 2^-19 of a rounding boundary) divides.
__device__ __forceinline__ uint32_t fp4_quant_quad(float4 v, uint32_t* scale_code) {
    float amax = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    constexpr float kSixthLo = 0x1.555554p-3f, kSixthHi = 0x1.555556p-3f;  // adjacent floats around 1/6
    uint32_t sc = e4m3_rn(amax * kSixthLo);
    if (sc != e4m3_rn(amax * kSixthHi)) sc = e4m3_rn(__fdiv_rn(amax, 6.0f));
    *scale_code = sc;
    const float s = e4m3_val(sc);
    if (s == 0.0f) return 0u;
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));  // s >= 2^-9: never subnormal
    const float rlo = r * (1.0f - 0x1p-19f), rhi = r * (1.0f + 0x1p-19f);
    const uint32_t lo = e2m1x2_rn(v.x * rlo, v.y * rlo) | (e2m1x2_rn(v.z * rlo, v.w * rlo) << 8);
    const uint32_t hi = e2m1x2_rn(v.x * rhi, v.y * rhi) | (e2m1x2_rn(v.z * rhi, v.w * rhi) << 8);
    if (lo == hi) return lo;
    const uint32_t c01 = e2m1x2_rn(__fdiv_rn(v.x, s), __fdiv_rn(v.y, s));
    const uint32_t c23 = e2m1x2_rn(__fdiv_rn(v.z, s), __fdiv_rn(v.w, s));
    return c01 | (c23 << 8);
}

// Eight e2m1 codes (nearest even, saturating to +-6) of v[0..7] scaled by
// m: element i in nibble i.
__device__ __forceinline__ uint32_t e2m1x8_rn(const float* v, float m) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(v[0] * m), "f"(v[1] * m), "f"(v[2] * m), "f"(v[3] * m), "f"(v[4] * m), "f"(v[5] * m),
          "f"(v[6] * m), "f"(v[7] * m));
    return out;
}

// max(|v_i|) over a block of 16 held by one thread: with fmaxf (NaN values
// ignored, as the FP4 scale takes them) or NaN-propagating (NaN iff some v_i
// is NaN, else the same value).
__device__ __forceinline__ float fmax_nan(float a, float b) {
    float d;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}
template <bool NAN_PROPAGATES>
__device__ __forceinline__ float absmax16(const float (&v)[16]) {
    auto mx = [](float a, float b) { return NAN_PROPAGATES ? fmax_nan(a, b) : fmaxf(a, b); };
    float m8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m8[i] = mx(fabsf(v[i]), fabsf(v[i + 8]));
#pragma unroll
    for (int i = 0; i < 4; ++i) m8[i] = mx(m8[i], m8[i + 4]);
    return mx(mx(m8[0], m8[2]), mx(m8[1], m8[3]));
}

// FP4 copy of one block of 16 contiguous values held by one thread: the
// scale and codes of fp4_quant_quad (the same bracketed quotients), with
// the block maximum (NaN values ignored) given or taken in registers.
// Returns the 64 code bits, element i in nibble i % 8 of word i / 8, and
// sets *scale_code.
__device__ __forceinline__ uint2 fp4_quant16(const float (&v)[16], float amax, uint32_t* scale_code) {
    constexpr float kSixthLo = 0x1.555554p-3f, kSixthHi = 0x1.555556p-3f;  // adjacent floats around 1/6
    uint32_t sc = e4m3_rn(amax * kSixthLo);
    if (sc != e4m3_rn(amax * kSixthHi)) sc = e4m3_rn(__fdiv_rn(amax, 6.0f));
    *scale_code = sc;
    const float s = e4m3_val(sc);
    if (s == 0.0f) return make_uint2(0u, 0u);
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));  // s >= 2^-9: never subnormal
    const float rlo = r * (1.0f - 0x1p-19f), rhi = r * (1.0f + 0x1p-19f);
    const uint2 lo = make_uint2(e2m1x8_rn(v, rlo), e2m1x8_rn(v + 8, rlo));
    const uint2 hi = make_uint2(e2m1x8_rn(v, rhi), e2m1x8_rn(v + 8, rhi));
    if (lo.x == hi.x && lo.y == hi.y) return lo;
    float q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = __fdiv_rn(v[i], s);
    return make_uint2(e2m1x8_rn(q, 1.0f), e2m1x8_rn(q + 8, 1.0f));
}

__device__ __forceinline__ uint2 fp4_quant16(const float (&v)[16], uint32_t* scale_code) {
    return fp4_quant16(v, absmax16<false>(v), scale_code);
}

}  // namespace rssm
