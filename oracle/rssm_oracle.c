/*
 * rssm_oracle.c -- plain fp64 CPU oracle for the replay-based SSM decode path.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library. The GPU library shares no code,
 * header, table or helper with it, and never calls it.
 *
 * Source of the method: the ReplaySSM article (devotd.net news page
 * "nvidia-replayssm-hybrid-model-ssm-decoding-state-buffer", English version),
 *   s1 "Store recent inputs instead of the full state"
 *   s3 "Roll back incorrect predictions using buffer positions"
 *   s4 "Prevent low-precision errors from accumulating again".
 * The article gives no formula. The concrete instance is a Mamba-2-style
 * selective SSM with one scalar decay per head:
 *     a_t  = exp(dt_t * A_h)
 *     h_t  = a_t * h_{t-1} + dt_t * x_t (outer) B_t        h: [head_dim P][d_state N]
 *     y_t  = h_t . C_t + D_h * x_t
 * B and C are shared by the H/G consecutive heads of a group.
 *
 * Everything is single-threaded and unblocked, in fp64, in the order the
 * definitions state. Every function here is pinned by a test in
 * tests/test_oracle_*.py against closed forms, special cases, brute force
 * or a library routine (none is "parity unpinned").
 *
 * Per-request layouts used here (independent of the GPU library's layouts):
 *   ckpt [H][P][N]   xb [Lcap][H][P]   Bb [Lcap][G][N]   dtb [Lcap][H]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Group of head h: contiguous groups of H/G heads each. */
static int group_of(int h, int H, int G) { return h / (H / G); }

/* ------------------------------------------------------------------------ */
/* 1. Conventional recurrence: the definition itself.                       */
/*    ReplaySSM article s1: the conventional scheme reads and writes the    */
/*    whole state for every token.                                          */
/* ------------------------------------------------------------------------ */

/* Runs T tokens of one request. h [H][P][N] is updated in place.
 * x [T][H][P], B and C [T][G][N], dt [T][H], A [H], D [H], y [T][H][P]. */
void oracle_conv_steps(int H, int P, int N, int G, int T, double *h,
                       const double *x, const double *B, const double *C,
                       const double *dt, const double *A, const double *D,
                       double *y)
{
    for (int t = 0; t < T; ++t) {
        const double *xt = x + (size_t)t * H * P;
        const double *Bt = B + (size_t)t * G * N;
        const double *Ct = C + (size_t)t * G * N;
        const double *dtt = dt + (size_t)t * H;
        double *yt = y + (size_t)t * H * P;
        for (int hh = 0; hh < H; ++hh) {
            int g = group_of(hh, H, G);
            double a = exp(dtt[hh] * A[hh]);
            for (int p = 0; p < P; ++p) {
                double *row = h + ((size_t)hh * P + p) * N;
                double xp = xt[(size_t)hh * P + p];
                double acc = 0.0;
                for (int n = 0; n < N; ++n) {
                    row[n] = a * row[n] + dtt[hh] * xp * Bt[(size_t)g * N + n];
                    acc += row[n] * Ct[(size_t)g * N + n];
                }
                yt[(size_t)hh * P + p] = acc + D[hh] * xp;
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* 2. Replay form: checkpoint + buffer of recent inputs.                    */
/*    ReplaySSM article s1: the state is the checkpoint from the start of   */
/*    the interval plus the inputs received since; each output reads the    */
/*    checkpoint, and the checkpoint is rewritten once the buffer is full.  */
/* ------------------------------------------------------------------------ */

static void put_entry(int H, int P, int N, int G, int slot, double *xb,
                      double *Bb, double *dtb, const double *x,
                      const double *B, const double *dt)
{
    memcpy(xb + (size_t)slot * H * P, x, sizeof(double) * (size_t)H * P);
    memcpy(Bb + (size_t)slot * G * N, B, sizeof(double) * (size_t)G * N);
    memcpy(dtb + (size_t)slot * H, dt, sizeof(double) * (size_t)H);
}

/* a_r of head hh for buffer slot r */
static double slot_decay(const double *dtb, const double *A, int H, int r, int hh)
{
    return exp(dtb[(size_t)r * H + hh] * A[hh]);
}

/* Output of the token held in slot t, whose C is Ct [G][N]:
 *   y[h,p] = (prod_{r=0..t} a_r) * sum_n ckpt[h,p,n] C[n]
 *          + sum_{s=0..t} (prod_{r=s+1..t} a_r) * dt_s * (B_s . C) * x_s[h,p]
 *          + D_h * x_t[h,p]                                                    */
static void replay_output(int H, int P, int N, int G, const double *ckpt,
                          const double *xb, const double *Bb, const double *dtb,
                          const double *A, const double *D, const double *Ct,
                          int t, double *y)
{
    double *w = (double *)malloc(sizeof(double) * (size_t)(t + 1));
    for (int hh = 0; hh < H; ++hh) {
        int g = group_of(hh, H, G);
        const double *Cg = Ct + (size_t)g * N;
        double decay = 1.0;
        for (int r = 0; r <= t; ++r) decay *= slot_decay(dtb, A, H, r, hh);
        for (int s = 0; s <= t; ++s) {
            double prod = 1.0;
            for (int r = s + 1; r <= t; ++r) prod *= slot_decay(dtb, A, H, r, hh);
            double bc = 0.0;
            for (int n = 0; n < N; ++n) bc += Bb[((size_t)s * G + g) * N + n] * Cg[n];
            w[s] = dtb[(size_t)s * H + hh] * prod * bc;
        }
        for (int p = 0; p < P; ++p) {
            const double *row = ckpt + ((size_t)hh * P + p) * N;
            double hc = 0.0;
            for (int n = 0; n < N; ++n) hc += row[n] * Cg[n];
            double acc = decay * hc;
            for (int s = 0; s <= t; ++s) acc += w[s] * xb[((size_t)s * H + hh) * P + p];
            y[(size_t)hh * P + p] = acc + D[hh] * xb[((size_t)t * H + hh) * P + p];
        }
    }
    free(w);
}

/* Standard decode of one token: append it at slot *pos, output it, advance.
 * Returns -1 (and changes nothing) when the buffer has no free slot. */
int oracle_replay_decode(int H, int P, int N, int G, int Lcap,
                         const double *ckpt, double *xb, double *Bb, double *dtb,
                         int *pos, const double *x, const double *B,
                         const double *C, const double *dt, const double *A,
                         const double *D, double *y)
{
    if (*pos < 0 || *pos >= Lcap) return -1;
    put_entry(H, P, N, G, *pos, xb, Bb, dtb, x, B, dt);
    replay_output(H, P, N, G, ckpt, xb, Bb, dtb, A, D, C, *pos, y);
    *pos += 1;
    return 0;
}

/* Fold the T = *pos buffered entries into state [H][P][N]:
 *   state[h,p,n] <- (prod_{r<T} a_r) state[h,p,n]
 *                 + sum_{s<T} (prod_{s<r<T} a_r) dt_s x_s[h,p] B_s[n]          */
static void fold_fp64(int H, int P, int N, int G, double *state,
                      const double *xb, const double *Bb, const double *dtb,
                      int T, const double *A)
{
    double *c = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    for (int hh = 0; hh < H; ++hh) {
        int g = group_of(hh, H, G);
        double decay = 1.0;
        for (int r = 0; r < T; ++r) decay *= slot_decay(dtb, A, H, r, hh);
        for (int s = 0; s < T; ++s) {
            double prod = 1.0;
            for (int r = s + 1; r < T; ++r) prod *= slot_decay(dtb, A, H, r, hh);
            c[s] = dtb[(size_t)s * H + hh] * prod;
        }
        for (int p = 0; p < P; ++p) {
            double *row = state + ((size_t)hh * P + p) * N;
            for (int n = 0; n < N; ++n) {
                double v = decay * row[n];
                for (int s = 0; s < T; ++s)
                    v += c[s] * xb[((size_t)s * H + hh) * P + p] * Bb[((size_t)s * G + g) * N + n];
                row[n] = v;
            }
        }
    }
    free(c);
}

/* Interval flush: fold every buffered entry into the checkpoint, empty the
 * buffer (ReplaySSM article s1: one checkpoint write per interval). */
void oracle_replay_flush(int H, int P, int N, int G, double *ckpt,
                         const double *xb, const double *Bb, const double *dtb,
                         int *pos, const double *A)
{
    fold_fp64(H, P, N, G, ckpt, xb, Bb, dtb, *pos, A);
    *pos = 0;
}

/* Speculative verify (ReplaySSM article s3): the ntok tokens (pending token
 * plus drafts) go into slots pos..pos+ntok-1, every one gets its output from
 * the checkpoint and the buffer, no state is produced and pos stays put.
 * x [ntok][H][P], B and C [ntok][G][N], dt [ntok][H], y [ntok][H][P].
 * Returns -1 (and changes nothing) when the slots do not fit. */
int oracle_replay_verify(int H, int P, int N, int G, int Lcap,
                         const double *ckpt, double *xb, double *Bb, double *dtb,
                         int pos, int ntok, const double *x, const double *B,
                         const double *C, const double *dt, const double *A,
                         const double *D, double *y)
{
    if (pos < 0 || ntok < 1 || pos + ntok > Lcap) return -1;
    for (int j = 0; j < ntok; ++j)
        put_entry(H, P, N, G, pos + j, xb, Bb, dtb, x + (size_t)j * H * P,
                  B + (size_t)j * G * N, dt + (size_t)j * H);
    for (int j = 0; j < ntok; ++j)
        replay_output(H, P, N, G, ckpt, xb, Bb, dtb, A, D,
                      C + (size_t)j * G * N, pos + j, y + (size_t)j * H * P);
    return 0;
}

/* Accept n drafts: the valid length grows by the pending token plus n. */
void oracle_replay_accept(int *pos, int n) { *pos += n + 1; }

/* ------------------------------------------------------------------------ */
/* 3. Counter-based random numbers: Philox4x32-10.                          */
/*    Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as      */
/*    1, 2, 3", SC'11, section 4 (Philox): ten rounds of two 32x32->64      */
/*    multiplies, key bumped by the Weyl constants between rounds.          */
/* ------------------------------------------------------------------------ */

void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += W0; k1 += W1; }
        uint64_t p0 = (uint64_t)M0 * c0;
        uint64_t p1 = (uint64_t)M1 * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* ------------------------------------------------------------------------ */
/* 4. Number formats. Written in exact double arithmetic on values.         */
/*    bf16: IEEE binary32 with the low 16 fraction bits dropped.            */
/*    e4m3: OCP 8-bit floating point (E4M3, "fn"): bias 7, no infinity,     */
/*          NaN = S.1111.111, largest finite 448, subnormal step 2^-9.      */
/*    e2m1: OCP Microscaling FP4 (E2M1): bias 1, values 0, 0.5, 1, 1.5, 2,  */
/*          3, 4, 6; no infinity or NaN.                                    */
/* ------------------------------------------------------------------------ */

double oracle_bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

double oracle_e4m3_value(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    return s ? -mag : mag;
}

double oracle_e2m1_value(uint8_t c)
{
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp((double)(2 + m), e - 2);
    return s ? -mag : mag;
}

/* Bit pattern of a representable e4m3 magnitude (0 or in [2^-9, 448]). */
static uint8_t e4m3_encode_exact(int neg, double mag)
{
    uint8_t bits;
    if (mag < ldexp(1.0, -6)) {
        bits = (uint8_t)(mag / ldexp(1.0, -9));
    } else {
        int e;
        double fr = frexp(mag, &e);           /* mag = fr * 2^e, fr in [0.5, 1) */
        int m = (int)((2.0 * fr - 1.0) * 8.0);
        bits = (uint8_t)(((e - 1 + 7) << 3) | m);
    }
    return (uint8_t)(neg ? (bits | 0x80) : bits);
}

/* Spacing of e4m3 values around magnitude a (0 < a < 448). */
static double e4m3_quantum(double a)
{
    if (a < ldexp(1.0, -6)) return ldexp(1.0, -9);
    int e;
    frexp(a, &e);
    return ldexp(1.0, e - 1 - 3);
}

/* Spacing of bf16 values around magnitude a (0 < a < 2^128). */
static double bf16_quantum(double a)
{
    if (a < ldexp(1.0, -126)) return ldexp(1.0, -133);
    int e;
    frexp(a, &e);
    return ldexp(1.0, e - 1 - 7);
}

/* Round to nearest, ties to even, saturating to +-448 (inf included). */
uint8_t oracle_e4m3_rne(float v)
{
    if (isnan(v)) return 0x7F;
    int neg = signbit(v) != 0;
    double a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(neg ? 0xFE : 0x7E);
    double q = e4m3_quantum(a);
    double r = nearbyint(a / q) * q;       /* default mode: ties to even */
    return e4m3_encode_exact(neg, r);
}

/* Round to nearest, ties to even, saturating to +-6. Finite inputs only. */
uint8_t oracle_e2m1_rne(float v)
{
    int neg = signbit(v) != 0;
    double a = fabs((double)v);
    int c;
    if (a >= 6.0) {
        c = 7;
    } else {
        double q = (a < 2.0) ? 0.5 : (a < 4.0 ? 1.0 : 2.0);
        double r = nearbyint(a / q) * q;
        static const double mags[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
        c = 0;
        for (int i = 0; i < 8; ++i)
            if (mags[i] == r) c = i;
    }
    return (uint8_t)(neg ? (c | 8) : c);
}

/* Stochastic rounding (ReplaySSM article s4: the update copy is rounded at
 * random to one of the two neighbouring representable values). With
 * |v| = q (m + f), m integer, f in [0,1), q the target spacing at |v|, the
 * magnitude rounds up iff r < floor(f * 2^32); the sign is kept. Thus
 * P(up) = floor(f 2^32) / 2^32 for a uniform 32-bit r. */
uint16_t oracle_sr_bf16(float v, uint32_t r)
{
    uint32_t u;
    memcpy(&u, &v, 4);
    if (isnan(v)) return (uint16_t)((u >> 16) | 0x0040);
    if (isinf(v)) return (uint16_t)(u >> 16);
    int neg = signbit(v) != 0;
    double a = fabs((double)v);
    if (a == 0.0) return (uint16_t)(neg ? 0x8000 : 0);
    double q = bf16_quantum(a);
    double m = floor(a / q);
    double f = a / q - m;
    double F = floor(ldexp(f, 32));
    double res = ((double)r < F) ? (m + 1.0) * q : m * q;
    float rf = (float)res;                  /* exact, or +inf past the top */
    uint32_t b;
    memcpy(&b, &rf, 4);
    b >>= 16;
    return (uint16_t)(neg ? (b | 0x8000) : b);
}

uint8_t oracle_sr_e4m3(float v, uint32_t r)
{
    if (isnan(v)) return 0x7F;
    int neg = signbit(v) != 0;
    double a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(neg ? 0xFE : 0x7E);
    if (a == 0.0) return (uint8_t)(neg ? 0x80 : 0);
    double q = e4m3_quantum(a);
    double m = floor(a / q);
    double f = a / q - m;
    double F = floor(ldexp(f, 32));
    double res = ((double)r < F) ? (m + 1.0) * q : m * q;
    return e4m3_encode_exact(neg, res);
}

/* FP4 output copy of 16 contiguous values: one e4m3 scale
 * s = e4m3_rne(amax / 6) (fp32 division), codes e2m1_rne(v_i / s) (fp32
 * division), all codes 0 when s is 0. Element 2k in the low nibble of
 * byte k, element 2k+1 in the high nibble. */
void oracle_fp4_quant16(const float *v, uint8_t *codes, uint8_t *scale)
{
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float m = fabsf(v[i]);
        if (m > amax) amax = m;
    }
    float sv = amax / 6.0f;
    uint8_t sc = oracle_e4m3_rne(sv);
    float s = (float)oracle_e4m3_value(sc);
    *scale = sc;
    for (int k = 0; k < 8; ++k) codes[k] = 0;
    if (s == 0.0f) return;
    for (int i = 0; i < 16; ++i) {
        float qv = v[i] / s;
        uint8_t c = oracle_e2m1_rne(qv);
        codes[i / 2] |= (uint8_t)((i & 1) ? (c << 4) : c);
    }
}

/* ------------------------------------------------------------------------ */
/* 5. Precision split (ReplaySSM article s4): a high-precision update copy  */
/*    that only the interval update reads, and a separate low-precision     */
/*    output copy that only the outputs read.                               */
/* ------------------------------------------------------------------------ */

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_E4M3 = 2, ORC_FP4 = 3 };

/* Values of a state copy of n_el elements: f32 (float), bf16 (uint16),
 * e4m3 (uint8), or FP4 codes + scales (16 elements per scale). */
void oracle_widen(int dtype, size_t n_el, const void *src, const uint8_t *scales, double *out)
{
    for (size_t i = 0; i < n_el; ++i) {
        switch (dtype) {
        case ORC_F32: out[i] = ((const float *)src)[i]; break;
        case ORC_BF16: out[i] = oracle_bf16_value(((const uint16_t *)src)[i]); break;
        case ORC_E4M3: out[i] = oracle_e4m3_value(((const uint8_t *)src)[i]); break;
        default: {
            uint8_t byte = ((const uint8_t *)src)[i / 2];
            uint8_t c = (uint8_t)((i & 1) ? (byte >> 4) : (byte & 15));
            out[i] = oracle_e2m1_value(c) * oracle_e4m3_value(scales[i / 16]);
        }
        }
    }
}

/* Stochastic rounding of one head's values v [P*N] into an update copy,
 * with random word (e mod 4) of Philox4x32-10 at counter
 * (e / 4, head, request, flush_count) and key (lo32(seed), hi32(seed)),
 * e = p * N + n. */
void oracle_sr_head(int dtype, uint64_t seed, uint32_t request, uint32_t head,
                    uint32_t flush_count, size_t n_el, const float *v, void *out)
{
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    for (size_t e = 0; e < n_el; ++e) {
        uint32_t ctr[4] = {(uint32_t)(e / 4), head, request, flush_count}, w[4];
        oracle_philox4x32_10(ctr, key, w);
        uint32_t r = w[e % 4];
        if (dtype == ORC_BF16) ((uint16_t *)out)[e] = oracle_sr_bf16(v[e], r);
        else ((uint8_t *)out)[e] = oracle_sr_e4m3(v[e], r);
    }
}

/* FP4 copy of n_el values (n_el a multiple of 16). */
void oracle_fp4_quant(size_t n_el, const float *v, uint8_t *codes, uint8_t *scales)
{
    for (size_t blk = 0; blk < n_el / 16; ++blk)
        oracle_fp4_quant16(v + blk * 16, codes + blk * 8, scales + blk);
}

/* Interval refresh of one request in split precision.
 *   upd_dtype: ORC_F32 / ORC_BF16 / ORC_E4M3 -- the update copy upd [H][P][N];
 *              ORC_FP4 -- the shared-copy control: codes/scales are both the
 *              update copy and the output copy.
 *   out_fp4:   write the FP4 output copy (codes [H][P][N/2], scales
 *              [H][P][N/16]) from the fp32 result.
 * Steps: widen the update copy; fold the *pos buffered entries in fp64;
 * round the result to fp32 (nearest even); write the update copy (fp32 as
 * is, bf16/e4m3 by stochastic rounding with counter flush_count, FP4 by
 * nearest rounding); write the FP4 output copy; pos <- 0; flush_count += 1.
 * v32_out (optional, [H][P][N]) receives the fp32 result. */
void oracle_lowprec_refresh(int H, int P, int N, int G, int upd_dtype, int out_fp4,
                            uint64_t seed, uint32_t request, uint32_t *flush_count,
                            void *upd, uint8_t *codes, uint8_t *scales,
                            const double *xb, const double *Bb, const double *dtb,
                            int *pos, const double *A, float *v32_out)
{
    size_t n_head = (size_t)P * N, n_all = (size_t)H * n_head;
    double *st = (double *)malloc(sizeof(double) * n_all);
    float *v32 = (float *)malloc(sizeof(float) * n_all);
    if (upd_dtype == ORC_FP4) oracle_widen(ORC_FP4, n_all, codes, scales, st);
    else oracle_widen(upd_dtype, n_all, upd, NULL, st);
    fold_fp64(H, P, N, G, st, xb, Bb, dtb, *pos, A);
    for (size_t i = 0; i < n_all; ++i) v32[i] = (float)st[i];
    if (upd_dtype == ORC_F32) {
        memcpy(upd, v32, sizeof(float) * n_all);
    } else if (upd_dtype == ORC_BF16 || upd_dtype == ORC_E4M3) {
        size_t el = (upd_dtype == ORC_BF16) ? 2 : 1;
        for (int hh = 0; hh < H; ++hh)
            oracle_sr_head(upd_dtype, seed, request, (uint32_t)hh, *flush_count, n_head,
                           v32 + (size_t)hh * n_head, (uint8_t *)upd + (size_t)hh * n_head * el);
    } else {
        oracle_fp4_quant(n_all, v32, codes, scales);
    }
    if (out_fp4 && upd_dtype != ORC_FP4) oracle_fp4_quant(n_all, v32, codes, scales);
    if (v32_out) memcpy(v32_out, v32, sizeof(float) * n_all);
    free(st);
    free(v32);
    *pos = 0;
    *flush_count += 1;
}
