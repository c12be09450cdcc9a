// rssm_kernels.cu -- sm_100a kernels of librssm.
//
// The hot path at d_state 128 (head_dim a multiple of 8) runs two
// persistent, warp-specialised kernels, one CTA per SM:
//   k_replay_pipe  decode, verify, fused decode + flush: a producer warp
//                  fills a ring of shared-memory stages with bulk copies of
//                  each (request, head) record and its B rows; consumer warp
//                  groups compute the outputs from shared memory;
//   k_fold_pipe    interval flush and precision-split refresh: the same
//                  producer/consumer ring over the requests that are due.
// Other shapes run one CTA of 256 threads per (request, head) tile
// (k_replay, k_fold), the tile brought in by one bulk copy issued first.
// k_prefill folds a prompt into the checkpoint; k_conv is the conventional
// per-token scheme kept for comparison. Rows are reduced across the lanes
// that hold their columns with shuffles; there are no float atomics, every
// result has a fixed summation order, and runs are bit-reproducible.
//
// Method: ReplaySSM article (devotd.net
// "nvidia-replayssm-hybrid-model-ssm-decoding-state-buffer"):
//   s1 "Store recent inputs instead of the full state"          -> k_replay_pipe, k_fold_pipe (k_replay, k_fold)
//   s3 "Roll back incorrect predictions using buffer positions" -> verify in k_replay_pipe, k_accept
//   s4 "Prevent low-precision errors from accumulating again"   -> refresh in k_fold_pipe, FP4 reads
//   conventional scheme of s1/s3 (in-run comparison)            -> k_conv
#include "rssm_device.cuh"
#include "rssm_internal.h"
#include "rssm_mma.cuh"
#include "rssm.h"

#include <atomic>
#include <type_traits>

namespace rssm {

__host__ __device__ inline uint32_t tile_bytes(int fmt, int P, int N) {
    const uint32_t n = static_cast<uint32_t>(P) * static_cast<uint32_t>(N);
    return fmt == kF32 ? 4u * n : fmt == kBF16 ? 2u * n : fmt == kE4M3 ? n : n / 2u;
}
__host__ __device__ inline uint32_t scale_bytes(int fmt, int P, int N) {
    return fmt == kFP4 ? static_cast<uint32_t>(P) * static_cast<uint32_t>(N) / 16u : 0u;
}
__host__ __device__ inline uint32_t align16(uint32_t x) { return (x + 15u) & ~15u; }

// Four consecutive state values (row r, column group c of 4) of a tile in
// shared memory, in format F.
template <int F>
__device__ __forceinline__ float4 tile_load4(const unsigned char* t, const unsigned char* sc, int r, int c,
                                             int N) {
    const int q = r * (N >> 2) + c;
    if constexpr (F == kF32) {
        return reinterpret_cast<const float4*>(t)[q];
    } else if constexpr (F == kBF16) {
        return bf16x4_val(reinterpret_cast<const uint2*>(t)[q]);
    } else if constexpr (F == kE4M3) {
        return e4m3x4_val(reinterpret_cast<const uint32_t*>(t)[q]);
    } else {
        return fp4x4_val(reinterpret_cast<const uint16_t*>(t)[q], e4m3_val(sc[q >> 2]));
    }
}

__device__ __forceinline__ void stream_store4(float* p, float4 v) { __stcs(reinterpret_cast<float4*>(p), v); }

// Last CTA of request b to finish moves the request's position. Thread 0
// calls it after the CTA's last use of pos[b]; no CTA ever waits for another.
__device__ __forceinline__ void request_done(uint32_t* arrive, int b, int nblk, int32_t* pos, int new_pos,
                                             uint32_t* flush_count, bool bump) {
    __threadfence();
    const uint32_t old = atomicAdd(&arrive[b], 1u);
    if (old == static_cast<uint32_t>(nblk - 1)) {
        arrive[b] = 0u;
        pos[b] = new_pos;
        if (bump) flush_count[b] += 1u;
    }
}

// Inclusive prefix sum over the lanes of one warp.
__device__ __forceinline__ float warp_prefix(float v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float t = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += t;
    }
    return v;
}

__host__ __device__ inline int round_up8(int x) { return (x + 7) & ~7; }

constexpr int kRB = 8;  // fold: rows per thread (register block)

// The fold of s1 as a register-blocked rank-T update:
//   v[r][c] = alpha * tile[r][c] + sum_{s<T} xw[s][r] * B_s[c],
// xw[s][r] = dt_s exp(A (S_T - S_s)) x_s[r] in shared memory with row stride
// xs = round_up8(P). A thread owns kRB consecutive rows and one group of 4
// columns, keeps their accumulators in registers and streams over s: per s
// one float4 of B (brow(s, c)) and two float4 of xw. emit(r, c, v, valid)
// is called by every lane for every owned row (valid = row in range).
template <typename BRow, typename Emit>
__device__ __forceinline__ void fold_tile(const float* s32, const float* s_xw, int xs, int P, int N, int lpr,
                                          int T, float alpha, BRow brow, Emit emit) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int lsh = __ffs(lpr) - 1;
    const int rpw = 32 >> lsh, col4 = lane & (lpr - 1), rsub = lane >> lsh;
    const int rows_per_pass = kWarps * rpw * kRB;
    for (int base = 0; base < P; base += rows_per_pass) {
        const int rb = base + (warp * rpw + rsub) * kRB;
        float2 acc2[4][4];  // rows paired for the packed FMAs
#pragma unroll
        for (int k = 0; k < kRB; ++k) {
            const int r = rb + k;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < P) {
                v = reinterpret_cast<const float4*>(s32)[r * (N >> 2) + col4];
                v.x *= alpha;
                v.y *= alpha;
                v.z *= alpha;
                v.w *= alpha;
            }
            acc2_set_row(acc2, k, v);
        }
        if (rb < P) {
#pragma unroll 2
            for (int s = 0; s < T; ++s) {
                const float4 bv = brow(s, col4);
                const float4* xw4 = reinterpret_cast<const float4*>(s_xw + s * xs + rb);
                const float4 xa = xw4[0], xb = xw4[1];
                const float2 w2[4] = {make_float2(xa.x, xa.y), make_float2(xa.z, xa.w), make_float2(xb.x, xb.y),
                                      make_float2(xb.z, xb.w)};
                rank1_8x4(acc2, w2, bv);
            }
        }
#pragma unroll
        for (int k = 0; k < kRB; ++k) emit(rb + k, col4, acc2_row(acc2, k), rb + k < P);
    }
}

// Eight consecutive input elements as raw bits (one or two 16-byte accesses).
template <typename TIn> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    uint4 u;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = *reinterpret_cast<const uint4*>(p); }
    __device__ __forceinline__ void store(__nv_bfloat16* p) const { *reinterpret_cast<uint4*>(p) = u; }
    __device__ __forceinline__ float4 lo() const { return bf16x4_val(make_uint2(u.x, u.y)); }
    __device__ __forceinline__ float4 hi() const { return bf16x4_val(make_uint2(u.z, u.w)); }
};
template <> struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p) {
        a = reinterpret_cast<const float4*>(p)[0];
        b = reinterpret_cast<const float4*>(p)[1];
    }
    __device__ __forceinline__ void store(float* p) const {
        reinterpret_cast<float4*>(p)[0] = a;
        reinterpret_cast<float4*>(p)[1] = b;
    }
    __device__ __forceinline__ float4 lo() const { return a; }
    __device__ __forceinline__ float4 hi() const { return b; }
};

// Sums 8 per-lane partials (rows 0..7 of a warp's block) over the 32 lanes
// with a transpose butterfly (9 shuffles instead of 40): lanes exchange the
// half of their rows that the partner keeps. Lane l returns the total of
// row (l >> 2) & 7. Fixed order, so the result is reproducible.
__device__ __forceinline__ float warp_reduce8(const float (&v)[8]) {
    const int lane = threadIdx.x & 31;
    const bool b16 = lane & 16, b8 = lane & 8, b4 = lane & 4;
    float w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = b16 ? v[i] : v[i + 4];
        const float keep = b16 ? v[i + 4] : v[i];
        w[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    float u[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b8 ? w[i] : w[i + 2];
        const float keep = b8 ? w[i + 2] : w[i];
        u[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    const float send = b4 ? u[0] : u[1];
    float z = (b4 ? u[1] : u[0]) + __shfl_xor_sync(0xffffffffu, send, 4);
    z += __shfl_xor_sync(0xffffffffu, z, 2);
    z += __shfl_xor_sync(0xffffffffu, z, 1);
    return z;
}

// Four floats back to the input element type (exact for values that came from it).
__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
    const uint2 u = make_uint2((__float_as_uint(v.x) >> 16) | (__float_as_uint(v.y) & 0xFFFF0000u),
                               (__float_as_uint(v.z) >> 16) | (__float_as_uint(v.w) & 0xFFFF0000u));
    *reinterpret_cast<uint2*>(p) = u;
}

// ---------------------------------------------------------------------------
// Replay decode / verify (s1, s3).
//   y_j = exp(A S_t) (h_ckpt C_j) + sum_{s<=t} dt_s exp(A (S_t - S_s)) (B_s . C_j) x_s + D x_t,
//   t = pos + j, for the ntok tokens of this call; S = prefix sum of the
//   buffered dt. The new tokens are appended at slots pos..pos+ntok-1.
//   While the tile streams in, the CTA stages x_s of every slot in shared
//   memory, forms the decay weights (warp 0) and the B_s . C_j products
//   (all warps), in two batches of independent loads (this call's inputs
//   with pos, then the buffered slots). After the tile lands, each row's
//   output is one reduction over the row's lanes of the h.C dot product and
//   the replay terms (lane l takes slots s = l mod lanes).
//   RF: format of the copy read (fp32 checkpoint, bf16/e4m3 update copy, or
//   FP4 copy). NT: compile-time bound on ntok. FUSED: the token that fills
//   the buffer also folds it into the fp32 checkpoint. WIDE: d_state 128 and
//   head_dim a multiple of 8 -- 16-byte staging, a warp owns 8 consecutive
//   rows, lane l is slot l, and the 8 rows reduce together (warp_reduce8).
// ---------------------------------------------------------------------------
// Minimum resident CTAs per SM the register allocation must allow.
__host__ __device__ constexpr int replay_min_blocks(int nt, int fused) {
    return fused ? 4 : (nt == 1 ? 6 : (nt <= kMidTok ? 4 : 3));
}

template <typename TIn, int RF, int NT, int FUSED, int WIDE>
__global__ void __launch_bounds__(kThreads, replay_min_blocks(NT, FUSED)) k_replay(const ReplayArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bar;
    __shared__ float s_w[NT][kMaxCap];  // dt_s exp(A (S_t - S_s)) for token j; 0 for s > t
    __shared__ float s_g[NT][kMaxCap];  // B_s . C_j
    __shared__ float s_decay[NT];       // exp(A S_t)
    __shared__ int s_pos;

    const int H = a.s.H, P = a.s.P, N = a.s.N, G = a.s.G, cap = a.s.cap;
    const int lpr = WIDE ? 32 : a.s.lpr;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x / H, h = blockIdx.x - b * H;
    const int hpg = H / G, g = h / hpg;
    const int ntok = a.ntok;
    const int lsh = __ffs(lpr) - 1;
    const int rpw = 32 >> lsh, col4 = lane & (lpr - 1), rsub = lane >> lsh;
    const int xs = round_up8(P);
    const size_t bh = static_cast<size_t>(b) * H + h;
    const size_t bg = static_cast<size_t>(b) * G + g;

    // per-CTA bases: token j adds j*HP (x, y), j*GN (B, C), j*H (dt); slot s adds s*P, s*N
    const size_t HP = static_cast<size_t>(H) * P, GN = static_cast<size_t>(G) * N;
    const TIn* xin = static_cast<const TIn*>(a.x) + static_cast<size_t>(b) * ntok * HP + static_cast<size_t>(h) * P;
    const TIn* Bin = static_cast<const TIn*>(a.B) + static_cast<size_t>(b) * ntok * GN + static_cast<size_t>(g) * N;
    const TIn* Cin = static_cast<const TIn*>(a.C) + static_cast<size_t>(b) * ntok * GN + static_cast<size_t>(g) * N;
    const float* dtin = a.dt + static_cast<size_t>(b) * ntok * H + h;
    float* yout = a.y + static_cast<size_t>(b) * ntok * HP + static_cast<size_t>(h) * P;
    unsigned char* rec = a.record + bh * a.rec.bytes;
    TIn* xb = reinterpret_cast<TIn*>(rec + a.rec.x);
    TIn* bb = static_cast<TIn*>(a.bbuf) + bg * cap * N;
    float* dtb = reinterpret_cast<float*>(rec + a.rec.dt);

    const uint32_t tb = tile_bytes(RF, P, N), sb = scale_bytes(RF, P, N);
    unsigned char* s_tile = smem;
    unsigned char* s_sc = smem + align16(tb);
    float* s_x = reinterpret_cast<float*>(smem + align16(tb) + align16(sb));  // [cap][xs]
    float* s_B = s_x + cap * xs;                                              // fused: [L][N]
    const uint32_t bar_a = smem_u32(&bar);

    if (tid == 0) {
        mbar_init(bar_a, 1);
        // the copy's values and (FP4) scales, contiguous in the record as here
        mbar_expect_tx(bar_a, tb + sb);
        bulk_g2s(smem_u32(s_tile), rec, tb + sb, bar_a);
        s_pos = a.pos[b];  // the only read of pos: every thread uses this copy
    }

    // ---- first loads: C rows, this call's x and dt (with the position, above)
    float4 c4[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j)
        c4[j] = (j < ntok) ? load4(Cin + j * GN + 4 * col4) : make_float4(0.f, 0.f, 0.f, 0.f);
    const int nq_new = WIDE ? (ntok * P) >> 3 : 0;  // 8-element chunks of this call's x
    __syncthreads();  // barrier initialised and pos read before anyone uses them

    const int pos = s_pos;
    const int T = pos + ntok;
    const bool ok = pos >= 0 && T <= cap;
    const bool fold_now = FUSED && RF == kF32 && NT == 1 && ok && T == a.s.L;
    if (!ok && tid == 0) set_error(a.err, (pos < 0 || pos > cap) ? RSSM_DEVERR_POS_RANGE : RSSM_DEVERR_CAPACITY);
    // past the barrier no thread of this CTA reads pos again; once every CTA
    // of the request has arrived, the last one moves it
    if (a.advance && ok && tid == kThreads - 32)
        request_done(a.arrive, b, H, a.pos, fold_now ? 0 : pos + 1, a.flush_count, fold_now);

    if (ok) {
        const float Ah = a.A[h];
        // ---- second loads (independent): the buffered slots s < pos and this
        // call's tokens -> shared memory; this call's tokens -> the buffer
        if constexpr (WIDE) {
            Raw8<TIn> xr;
            if (tid < nq_new) {
                const int e = tid << 3, j = e / P, p = e - j * P;
                xr.load(xin + j * HP + p);
            }
            for (int q = tid; q < ((pos * P) >> 3); q += kThreads) {
                const int e = q << 3, sl = e / P, p = e - sl * P;
                Raw8<TIn> r;
                r.load(xb + e);
                float4* d = reinterpret_cast<float4*>(s_x + sl * xs + p);
                d[0] = r.lo();
                d[1] = r.hi();
            }
            if (tid < nq_new) {
                const int e = tid << 3, j = e / P, p = e - j * P;
                float4* d = reinterpret_cast<float4*>(s_x + (pos + j) * xs + p);
                d[0] = xr.lo();
                d[1] = xr.hi();
                xr.store(xb + (pos + j) * P + p);
            }
            for (int q = tid + kThreads; q < nq_new; q += kThreads) {  // many tokens
                const int e = q << 3, j = e / P, p = e - j * P;
                Raw8<TIn> r;
                r.load(xin + j * HP + p);
                float4* d = reinterpret_cast<float4*>(s_x + (pos + j) * xs + p);
                d[0] = r.lo();
                d[1] = r.hi();
                r.store(xb + (pos + j) * P + p);
            }
        } else {
            constexpr int kNew = 2;
            TIn xn[kNew];
#pragma unroll
            for (int k = 0; k < kNew; ++k) {
                const int i = tid + k * kThreads;
                xn[k] = (i < ntok * P) ? xin[(i / P) * HP + (i % P)] : TIn(0.f);
            }
            constexpr int kOld = 4;
            for (int base = 0; base < pos * P; base += kOld * kThreads) {
                float xo[kOld];
#pragma unroll
                for (int k = 0; k < kOld; ++k) {
                    const int i = base + tid + k * kThreads;
                    xo[k] = (i < pos * P) ? to_f32(xb[i]) : 0.f;
                }
#pragma unroll
                for (int k = 0; k < kOld; ++k) {
                    const int i = base + tid + k * kThreads;
                    if (i < pos * P) s_x[(i / P) * xs + (i % P)] = xo[k];
                }
            }
#pragma unroll
            for (int k = 0; k < kNew; ++k) {
                const int i = tid + k * kThreads;
                if (i < ntok * P) {
                    const int j = i / P, p = i - j * P;
                    s_x[(pos + j) * xs + p] = to_f32(xn[k]);
                    xb[(pos + j) * P + p] = xn[k];
                }
            }
            for (int i = tid + kNew * kThreads; i < ntok * P; i += kThreads) {  // large head_dim or many tokens
                const int j = i / P, p = i - j * P;
                const TIn v = xin[j * HP + p];
                s_x[(pos + j) * xs + p] = to_f32(v);
                xb[(pos + j) * P + p] = v;
            }
        }
        if (warp == 0) {
            const float dnew = (lane >= pos && lane < T) ? dtin[(lane - pos) * H] : 0.f;
            const float dts = (lane < pos) ? dtb[lane] : dnew;
            if (lane >= pos && lane < T) dtb[lane] = dnew;
            const float Sx = warp_prefix(dts);
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                if (j < ntok) {
                    const float St = __shfl_sync(0xffffffffu, Sx, pos + j);
                    s_w[j][lane] = (lane <= pos + j) ? dts * expf(Ah * (St - Sx)) : 0.f;
                    if (lane == 0) s_decay[j] = expf(Ah * St);
                }
            }
        }
        // g[j][s] = B_s . C_j; the group's first head appends this call's B rows
        const bool leader = (h == g * hpg);
        for (int s0 = warp * rpw; s0 < T; s0 += 2 * kWarps * rpw) {
            const int sa = s0 + rsub, sb2 = s0 + kWarps * rpw + rsub;
            auto bload = [&](int sl) {
                if (sl >= T) return make_float4(0.f, 0.f, 0.f, 0.f);
                return (sl < pos) ? load4(bb + sl * N + 4 * col4) : load4(Bin + (sl - pos) * GN + 4 * col4);
            };
            const float4 bva = bload(sa), bvb = bload(sb2);
            if (leader) {
                if (sa >= pos && sa < T) store4(bb + sa * N + 4 * col4, bva);
                if (sb2 >= pos && sb2 < T) store4(bb + sb2 * N + 4 * col4, bvb);
            }
            if (fold_now) {
                if (sa < T) reinterpret_cast<float4*>(s_B)[sa * (N >> 2) + col4] = bva;
                if (sb2 < T) reinterpret_cast<float4*>(s_B)[sb2 * (N >> 2) + col4] = bvb;
            }
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                if (j < ntok) {
                    const float da = group_sum(dot4(bva, c4[j]), lpr);
                    const float db = group_sum(dot4(bvb, c4[j]), lpr);
                    if (col4 == 0) {
                        if (sa < T) s_g[j][sa] = da;
                        if (sb2 < T) s_g[j][sb2] = db;
                    }
                }
            }
        }
    }

    // one thread waits for the tile; the barrier publishes it (and the
    // staged rows, weights and dot products) to the whole CTA
    bool arrived = true;
    if (tid == 0) arrived = mbar_wait_bounded(bar_a, 0, kWaitNs);
    if (__syncthreads_or(!arrived)) {
        if (tid == 0) {
            set_error(a.err, RSSM_DEVERR_TIMEOUT);
            mbar_wait_bounded(bar_a, 0, kWaitNs);
        }
        return;
    }
    if (!ok) return;

    const float Dh = a.D[h];
    if constexpr (WIDE) {
        // warp w owns rows r0..r0+7; lane l adds slot l's replay term to every row
        for (int r0 = warp * 8; r0 < P; r0 += kWarps * 8) {
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                if (j < ntok) {
                    const int t = pos + j;
                    const float dec = s_decay[j];
                    float part[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const float4 hv = (r0 + k < P) ? tile_load4<RF>(s_tile, s_sc, r0 + k, lane, N)
                                                       : make_float4(0.f, 0.f, 0.f, 0.f);
                        part[k] = dec * dot4(hv, c4[j]);
                    }
                    if (lane <= t) {
                        const float coef = s_w[j][lane] * s_g[j][lane];
                        const float4* xv = reinterpret_cast<const float4*>(s_x + lane * xs + r0);
                        const float4 xa = xv[0], xc = xv[1];
                        part[0] = fmaf(coef, xa.x, part[0]);
                        part[1] = fmaf(coef, xa.y, part[1]);
                        part[2] = fmaf(coef, xa.z, part[2]);
                        part[3] = fmaf(coef, xa.w, part[3]);
                        part[4] = fmaf(coef, xc.x, part[4]);
                        part[5] = fmaf(coef, xc.y, part[5]);
                        part[6] = fmaf(coef, xc.z, part[6]);
                        part[7] = fmaf(coef, xc.w, part[7]);
                    }
                    const float z = warp_reduce8(part);
                    const int r = r0 + ((lane >> 2) & 7);
                    if ((lane & 3) == 0 && r < P) yout[j * HP + r] = fmaf(Dh, s_x[t * xs + r], z);
                }
            }
        }
    } else {
        for (int r0 = warp * rpw; r0 < P; r0 += kWarps * rpw) {
            const int r = r0 + rsub;
            const bool valid = r < P;
            const float4 hv = valid ? tile_load4<RF>(s_tile, s_sc, r, col4, N) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                if (j < ntok) {
                    const int t = pos + j;
                    float part = s_decay[j] * dot4(hv, c4[j]);
                    if (valid)
                        for (int sl = col4; sl <= t; sl += lpr)
                            part = fmaf(s_w[j][sl] * s_g[j][sl], s_x[sl * xs + r], part);
                    const float sum = group_sum(part, lpr);
                    if (valid && col4 == 0) yout[j * HP + r] = fmaf(Dh, s_x[t * xs + r], sum);
                }
            }
        }
    }

    if constexpr (RF == kF32 && NT == 1 && FUSED) {
        if (fold_now) {
            // fused flush: the token that fills the buffer folds it into the
            // checkpoint from the tile, x rows and B rows already in shared memory.
            float* dst = reinterpret_cast<float*>(rec);
            auto brow = [&](int sl, int c) {
                const float w = s_w[0][sl];
                const float4 v = reinterpret_cast<const float4*>(s_B + sl * N)[c];
                return make_float4(w * v.x, w * v.y, w * v.z, w * v.w);
            };
            auto emit = [&](int r, int c, float4 v, bool valid) {
                if (valid) stream_store4(dst + r * N + 4 * c, v);
            };
            fold_tile(reinterpret_cast<const float*>(s_tile), s_x, xs, P, N, lpr, T, s_decay[0], brow, emit);
        }
    }
}

// ---------------------------------------------------------------------------
// Persistent, warp-specialised replay decode / verify for d_state 128 and
// head_dim a multiple of 8. One CTA per SM walks the tiles
// t = blockIdx.x + k * gridDim.x ((request, head) = (t / H, t % H)).
// A producer warp (one lane per tile, a batch of tiles per pass) reads each
// tile's position a batch ahead and brings the tile's state into a ring of
// shared-memory stages with two bulk copies (the
// record prefix -- copy, dt row and buffered x rows -- and the buffered B
// rows; completion on the stage's "full" mbarrier). Consumer warps compute
// the outputs from shared memory only and release the stage (its "empty"
// mbarrier). This call's x, B and C rows come from the consumers
// themselves, one tile ahead (cp.async into a per-group double buffer).
// The HBM stream never waits for a tile's arithmetic, and a tile's
// arithmetic never waits for HBM latency. Every wait is bounded by
// %globaltimer; a timeout sets the error word.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t fdiv(uint32_t x, const FastDiv& f) { return (__umulhi(x, f.mul) + x) >> f.shr; }

// Programmatic dependent launch (the persistent kernels are launched with
// programmatic stream serialization): let the next kernel on the stream start
// launching now -- its CTAs take an SM once this kernel's CTA there exits --
// and wait until the previous kernel's writes are visible before reading any
// global memory. Both are no-ops for a plain launch.
__device__ __forceinline__ void pdl_prologue() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Barrier of one consumer group of nthr threads (named barrier 1 + gi),
// returning the OR of v.
__device__ __forceinline__ int group_sync_or(int gi, int nthr, int v) {
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.s32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.s32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(v), "r"(1 + gi), "r"(nthr)
        : "memory");
    return r;
}

__device__ __forceinline__ void group_sync(int gi, int nthr) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + gi), "r"(nthr) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Consumer groups of the pipelined kernel and warps per group. Groups work
// on different tiles at once, which hides the latency chain of one tile
// (barriers, shared-memory loads, shuffle reductions). The fp32 copy fills a
// 39 KB stage per tile at the shapes served, so few tiles fit in shared
// memory: three groups of four warps. Verify (K+1 tokens per tile) takes
// three groups of four warps for every copy (two groups for more than kMidTok
// tokens, whose registers would spill). Decode of the smaller copies has room
// for many tiles: bf16 seven groups of two warps; e4m3 and FP4 fifteen groups
// of one warp, each tile worked by one warp without group barriers. Fifteen
// consumer warps + the producer are 16 warps, the block size at which the
// register budget stays 128 per thread (13 warps get the same), and group
// 14 uses the last named barrier (15). (B200, FP4 decode: 93 us with 12 x 1,
// 102 us with 6 x 2, 114 us with 8 x 1 in the first form of the kernel;
// 43.1 -> 40.2 us from 12 x 1 to 15 x 1 in the current one; FP4 verify
// 1163 us with 12 x 1, 934 us with 3 x 4.)
__host__ __device__ constexpr int pipe_groups(int nt, int rf) {
    return nt > 1 ? (nt <= kMidTok ? 3 : 2) : (rf == kF32 ? 3 : (rf == kBF16 ? 7 : 15));
}
__host__ __device__ constexpr int pipe_cwarps(int nt, int rf) {
    return nt > 1 ? 4 : (rf == kF32 ? 4 : (rf == kBF16 ? 2 : 1));
}
// The FP4-reading decode's producer also brings this call's x, B and C rows
// with the stage (its consumers are single warps, for which fetching them is
// a long step of each tile); the other forms fetch them in the consumers.
__host__ __device__ constexpr bool pipe_rows_in_stage(int nt, int rf, int fused) {
    return nt == 1 && rf == kFP4 && !fused;
}
__host__ __device__ constexpr int pipe_threads(int nt, int rf) {
    return (pipe_groups(nt, rf) * pipe_cwarps(nt, rf) + 1) * 32;
}
// Static shared memory of k_replay_pipe<*, rf, nt, *>: per-group weights,
// B.C products and decays, the stage barriers, the abort flag (plus slack for
// what the compiler adds); the dynamic stages get the rest.
__host__ __device__ constexpr size_t pipe_static_smem(int nt, int rf) {
    return static_cast<size_t>(pipe_groups(nt, rf)) * nt * (2 * kMaxCap + 1) * 4 + 2 * kPipeStagesMax * 8 + 1024 +
           (nt == 1 && rf == kFP4 ? static_cast<size_t>(pipe_groups(nt, rf)) * kMaxHeadDim * 4 : 0);
}

// ---------------------------------------------------------------------------
// Tensor-core dot products of k_replay_pipe (bf16 inputs, d_state 128; the
// operand layouts and precision are described in rssm_mma.cuh). Lane
// 4 g + t owns the 32 columns 32t..32t+31 of a row, in four 8-column chunks.
// ---------------------------------------------------------------------------
constexpr int kD128 = 128;

// The four 8-column chunks (bf16) of a 128-column row that lane t owns;
// chunk c read from position (c + t) & 3 when rot (spreads the banks of rows
// 256 B apart), else c. Zeros for a null row.
__device__ __forceinline__ void load_bf16_chunks(uint4 (&dst)[4], const __nv_bfloat16* row, int t, bool rot) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int pc = rot ? ((c + t) & 3) : c;
        dst[c] = row ? *reinterpret_cast<const uint4*>(row + 32 * t + 8 * pc) : make_uint4(0u, 0u, 0u, 0u);
    }
}

// g[j][s] = B_s . C_j for the slots s0..s0+15 below T and the tokens j < ntok,
// by one warp: product rows = slots, k = d_state, columns = tokens. Slot s
// is the stage's row br + s N (s < pos) or this call's row nb + (s - pos) N.
// s_g: [tokens][kMaxCap].
__device__ __forceinline__ void bc_products_mma(const __nv_bfloat16* br, const __nv_bfloat16* nb,
                                                const __nv_bfloat16* nc, int pos, int T, int ntok, int s0,
                                                float* s_g) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    auto row_of = [&](int sl) -> const __nv_bfloat16* {
        return sl < pos ? br + sl * kD128 : (sl < T ? nb + (sl - pos) * kD128 : nullptr);
    };
    uint4 cb[4], r0[4], r1[4];
    load_bf16_chunks(cb, g < ntok ? nc + g * kD128 : nullptr, t, true);
    load_bf16_chunks(r0, row_of(s0 + g), t, true);
    load_bf16_chunks(r1, row_of(s0 + g + 8), t, true);
    float d[4] = {0.f, 0.f, 0.f, 0.f}, e[4] = {0.f, 0.f, 0.f, 0.f};  // two independent chains
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        mma_bf16(d, r0[c].x, r1[c].x, r0[c].y, r1[c].y, cb[c].x, cb[c].y);
        mma_bf16(e, r0[c].z, r1[c].z, r0[c].w, r1[c].w, cb[c].z, cb[c].w);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) d[i] += e[i];
    const int sa = s0 + g, sb = s0 + g + 8, j0 = 2 * t, j1 = 2 * t + 1;
    if (sa < T) {
        if (j0 < ntok) s_g[j0 * kMaxCap + sa] = d[0];
        if (j1 < ntok) s_g[j1 * kMaxCap + sa] = d[1];
    }
    if (sb < T) {
        if (j0 < ntok) s_g[j0 * kMaxCap + sb] = d[2];
        if (j1 < ntok) s_g[j1 * kMaxCap + sb] = d[3];
    }
}

// Whether a copy format reads its rows in rotated chunk order (rows 256 B or
// 512 B apart) or in order (128 B / 64 B rows spread the banks already).
__host__ __device__ constexpr bool hc_rotated(int rf) { return rf == kF32 || rf == kBF16; }

// B operand of h . C_j for lane (g, t): token j = g, from the lane's chunks of
// C_g (bf16, cb); bfrag[4 c + u] stands for columns 2u, 2u + 1 of chunk c.
// F32 and BF16: the bf16 words as they are (the tf32 steps take each half as
// an fp32 value); E4M3 / FP4: f16 pairs. For the k16 steps, bfrag[2 m],
// bfrag[2 m + 1] are b0, b1 of step m.
template <int RF>
__device__ __forceinline__ void hc_bfrag(const uint4 (&cb)[4], uint32_t (&bfrag)[16]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint32_t w[4] = {cb[c].x, cb[c].y, cb[c].z, cb[c].w};
#pragma unroll
        for (int u = 0; u < 4; ++u) bfrag[4 * c + u] = (RF == kF32 || RF == kBF16) ? w[u] : bf16x2_to_f16x2(w[u]);
    }
}

// d += h . C for the rows R0 + g (d0, d1) and R0 + g + 8 (d2, d3) of a stage
// tile (format RF, d_state 128), columns j = 2t, 2t+1 of the product: the
// tokens (bfrag from hc_bfrag) or, for the FP4 decode, the scale blocks
// (bfrag zero except in column g = block). SCALE_A: multiply FP4 codes by
// their block scale before the product (verify); else the product is of the
// bare codes (the decode applies the scales per block afterwards). Rows at or
// past P read as zero.
template <int RF, bool SCALE_A>
__device__ __forceinline__ void hc_mma(const unsigned char* tile, const unsigned char* sc, int R0, int P,
                                       const uint32_t (&bfrag)[16], float (&d_out)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    // two independent accumulation chains (even / odd steps), added at the end
    float d[4] = {0.f, 0.f, 0.f, 0.f}, e[4] = {0.f, 0.f, 0.f, 0.f};
    const int ra = R0 + g, rb = R0 + g + 8;
    const bool va = ra < P, vb = rb < P;
    if constexpr (RF == kF32) {
        const float* pa = reinterpret_cast<const float*>(tile) + ra * kD128 + 32 * t;
        const float* pb = reinterpret_cast<const float*>(tile) + rb * kD128 + 32 * t;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int pc = 8 * ((c + t) & 3);
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 a0 = va ? *reinterpret_cast<const float4*>(pa + pc) : z;
            const float4 a1 = va ? *reinterpret_cast<const float4*>(pa + pc + 4) : z;
            const float4 b0 = vb ? *reinterpret_cast<const float4*>(pb + pc) : z;
            const float4 b1 = vb ? *reinterpret_cast<const float4*>(pb + pc + 4) : z;
            const float ra8[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float rb8[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                uint32_t h0, l0, h1, l1, h2, l2, h3, l3;
                tf32_split(ra8[2 * u], h0, l0);      // row g, k lo
                tf32_split(rb8[2 * u], h1, l1);      // row g + 8, k lo
                tf32_split(ra8[2 * u + 1], h2, l2);  // row g, k hi
                tf32_split(rb8[2 * u + 1], h3, l3);  // row g + 8, k hi
                // step 4c + u: k lo = column 2u of the chunk, k hi = column 2u + 1
                const uint32_t q0 = bf16lo_bits(bfrag[4 * c + u]), q1 = bf16hi_bits(bfrag[4 * c + u]);
                mma_tf32(d, h0, h1, h2, h3, q0, q1);
                mma_tf32(e, l0, l1, l2, l3, q0, q1);
            }
        }
    } else if constexpr (RF == kBF16) {
        uint4 u0[4], u1[4];
        const __nv_bfloat16* rows = reinterpret_cast<const __nv_bfloat16*>(tile);
        load_bf16_chunks(u0, va ? rows + ra * kD128 : nullptr, t, true);
        load_bf16_chunks(u1, vb ? rows + rb * kD128 : nullptr, t, true);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            mma_bf16(d, u0[c].x, u1[c].x, u0[c].y, u1[c].y, bfrag[4 * c], bfrag[4 * c + 1]);
            mma_bf16(e, u0[c].z, u1[c].z, u0[c].w, u1[c].w, bfrag[4 * c + 2], bfrag[4 * c + 3]);
        }
    } else if constexpr (RF == kE4M3) {
        // 32 codes of a row per lane: two 16-byte words, chunk c = word half c & 1 of e[c >> 1]
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        const uint4 ea0 = va ? *reinterpret_cast<const uint4*>(tile + ra * kD128 + 32 * t) : z;
        const uint4 ea1 = va ? *reinterpret_cast<const uint4*>(tile + ra * kD128 + 32 * t + 16) : z;
        const uint4 eb0 = vb ? *reinterpret_cast<const uint4*>(tile + rb * kD128 + 32 * t) : z;
        const uint4 eb1 = vb ? *reinterpret_cast<const uint4*>(tile + rb * kD128 + 32 * t + 16) : z;
        const uint32_t wa[8] = {ea0.x, ea0.y, ea0.z, ea0.w, ea1.x, ea1.y, ea1.z, ea1.w};
        const uint32_t wb[8] = {eb0.x, eb0.y, eb0.z, eb0.w, eb1.x, eb1.y, eb1.z, eb1.w};
#pragma unroll
        for (int m = 0; m < 8; ++m) {  // step m: codes 4m..4m+3 of the lane's 32
            uint32_t a0, a2, a1, a3;
            e4m3x4_h2(wa[m], a0, a2);
            e4m3x4_h2(wb[m], a1, a3);
            if (m & 1)
                mma_f16(e, a0, a1, a2, a3, bfrag[2 * m], bfrag[2 * m + 1]);
            else
                mma_f16(d, a0, a1, a2, a3, bfrag[2 * m], bfrag[2 * m + 1]);
        }
    } else {
        // FP4: 32 codes of a row per lane in one 16-byte word; scales of the
        // lane's two blocks (2t, 2t + 1) in one 16-bit word
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        const uint4 qa = va ? *reinterpret_cast<const uint4*>(tile + ra * (kD128 / 2) + 16 * t) : z;
        const uint4 qb = vb ? *reinterpret_cast<const uint4*>(tile + rb * (kD128 / 2) + 16 * t) : z;
        const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w}, wb[4] = {qb.x, qb.y, qb.z, qb.w};
        uint32_t sa = 0u, sb = 0u;
        if constexpr (SCALE_A) {
            sa = va ? e4m3x2_h2(*reinterpret_cast<const uint16_t*>(sc + ra * (kD128 / 16) + 2 * t)) : 0u;
            sb = vb ? e4m3x2_h2(*reinterpret_cast<const uint16_t*>(sc + rb * (kD128 / 16) + 2 * t)) : 0u;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // chunk c: codes 8c..8c+7 (block 2t + c / 2)
            uint32_t ha[4], hb[4];
            e2m1x8_h2(wa[c], ha);
            e2m1x8_h2(wb[c], hb);
            if constexpr (SCALE_A) {
                const uint32_t s2a = (c < 2) ? h2_dup_lo(sa) : h2_dup_hi(sa);
                const uint32_t s2b = (c < 2) ? h2_dup_lo(sb) : h2_dup_hi(sb);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    ha[k] = hmul2_u32(ha[k], s2a);
                    hb[k] = hmul2_u32(hb[k], s2b);
                }
            }
            mma_f16(d, ha[0], hb[0], ha[1], hb[1], bfrag[4 * c], bfrag[4 * c + 1]);
            mma_f16(e, ha[2], hb[2], ha[3], hb[3], bfrag[4 * c + 2], bfrag[4 * c + 3]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) d_out[i] += d[i] + e[i];
}

// d += the bare code . C block sums of the FP4 decode for rows g (qa) and
// g + 8 (qb): the lane's 32 codes of each row in one 16-byte word; bfrag
// holds C only in the column of the block a step's k falls in.
__device__ __forceinline__ void fp4_codes_mma(const uint4& qa, const uint4& qb, const uint32_t (&bfrag)[16],
                                              float (&d_out)[4]) {
    float d[4] = {0.f, 0.f, 0.f, 0.f}, e[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w}, wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t ha[4], hb[4];
        e2m1x8_h2(wa[c], ha);
        e2m1x8_h2(wb[c], hb);
        mma_f16(d, ha[0], hb[0], ha[1], hb[1], bfrag[4 * c], bfrag[4 * c + 1]);
        mma_f16(e, ha[2], hb[2], ha[3], hb[3], bfrag[4 * c + 2], bfrag[4 * c + 3]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) d_out[i] += d[i] + e[i];
}

// Replay terms of the verify: d += sum_s coef[j][s] x_s[row] for the rows
// R0 + g, R0 + g + 8 and the tokens j = 2t, 2t+1, over the slots below T
// (tf32 k8 steps of 8 slots; x exact, coef split hi + lo in cfrag). xrow[2q]
// / xrow[2q + 1]: this lane's slot rows 8q + t / 8q + t + 4 (0 past T).
__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void replay_mma(const uint32_t (&xrow)[kMaxCap / 4], int T, int P, int R0,
                                           const uint32_t (&cfrag)[16], float (&d_out)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2;
    const int ra = min(R0 + g, P - 1), rb = min(R0 + g + 8, P - 1);  // rows past P: read and discarded
    float d[4] = {0.f, 0.f, 0.f, 0.f}, e[4] = {0.f, 0.f, 0.f, 0.f};
    // xrow[i]: shared-memory address of the slot's x row (bf16), 0 past T
    auto xb = [&](int i, int r) -> uint32_t { return xrow[i] ? lds_u16(xrow[i] + 2u * r) << 16 : 0u; };
#pragma unroll
    for (int q = 0; q < kMaxCap / 8; ++q) {
        if (8 * q < T) {
            const uint32_t a0 = xb(2 * q, ra), a1 = xb(2 * q, rb), a2 = xb(2 * q + 1, ra), a3 = xb(2 * q + 1, rb);
            mma_tf32(d, a0, a1, a2, a3, cfrag[4 * q], cfrag[4 * q + 1]);
            mma_tf32(e, a0, a1, a2, a3, cfrag[4 * q + 2], cfrag[4 * q + 3]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) d_out[i] += d[i] + e[i];
}

// Stage meta (int words): the position and the index k of the tile the
// stage holds (-1 before its first use).
constexpr int kMetaPos = 0, kMetaTile = 1;
constexpr int kProdBatch = 8;  // most tiles the producer warp issues per pass (one per lane)
constexpr int kProdDiv = 3;    // ... and at most a third of the stages

template <typename TIn, int RF, int NT, int FUSED>
__global__ void __launch_bounds__(pipe_threads(NT, RF), 1) k_replay_pipe(const ReplayArgs a, const PipeLayout lay) {
    constexpr int CG = pipe_groups(NT, RF), CW = pipe_cwarps(NT, RF), CT = CW * 32;
    static_assert(!FUSED || (RF == kF32 && NT == 1), "the fused fold is for fp32 decode");
    // bf16 inputs: verify (every copy format) and the FP4 decode form their
    // dot products on the tensor cores
    constexpr bool kMma = std::is_same<TIn, __nv_bfloat16>::value && (NT > 1 || RF == kFP4);
    constexpr bool kRowsInStage = pipe_rows_in_stage(NT, RF, FUSED);
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full_bar[kPipeStagesMax];
    __shared__ __align__(8) uint64_t empty_bar[kPipeStagesMax];
    __shared__ float s_w[CG][NT][kMaxCap];  // dt_s exp(A (S_t - S_s)) for token j; 0 for s > t
    __shared__ float s_g[CG][NT][kMaxCap];  // B_s . C_j
    __shared__ float s_decay[CG][NT];       // exp(A S_t)
    __shared__ float s_rep[kMma && NT == 1 ? CG : 1][kMma && NT == 1 ? kMaxHeadDim : 1];  // FP4 decode: replay terms
    __shared__ volatile int s_abort;

    const int H = a.s.H, P = a.s.P, N = a.s.N, G = a.s.G, cap = a.s.cap;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ntok = a.ntok, S = lay.stages;
    const int ntiles = a.s.batch * H;
    const size_t HP = static_cast<size_t>(H) * P, GN = static_cast<size_t>(G) * N;
    constexpr int es = static_cast<int>(sizeof(TIn));

    pdl_prologue();
    if (tid == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(smem_u32(&full_bar[st]), 1);
            mbar_init(smem_u32(&empty_bar[st]), CW);
            reinterpret_cast<int*>(smem + static_cast<size_t>(st) * lay.stage_bytes + lay.meta)[kMetaTile] = -1;
        }
        s_abort = 0;
    }
    __syncthreads();

    if (warp == CG * CW) {
        // ------------------------------------------------------------ producer
        // Only what the copies need, for nb tiles per pass: lane i takes tile
        // kb + i of the batch kb.. -- its position (loaded one batch ahead),
        // its stage, the record and B-row addresses -- so one pass of the
        // warp's instructions issues the copies of nb tiles. A batch waits
        // for its nb stages together, so nb is a third of the ring (the rest
        // stays in flight meanwhile); the lanes of a batch never share a
        // stage. Everything else is the consumers' work.
        const int nb = S / kProdDiv < 1 ? 1 : (S / kProdDiv > kProdBatch ? kProdBatch : S / kProdDiv);
        const bool lane_on = lane < nb;
        auto tile_of = [&](int k) { return blockIdx.x + static_cast<uint32_t>(k) * gridDim.x; };
        auto load_pos = [&](int k) {
            const uint32_t t = tile_of(k);
            return (lane_on && t < static_cast<uint32_t>(ntiles)) ? a.pos[fdiv(t, lay.divH)] : 0;
        };
        const size_t brow_bytes = static_cast<size_t>(cap) * N * es;
        int pnext = load_pos(lane);
        int st = lane, use = 0;  // stage of tile kb + lane and its use count
        int kb = 0;
        bool aborted = false;
        for (; tile_of(kb) < static_cast<uint32_t>(ntiles); kb += nb) {
            const int k = kb + lane;
            const uint32_t t = tile_of(k);
            const bool mine = lane_on && t < static_cast<uint32_t>(ntiles);
            const int pos = pnext;
            pnext = load_pos(k + nb);
            bool fail = false;
            if (mine && use > 0) fail = !mbar_wait_bounded(smem_u32(&empty_bar[st]), (use - 1) & 1, kWaitNs);
            if (fail) {
                set_error(a.err, RSSM_DEVERR_TIMEOUT);
                s_abort = 1;
            }
            // one decision for the whole warp, before any copy of the batch
            if (__any_sync(0xffffffffu, fail || s_abort)) {
                aborted = true;
                break;
            }
            if (mine) {
                const int b = fdiv(t, lay.divH), h = static_cast<int>(t) - b * H;
                unsigned char* sp = smem + static_cast<size_t>(st) * lay.stage_bytes;
                const uint32_t fb = smem_u32(&full_bar[st]);
                int* meta = reinterpret_cast<int*>(sp + lay.meta);
                meta[kMetaPos] = pos;
                reinterpret_cast<volatile int*>(meta)[kMetaTile] = k;
                const bool ok = pos >= 0 && pos + ntok <= cap;
                // record prefix: copy, scales, dt row and x rows 0..pos-1
                const uint32_t nrec = a.rec.x + static_cast<uint32_t>(pos * P * es);
                const uint32_t nbr = static_cast<uint32_t>(pos * N * es);
                const uint32_t nnew = kRowsInStage ? static_cast<uint32_t>(ntok * (P + 2 * N) * es) : 0u;
                mbar_expect_tx(fb, ok ? nrec + nbr + nnew : 0u);  // nothing to copy for a bad position
                if (ok) {
                    bulk_g2s(smem_u32(sp), a.record + static_cast<size_t>(t) * a.rec.bytes, nrec, fb);
                    const int g = fdiv(h, lay.divHpg);
                    const size_t bg = static_cast<size_t>(b) * G + g;
                    if (nbr > 0)
                        bulk_g2s(smem_u32(sp + lay.brows), static_cast<const unsigned char*>(a.bbuf) + bg * brow_bytes,
                                 nbr, fb);
                    if constexpr (kRowsInStage) {  // this call's x, B and C rows (one token)
                        const uint32_t rw = smem_u32(sp + lay.rows);
                        bulk_g2s(rw, static_cast<const TIn*>(a.x) + static_cast<size_t>(t) * P, P * es, fb);
                        bulk_g2s(rw + lay.nb_off, static_cast<const TIn*>(a.B) + bg * N, N * es, fb);
                        bulk_g2s(rw + lay.nc_off, static_cast<const TIn*>(a.C) + bg * N, N * es, fb);
                    }
                }
            }
            st += nb;
            if (st >= S) {
                st -= S;
                ++use;
            }
            __syncwarp();
        }
        if (aborted && lane == 0) {
            // let every copy this warp issued land before the CTA can exit:
            // tiles 0..kb-1 were issued, the last S of them may be in flight
            for (int kk = kb - 1; kk >= 0 && kk > kb - 1 - S; --kk)
                mbar_wait_bounded(smem_u32(&full_bar[kk % S]), (kk / S) & 1, kWaitNs);
        }
        return;
    }

    // --------------------------------------------------------------- consumers
    // Group gi takes tiles k = gi, gi + CG, ...; its CW warps: warps 0..3
    // form the B.C products (8 slots each), warp CW-1 the decay weights and
    // the request's arrival, warp 2 appends this call's x and B to the
    // buffer, all of them 8 rows at a time of the output.
    const int gi = warp / CW, cw = warp - gi * CW;
    const int ctid = tid - gi * CT;
    unsigned char* nbase = smem + static_cast<size_t>(S) * lay.stage_bytes + static_cast<size_t>(gi) * 2 * lay.newrows;
    // fused fold: w_s x_s in fp32, [cap][P], per group after the row buffers
    float* s_xw = reinterpret_cast<float*>(smem + static_cast<size_t>(S) * lay.stage_bytes +
                                           static_cast<size_t>(CG) * 2 * lay.newrows +
                                           static_cast<size_t>(gi) * lay.xw_bytes);
    // this call's rows of tile kk -> buf: [ntok][P] x, [ntok][N] B, [ntok][N] C in
    // 16-byte chunks, then the scalars dt [ntok], A_h, D_h at nd_off
    const int xc = (P * es) >> 4, bc = (N * es) >> 4;  // 16-byte chunks of an x row, of a B or C row
    const float inv_xc = 1.0f / static_cast<float>(xc);
    auto prefetch = [&](int kk, unsigned char* buf) {
        const uint32_t t = blockIdx.x + static_cast<uint32_t>(kk) * gridDim.x;
        if (t < static_cast<uint32_t>(ntiles)) {
            const int b = fdiv(t, lay.divH), h = t - b * H, g = fdiv(h, lay.divHpg);
            const size_t b0 = static_cast<size_t>(b) * ntok;
            const unsigned char* xs = reinterpret_cast<const unsigned char*>(
                static_cast<const TIn*>(a.x) + b0 * HP + static_cast<size_t>(h) * P);
            const unsigned char* bs = reinterpret_cast<const unsigned char*>(
                static_cast<const TIn*>(a.B) + b0 * GN + static_cast<size_t>(g) * N);
            const unsigned char* cs = reinterpret_cast<const unsigned char*>(
                static_cast<const TIn*>(a.C) + b0 * GN + static_cast<size_t>(g) * N);
            // every token's chunks in one branch-free sweep, so a warp issues
            // its copies in a few instructions: chunks [0, ntok xc) are the x
            // rows, then ntok bc of B rows, then ntok bc of C rows. Warps 1 and
            // 2 issue them (warp 0 starts the B.C products at once, warp CW-1
            // forms the weights): verify 571 -> 538 us; one divergent cp.async
            // per row kind and token had taken ~2,200 cycles per tile.
            {
                const int nxc = ntok * xc, nbc = ntok * bc;
                const int bsh = bc == 16 ? 4 : 5;  // bc = 128 es / 16
                constexpr int pf0 = CW > 2 ? 32 : 0, pfn = CW > 2 ? 64 : CT;
                for (int c = ctid - pf0; ctid >= pf0 && ctid < pf0 + pfn && c < nxc + 2 * nbc; c += pfn) {
                    const bool isx = c < nxc;
                    const int cb = c - nxc;
                    const bool isb = !isx && cb < nbc;
                    const int cc = isb ? cb : cb - nbc;
                    const int jx = static_cast<int>((static_cast<float>(c) + 0.5f) * inv_xc);  // c / xc, exact (c < 2^10)
                    const int j = isx ? jx : (cc >> bsh), q = isx ? c - jx * xc : (cc & (bc - 1));
                    const unsigned char* src = isx ? xs + static_cast<size_t>(j) * HP * es
                                                   : (isb ? bs : cs) + static_cast<size_t>(j) * GN * es;
                    const uint32_t dof = isx ? static_cast<uint32_t>(j * P * es)
                                             : (isb ? lay.nb_off : lay.nc_off) + static_cast<uint32_t>(j * N * es);
                    cp_async16(smem_u32(buf) + dof + 16u * q, src + 16 * q);
                }
            }
            if (ctid < ntok + 2) {  // scalars, 4 bytes each: dt of each token, A_h, D_h
                const int i = ctid;
                const float* src = i < ntok ? a.dt + (b0 + i) * H + h : (i == ntok ? a.A + h : a.D + h);
                const uint32_t dst = smem_u32(buf + lay.nd_off + 4 * (i < ntok ? i : kMaxTok + (i - ntok)));
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
            }
        }
        cp_async_commit();  // one group per tile, empty past the last tile
    };
    // rows of this group's first tile; each tile then fetches the next one's
    if constexpr (!kRowsInStage) prefetch(gi, nbase);
    const uint32_t step = static_cast<uint32_t>(CG) * gridDim.x;
    const int dh = static_cast<int>(step % static_cast<uint32_t>(H)), db = static_cast<int>(step / H);
    const uint32_t t0 = blockIdx.x + static_cast<uint32_t>(gi) * gridDim.x;
    int b = fdiv(t0, lay.divH), h = static_cast<int>(t0) - b * H;
    int st = gi, use = 0;
    while (st >= S) {
        st -= S;
        ++use;
    }
    // deferred arrival (warp CW-1, lane 0): the returned count is checked one tile later
    int pend_b = -1, pend_new = 0;
    bool pend_bump = false;
    uint32_t pend_old = 0;
    int it = 0;
    for (int k = gi; t0 + static_cast<uint32_t>(it) * step < static_cast<uint32_t>(ntiles); k += CG, ++it) {
        const int g = fdiv(h, lay.divHpg);
        const size_t bh = static_cast<size_t>(b) * H + h, bg = static_cast<size_t>(b) * G + g;
        const unsigned char* sp = smem + static_cast<size_t>(st) * lay.stage_bytes;
        // rows with the stage: this call's scalars of the tile, loaded before
        // the waits so that they arrive meanwhile (dt of token `lane`, A_h, D_h)
        float dtl = 0.f, Ahr = 0.f, Dhr = 0.f;
        if constexpr (kRowsInStage) {
            dtl = lane < ntok ? a.dt[(static_cast<size_t>(b) * ntok + lane) * H + h] : 0.f;
            Ahr = a.A[h];
            Dhr = a.D[h];
        }
        int stop = 0;
        if (ctid == 0) {
            stop = s_abort;
            // The stage's previous use may belong to another group and still
            // be in flight; once the producer has tagged the stage with this
            // tile, that use has landed and the parity below names this one.
            const volatile int* tag = reinterpret_cast<const volatile int*>(sp + lay.meta) + kMetaTile;
            if (!stop && !smem_wait_eq_bounded(tag, k, kWaitNs)) {
                set_error(a.err, RSSM_DEVERR_TIMEOUT);  // never tagged: nothing was issued for it
                s_abort = 1;
                stop = 1;
            }
            if (!stop && !mbar_wait_bounded(smem_u32(&full_bar[st]), use & 1, kWaitNs)) {
                set_error(a.err, RSSM_DEVERR_TIMEOUT);
                s_abort = 1;
                stop = 1;
                mbar_wait_bounded(smem_u32(&full_bar[st]), use & 1, kWaitNs);  // copies in flight
            }
        }
        if constexpr (!kRowsInStage) cp_async_wait_all();  // this tile's rows
        // the stage and this tile's rows have landed; this group's previous
        // readers of s_w / s_g and of the row buffers are done
        if (group_sync_or(gi, CT, stop)) break;
        // the next tile's rows, into the buffer the previous tile used (its
        // readers all passed the barrier above); they land while this tile works
        if constexpr (!kRowsInStage) prefetch(k + CG, nbase + ((it + 1) & 1) * lay.newrows);
        bool released = false;  // the stage went back to the producer before the tile's end
        const unsigned char* nr = kRowsInStage ? sp + lay.rows : nbase + (it & 1) * lay.newrows;
        const float* sc4 = reinterpret_cast<const float*>(nr + lay.nd_off);  // row buffers: dt [8], A, D
        const int pos = reinterpret_cast<const int*>(sp + lay.meta)[kMetaPos];
        const int T = pos + ntok;
        const bool ok = pos >= 0 && T <= cap;
        const TIn* xr = reinterpret_cast<const TIn*>(sp + a.rec.x);     // slot s < pos: xr + s*P
        const TIn* br = reinterpret_cast<const TIn*>(sp + lay.brows);   // slot s < pos: br + s*N
        const TIn* nx = reinterpret_cast<const TIn*>(nr);               // token j: nx + j*P
        const TIn* nb = reinterpret_cast<const TIn*>(nr + lay.nb_off);  // token j: nb + j*N
        const TIn* nc = reinterpret_cast<const TIn*>(nr + lay.nc_off);  // token j: nc + j*N
        unsigned char* rec = a.record + bh * a.rec.bytes;
        float4 c4[NT];
        if (!ok) {
            if (ctid == 0) set_error(a.err, (pos < 0 || pos > cap) ? RSSM_DEVERR_POS_RANGE : RSSM_DEVERR_CAPACITY);
        } else {
#pragma unroll
            for (int j = 0; j < NT; ++j)
                c4[j] = (j < ntok) ? load4(nc + j * N + 4 * lane) : make_float4(0.f, 0.f, 0.f, 0.f);
            // a tile that folds (fused flush) needs neither the B.C products nor
            // the replay rows: its output comes from the folded state
            const bool fold_now = FUSED && T == a.s.L;
            if constexpr (kMma) {
                // B_s . C_j on the tensor cores, 16 slots per warp
                for (int s0 = 16 * cw; s0 < T; s0 += 16 * CW)
                    bc_products_mma(reinterpret_cast<const __nv_bfloat16*>(br),
                                    reinterpret_cast<const __nv_bfloat16*>(nb),
                                    reinterpret_cast<const __nv_bfloat16*>(nc), pos, T, ntok, s0, &s_g[gi][0][0]);
            }
            for (int s0 = cw * 8; !kMma && !fold_now && s0 < T; s0 += CW * 8) {
                // B_s . C_j for slots s0..s0+7, reduced together; the 8 B rows
                // are read once for all tokens
                float4 bv[8];
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const int sl = s0 + kk;
                    const TIn* row = (sl < pos) ? br + sl * N : nb + (sl - pos) * N;
                    bv[kk] = (sl < T) ? load4(row + 4 * lane) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    if (j < ntok) {
                        float part[8];
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) part[kk] = dot4(bv[kk], c4[j]);
                        const float z = warp_reduce8(part);
                        const int sl = s0 + ((lane >> 2) & 7);
                        if ((lane & 3) == 0 && sl < T) s_g[gi][j][sl] = z;
                    }
                }
            }
            if (cw == CW - 1) {
                const float* dtrow = reinterpret_cast<const float*>(sp + a.rec.dt);
                float dnv;
                if constexpr (kRowsInStage)
                    dnv = __shfl_sync(0xffffffffu, dtl, (lane - pos) & 31);
                else
                    dnv = (lane >= pos && lane < T) ? sc4[lane - pos] : 0.f;
                const float dnew = (lane >= pos && lane < T) ? dnv : 0.f;
                const float dts = (lane < pos) ? dtrow[lane] : dnew;
                if (lane >= pos && lane < T) reinterpret_cast<float*>(rec + a.rec.dt)[lane] = dnew;
                const float Sx = warp_prefix(dts);
                const float Ah = kRowsInStage ? Ahr : sc4[kMaxTok];
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    if (j < ntok) {
                        const float St = __shfl_sync(0xffffffffu, Sx, pos + j);
                        s_w[gi][j][lane] = (lane <= pos + j) ? dts * expf(Ah * (St - Sx)) : 0.f;
                        if (lane == 0) s_decay[gi][j] = expf(Ah * St);
                    }
                }
                if (a.advance && lane == 0) {
                    // every CTA read pos[b] before it processed b's tiles; the
                    // request's last arrival moves it (to 0 after a fused fold)
                    if (pend_b >= 0 && pend_old == static_cast<uint32_t>(H - 1)) {
                        a.arrive[pend_b] = 0u;
                        a.pos[pend_b] = pend_new;
                        if (pend_bump) a.flush_count[pend_b] += 1u;
                    }
                    pend_b = b;
                    pend_bump = FUSED && T == a.s.L;
                    pend_new = pend_bump ? 0 : pos + 1;
                    pend_old = atomicAdd(&a.arrive[b], 1u);
                }
            }
            if (!fold_now && cw == (CW >= 3 ? 2 : 0)) {
                // append this call's x (and, for the group's first head, B) to the buffer
                const int xq = ntok * xc, bq = ntok * bc;
                uint4* xdst = reinterpret_cast<uint4*>(rec + a.rec.x + static_cast<size_t>(pos) * P * es);
                for (int q = lane; q < xq; q += 32) xdst[q] = reinterpret_cast<const uint4*>(nx)[q];
                if (h == g * (H / G)) {
                    uint4* bdst = reinterpret_cast<uint4*>(static_cast<TIn*>(a.bbuf) + (bg * cap + pos) * N);
                    for (int q = lane; q < bq; q += 32) bdst[q] = reinterpret_cast<const uint4*>(nb)[q];
                }
            }
        }
        group_sync(gi, CT);  // s_w, s_g, s_decay ready
        if (ok && !(FUSED && T == a.s.L)) {
            const unsigned char* tile = sp;
            const unsigned char* sc = sp + a.rec.scales;
            const float Dh = kRowsInStage ? Dhr : sc4[kMaxTok + 1];
            float* yout = a.y + static_cast<size_t>(b) * ntok * HP + static_cast<size_t>(h) * P;
            const TIn* xrow = (lane < pos) ? xr + lane * P : nx + (lane - pos) * P;  // slot `lane`
            // partials of rows r0..r0+7 for token j: lane l holds columns 4l..4l+3
            // of h.C and slot l's replay term (zeros past the last row)
            auto partials = [&](int r0, const float4& cj, float dec, float coef, bool term, float (&part)[8]) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    if constexpr (RF == kFP4) {
                        // codes . C first, then one multiply by the block scale
                        const int q = (r0 + kk) * (N >> 2) + lane;
                        part[kk] = (r0 + kk < P) ? (dec * e4m3_val(sc[q >> 2])) *
                                                       dot4(e2m1x4_val(reinterpret_cast<const uint16_t*>(tile)[q]), cj)
                                                 : 0.f;
                    } else {
                        const float4 hv = (r0 + kk < P) ? tile_load4<RF>(tile, sc, r0 + kk, lane, N)
                                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                        part[kk] = dec * dot4(hv, cj);
                    }
                }
                if (term && r0 < P) {
                    Raw8<TIn> xv;
                    xv.load(xrow + r0);
                    const float4 xa = xv.lo(), xb = xv.hi();
                    part[0] = fmaf(coef, xa.x, part[0]);
                    part[1] = fmaf(coef, xa.y, part[1]);
                    part[2] = fmaf(coef, xa.z, part[2]);
                    part[3] = fmaf(coef, xa.w, part[3]);
                    part[4] = fmaf(coef, xb.x, part[4]);
                    part[5] = fmaf(coef, xb.y, part[5]);
                    part[6] = fmaf(coef, xb.z, part[6]);
                    part[7] = fmaf(coef, xb.w, part[7]);
                }
            };
            if constexpr (kMma && NT == 1) {
                // FP4 decode on the tensor cores: the product's 8 columns are the
                // 8 scale blocks of a row (B holds C in the column of the block
                // its k falls in), so lane (g, t) receives the bare code . C sums
                // of blocks 2t, 2t + 1 of rows g and g + 8 and scales them; its
                // replay terms (slots t, t + 4, ...) join before the row's four
                // lanes add up.
                const int g = lane >> 2, t = lane & 3;
                uint4 cb[4];
                load_bf16_chunks(cb, reinterpret_cast<const __nv_bfloat16*>(nc), t, false);
                uint32_t bf[16];
                hc_bfrag<kFP4>(cb, bf);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const bool mine = g == 2 * t + (c >> 1);
#pragma unroll
                    for (int u = 0; u < 4; ++u) bf[4 * c + u] = mine ? bf[4 * c + u] : 0u;
                }
                const float dec = s_decay[gi][0];
                // replay terms sum_{s <= pos} coef_s x_s[p] of every row: lane l
                // takes rows 2l, 2l + 1 (+ 64 ...), one 32-bit load of x per slot
                float* rep = s_rep[gi];
                for (int p0 = 2 * (lane + 32 * cw); p0 < P; p0 += 64 * CW) {
                    float r0 = 0.f, r1 = 0.f;
                    for (int sl = 0; sl <= pos; ++sl) {
                        const float cfs = s_w[gi][0][sl] * s_g[gi][0][sl];
                        const uint32_t w2 = *reinterpret_cast<const uint32_t*>((sl < pos ? xr + sl * P : nx) + p0);
                        r0 = fmaf(cfs, __uint_as_float(bf16lo_bits(w2)), r0);
                        r1 = fmaf(cfs, __uint_as_float(bf16hi_bits(w2)), r1);
                    }
                    rep[p0] = r0;
                    rep[p0 + 1] = r1;
                }
                if constexpr (CW == 1)
                    __syncwarp();
                else
                    group_sync(gi, CT);
                // rows R0 + g, R0 + g + 8: scale the two block sums, add the row's
                // four lanes, then the replay term and D x
                // (xa, xb: this call's x of the two rows)
                auto finish = [&](int R0, const float (&d)[4], uint32_t s2a, uint32_t s2b, float xa, float xb) {
                    const int ra = R0 + g, rb = ra + 8;
                    const float2 sa = h2_f2(s2a), sb = h2_f2(s2b);
                    float pa = fmaf(sa.x, d[0], sa.y * d[1]);
                    float pb = fmaf(sb.x, d[2], sb.y * d[3]);
                    pa += __shfl_xor_sync(0xffffffffu, pa, 1);
                    pb += __shfl_xor_sync(0xffffffffu, pb, 1);
                    pa += __shfl_xor_sync(0xffffffffu, pa, 2);
                    pb += __shfl_xor_sync(0xffffffffu, pb, 2);
                    if (t == 0) {
                        if (ra < P) yout[ra] = fmaf(Dh, xa, fmaf(dec, pa, rep[ra]));
                        if (rb < P) yout[rb] = fmaf(Dh, xb, fmaf(dec, pb, rep[rb]));
                    }
                };
                auto scales2 = [&](int r) -> uint32_t {  // e4m3 scales of blocks 2t, 2t + 1 of row r as f16
                    return r < P ? e4m3x2_h2(*reinterpret_cast<const uint16_t*>(sc + r * (N >> 4) + 2 * t)) : 0u;
                };
                if (CW == 1 && P <= 64) {
                    // the lane's codes, scales and x (this call's, of its rows) of
                    // every row group into registers, then the stage goes back to
                    // the producer before the products
                    uint4 qa[4], qb[4];
                    uint32_t s2a[4], s2b[4], xab[4];
#pragma unroll
                    for (int rg = 0; rg < 4; ++rg) {
                        const int ra = 16 * rg + g, rb = ra + 8;
                        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                        qa[rg] = ra < P ? *reinterpret_cast<const uint4*>(tile + ra * (kD128 / 2) + 16 * t) : z;
                        qb[rg] = rb < P ? *reinterpret_cast<const uint4*>(tile + rb * (kD128 / 2) + 16 * t) : z;
                        s2a[rg] = scales2(ra);
                        s2b[rg] = scales2(rb);
                        const uint16_t* xw = reinterpret_cast<const uint16_t*>(nx);
                        xab[rg] = (ra < P ? xw[ra] : 0u) | ((rb < P ? static_cast<uint32_t>(xw[rb]) : 0u) << 16);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&empty_bar[st]));
                    released = true;
#pragma unroll
                    for (int rg = 0; rg < 4; ++rg) {
                        if (16 * rg < P) {
                            float d[4] = {0.f, 0.f, 0.f, 0.f};
                            fp4_codes_mma(qa[rg], qb[rg], bf, d);
                            finish(16 * rg, d, s2a[rg], s2b[rg], __uint_as_float(xab[rg] << 16),
                                   __uint_as_float(xab[rg] & 0xFFFF0000u));
                        }
                    }
                } else {
                    for (int R0 = 16 * cw; R0 < P; R0 += 16 * CW) {
                        float d[4] = {0.f, 0.f, 0.f, 0.f};
                        hc_mma<kFP4, false>(tile, sc, R0, P, bf, d);
                        const int ra = R0 + g, rb = ra + 8;
                        finish(R0, d, scales2(ra), scales2(rb), ra < P ? to_f32(nx[ra]) : 0.f,
                               rb < P ? to_f32(nx[rb]) : 0.f);
                    }
                }
            } else if constexpr (kMma) {
                // verify on the tensor cores: lane (g, t) receives h . C_j and the
                // replay sums of rows g, g + 8 for the tokens j = 2t, 2t + 1
                const int g = lane >> 2, t = lane & 3;
                uint4 cb[4];
                load_bf16_chunks(cb, g < ntok ? reinterpret_cast<const __nv_bfloat16*>(nc) + g * kD128 : nullptr, t,
                                 hc_rotated(RF));
                uint32_t bf[16];
                hc_bfrag<RF>(cb, bf);
                // coef of token g for the slots 8q + t (b0) and 8q + t + 4 (b1), hi + lo
                uint32_t cfr[16];
#pragma unroll
                for (int q = 0; q < kMaxCap / 8; ++q) {
                    const int s0 = 8 * q + t, s1 = s0 + 4;
                    const float c0 = (g < ntok && s0 <= pos + g) ? s_w[gi][g][s0] * s_g[gi][g][s0] : 0.f;
                    const float c1 = (g < ntok && s1 <= pos + g) ? s_w[gi][g][s1] * s_g[gi][g][s1] : 0.f;
                    tf32_split(c0, cfr[4 * q], cfr[4 * q + 2]);
                    tf32_split(c1, cfr[4 * q + 1], cfr[4 * q + 3]);
                }
                const int j0 = 2 * t, j1 = 2 * t + 1;
                const float dec0 = j0 < ntok ? s_decay[gi][j0] : 0.f, dec1 = j1 < ntok ? s_decay[gi][j1] : 0.f;
                // this lane's slot rows for the replay steps: 8q + t and 8q + t + 4
                uint32_t xrow[kMaxCap / 4];
#pragma unroll
                for (int i = 0; i < kMaxCap / 4; ++i) {
                    const int sl = 8 * (i >> 1) + t + 4 * (i & 1);
                    xrow[i] = sl < pos ? smem_u32(xr + sl * P) : (sl < T ? smem_u32(nx + (sl - pos) * P) : 0u);
                }
                for (int R0 = 16 * cw; R0 < P; R0 += 16 * CW) {
                    float dh[4] = {0.f, 0.f, 0.f, 0.f}, dx[4] = {0.f, 0.f, 0.f, 0.f};
                    hc_mma<RF, true>(tile, sc, R0, P, bf, dh);
                    replay_mma(xrow, T, P, R0, cfr, dx);
                    const int ra = R0 + g, rb = ra + 8;
                    if (ra < P) {
                        if (j0 < ntok) yout[j0 * HP + ra] = fmaf(Dh, to_f32(nx[j0 * P + ra]), fmaf(dec0, dh[0], dx[0]));
                        if (j1 < ntok) yout[j1 * HP + ra] = fmaf(Dh, to_f32(nx[j1 * P + ra]), fmaf(dec1, dh[1], dx[1]));
                    }
                    if (rb < P) {
                        if (j0 < ntok) yout[j0 * HP + rb] = fmaf(Dh, to_f32(nx[j0 * P + rb]), fmaf(dec0, dh[2], dx[2]));
                        if (j1 < ntok) yout[j1 * HP + rb] = fmaf(Dh, to_f32(nx[j1 * P + rb]), fmaf(dec1, dh[3], dx[3]));
                    }
                }
            } else if constexpr (RF == kFP4 && NT == 1) {
                // FP4 decode: lane l takes row r0 + l/4 and columns 32 (l % 4) ..
                // +31 of an 8-row block: one 16-byte load of codes and one of
                // two scales per row, codes.C per 16 columns times the block
                // scale, and the replay terms of slots l % 4, l % 4 + 4, ...;
                // the row's 4 lanes then add up with two shuffles
                const int sg = lane & 3, rl = lane >> 2;
                float cv[32];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    Raw8<TIn> r8;
                    r8.load(nc + 32 * sg + 8 * i);
                    const float4 lo = r8.lo(), hi = r8.hi();
                    cv[8 * i + 0] = lo.x;
                    cv[8 * i + 1] = lo.y;
                    cv[8 * i + 2] = lo.z;
                    cv[8 * i + 3] = lo.w;
                    cv[8 * i + 4] = hi.x;
                    cv[8 * i + 5] = hi.y;
                    cv[8 * i + 6] = hi.z;
                    cv[8 * i + 7] = hi.w;
                }
                const float dec = s_decay[gi][0];
                float cf[kMaxCap / 4];
#pragma unroll
                for (int m = 0; m < kMaxCap / 4; ++m) {
                    const int sl = sg + 4 * m;
                    cf[m] = (sl <= pos) ? s_w[gi][0][sl] * s_g[gi][0][sl] : 0.f;
                }
                for (int r0 = cw * 8; r0 < P; r0 += CW * 8) {
                    const int r = r0 + rl;
                    const uint4 q4 = *reinterpret_cast<const uint4*>(tile + r * (N >> 1) + 16 * sg);
                    const float2 s2 =
                        h2_f2(e4m3x2_h2(*reinterpret_cast<const uint16_t*>(sc + r * (N >> 4) + 2 * sg)));
                    const float a0 = e2m1x8_dot(q4.x, cv, 0.f) + e2m1x8_dot(q4.y, cv + 8, 0.f);
                    const float a1 = e2m1x8_dot(q4.z, cv + 16, 0.f) + e2m1x8_dot(q4.w, cv + 24, 0.f);
                    float part = dec * fmaf(s2.x, a0, s2.y * a1);
#pragma unroll
                    for (int m = 0; m < kMaxCap / 4; ++m) {
                        const int sl = sg + 4 * m;
                        if (sl <= pos) part = fmaf(cf[m], to_f32((sl < pos ? xr + sl * P : nx)[r]), part);
                    }
                    part += __shfl_xor_sync(0xffffffffu, part, 1);
                    part += __shfl_xor_sync(0xffffffffu, part, 2);
                    if (sg == 0) yout[r] = fmaf(Dh, to_f32(nx[r]), part);
                }
            } else if constexpr (NT > 1) {
                // verify: one 8-row block at a time; its tile rows and x
                // values are read once for all tokens
                for (int r0 = cw * 8; r0 < P; r0 += CW * 8) {
                    float4 hv[8];
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) hv[kk] = tile_load4<RF>(tile, sc, r0 + kk, lane, N);
                    float xv8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    if (lane < T) {  // slot `lane` exists (its row lies in the stage or this call's rows)
                        Raw8<TIn> xv;
                        xv.load(xrow + r0);
                        const float4 xa = xv.lo(), xb = xv.hi();
                        xv8[0] = xa.x; xv8[1] = xa.y; xv8[2] = xa.z; xv8[3] = xa.w;
                        xv8[4] = xb.x; xv8[5] = xb.y; xv8[6] = xb.z; xv8[7] = xb.w;
                    }
                    const int rr = r0 + ((lane >> 2) & 7);
#pragma unroll
                    for (int j = 0; j < NT; ++j) {
                        if (j < ntok) {
                            const int tt = pos + j;
                            const float dec = s_decay[gi][j];
                            const float4 cd = make_float4(dec * c4[j].x, dec * c4[j].y, dec * c4[j].z, dec * c4[j].w);
                            const float coef = (lane <= tt) ? s_w[gi][j][lane] * s_g[gi][j][lane] : 0.f;
                            float part[8];
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk) part[kk] = fmaf(coef, xv8[kk], dot4(hv[kk], cd));
                            const float z = warp_reduce8(part);
                            if ((lane & 3) == 0) yout[j * HP + rr] = fmaf(Dh, to_f32(nx[j * P + rr]), z);
                        }
                    }
                }
            }
            // decode: two 8-row blocks per pass, so their reductions overlap
            for (int r0 = cw * 8; NT == 1 && RF != kFP4 && r0 < P; r0 += 2 * CW * 8) {
                const int r1 = r0 + CW * 8;
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    if (j < ntok) {
                        const int tt = pos + j;
                        const float dec = s_decay[gi][j];
                        const bool term = lane <= tt;
                        const float coef = term ? s_w[gi][j][lane] * s_g[gi][j][lane] : 0.f;
                        float pa[8], pb[8];
                        partials(r0, c4[j], dec, coef, term, pa);
                        partials(r1, c4[j], dec, coef, term, pb);
                        const float za = warp_reduce8(pa), zb = warp_reduce8(pb);
                        const int ra = r0 + ((lane >> 2) & 7), rb = r1 + ((lane >> 2) & 7);
                        if ((lane & 3) == 0) {
                            if (ra < P) yout[j * HP + ra] = fmaf(Dh, to_f32(nx[j * P + ra]), za);
                            if (rb < P) yout[j * HP + rb] = fmaf(Dh, to_f32(nx[j * P + rb]), zb);
                        }
                    }
                }
            }
        }
        if constexpr (FUSED != 0) {
            if (ok && T == a.s.L) {  // uniform over the group: the token that fills the buffer folds it
                // h <- exp(A S_T) h + sum_s w_s x_s B_s^T with w_s = s_w[gi][0][s]
                // (t = pos = T - 1), written over the checkpoint in the record.
                // The folded state is h_t itself, so y_t = h_t C_t + D x_t.
                const int x8 = P >> 3;
                for (int c = ctid; c < T * x8; c += CT) {
                    const int sl = c / x8, p8 = (c - sl * x8) << 3;
                    Raw8<TIn> r;
                    r.load((sl < pos ? xr + sl * P : nx) + p8);
                    const float w = s_w[gi][0][sl];
                    const float4 lo = r.lo(), hi = r.hi();
                    float4* d = reinterpret_cast<float4*>(s_xw + sl * P + p8);
                    d[0] = make_float4(w * lo.x, w * lo.y, w * lo.z, w * lo.w);
                    d[1] = make_float4(w * hi.x, w * hi.y, w * hi.z, w * hi.w);
                }
                group_sync(gi, CT);
                const float alpha = s_decay[gi][0];
                float* ck = reinterpret_cast<float*>(rec);
                for (int r0 = cw * kRB; r0 < P; r0 += CW * kRB) {
                    // acc = alpha h, then the slots in order (as the flush kernels)
                    float2 acc2[4][4];
#pragma unroll
                    for (int kk = 0; kk < kRB; ++kk) {
                        const float4 hv = reinterpret_cast<const float4*>(sp)[(r0 + kk) * (N >> 2) + lane];
                        acc2_set_row(acc2, kk, make_float4(alpha * hv.x, alpha * hv.y, alpha * hv.z, alpha * hv.w));
                    }
#pragma unroll 2
                    for (int sl = 0; sl < T; ++sl) {
                        const float4 bv = load4((sl < pos ? br + sl * N : nb) + 4 * lane);
                        const float4* xw4 = reinterpret_cast<const float4*>(s_xw + sl * P + r0);
                        const float4 xa = xw4[0], xb = xw4[1];
                        const float2 w2[4] = {make_float2(xa.x, xa.y), make_float2(xa.z, xa.w),
                                              make_float2(xb.x, xb.y), make_float2(xb.z, xb.w)};
                        rank1_8x4(acc2, w2, bv);
                    }
                    float part[kRB];
#pragma unroll
                    for (int kk = 0; kk < kRB; ++kk) {
                        const float4 v = acc2_row(acc2, kk);
                        stream_store4(ck + (r0 + kk) * N + 4 * lane, v);
                        part[kk] = dot4(v, c4[0]);
                    }
                    const float z = warp_reduce8(part);
                    const int r = r0 + ((lane >> 2) & 7);
                    if ((lane & 3) == 0)
                        a.y[static_cast<size_t>(b) * HP + static_cast<size_t>(h) * P + r] =
                            fmaf(sc4[kMaxTok + 1], to_f32(nx[r]), z);
                }
            }
        }
        __syncwarp();
        if (lane == 0 && !released) mbar_arrive(smem_u32(&empty_bar[st]));
        h += dh;
        b += db;
        if (h >= H) {
            h -= H;
            ++b;
        }
        st += CG;
        while (st >= S) {
            st -= S;
            ++use;
        }
    }
    cp_async_wait_all();  // no copy of this thread outlives the CTA
    if (cw == CW - 1 && lane == 0 && pend_b >= 0 && pend_old == static_cast<uint32_t>(H - 1)) {
        a.arrive[pend_b] = 0u;  // the last pending arrival of this group
        a.pos[pend_b] = pend_new;
        if (pend_bump) a.flush_count[pend_b] += 1u;
    }
}

// ---------------------------------------------------------------------------
// Fold of the buffer into the update copy: flush (s1) and precision-split
// refresh (s4). UF: format of the update copy (read and written); OUT4: also
// write the FP4 output copy from the fp32 result.
// ---------------------------------------------------------------------------
template <typename TIn, int UF, int OUT4>
__global__ void __launch_bounds__(kThreads, 4) k_fold(const FoldArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bar;
    __shared__ float s_cw[kMaxCap];
    __shared__ float s_alpha;
    __shared__ int s_pos;
    __shared__ uint32_t s_fc;

    const int H = a.s.H, P = a.s.P, N = a.s.N, G = a.s.G, cap = a.s.cap, lpr = a.s.lpr;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x / H, h = blockIdx.x - b * H;
    const int g = h / (H / G);
    const int xs = round_up8(P);
    const size_t bh = static_cast<size_t>(b) * H + h;

    const uint32_t tb = tile_bytes(UF, P, N), sb = scale_bytes(UF, P, N);
    unsigned char* s_in = smem;
    unsigned char* s_insc = smem + align16(tb);
    unsigned char* after_in = smem + align16(tb) + align16(sb);
    float* s32 = (UF == kF32) ? reinterpret_cast<float*>(s_in) : reinterpret_cast<float*>(after_in);
    float* s_B = reinterpret_cast<float*>(after_in + (UF == kF32 ? 0u : 4u * P * N));  // [cap][N]
    float* s_x = s_B + cap * N;                                                        // [cap][xs]
    const uint32_t bar_a = smem_u32(&bar);

    if (tid == 0) {
        // the only reads of pos and flush_count: every thread uses these copies
        const int p0 = a.pos[b];
        s_pos = p0;
        s_fc = a.flush_count[b];
        const bool go0 = p0 >= 0 && p0 <= cap && ((p0 >= a.s.L) || (a.mode >= 1 && p0 > 0) || (a.mode == 2));
        if (go0) {
            // values and (FP4, in the record) scales: contiguous, as here
            mbar_init(bar_a, 1);
            mbar_expect_tx(bar_a, tb + sb);
            bulk_g2s(smem_u32(s_in), a.upd + bh * a.upd_stride, tb + sb, bar_a);
        }
    }
    __syncthreads();
    const int pos = s_pos;
    const uint32_t fc = s_fc;
    if (pos < 0 || pos > cap) {
        if (tid == 0) set_error(a.err, RSSM_DEVERR_POS_RANGE);
        return;
    }
    const bool go = (pos >= a.s.L) || (a.mode >= 1 && pos > 0) || (a.mode == 2);
    if (!go) return;
    const int T = pos;
    // past the barrier no thread of this CTA reads pos or flush_count again;
    // once every CTA of the request has arrived, the last one resets them
    if (tid == kThreads - 32) request_done(a.arrive, b, H, a.pos, 0, a.flush_count, true);

    unsigned char* rec = a.record + bh * a.rec.bytes;
    unsigned char* upd = a.upd + bh * a.upd_stride;
    const TIn* bb = static_cast<const TIn*>(a.bbuf);
    const float Ah = a.A[h];
    // one round of independent loads: B rows, x rows (16-byte chunks when the
    // rows allow it), dt
    const TIn* bbg = bb + (static_cast<size_t>(b) * G + g) * cap * N;
    const TIn* xbh = reinterpret_cast<const TIn*>(rec + a.rec.x);
    for (int q = tid; q < ((T * N) >> 3); q += kThreads) {
        Raw8<TIn> r;
        r.load(bbg + (q << 3));
        reinterpret_cast<float4*>(s_B)[2 * q] = r.lo();
        reinterpret_cast<float4*>(s_B)[2 * q + 1] = r.hi();
    }
    if ((P & 7) == 0) {
        for (int q = tid; q < ((T * P) >> 3); q += kThreads) {
            const int e = q << 3, sl = e / P, p = e - sl * P;
            Raw8<TIn> r;
            r.load(xbh + e);
            float4* d = reinterpret_cast<float4*>(s_x + sl * xs + p);
            d[0] = r.lo();
            d[1] = r.hi();
        }
    } else {
        for (int i = tid; i < T * P; i += kThreads) s_x[(i / P) * xs + (i % P)] = to_f32(xbh[i]);
    }
    if (warp == 0) {
        const float dts = (lane < T) ? reinterpret_cast<const float*>(rec + a.rec.dt)[lane] : 0.f;
        const float Sx = warp_prefix(dts);
        const float Stot = T > 0 ? __shfl_sync(0xffffffffu, Sx, T - 1) : 0.f;
        s_cw[lane] = (lane < T) ? dts * expf(Ah * (Stot - Sx)) : 0.f;
        if (lane == 0) s_alpha = expf(Ah * Stot);
    }

    // one thread waits for the tile; the barrier publishes it to the CTA
    bool arrived = true;
    if (tid == 0) arrived = mbar_wait_bounded(bar_a, 0, kWaitNs);
    if (__syncthreads_or(!arrived)) {
        if (tid == 0) {
            set_error(a.err, RSSM_DEVERR_TIMEOUT);
            mbar_wait_bounded(bar_a, 0, kWaitNs);
        }
        return;
    }
    if constexpr (UF != kF32) {
        const int nq = P * (N >> 2);
        for (int q = tid; q < nq; q += kThreads) {
            const int r = q / (N >> 2), c = q - r * (N >> 2);
            reinterpret_cast<float4*>(s32)[q] = tile_load4<UF>(s_in, s_insc, r, c, N);
        }
        __syncthreads();
    }

    const PhiloxKeys pkeys = philox_keys(a.seed);
    auto brow = [&](int s, int c) {
        const float w = s_cw[s];
        const float4 v = reinterpret_cast<const float4*>(s_B + s * N)[c];
        return make_float4(w * v.x, w * v.y, w * v.z, w * v.w);
    };
    auto emit = [&](int r, int c, float4 v, bool valid) {
        const uint32_t e = static_cast<uint32_t>(r * N + 4 * c);  // element of v.x within the head
        if constexpr (UF == kF32) {
            if (valid) stream_store4(reinterpret_cast<float*>(upd) + e, v);
        } else if constexpr (UF == kBF16 || UF == kE4M3) {
            if (valid) {
                // Philox counter (e/4, head, request, flush_count)
                const uint4 rw = philox4x32_10(make_uint4(e >> 2, h, b, fc), pkeys);
                if constexpr (UF == kBF16) {
                    const uint2 w = make_uint2(sr_bf16x2(v.x, v.y, rw.x, rw.y), sr_bf16x2(v.z, v.w, rw.z, rw.w));
                    *reinterpret_cast<uint2*>(upd + 2u * e) = w;
                } else {
                    const uint32_t w = sr_e4m3(v.x, rw.x) | (sr_e4m3(v.y, rw.y) << 8) |
                                       (sr_e4m3(v.z, rw.z) << 16) | (sr_e4m3(v.w, rw.w) << 24);
                    *reinterpret_cast<uint32_t*>(upd + e) = w;
                }
            }
        } else {
            // the shared FP4 copy lives in the record: scales at rec.scales
            uint32_t sc;
            const uint32_t codes = fp4_quant_quad(v, &sc);
            if (valid) {
                *reinterpret_cast<uint16_t*>(upd + e / 2) = static_cast<uint16_t>(codes);
                if ((c & 3) == 0) upd[a.rec.scales + e / 16] = static_cast<uint8_t>(sc);
            }
        }
        if constexpr (OUT4 != 0) {
            uint32_t sc;
            const uint32_t codes = fp4_quant_quad(v, &sc);
            if (valid) {
                *reinterpret_cast<uint16_t*>(rec + e / 2) = static_cast<uint16_t>(codes);
                if ((c & 3) == 0) rec[a.rec.scales + e / 16] = static_cast<uint8_t>(sc);
            }
        }
    };
    fold_tile(s32, s_x, xs, P, N, lpr, T, s_alpha, brow, emit);
}

// ---------------------------------------------------------------------------
// Persistent, warp-specialised fold (flush and refresh) for d_state 128 and
// head_dim a multiple of 8. The producer warp walks the CTA's tiles, skips
// the requests that are not due, and brings each due tile into a stage: its
// update copy and, from the record, dt and the x rows 0..pos-1 (one bulk copy
// when the update copy is the record's own copy), plus the group's B rows.
// Consumer groups take the due tiles in turn (stage sequence q = gi, gi+CG,
// ...; the producer ends each group's sequence with a tile index of -1):
// weights, B and w_s x_s to fp32 in the group's scratch, then the rank-T
// update 8 rows x 4 columns per thread and the format's epilogue, stored
// straight from registers.
// ---------------------------------------------------------------------------
struct FoldPipeLayout {
    uint32_t stage_bytes, st_dt, st_x, brows, meta, scratch;
    int stages;
    FastDiv divH, divHpg;
};

// meta words of a fold stage: tile index (-1: end), position, flush count, A_h, tag
constexpr int kFMetaTile = 0, kFMetaPos = 1, kFMetaFc = 2, kFMetaA = 3, kFMetaTag = 4;

// Consumer groups of four warps: three for the fp32 flush (bound by HBM;
// B200: 190 us with 3 groups, 196 with 4), four for the low-precision
// refreshes, which are bound by issue (Philox draws, rounding, FP4
// quantisation; bf16 refresh 478 -> 430 us with 4 groups).
__host__ __device__ constexpr int fold_groups(int uf) { return uf == kF32 ? 3 : 5; }
__host__ __device__ constexpr int fold_cwarps(int uf) { return (void)uf, 4; }
__host__ __device__ constexpr int fold_threads(int uf) { return (fold_groups(uf) * fold_cwarps(uf) + 1) * 32; }

template <typename TIn, int UF, int OUT4>
__global__ void __launch_bounds__(fold_threads(UF), 1) k_fold_pipe(const FoldArgs a, const FoldPipeLayout lay) {
    constexpr int CG = fold_groups(UF), CW = fold_cwarps(UF), CT = CW * 32;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full_bar[kPipeStagesMax];
    __shared__ __align__(8) uint64_t empty_bar[kPipeStagesMax];
    __shared__ float s_cw[CG][kMaxCap];  // dt_s exp(A (S_T - S_s))
    __shared__ float s_alpha[CG];        // exp(A S_T)
    __shared__ volatile int s_abort;

    const int H = a.s.H, P = a.s.P, N = a.s.N, G = a.s.G, cap = a.s.cap, L = a.s.L;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int S = lay.stages;
    const int ntiles = a.s.batch * H;
    constexpr int es = static_cast<int>(sizeof(TIn));
    const uint32_t tbu = tile_bytes(UF, P, N) + scale_bytes(UF, P, N);  // update copy (+ FP4 scales)
    const bool in_record = a.upd == a.record;

    pdl_prologue();
    if (tid == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(smem_u32(&full_bar[st]), 1);
            mbar_init(smem_u32(&empty_bar[st]), CW);
            reinterpret_cast<int*>(smem + static_cast<size_t>(st) * lay.stage_bytes + lay.meta)[kFMetaTag] = -1;
        }
        s_abort = 0;
    }
    __syncthreads();

    if (warp == CG * CW) {
        // ------------------------------------------------------------ producer
        int p0 = 0, p1 = 0;
        uint32_t f0 = 0, f1 = 0;
        float A0 = 0.f, A1 = 0.f;
        auto fetch = [&](int kbase, int& pp, uint32_t& ff, float& AA) {
            const uint32_t tt = blockIdx.x + static_cast<uint32_t>(kbase + lane) * gridDim.x;
            if (tt < static_cast<uint32_t>(ntiles)) {
                const int bb = fdiv(tt, lay.divH);
                pp = a.pos[bb];
                ff = a.flush_count[bb];
                AA = a.A[tt - bb * H];
            }
        };
        fetch(0, p0, f0, A0);
        fetch(32, p1, f1, A1);
        int q = 0, st = 0, use = 0;  // stage sequence of the due tiles
        int q_issued = -1;
        bool aborted = false;
        // takes the next stage; false when the kernel is aborting
        auto take_stage = [&]() {
            int live = 1;
            if (lane == 0) {
                if (use > 0 && !mbar_wait_bounded(smem_u32(&empty_bar[st]), (use - 1) & 1, kWaitNs)) {
                    set_error(a.err, RSSM_DEVERR_TIMEOUT);
                    s_abort = 1;
                }
                live = !s_abort;
            }
            return __shfl_sync(0xffffffffu, live, 0) != 0;
        };
        auto next_stage = [&]() {
            q_issued = q;
            ++q;
            if (++st == S) {
                st = 0;
                ++use;
            }
        };
        for (int k = 0; blockIdx.x + static_cast<uint32_t>(k) * gridDim.x < static_cast<uint32_t>(ntiles); ++k) {
            const uint32_t t = blockIdx.x + static_cast<uint32_t>(k) * gridDim.x;
            const bool cur = (k >> 5) & 1;
            const int sel = k & 31;
            if (sel == 0 && k > 0) {
                if (cur)
                    fetch(k + 32, p0, f0, A0);
                else
                    fetch(k + 32, p1, f1, A1);
            }
            int pos;
            uint32_t fc;
            float Ah;
            if (cur) {
                pos = __shfl_sync(0xffffffffu, p1, sel);
                fc = __shfl_sync(0xffffffffu, f1, sel);
                Ah = __shfl_sync(0xffffffffu, A1, sel);
            } else {
                pos = __shfl_sync(0xffffffffu, p0, sel);
                fc = __shfl_sync(0xffffffffu, f0, sel);
                Ah = __shfl_sync(0xffffffffu, A0, sel);
            }
            if (pos < 0 || pos > cap) {
                if (lane == 0) set_error(a.err, RSSM_DEVERR_POS_RANGE);
                continue;
            }
            if (!((pos >= L) || (a.mode >= 1 && pos > 0) || (a.mode == 2))) continue;  // not due
            if (!take_stage()) {
                aborted = true;
                break;
            }
            if (lane == 0) {
                unsigned char* sp = smem + static_cast<size_t>(st) * lay.stage_bytes;
                const uint32_t fb = smem_u32(&full_bar[st]);
                int* meta = reinterpret_cast<int*>(sp + lay.meta);
                meta[kFMetaTile] = static_cast<int>(t);
                meta[kFMetaPos] = pos;
                meta[kFMetaFc] = static_cast<int>(fc);
                reinterpret_cast<float*>(meta)[kFMetaA] = Ah;
                reinterpret_cast<volatile int*>(meta)[kFMetaTag] = q;
                const int b = fdiv(t, lay.divH), h = static_cast<int>(t) - b * H;
                const unsigned char* rec = a.record + static_cast<size_t>(t) * a.rec.bytes;
                const uint32_t nx = static_cast<uint32_t>(pos * P * es), nb = static_cast<uint32_t>(pos * N * es);
                const uint32_t ndx = (a.rec.x - a.rec.dt) + nx;  // dt row and x rows, contiguous in the record
                mbar_expect_tx(fb, (in_record ? a.rec.x + nx : tbu + ndx) + nb);
                if (in_record) {
                    bulk_g2s(smem_u32(sp), rec, a.rec.x + nx, fb);
                } else {
                    bulk_g2s(smem_u32(sp), a.upd + static_cast<size_t>(t) * a.upd_stride, tbu, fb);
                    bulk_g2s(smem_u32(sp + lay.st_dt), rec + a.rec.dt, ndx, fb);
                }
                if (nb > 0) {
                    const size_t bg = static_cast<size_t>(b) * G + fdiv(h, lay.divHpg);
                    bulk_g2s(smem_u32(sp + lay.brows),
                             static_cast<const unsigned char*>(a.bbuf) + bg * static_cast<size_t>(cap) * N * es, nb,
                             fb);
                }
            }
            next_stage();
            __syncwarp();
        }
        // one end marker per consumer group
        for (int e = 0; e < CG && !aborted; ++e) {
            if (!take_stage()) {
                aborted = true;
                break;
            }
            if (lane == 0) {
                unsigned char* sp = smem + static_cast<size_t>(st) * lay.stage_bytes;
                int* meta = reinterpret_cast<int*>(sp + lay.meta);
                meta[kFMetaTile] = -1;
                reinterpret_cast<volatile int*>(meta)[kFMetaTag] = q;
                mbar_expect_tx(smem_u32(&full_bar[st]), 0u);
            }
            next_stage();
            __syncwarp();
        }
        if (aborted && lane == 0) {
            for (int qq = q_issued; qq >= 0 && qq > q_issued - S; --qq)
                mbar_wait_bounded(smem_u32(&full_bar[qq % S]), (qq / S) & 1, kWaitNs);
        }
        return;
    }

    // --------------------------------------------------------------- consumers
    const int gi = warp / CW, cw = warp - gi * CW;
    const int ctid = tid - gi * CT;
    const PhiloxKeys pkeys = philox_keys(a.seed);
    float* s_Bf = reinterpret_cast<float*>(smem + static_cast<size_t>(S) * lay.stage_bytes +
                                           static_cast<size_t>(gi) * lay.scratch);  // [T][N]
    float* s_xw = s_Bf + cap * N;                                                    // [T][P]
    const int bq = N / 8, xq = P / 8;  // 8-element chunks per B row / x row
    int st = gi, use = 0;
    while (st >= S) {
        st -= S;
        ++use;
    }
    int pend_b = -1;
    uint32_t pend_old = 0;
    for (int q = gi;; q += CG) {
        const unsigned char* sp = smem + static_cast<size_t>(st) * lay.stage_bytes;
        const int* meta = reinterpret_cast<const int*>(sp + lay.meta);
        int stop = 0;
        if (ctid == 0) {
            stop = s_abort;
            const volatile int* tag = reinterpret_cast<const volatile int*>(meta) + kFMetaTag;
            if (!stop && !smem_wait_eq_bounded(tag, q, kWaitNs)) {
                set_error(a.err, RSSM_DEVERR_TIMEOUT);
                s_abort = 1;
                stop = 1;
            }
            if (!stop && !mbar_wait_bounded(smem_u32(&full_bar[st]), use & 1, kWaitNs)) {
                set_error(a.err, RSSM_DEVERR_TIMEOUT);
                s_abort = 1;
                stop = 1;
                mbar_wait_bounded(smem_u32(&full_bar[st]), use & 1, kWaitNs);
            }
        }
        if (group_sync_or(gi, CT, stop)) break;
        const int t = meta[kFMetaTile];
        if (t < 0) {  // end of this group's sequence: hand the stage back and stop
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&empty_bar[st]));
            break;
        }
        const int T = meta[kFMetaPos];
        const uint32_t fc = static_cast<uint32_t>(meta[kFMetaFc]);
        const float Ah = reinterpret_cast<const float*>(meta)[kFMetaA];
        const int b = fdiv(static_cast<uint32_t>(t), lay.divH), h = t - b * H;
        const TIn* xr = reinterpret_cast<const TIn*>(sp + lay.st_x);
        const TIn* br = reinterpret_cast<const TIn*>(sp + lay.brows);
        if (cw == CW - 1) {
            const float dts = (lane < T) ? reinterpret_cast<const float*>(sp + lay.st_dt)[lane] : 0.f;
            const float Sx = warp_prefix(dts);
            const float Stot = T > 0 ? __shfl_sync(0xffffffffu, Sx, T - 1) : 0.f;
            s_cw[gi][lane] = (lane < T) ? dts * expf(Ah * (Stot - Sx)) : 0.f;
            if (lane == 0) s_alpha[gi] = expf(Ah * Stot);
            if (lane == 0) {
                // every CTA read pos[b] before processing b's tiles; the last arrival resets it
                if (pend_b >= 0 && pend_old == static_cast<uint32_t>(H - 1)) {
                    a.arrive[pend_b] = 0u;
                    a.pos[pend_b] = 0;
                    a.flush_count[pend_b] += 1u;
                }
                pend_b = b;
                pend_old = atomicAdd(&a.arrive[b], 1u);
            }
        } else {
            // B rows to fp32
            for (int c = ctid; c < T * bq; c += (CW - 1) * 32) {
                Raw8<TIn> r;
                r.load(br + c * 8);
                reinterpret_cast<float4*>(s_Bf)[2 * c] = r.lo();
                reinterpret_cast<float4*>(s_Bf)[2 * c + 1] = r.hi();
            }
        }
        group_sync(gi, CT);  // weights and B ready
        const float alpha = s_alpha[gi];
        for (int c = ctid; c < T * xq; c += CT) {
            const int sl = c / xq;
            const float w = s_cw[gi][sl];
            Raw8<TIn> r;
            r.load(xr + c * 8);
            const float4 lo = r.lo(), hi = r.hi();
            reinterpret_cast<float4*>(s_xw)[2 * c] = make_float4(w * lo.x, w * lo.y, w * lo.z, w * lo.w);
            reinterpret_cast<float4*>(s_xw)[2 * c + 1] = make_float4(w * hi.x, w * hi.y, w * hi.z, w * hi.w);
        }
        group_sync(gi, CT);  // w_s x_s ready
        const unsigned char* tile = sp;
        const unsigned char* tsc = sp + (in_record ? a.rec.scales : align16(tile_bytes(UF, P, N)));
        unsigned char* upd = a.upd + static_cast<size_t>(t) * a.upd_stride;
        unsigned char* rec = a.record + static_cast<size_t>(t) * a.rec.bytes;
        for (int r0 = cw * kRB; r0 < P; r0 += CW * kRB) {
            // acc = alpha h, then the slots in order (the one-CTA fold's order),
            // rows paired for the packed FMAs
            float2 acc2[4][4];
#pragma unroll
            for (int kk = 0; kk < kRB; ++kk) {
                const float4 hv = tile_load4<UF>(tile, tsc, r0 + kk, lane, N);
                acc2_set_row(acc2, kk, make_float4(alpha * hv.x, alpha * hv.y, alpha * hv.z, alpha * hv.w));
            }
#pragma unroll 2
            for (int sl = 0; sl < T; ++sl) {
                const float4 bv = reinterpret_cast<const float4*>(s_Bf + sl * N)[lane];
                const float4* xw4 = reinterpret_cast<const float4*>(s_xw + sl * P + r0);
                const float4 xa = xw4[0], xb = xw4[1];
                const float2 w2[4] = {make_float2(xa.x, xa.y), make_float2(xa.z, xa.w), make_float2(xb.x, xb.y),
                                      make_float2(xb.z, xb.w)};
                rank1_8x4(acc2, w2, bv);
            }
#pragma unroll
            for (int kk = 0; kk < kRB; ++kk) {
                const int r = r0 + kk;
                const float4 v = acc2_row(acc2, kk);
                const uint32_t e = static_cast<uint32_t>(r * N + 4 * lane);  // element of v.x within the head
                if constexpr (UF == kF32) {
                    stream_store4(reinterpret_cast<float*>(upd) + e, v);
                } else if constexpr (UF == kBF16 || UF == kE4M3) {
                    const uint4 rw = philox4x32_10(make_uint4(e >> 2, h, b, fc), pkeys);
                    if constexpr (UF == kBF16) {
                        const uint2 wv = make_uint2(sr_bf16x2(v.x, v.y, rw.x, rw.y), sr_bf16x2(v.z, v.w, rw.z, rw.w));
                        *reinterpret_cast<uint2*>(upd + 2u * e) = wv;
                    } else {
                        const uint32_t wv = sr_e4m3(v.x, rw.x) | (sr_e4m3(v.y, rw.y) << 8) |
                                            (sr_e4m3(v.z, rw.z) << 16) | (sr_e4m3(v.w, rw.w) << 24);
                        *reinterpret_cast<uint32_t*>(upd + e) = wv;
                    }
                } else {
                    uint32_t scv;
                    const uint32_t codes = fp4_quant_quad(v, &scv);
                    *reinterpret_cast<uint16_t*>(upd + e / 2) = static_cast<uint16_t>(codes);
                    if ((lane & 3) == 0) upd[a.rec.scales + e / 16] = static_cast<uint8_t>(scv);
                }
                if constexpr (OUT4 != 0) {
                    uint32_t scv;
                    const uint32_t codes = fp4_quant_quad(v, &scv);
                    *reinterpret_cast<uint16_t*>(rec + e / 2) = static_cast<uint16_t>(codes);
                    if ((lane & 3) == 0) rec[a.rec.scales + e / 16] = static_cast<uint8_t>(scv);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty_bar[st]));
        st += CG;
        while (st >= S) {
            st -= S;
            ++use;
        }
    }
    if (cw == CW - 1 && lane == 0 && pend_b >= 0 && pend_old == static_cast<uint32_t>(H - 1)) {
        a.arrive[pend_b] = 0u;  // the last pending arrival of this group
        a.pos[pend_b] = 0;
        a.flush_count[pend_b] += 1u;
    }
}

// ---------------------------------------------------------------------------
// Prefill: the prompt folded into the fp32 checkpoint, kPrefillChunk tokens
// at a time, with the fold of s1 (an interval flush of each chunk). One CTA
// per tile keeps the tile in shared memory across chunks: per chunk the B
// rows (fp32), the x rows and the weights dt_s exp(A (S_chunk - S_s)) are
// staged, then the register-blocked rank-T update writes the tile back (the
// last chunk writes the record).
// ---------------------------------------------------------------------------
constexpr int kPrefillChunk = 16;

template <typename TIn>
__global__ void __launch_bounds__(kThreads, 2) k_prefill(const PrefillArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bar;
    __shared__ float s_cw[kPrefillChunk];
    __shared__ float s_alpha;
    __shared__ int s_pos;

    const int H = a.s.H, P = a.s.P, N = a.s.N, G = a.s.G, lpr = a.s.lpr, batch = a.s.batch;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x / H, h = blockIdx.x - b * H;
    const int g = h / (H / G);
    const int xs = round_up8(P);
    const size_t bh = static_cast<size_t>(b) * H + h;
    float* s32 = reinterpret_cast<float*>(smem);  // [P][N]
    float* s_B = s32 + P * N;                      // [chunk][N]
    float* s_x = s_B + kPrefillChunk * N;          // [chunk][xs]
    unsigned char* rec = a.record + bh * a.rec.bytes;
    const uint32_t tb = 4u * static_cast<uint32_t>(P * N);
    const uint32_t bar_a = smem_u32(&bar);

    if (tid == 0) {
        const int p0 = a.pos[b];  // the only read of pos
        s_pos = p0;
        if (p0 == 0 && a.T0 > 0) {
            mbar_init(bar_a, 1);
            mbar_expect_tx(bar_a, tb);
            bulk_g2s(smem_u32(s32), rec, tb, bar_a);
        }
    }
    __syncthreads();
    if (s_pos != 0) {
        if (tid == 0) set_error(a.err, RSSM_DEVERR_POS_RANGE);
        return;
    }
    if (a.T0 <= 0) return;
    bool arrived = true;
    if (tid == 0) arrived = mbar_wait_bounded(bar_a, 0, kWaitNs);
    if (__syncthreads_or(!arrived)) {
        if (tid == 0) {
            set_error(a.err, RSSM_DEVERR_TIMEOUT);
            mbar_wait_bounded(bar_a, 0, kWaitNs);
        }
        return;
    }
    const float Ah = a.A[h];
    const size_t HP = static_cast<size_t>(H) * P, GN = static_cast<size_t>(G) * N;
    const TIn* xin = static_cast<const TIn*>(a.x) + static_cast<size_t>(b) * HP + static_cast<size_t>(h) * P;
    const TIn* Bin = static_cast<const TIn*>(a.B) + static_cast<size_t>(b) * GN + static_cast<size_t>(g) * N;
    const size_t xstep = static_cast<size_t>(batch) * HP, bstep = static_cast<size_t>(batch) * GN;
    const int n8 = N >> 3;
    for (int t0 = 0; t0 < a.T0; t0 += kPrefillChunk) {
        const int T = a.T0 - t0 < kPrefillChunk ? a.T0 - t0 : kPrefillChunk;
        for (int q = tid; q < T * n8; q += kThreads) {
            const int sl = q / n8, c8 = (q - sl * n8) << 3;
            Raw8<TIn> r;
            r.load(Bin + static_cast<size_t>(t0 + sl) * bstep + c8);
            float4* d = reinterpret_cast<float4*>(s_B + sl * N + c8);
            d[0] = r.lo();
            d[1] = r.hi();
        }
        for (int i = tid; i < T * P; i += kThreads) {
            const int sl = i / P, p = i - sl * P;
            s_x[sl * xs + p] = to_f32(xin[static_cast<size_t>(t0 + sl) * xstep + p]);
        }
        if (warp == 0) {
            const float dts = (lane < T) ? a.dt[(static_cast<size_t>(t0 + lane) * batch + b) * H + h] : 0.f;
            const float Sx = warp_prefix(dts);
            const float Stot = __shfl_sync(0xffffffffu, Sx, T - 1);
            if (lane < kPrefillChunk) s_cw[lane] = (lane < T) ? dts * expf(Ah * (Stot - Sx)) : 0.f;
            if (lane == 0) s_alpha = expf(Ah * Stot);
        }
        __syncthreads();  // chunk staged; the previous chunk's tile writes are visible
        const bool last = t0 + kPrefillChunk >= a.T0;
        auto brow = [&](int sl, int c) {
            const float w = s_cw[sl];
            const float4 v = reinterpret_cast<const float4*>(s_B + sl * N)[c];
            return make_float4(w * v.x, w * v.y, w * v.z, w * v.w);
        };
        auto emit = [&](int r, int c, float4 v, bool valid) {
            if (!valid) return;
            if (last)
                stream_store4(reinterpret_cast<float*>(rec) + r * N + 4 * c, v);
            else
                reinterpret_cast<float4*>(s32)[r * (N >> 2) + c] = v;
        };
        fold_tile(s32, s_x, xs, P, N, lpr, T, s_alpha, brow, emit);
        __syncthreads();  // every reader of this chunk's staging is done
    }
}

// ---------------------------------------------------------------------------
// Prefill on the tensor cores (bf16 inputs, d_state 128, head_dim a multiple
// of 16 up to 64). The fold of a whole prompt is one contraction per
// (request, head):
//   h_T = exp(A S) h_0 + sum_{t < T0} w_t x_t B_t^T,   w_t = dt_t exp(A R_t),
//   R_t = sum_{t < r < T0} dt_r (the decay from token t to the end), S = R_{-1},
// i.e. h_T - exp(A S) h_0 = X_w^T B with X_w[t][p] = w_t x_t[p] (K = T0).
// One CTA of 8 warps per tile walks the prompt in chunks of 64 tokens from
// the last to the first, so R_t is a running suffix sum (no cancellation).
// Per chunk: the x rows, B rows and dt land by cp.async (double-buffered,
// the next chunk while this one computes); every warp forms the chunk's w_t
// itself (the same arithmetic in each, so no barrier waits on it); all threads
// split w_t x_t[p] into bf16 hi + mid + lo parts (x_w to ~2^-27; B is bf16,
// exact; a two-part split, ~2^-17, left the checkpoint of a 512-token prompt
// 1.5e-4 of its rms from the recurrence); warp w accumulates rows 16 (w % 4)..
// of the product against the
// 64 columns 64 (w / 4).. with mma.sync bf16 m16n8k16, operands from shared
// memory by ldmatrix (rows XOR-swizzled by 16-byte chunk, conflict-free).
// ---------------------------------------------------------------------------
constexpr int kPfChunk = 64;                                 // prompt tokens per chunk
constexpr int kPfThreads = 256;
constexpr uint32_t kPfX = kPfChunk * 64 * 2;                 // x rows [64][64] bf16
constexpr uint32_t kPfB = kPfChunk * kD128 * 2;              // B rows [64][128] bf16 (swizzled)
constexpr uint32_t kPfBuf = kPfX + kPfB + kPfChunk * 4;      // + dt [64]
constexpr uint32_t kPfA = kPfChunk * 64 * 2;                 // x_w hi, mid or lo [64 tokens][64 rows] (swizzled)
constexpr size_t kPfSmem = 2 * static_cast<size_t>(kPfBuf) + 3 * kPfA;

__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16u : 0u)
                 : "memory");
}
__device__ __forceinline__ void cp_async4_zfill(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4u : 0u)
                 : "memory");
}

__global__ void __launch_bounds__(kPfThreads, 3) k_prefill_mma(const PrefillArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int s_pos;
    const int H = a.s.H, P = a.s.P, G = a.s.G, batch = a.s.batch, T0 = a.T0;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x / H, h = blockIdx.x - b * H, g = h / (H / G);
    unsigned char* rec = a.record + (static_cast<size_t>(b) * H + h) * a.rec.bytes;
    unsigned char* aw_hi = smem + 2 * kPfBuf;
    unsigned char* aw_md = aw_hi + kPfA;
    unsigned char* aw_lo = aw_md + kPfA;

    if (tid == 0) s_pos = a.pos[b];  // the only read of pos
    __syncthreads();
    if (s_pos != 0) {
        if (tid == 0) set_error(a.err, RSSM_DEVERR_POS_RANGE);
        return;
    }
    if (T0 <= 0) return;
    const size_t HP = static_cast<size_t>(H) * P, GN = static_cast<size_t>(G) * kD128;
    const __nv_bfloat16* xin = static_cast<const __nv_bfloat16*>(a.x) + static_cast<size_t>(b) * HP +
                               static_cast<size_t>(h) * P;
    const __nv_bfloat16* Bin = static_cast<const __nv_bfloat16*>(a.B) + static_cast<size_t>(b) * GN +
                               static_cast<size_t>(g) * kD128;
    const size_t xstep = static_cast<size_t>(batch) * HP, bstep = static_cast<size_t>(batch) * GN;
    const int nchunk = (T0 + kPfChunk - 1) / kPfChunk;

    // chunk c (tokens 64c ..) into buffer `buf`: x rows (P bf16), B rows
    // (chunk j of token k at (j ^ (k & 7))), dt; zeros past T0
    auto fetch = [&](int c, int buf) {
        unsigned char* base = smem + static_cast<size_t>(buf) * kPfBuf;
        const int t0 = c * kPfChunk;
        const int xq = P / 8;  // 16-byte chunks per x row
        for (int i = tid; i < kPfChunk * 16; i += kPfThreads) {  // B: 16 chunks per token
            const int k = i >> 4, j = i & 15, t = t0 + k;
            const bool ok = t < T0;
            cp_async16_zfill(smem_u32(base + kPfX + k * (kD128 * 2) + 16 * (j ^ (k & 7))),
                             Bin + static_cast<size_t>(ok ? t : t0) * bstep + 8 * j, ok);
        }
        for (int i = tid; i < kPfChunk * xq; i += kPfThreads) {
            const int k = i / xq, j = i - k * xq, t = t0 + k;
            const bool ok = t < T0;
            cp_async16_zfill(smem_u32(base + k * 128 + 16 * j), xin + static_cast<size_t>(ok ? t : t0) * xstep + 8 * j,
                             ok);
        }
        if (tid < kPfChunk) {
            const int t = t0 + tid;
            const bool ok = t < T0;
            cp_async4_zfill(smem_u32(base + kPfX + kPfB + 4 * tid),
                            a.dt + (static_cast<size_t>(ok ? t : t0) * batch + b) * H + h, ok);
        }
        cp_async_commit();
    };

    const float Ah = a.A[h];
    float carry = 0.f;  // sum of dt over the chunks already folded (warp 0)
    const int mt = warp & 3, nh = warp >> 2;
    const int R0 = 16 * mt;
    const bool rows_live = R0 < P;
    float acc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

    fetch(nchunk - 1, (nchunk - 1) & 1);
    for (int c = nchunk - 1; c >= 0; --c) {
        const int buf = c & 1;
        unsigned char* base = smem + static_cast<size_t>(buf) * kPfBuf;
        cp_async_wait_all();
        __syncthreads();  // chunk c landed; the previous chunk's readers are done
        if (c > 0) fetch(c - 1, buf ^ 1);
        {
            // w_t = dt_t exp(A R_t), formed by every warp alike (no barrier):
            // lane l takes tokens l and l + 32 of the chunk
            const float* dts = reinterpret_cast<const float*>(base + kPfX + kPfB);
            const float v0 = dts[lane], v1 = dts[lane + 32];
            float s0 = v0, s1 = v1;  // inclusive suffix sums within each half
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float u0 = __shfl_down_sync(0xffffffffu, s0, off);
                const float u1 = __shfl_down_sync(0xffffffffu, s1, off);
                if (lane + off < 32) {
                    s0 += u0;
                    s1 += u1;
                }
            }
            const float tot1 = __shfl_sync(0xffffffffu, s1, 0), tot0 = __shfl_sync(0xffffffffu, s0, 0);
            // R_t = (later chunks) + (later tokens of this chunk), exclusive of t
            const float w1 = v1 * expf(Ah * (carry + (s1 - v1)));
            const float w0 = v0 * expf(Ah * ((carry + tot1) + (s0 - v0)));
            carry = (carry + tot1) + tot0;
            // x_w = w_t x_t[p] as bf16 hi + mid + lo: thread -> token tid / 4, rows 16 (tid % 4) ..
            const int k = tid >> 2, p0 = 16 * (tid & 3);
            const float wa = __shfl_sync(0xffffffffu, w0, k & 31), wb = __shfl_sync(0xffffffffu, w1, k & 31);
            const float w = k < 32 ? wa : wb;  // uniform over the warp
            uint32_t hi[8], md[8], lo[8];
            if (p0 < P) {
                const uint4 u0 = *reinterpret_cast<const uint4*>(base + k * 128 + 2 * p0);
                const uint4 u1 = *reinterpret_cast<const uint4*>(base + k * 128 + 2 * p0 + 16);
                const uint32_t xw[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float f0 = w * __uint_as_float(bf16lo_bits(xw[q]));
                    const float f1 = w * __uint_as_float(bf16hi_bits(xw[q]));
                    const uint32_t hh = f32x2_to_bf16x2(f0, f1);
                    hi[q] = hh;
                    // the residuals below hi, then below mid, are exact in fp32
                    const float r0 = f0 - __uint_as_float(bf16lo_bits(hh)), r1 = f1 - __uint_as_float(bf16hi_bits(hh));
                    const uint32_t mm = f32x2_to_bf16x2(r0, r1);
                    md[q] = mm;
                    lo[q] = f32x2_to_bf16x2(r0 - __uint_as_float(bf16lo_bits(mm)), r1 - __uint_as_float(bf16hi_bits(mm)));
                }
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) hi[q] = md[q] = lo[q] = 0u;
            }
            const int c0 = p0 >> 3;  // 16-byte chunk of the row
            uint4* dh0 = reinterpret_cast<uint4*>(aw_hi + k * 128 + 16 * (c0 ^ (k & 7)));
            uint4* dh1 = reinterpret_cast<uint4*>(aw_hi + k * 128 + 16 * ((c0 + 1) ^ (k & 7)));
            uint4* dm0 = reinterpret_cast<uint4*>(aw_md + k * 128 + 16 * (c0 ^ (k & 7)));
            uint4* dm1 = reinterpret_cast<uint4*>(aw_md + k * 128 + 16 * ((c0 + 1) ^ (k & 7)));
            uint4* dl0 = reinterpret_cast<uint4*>(aw_lo + k * 128 + 16 * (c0 ^ (k & 7)));
            uint4* dl1 = reinterpret_cast<uint4*>(aw_lo + k * 128 + 16 * ((c0 + 1) ^ (k & 7)));
            *dh0 = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *dh1 = make_uint4(hi[4], hi[5], hi[6], hi[7]);
            *dm0 = make_uint4(md[0], md[1], md[2], md[3]);
            *dm1 = make_uint4(md[4], md[5], md[6], md[7]);
            *dl0 = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            *dl1 = make_uint4(lo[4], lo[5], lo[6], lo[7]);
        }
        __syncthreads();  // x_w ready
        if (rows_live) {
            const int j = lane >> 3, r = lane & 7;
#pragma unroll
            for (int ks = 0; ks < kPfChunk / 16; ++ks) {
                // A (rows R0.., tokens 16 ks..): matrix j = (rows 8 (j & 1).., tokens 8 (j >> 1)..)
                const int ka = 16 * ks + r + 8 * (j >> 1), pc = (R0 >> 3) + (j & 1);
                uint32_t ah[4], am[4], al[4];
                ldsm_x4_trans(smem_u32(aw_hi + ka * 128 + 16 * (pc ^ (ka & 7))), ah[0], ah[1], ah[2], ah[3]);
                ldsm_x4_trans(smem_u32(aw_md + ka * 128 + 16 * (pc ^ (ka & 7))), am[0], am[1], am[2], am[3]);
                ldsm_x4_trans(smem_u32(aw_lo + ka * 128 + 16 * (pc ^ (ka & 7))), al[0], al[1], al[2], al[3]);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    // B of n-tiles 8 nh + 2q, + 1: matrix j = (tokens 8 (j & 1).., n-tile 2q + (j >> 1))
                    const int kb = 16 * ks + r + 8 * (j & 1), ncn = 8 * nh + 2 * q + (j >> 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_trans(smem_u32(base + kPfX + kb * (kD128 * 2) + 16 * (ncn ^ (kb & 7))), b0, b1, b2, b3);
                    mma_bf16(acc[2 * q], ah[0], ah[1], ah[2], ah[3], b0, b1);
                    mma_bf16(acc[2 * q], am[0], am[1], am[2], am[3], b0, b1);
                    mma_bf16(acc[2 * q], al[0], al[1], al[2], al[3], b0, b1);
                    mma_bf16(acc[2 * q + 1], ah[0], ah[1], ah[2], ah[3], b2, b3);
                    mma_bf16(acc[2 * q + 1], am[0], am[1], am[2], am[3], b2, b3);
                    mma_bf16(acc[2 * q + 1], al[0], al[1], al[2], al[3], b2, b3);
                }
            }
        }
    }
    // h_T = exp(A S) h_0 + acc, S = the prompt's dt sum (each warp's carry)
    const float alpha = expf(Ah * carry);
    if (rows_live) {
        const int gq = lane >> 2, tq = lane & 3;
        float* hrow = reinterpret_cast<float*>(rec);
#pragma unroll
        for (int jn = 0; jn < 8; ++jn) {
            const int n = 64 * nh + 8 * jn + 2 * tq;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int r = R0 + gq + 8 * half;
                float2* pp = reinterpret_cast<float2*>(hrow + static_cast<size_t>(r) * kD128 + n);
                const float2 h0 = *pp;
                *pp = make_float2(fmaf(alpha, h0.x, acc[jn][2 * half]), fmaf(alpha, h0.y, acc[jn][2 * half + 1]));
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Prefill on the 5th-generation tensor cores (tcgen05; bf16 inputs, d_state
// 128, head_dim 64, an even number of heads per group). The same
// contraction as k_prefill_mma, h_T - exp(A S) h_0 = X_w^T B, for two heads
// of one group at once: the 128-row operand stacks their X_w (rows 0..63 the
// first head's head_dim, 64..127 the second's) and both use the group's B.
// One CTA of 8 warps per (request, head pair) walks the prompt in chunks of
// 32 tokens from the last to the first (R_t a running suffix sum):
//  - cp.async brings the chunk's B rows straight into the MMA's B operand
//    layout, the two heads' x rows and dt (double-buffered);
//  - warps 0-3 form the first head's w_t, warps 4-7 the second's (each warp
//    alike, no barrier), and every thread splits w_t x_t[p] into bf16
//    hi + mid + lo (x_w to ~2^-27) into the A operand;
//  - one thread issues tcgen05.mma (M128 N128 K16, bf16 x bf16 -> fp32, A and
//    B MN-major in 128-byte-swizzled atoms of 8 rows) into a 128-column fp32
//    accumulator in tensor memory, 2 K-steps x 3 parts per chunk, and
//    tcgen05.commit signals an mbarrier when they have read their operands;
//  - after the last chunk each warp reads its 32 accumulator rows x 64
//    columns with tcgen05.ld, adds exp(A S) h_0 and writes the checkpoint.
// Tensor memory is allocated after the request's position check and freed on
// every path that allocated it; every wait is bounded.
// ---------------------------------------------------------------------------
constexpr int kUmChunk = 32;                                          // prompt tokens per chunk
constexpr int kUmThreads = 256;
constexpr uint32_t kUmB = 2u * kUmChunk * 128u;                       // B operand: 2 column blocks x chunk x 128 B
constexpr uint32_t kUmX = 2u * kUmChunk * 128u;                       // x rows: 2 heads x chunk x 64 bf16
constexpr uint32_t kUmBuf = (kUmB + kUmX + 2u * kUmChunk * 4u + 1023u) & ~1023u;  // + dt [2 heads][chunk]; atom-aligned
constexpr uint32_t kUmA = 2u * kUmChunk * 128u;                       // one A part: 2 heads x chunk x 128 B
constexpr size_t kUmSmem = 1024 + 2 * static_cast<size_t>(kUmBuf) + 3 * static_cast<size_t>(kUmA);
constexpr uint32_t kUmCols = 128;                                     // tensor-memory columns (fp32 D, N = 128)

// Shared-memory matrix descriptor of a 128-byte-swizzled operand (start
// address, leading and stride byte offsets in 16-byte units, descriptor
// version 1, layout type 2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: fp32 accumulator, bf16 A and B, both MN-major,
// N = 128 (n_dim = N / 8), M = 128 (m_dim = M / 16).
constexpr uint32_t kUmIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) | ((128u >> 3) << 17) |
                              ((128u >> 4) << 24);

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(kUmIdesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// 16 consecutive fp32 columns of this thread's accumulator row (lane quadrant of the warp).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__global__ void __launch_bounds__(kUmThreads, 3) k_prefill_umma(const PrefillArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t mma_bar;
    __shared__ uint32_t s_tmem;
    __shared__ float s_alpha[2];
    __shared__ int s_pos;
    const int H = a.s.H, G = a.s.G, batch = a.s.batch, T0 = a.T0;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int pairs = H >> 1;
    const int b = blockIdx.x / pairs, h0 = 2 * (blockIdx.x - b * pairs), g = h0 / (H / G);
    // operand buffers on a 1024-byte boundary (the swizzle atoms)
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (sbase - smem_u32(smem_raw));
    const uint32_t s_a = sbase + 2 * kUmBuf;  // A parts: hi, mid, lo, kUmA bytes each

    if (tid == 0) s_pos = a.pos[b];  // the only read of pos
    __syncthreads();
    if (s_pos != 0) {
        if (tid == 0) set_error(a.err, RSSM_DEVERR_POS_RANGE);
        return;
    }
    if (T0 <= 0) return;
    if (warp == 0) {  // tensor memory for the accumulator (one warp allocates and frees)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(kUmCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) mbar_init(smem_u32(&mma_bar), 1);
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = s_tmem;

    const size_t HP = static_cast<size_t>(H) * 64, GN = static_cast<size_t>(G) * kD128;
    const __nv_bfloat16* xin = static_cast<const __nv_bfloat16*>(a.x) + static_cast<size_t>(b) * HP + h0 * 64;
    const __nv_bfloat16* Bin = static_cast<const __nv_bfloat16*>(a.B) + static_cast<size_t>(b) * GN +
                               static_cast<size_t>(g) * kD128;
    const size_t xstep = static_cast<size_t>(batch) * HP, bstep = static_cast<size_t>(batch) * GN;
    const int nchunk = (T0 + kUmChunk - 1) / kUmChunk;

    // chunk c (tokens 32c ..) into buffer `buf`: B rows in the operand layout
    // (column block n / 64, token row k, 16-byte chunk (n % 64) / 8 ^ (k & 7)),
    // the two heads' x rows [head][k][64], dt [head][k]; zeros past T0
    auto fetch = [&](int c, int buf) {
        const uint32_t base = sbase + static_cast<uint32_t>(buf) * kUmBuf;
        const int t0 = c * kUmChunk;
        for (int i = tid; i < kUmChunk * 16; i += kUmThreads) {
            const int k = i >> 4, j = i & 15, t = t0 + k;
            const bool ok = t < T0;
            const uint32_t dst = base + (j >> 3) * (kUmChunk * 128) + k * 128 + 16 * ((j & 7) ^ (k & 7));
            cp_async16_zfill(dst, Bin + static_cast<size_t>(ok ? t : t0) * bstep + 8 * j, ok);
        }
        for (int i = tid; i < kUmChunk * 16; i += kUmThreads) {
            const int k = i >> 4, j = i & 15, t = t0 + k;  // j: head j / 8, 16-byte chunk j % 8 of its row
            const bool ok = t < T0;
            const uint32_t dst = base + kUmB + (j >> 3) * (kUmChunk * 128) + k * 128 + 16 * ((j & 7) ^ (k & 7));
            cp_async16_zfill(dst, xin + static_cast<size_t>(ok ? t : t0) * xstep + 8 * j, ok);
        }
        if (tid < 2 * kUmChunk) {
            const int hh = tid / kUmChunk, k = tid % kUmChunk, t = t0 + k;
            const bool ok = t < T0;
            cp_async4_zfill(base + kUmB + kUmX + 4 * (hh * kUmChunk + k),
                            a.dt + (static_cast<size_t>(ok ? t : t0) * batch + b) * H + h0 + hh, ok);
        }
        cp_async_commit();
    };

    const int wh = warp >> 2;  // the head whose weights this warp forms
    const float Ah = a.A[h0 + wh];
    float carry = 0.f;  // dt sum of the chunks already folded (this warp's head)
    bool timed_out = false;

    fetch(nchunk - 1, (nchunk - 1) & 1);
    for (int c = nchunk - 1, i = 0; c >= 0; --c, ++i) {
        const int buf = c & 1;
        const uint32_t base = sbase + static_cast<uint32_t>(buf) * kUmBuf;
        const unsigned char* gbase = smem + static_cast<size_t>(buf) * kUmBuf;
        cp_async_wait_all();
        // the previous chunk's MMAs have read the A parts and their B buffer
        if (i > 0 && !mbar_wait_bounded(smem_u32(&mma_bar), (i - 1) & 1, kWaitNs)) timed_out = true;
        __syncthreads();  // chunk c landed for every thread; the buffers above are free
        if (c > 0) fetch(c - 1, buf ^ 1);
        // w_t = dt_t exp(A R_t) of this warp's head: lane l takes token l
        const float* dts = reinterpret_cast<const float*>(gbase + kUmB + kUmX) + wh * kUmChunk;
        const float v = dts[lane];
        float s = v;  // inclusive suffix sum
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float u = __shfl_down_sync(0xffffffffu, s, off);
            if (lane + off < 32) s += u;
        }
        const float tot = __shfl_sync(0xffffffffu, s, 0);
        const float wl = v * expf(Ah * (carry + (s - v)));
        carry += tot;
        {
            // x_w = w_t x_t[p] as bf16 hi + mid + lo: thread -> head tid / 128,
            // token (tid % 128) / 4, rows 16 (tid % 4) .. + 15
            const int hh = tid >> 7, k = (tid & 127) >> 2, p0 = 16 * (tid & 3);
            const float w = __shfl_sync(0xffffffffu, wl, k);  // warps of head hh hold its weights
            // (x rows are staged with 16-byte chunk (p / 8) ^ (k & 7), conflict-free here)
            const unsigned char* xrow = gbase + kUmB + hh * (kUmChunk * 128) + k * 128;
            const uint4 u0 = *reinterpret_cast<const uint4*>(xrow + 16 * ((p0 >> 3) ^ (k & 7)));
            const uint4 u1 = *reinterpret_cast<const uint4*>(xrow + 16 * (((p0 >> 3) + 1) ^ (k & 7)));
            const uint32_t xw[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            uint32_t hi[8], md[8], lo[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float f0 = w * __uint_as_float(bf16lo_bits(xw[q]));
                const float f1 = w * __uint_as_float(bf16hi_bits(xw[q]));
                const uint32_t hh2 = f32x2_to_bf16x2(f0, f1);
                hi[q] = hh2;
                const float r0 = f0 - __uint_as_float(bf16lo_bits(hh2)), r1 = f1 - __uint_as_float(bf16hi_bits(hh2));
                const uint32_t mm = f32x2_to_bf16x2(r0, r1);
                md[q] = mm;
                lo[q] = f32x2_to_bf16x2(r0 - __uint_as_float(bf16lo_bits(mm)), r1 - __uint_as_float(bf16hi_bits(mm)));
            }
            // A part layout: [head][token k][128 B], 16-byte chunk (p / 8) ^ (k & 7)
            const int c0 = p0 >> 3;
            const uint32_t row = static_cast<uint32_t>(hh * (kUmChunk * 128) + k * 128);
            const uint32_t d0 = row + 16 * (c0 ^ (k & 7)), d1 = row + 16 * ((c0 + 1) ^ (k & 7));
            unsigned char* ap = smem + (s_a - sbase);
            *reinterpret_cast<uint4*>(ap + d0) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(ap + d1) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
            *reinterpret_cast<uint4*>(ap + kUmA + d0) = make_uint4(md[0], md[1], md[2], md[3]);
            *reinterpret_cast<uint4*>(ap + kUmA + d1) = make_uint4(md[4], md[5], md[6], md[7]);
            *reinterpret_cast<uint4*>(ap + 2 * kUmA + d0) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            *reinterpret_cast<uint4*>(ap + 2 * kUmA + d1) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
        }
        // the operands written by ordinary stores and cp.async, visible to the tensor cores
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        if (tid == 0) {
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
            for (int ks = 0; ks < kUmChunk / 16; ++ks) {
                // K-step: 16 tokens = two 8-row atoms (SBO 1024 B); A: head blocks
                // 64 rows apart in M (LBO = chunk x 128 B); B: column blocks of 64
#pragma unroll
                for (int part = 0; part < 3; ++part) {
                    const uint64_t ad = umma_desc_sw128(s_a + part * kUmA + ks * 2048, kUmChunk * 128, 1024);
                    const uint64_t bd = umma_desc_sw128(base + ks * 2048, kUmChunk * 128, 1024);
                    umma_f16(tmem, ad, bd, (i > 0 || ks > 0 || part > 0) ? 1u : 0u);
                }
            }
            umma_commit(smem_u32(&mma_bar));
        }
    }
    // the last chunk's products complete
    if (!mbar_wait_bounded(smem_u32(&mma_bar), (nchunk - 1) & 1, kWaitNs)) timed_out = true;
    if (lane == 0 && (warp == 0 || warp == 4)) s_alpha[wh] = expf(Ah * carry);
    if (timed_out) set_error(a.err, RSSM_DEVERR_TIMEOUT);
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    {
        // warp w reads accumulator lanes 32 (w % 4) .. (rows = head_dim rows of
        // head (w % 4) / 2) and columns 64 (w / 4) ..
        const int q = warp & 3, half = warp >> 2;
        const int r = 32 * q + lane, hh = r >> 6, p = r & 63;
        const float alpha = s_alpha[hh];
        float* hrow = reinterpret_cast<float*>(a.record + (static_cast<size_t>(b) * H + h0 + hh) * a.rec.bytes) +
                      static_cast<size_t>(p) * kD128;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            const int col = 64 * half + 16 * cc;
            float d[16];
            tmem_ld16(tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(col), d);
            float4* hp = reinterpret_cast<float4*>(hrow + col);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
                const float4 h = hp[v4];
                hp[v4] = make_float4(fmaf(alpha, h.x, d[4 * v4]), fmaf(alpha, h.y, d[4 * v4 + 1]),
                                     fmaf(alpha, h.z, d[4 * v4 + 2]), fmaf(alpha, h.w, d[4 * v4 + 3]));
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kUmCols) : "memory");
    }
}

// ---------------------------------------------------------------------------
// Low-precision refresh with the fold on the 5th-generation tensor cores
// (bf16 inputs, d_state 128, head_dim 64, an even number of heads per
// group). The fold of s1, v = exp(A S_T) h_0 + X_w^T B with X_w[s][p] =
// dt_s exp(A (S_T - S_s)) x_s[p], is a K = T contraction; two heads of one
// group share the request's B rows and position, so a head pair is one
// M128 N128 tcgen05.mma per 16 buffered tokens (rows 0..63 the first head's
// head_dim, 64..127 the second's). One persistent CTA per SM: a producer
// warp brings each due pair into a stage (both update copies, dt and x
// rows, the group's B rows; bulk copies on an mbarrier ring, as in
// k_fold_pipe) and consumer groups of four or eight warps take the pairs in
// turn:
//  - every warp forms both heads' weights (no barrier), then the group
//    builds one K-step's operands: X_w split into bf16 hi + mid + lo
//    (~2^-27 relative) and the B rows (exact in bf16), MN-major in
//    128-byte-swizzled atoms, zero past T;
//  - one thread issues the three MMAs into the group's 128-column fp32
//    accumulator in tensor memory and commits them to the group's mbarrier;
//  - each thread then owns one accumulator row, or half of one with eight
//    warps (warp w reads lanes 32 (w % 4) ..): 16 columns at a time it reads
//    the row with tcgen05.ld, adds exp(A S_T) h_0 from the stage and runs the
//    format's epilogue -- a Philox draw per 4 consecutive columns and the
//    stochastic rounding, an FP4 block of 16 columns quantised in registers
//    (for e4m3 the block's NaN-propagating max also decides whether any of
//    its values needs the rounding's special cases) -- storing straight to
//    global memory.
// Every wait is bounded; tensor memory is allocated once per CTA and freed
// on every path.
// ---------------------------------------------------------------------------
struct FoldUmmaLayout {
    uint32_t hb;           // one head's block in a stage: update copy (+ scales), dt row, x rows
    uint32_t st_dt, st_x;  // offsets of the dt row and the x rows in a head block
    uint32_t brows;        // the group's B rows [cap][128] (bf16), after the two head blocks
    uint32_t meta;
    uint32_t stage_bytes;
    int stages;
    FastDiv divPr;    // head pair -> request (H / 2 pairs per request)
    FastDiv divHpg;   // head -> group
    PhiloxKeys keys;  // the ten round keys of the seed (read from the parameter space)
};

constexpr int kFuK = 16;                        // buffered tokens per MMA K-step
constexpr uint32_t kFuPart = 2u * kFuK * 128u;  // one A part: 2 heads x 16 tokens x 128 B
constexpr uint32_t kFuOps = 4u * kFuPart;       // A hi, mid, lo + B (2 column blocks x 16 tokens x 128 B)
// meta words of a stage: pair index (-1: end), position, flush count, A of both heads, tag
constexpr int kUMetaPair = 0, kUMetaPos = 1, kUMetaFc = 2, kUMetaA0 = 3, kUMetaTag = 5;

// Consumer groups per update format and warps per group (4: a thread owns
// a whole row; 8: half a row, the two halves of the row's columns on warps
// w and w + 4). A group holds its stage for the whole pair, so there must be
// at least as many stages as groups (bf16 stages are ~41 KB). B200, split_b256
// refresh: bf16 3 x 4 warps 234 us (3 x 8: 246); e4m3 3 x 8 306 us (4 x 4:
// 366 before the epilogue loop was unrolled by 2); FP4 4 x 4 91 us (3 x 8: 96).
__host__ __device__ constexpr int fu_groups(int uf) { return uf == kF32 ? 2 : (uf == kFP4 ? 4 : 3); }
__host__ __device__ constexpr int fu_cwarps(int uf) { return uf == kE4M3 ? 8 : 4; }
__host__ __device__ constexpr int fu_threads(int uf) { return (fu_cwarps(uf) * fu_groups(uf) + 1) * 32; }
__host__ __device__ constexpr uint32_t fu_cols(int uf) { return fu_groups(uf) <= 2 ? 256u : 512u; }

// 16 consecutive values (row p, columns 16 cc ..) of a 64 x 128 tile in
// shared memory, in format F (FP4: codes, and the block scales at sc).
template <int F>
__device__ __forceinline__ void row16_load(const unsigned char* t, const unsigned char* sc, int p, int cc,
                                           float (&v)[16]) {
    if constexpr (F == kF32) {
        const float4* q = reinterpret_cast<const float4*>(t + p * 512 + cc * 64);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 f = q[i];
            v[4 * i] = f.x;
            v[4 * i + 1] = f.y;
            v[4 * i + 2] = f.z;
            v[4 * i + 3] = f.w;
        }
    } else if constexpr (F == kBF16) {
        const uint4* q = reinterpret_cast<const uint4*>(t + p * 256 + cc * 32);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint4 u = q[i];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                v[8 * i + 2 * k] = __uint_as_float(w[k] << 16);
                v[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
            }
        }
    } else if constexpr (F == kE4M3) {
        const uint4 u = *reinterpret_cast<const uint4*>(t + p * 128 + cc * 16);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float4 f = e4m3x4_val(w[k]);
            v[4 * k] = f.x;
            v[4 * k + 1] = f.y;
            v[4 * k + 2] = f.z;
            v[4 * k + 3] = f.w;
        }
    } else {
        const uint2 u = *reinterpret_cast<const uint2*>(t + p * 64 + cc * 8);
        const float s = e4m3_val(sc[p * 8 + cc]);
        e2m1x8_val(u.x, s, v);
        e2m1x8_val(u.y, s, v + 8);
    }
}

template <int UF, int OUT4>
__global__ void __launch_bounds__(fu_threads(UF), 1) k_fold_umma(const FoldArgs a, const __grid_constant__ FoldUmmaLayout lay) {
    constexpr int CG = fu_groups(UF), CW = fu_cwarps(UF), CT = CW * 32;
    constexpr int NCC = 8 * 4 / CW;  // 16-column steps per thread
    static_assert(CW == 4 || CW == 8, "a group covers the 128 accumulator lanes with 4 or 8 warps");
    static_assert(128 * CG <= static_cast<int>(fu_cols(UF)), "each group's 128 accumulator columns are allocated");
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kPipeStagesMax];
    __shared__ __align__(8) uint64_t empty_bar[kPipeStagesMax];
    __shared__ __align__(8) uint64_t mma_bar[CG];
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_abort;

    const int H = a.s.H, G = a.s.G, cap = a.s.cap, L = a.s.L;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int S = lay.stages;
    const int hp = H >> 1;  // head pairs per request
    const int npairs = a.s.batch * hp;
    const uint32_t tbu = tile_bytes(UF, 64, kD128) + scale_bytes(UF, 64, kD128);
    const bool in_record = a.upd == a.record;
    // the groups' operand areas (1024-byte swizzle atoms) first, then the stages
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (sbase - smem_u32(smem_raw));
    unsigned char* stg = smem + CG * kFuOps;

    pdl_prologue();
    if (warp == 0) {  // one warp allocates the accumulators (128 columns per group) and frees them
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(fu_cols(UF))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 32) {
        for (int st = 0; st < S; ++st) {
            mbar_init(smem_u32(&full_bar[st]), 1);
            mbar_init(smem_u32(&empty_bar[st]), CW);
            reinterpret_cast<int*>(stg + static_cast<size_t>(st) * lay.stage_bytes + lay.meta)[kUMetaTag] = -1;
        }
        for (int g = 0; g < CG; ++g) mbar_init(smem_u32(&mma_bar[g]), 1);
        s_abort = 0;
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = s_tmem;

    if (warp == CG * CW) {
        // ------------------------------------------------------------ producer
        int p0 = 0, p1 = 0;
        uint32_t f0 = 0, f1 = 0;
        float2 A0 = make_float2(0.f, 0.f), A1 = A0;
        auto fetch = [&](int kbase, int& pp, uint32_t& ff, float2& AA) {
            const uint32_t u = blockIdx.x + static_cast<uint32_t>(kbase + lane) * gridDim.x;
            if (u < static_cast<uint32_t>(npairs)) {
                const int bb = fdiv(u, lay.divPr);
                const int hh = 2 * (static_cast<int>(u) - bb * hp);
                pp = a.pos[bb];
                ff = a.flush_count[bb];
                AA = make_float2(a.A[hh], a.A[hh + 1]);
            }
        };
        fetch(0, p0, f0, A0);
        fetch(32, p1, f1, A1);
        int q = 0, st = 0, use = 0;  // stage sequence of the due pairs
        int q_issued = -1;
        bool aborted = false;
        auto take_stage = [&]() {
            int live = 1;
            if (lane == 0) {
                if (use > 0 && !mbar_wait_bounded(smem_u32(&empty_bar[st]), (use - 1) & 1, kWaitNs)) {
                    set_error(a.err, RSSM_DEVERR_TIMEOUT);
                    s_abort = 1;
                }
                live = !s_abort;
            }
            return __shfl_sync(0xffffffffu, live, 0) != 0;
        };
        auto next_stage = [&]() {
            q_issued = q;
            ++q;
            if (++st == S) {
                st = 0;
                ++use;
            }
        };
        for (int k = 0; blockIdx.x + static_cast<uint32_t>(k) * gridDim.x < static_cast<uint32_t>(npairs); ++k) {
            const uint32_t u = blockIdx.x + static_cast<uint32_t>(k) * gridDim.x;
            const bool cur = (k >> 5) & 1;
            const int sel = k & 31;
            if (sel == 0 && k > 0) {
                if (cur)
                    fetch(k + 32, p0, f0, A0);
                else
                    fetch(k + 32, p1, f1, A1);
            }
            const int pos = __shfl_sync(0xffffffffu, cur ? p1 : p0, sel);
            const uint32_t fc = __shfl_sync(0xffffffffu, cur ? f1 : f0, sel);
            const float Aa = __shfl_sync(0xffffffffu, cur ? A1.x : A0.x, sel);
            const float Ab = __shfl_sync(0xffffffffu, cur ? A1.y : A0.y, sel);
            if (pos < 0 || pos > cap) {
                if (lane == 0) set_error(a.err, RSSM_DEVERR_POS_RANGE);
                continue;
            }
            if (!((pos >= L) || (a.mode >= 1 && pos > 0) || (a.mode == 2))) continue;  // not due
            if (!take_stage()) {
                aborted = true;
                break;
            }
            if (lane == 0) {
                unsigned char* sp = stg + static_cast<size_t>(st) * lay.stage_bytes;
                const uint32_t fb = smem_u32(&full_bar[st]);
                int* meta = reinterpret_cast<int*>(sp + lay.meta);
                meta[kUMetaPair] = static_cast<int>(u);
                meta[kUMetaPos] = pos;
                meta[kUMetaFc] = static_cast<int>(fc);
                reinterpret_cast<float*>(meta)[kUMetaA0] = Aa;
                reinterpret_cast<float*>(meta)[kUMetaA0 + 1] = Ab;
                reinterpret_cast<volatile int*>(meta)[kUMetaTag] = q;
                const int b = fdiv(u, lay.divPr), h0 = 2 * (static_cast<int>(u) - b * hp);
                const size_t t0 = static_cast<size_t>(b) * H + h0;
                const uint32_t nx = static_cast<uint32_t>(pos) * 128u, nb = static_cast<uint32_t>(pos) * 256u;
                const uint32_t ndx = (a.rec.x - a.rec.dt) + nx;  // dt row and x rows, contiguous in the record
                const uint32_t per = in_record ? a.rec.x + nx : tbu + ndx;
                mbar_expect_tx(fb, 2u * per + nb);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const unsigned char* rec = a.record + (t0 + j) * a.rec.bytes;
                    unsigned char* hbp = sp + j * lay.hb;
                    if (in_record) {
                        bulk_g2s(smem_u32(hbp), rec, a.rec.x + nx, fb);
                    } else {
                        bulk_g2s(smem_u32(hbp), a.upd + (t0 + j) * a.upd_stride, tbu, fb);
                        bulk_g2s(smem_u32(hbp + lay.st_dt), rec + a.rec.dt, ndx, fb);
                    }
                }
                if (nb > 0) {
                    const size_t bg = static_cast<size_t>(b) * G + fdiv(static_cast<uint32_t>(h0), lay.divHpg);
                    bulk_g2s(smem_u32(sp + lay.brows),
                             static_cast<const unsigned char*>(a.bbuf) + bg * static_cast<size_t>(cap) * 256u, nb, fb);
                }
            }
            next_stage();
            __syncwarp();
        }
        // one end marker per consumer group
        for (int e = 0; e < CG && !aborted; ++e) {
            if (!take_stage()) {
                aborted = true;
                break;
            }
            if (lane == 0) {
                unsigned char* sp = stg + static_cast<size_t>(st) * lay.stage_bytes;
                int* meta = reinterpret_cast<int*>(sp + lay.meta);
                meta[kUMetaPair] = -1;
                reinterpret_cast<volatile int*>(meta)[kUMetaTag] = q;
                mbar_expect_tx(smem_u32(&full_bar[st]), 0u);
            }
            next_stage();
            __syncwarp();
        }
        if (aborted && lane == 0) {
            for (int qq = q_issued; qq >= 0 && qq > q_issued - S; --qq)
                mbar_wait_bounded(smem_u32(&full_bar[qq % S]), (qq / S) & 1, kWaitNs);
        }
        return;
    }

    // --------------------------------------------------------------- consumers
    const int gi = warp / CW, cw = warp - gi * CW, ctid = tid - gi * CT;
    const PhiloxKeys& pkeys = lay.keys;
    unsigned char* ops = smem + gi * kFuOps;
    const uint32_t ops_u = sbase + gi * kFuOps;
    const uint32_t tacc = tmem + 128u * gi;                                     // the group's accumulator
    // this thread's row (accumulator lane 32 (cw % 4) + lane: head jr, row pr)
    // and its columns, 16 cc0 .. 16 (cc0 + NCC) - 1
    const int jr = (32 * (cw & 3) + lane) >> 6, pr = (32 * (cw & 3) + lane) & 63, cc0 = (cw >> 2) * NCC;
    const uint32_t trow = tacc + (static_cast<uint32_t>(32 * (cw & 3)) << 16);  // this warp's lanes
    const uint32_t mbar = smem_u32(&mma_bar[gi]);
    uint32_t ncommit = 0;
    bool timed_out = false;
    int st = gi, use = 0;
    while (st >= S) {
        st -= S;
        ++use;
    }
    int pend_b = -1;
    uint32_t pend_old = 0;
    for (int q = gi;; q += CG) {
        unsigned char* sp = stg + static_cast<size_t>(st) * lay.stage_bytes;
        const int* meta = reinterpret_cast<const int*>(sp + lay.meta);
        int stop = 0;
        if (ctid == 0) {
            stop = s_abort;
            const volatile int* tag = reinterpret_cast<const volatile int*>(meta) + kUMetaTag;
            if (!stop && !smem_wait_eq_bounded(tag, q, kWaitNs)) {
                set_error(a.err, RSSM_DEVERR_TIMEOUT);
                s_abort = 1;
                stop = 1;
            }
            if (!stop && !mbar_wait_bounded(smem_u32(&full_bar[st]), use & 1, kWaitNs)) {
                set_error(a.err, RSSM_DEVERR_TIMEOUT);
                s_abort = 1;
                stop = 1;
                mbar_wait_bounded(smem_u32(&full_bar[st]), use & 1, kWaitNs);
            }
        }
        if (group_sync_or(gi, CT, stop)) break;
        const int u = meta[kUMetaPair];
        if (u < 0) {  // end of this group's sequence: hand the stage back and stop
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&empty_bar[st]));
            break;
        }
        const int T = meta[kUMetaPos];
        const uint32_t fc = static_cast<uint32_t>(meta[kUMetaFc]);
        const int b = fdiv(static_cast<uint32_t>(u), lay.divPr), h0 = 2 * (u - b * hp);
        // both heads' weights dt_s exp(A_j (S_T - S_s)) and exp(A_j S_T), in
        // every warp (no barrier): lane l takes buffered token l (T <= 32)
        float wl[2], alpha2[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const float Aj = reinterpret_cast<const float*>(meta)[kUMetaA0 + j];
            const float dts = (lane < T) ? reinterpret_cast<const float*>(sp + j * lay.hb + lay.st_dt)[lane] : 0.f;
            const float Sx = warp_prefix(dts);
            const float Stot = T > 0 ? __shfl_sync(0xffffffffu, Sx, T - 1) : 0.f;
            wl[j] = (lane < T) ? dts * expf(Aj * (Stot - Sx)) : 0.f;
            alpha2[j] = expf(Aj * Stot);
        }
        if (cw == 0 && lane == 0) {
            // every CTA read pos[b] before processing b's pairs; the last arrival resets it
            if (pend_b >= 0 && pend_old == static_cast<uint32_t>(H - 2)) {
                a.arrive[pend_b] = 0u;
                a.pos[pend_b] = 0;
                a.flush_count[pend_b] += 1u;
            }
            pend_b = b;
            pend_old = atomicAdd(&a.arrive[b], 2u);
        }
        const int nks = (T + kFuK - 1) / kFuK;
        for (int ks = 0; ks < nks; ++ks) {
            // the previous K-step's MMAs have read the operands
            if (ks > 0 && !mbar_wait_bounded(mbar, (ncommit - 1) & 1, kWaitNs)) timed_out = true;
            // B operand: tokens 16 ks .. (zero past T) as column block n / 64,
            // token row k, 16-byte chunk (n % 64) / 8 ^ (k & 7)
            for (int i = ctid; i < kFuK * 16; i += CT) {
                const int k = i >> 4, jn = i & 15, s = kFuK * ks + k;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (s < T) v = *reinterpret_cast<const uint4*>(sp + lay.brows + s * 256 + 16 * jn);
                *reinterpret_cast<uint4*>(ops + 3 * kFuPart + (jn >> 3) * (kFuK * 128) + k * 128 +
                                          16 * ((jn & 7) ^ (k & 7))) = v;
            }
            // A parts, x_w = w_s x_s[p] as bf16 hi + mid + lo, 8 rows at a time:
            // item -> head i / 128, token (i / 8) % 16, rows 8 (i % 8) .. + 7
            for (int i = ctid; i < 2 * kFuK * 8; i += CT) {
                const int hh = i >> 7, k = (i >> 3) & (kFuK - 1), c = i & 7, s = kFuK * ks + k;
                const float w0 = __shfl_sync(0xffffffffu, wl[0], s), w1 = __shfl_sync(0xffffffffu, wl[1], s);
                uint4 xv = make_uint4(0u, 0u, 0u, 0u);
                float w = 0.f;
                if (s < T) {
                    w = hh ? w1 : w0;
                    xv = *reinterpret_cast<const uint4*>(sp + hh * lay.hb + lay.st_x + s * 128 + 16 * c);
                }
                const uint32_t xr[4] = {xv.x, xv.y, xv.z, xv.w};
                uint32_t hi[4], md[4], lo[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float f0 = w * __uint_as_float(bf16lo_bits(xr[q]));
                    const float f1 = w * __uint_as_float(bf16hi_bits(xr[q]));
                    const uint32_t hh2 = f32x2_to_bf16x2(f0, f1);
                    hi[q] = hh2;
                    const float r0 = f0 - __uint_as_float(bf16lo_bits(hh2)), r1 = f1 - __uint_as_float(bf16hi_bits(hh2));
                    const uint32_t mm = f32x2_to_bf16x2(r0, r1);
                    md[q] = mm;
                    lo[q] = f32x2_to_bf16x2(r0 - __uint_as_float(bf16lo_bits(mm)), r1 - __uint_as_float(bf16hi_bits(mm)));
                }
                // A part layout: [head][token k][128 B], 16-byte chunk (p / 8) ^ (k & 7)
                const uint32_t d = static_cast<uint32_t>(hh * (kFuK * 128) + k * 128 + 16 * (c ^ (k & 7)));
                *reinterpret_cast<uint4*>(ops + d) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4*>(ops + kFuPart + d) = make_uint4(md[0], md[1], md[2], md[3]);
                *reinterpret_cast<uint4*>(ops + 2 * kFuPart + d) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            // the operands written by ordinary stores, visible to the tensor cores
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            group_sync(gi, CT);
            if (ctid == 0) {
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                // A: head blocks 64 rows apart in M (LBO = 16 x 128 B), 8-token atoms
                // (SBO 1024 B); B: column blocks of 64 (LBO), 8-token atoms (SBO)
                const uint64_t bd = umma_desc_sw128(ops_u + 3 * kFuPart, kFuK * 128, 1024);
#pragma unroll
                for (int part = 0; part < 3; ++part)
                    umma_f16(tacc, umma_desc_sw128(ops_u + part * kFuPart, kFuK * 128, 1024), bd,
                             (ks > 0 || part > 0) ? 1u : 0u);
                umma_commit(mbar);
            }
            ++ncommit;
        }
        if (nks > 0) {
            if (!mbar_wait_bounded(mbar, (ncommit - 1) & 1, kWaitNs)) timed_out = true;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        }
        __syncwarp();  // converged for the warp-wide accumulator reads
        {
            // this thread's part of its row: v = exp(A S_T) h_0 + acc, 16 columns at a time
            const float alpha = jr ? alpha2[1] : alpha2[0];
            const int hj = h0 + jr;
            const size_t tj = static_cast<size_t>(b) * H + hj;
            const unsigned char* tile = sp + jr * lay.hb;
            const unsigned char* tsc = tile + (in_record ? a.rec.scales : align16(tile_bytes(UF, 64, kD128)));
            unsigned char* updj = a.upd + tj * a.upd_stride;
            unsigned char* recj = a.record + tj * a.rec.bytes;
            uint32_t su0 = 0u, su1 = 0u, so0 = 0u, so1 = 0u;  // the FP4 block scales (update, output copy)
            const PhiloxFixed pfix = philox_fixed(static_cast<uint32_t>(hj), static_cast<uint32_t>(b), fc, pkeys);
            // unrolled by 2 only: the fully unrolled epilogue (32 Philox draws)
            // outgrew the instruction cache (bf16 refresh 310 -> 234 us)
#pragma unroll 2
            for (int c8 = 0; c8 < NCC; ++c8) {
                const int cc = cc0 + c8;
                float v[16];
                if (nks > 0) {
                    tmem_ld16(trow + 16u * cc, v);
                } else {
                    // nothing buffered: fma(alpha, h, -0) is alpha h exactly, signed zeros included
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = -0.0f;
                }
                {
                    float h[16];
                    row16_load<UF>(tile, tsc, pr, cc, h);
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = fmaf(alpha, h[i], v[i]);
                }
                const uint32_t e0 = static_cast<uint32_t>(pr * kD128 + 16 * cc);  // element of v[0] in the head
                float amax = 0.f;  // the block's max |v| (FP4 scale)
                if constexpr (UF == kF32) {
                    float* o = reinterpret_cast<float*>(updj) + e0;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        stream_store4(o + 4 * i, make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]));
                } else if constexpr (UF == kBF16 || UF == kE4M3) {
                    // e4m3: the block's NaN-propagating |max| (shared with the FP4
                    // scale below); below 448, no value of the block needs the
                    // rounding's special cases (NaN, infinity, saturation). (bf16
                    // keeps its per-value NaN select: a block test measured slower.)
                    bool plain = false;
                    if constexpr (UF == kE4M3) {
                        amax = absmax16<true>(v);
                        plain = amax < 448.0f;
                    }
                    uint32_t wv[UF == kBF16 ? 8 : 4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        // Philox counter (e/4, head, request, flush_count)
                        const uint4 rw = philox4x32_10((e0 >> 2) + i, pfix, pkeys);
                        if constexpr (UF == kBF16) {
                            wv[2 * i] = sr_bf16x2(v[4 * i], v[4 * i + 1], rw.x, rw.y);
                            wv[2 * i + 1] = sr_bf16x2(v[4 * i + 2], v[4 * i + 3], rw.z, rw.w);
                        } else if (plain) {
                            wv[i] = sr_e4m3_in_range(v[4 * i], rw.x) | (sr_e4m3_in_range(v[4 * i + 1], rw.y) << 8) |
                                    (sr_e4m3_in_range(v[4 * i + 2], rw.z) << 16) |
                                    (sr_e4m3_in_range(v[4 * i + 3], rw.w) << 24);
                        } else {
                            wv[i] = sr_e4m3(v[4 * i], rw.x) | (sr_e4m3(v[4 * i + 1], rw.y) << 8) |
                                    (sr_e4m3(v[4 * i + 2], rw.z) << 16) | (sr_e4m3(v[4 * i + 3], rw.w) << 24);
                        }
                    }
                    if constexpr (UF == kBF16) {
                        uint4* o = reinterpret_cast<uint4*>(updj + 2u * e0);
                        o[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                        o[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
                    } else {
                        *reinterpret_cast<uint4*>(updj + e0) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                    }
                } else {
                    uint32_t scv;
                    *reinterpret_cast<uint2*>(updj + e0 / 2) = fp4_quant16(v, &scv);
                    if (c8 < 4)
                        su0 |= scv << (8 * c8);
                    else
                        su1 |= scv << (8 * (c8 - 4));
                }
                if constexpr (OUT4 != 0) {
                    uint32_t scv;
                    if constexpr (UF == kE4M3) {
                        if (amax != amax) amax = absmax16<false>(v);  // a NaN value: the scale ignores it
                    } else {
                        amax = absmax16<false>(v);
                    }
                    *reinterpret_cast<uint2*>(recj + e0 / 2) = fp4_quant16(v, amax, &scv);
                    if (c8 < 4)
                        so0 |= scv << (8 * c8);
                    else
                        so1 |= scv << (8 * (c8 - 4));
                }
            }
            // the block scales of this thread's columns: bytes cc0 .. cc0 + NCC - 1 of the row's 8
            if constexpr (UF == kFP4) {
                if constexpr (NCC == 8)
                    *reinterpret_cast<uint2*>(updj + a.rec.scales + pr * 8) = make_uint2(su0, su1);
                else
                    *reinterpret_cast<uint32_t*>(updj + a.rec.scales + pr * 8 + cc0) = su0;
            }
            if constexpr (OUT4 != 0) {
                if constexpr (NCC == 8)
                    *reinterpret_cast<uint2*>(recj + a.rec.scales + pr * 8) = make_uint2(so0, so1);
                else
                    *reinterpret_cast<uint32_t*>(recj + a.rec.scales + pr * 8 + cc0) = so0;
            }
        }
        if (timed_out) {  // any thread whose wait ran out (first error wins)
            set_error(a.err, RSSM_DEVERR_TIMEOUT);
            s_abort = 1;
        }
        // the accumulator reads done before the group's next MMA; the stage back to the producer
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty_bar[st]));
        st += CG;
        while (st >= S) {
            st -= S;
            ++use;
        }
    }
    if (cw == 0 && lane == 0 && pend_b >= 0 && pend_old == static_cast<uint32_t>(H - 2)) {
        a.arrive[pend_b] = 0u;  // the last pending arrival of this group
        a.pos[pend_b] = 0;
        a.flush_count[pend_b] += 1u;
    }
    // no MMA of the group in flight (a timed-out wait is retried once), then
    // every consumer is past its last accumulator read: free tensor memory
    if (timed_out && ncommit > 0) mbar_wait_bounded(mbar, (ncommit - 1) & 1, kWaitNs);
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    asm volatile("bar.sync %0, %1;" ::"r"(CG + 1), "r"(CG * CT) : "memory");
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(fu_cols(UF)) : "memory");
    }
}

// ---------------------------------------------------------------------------
// Conventional scheme (in-run comparison, s1/s3): per token
//   h <- exp(dt A) h + dt x B^T, write h, y = h C + D x.
// VERIFY: read copy cur[b], write the state after token j to copy j.
// ---------------------------------------------------------------------------
template <typename TIn, int NT, int VERIFY>
__global__ void __launch_bounds__(kThreads, VERIFY ? (NT <= kMidTok ? 3 : 2) : 6) k_conv(const ConvArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bar;

    const int H = a.s.H, P = a.s.P, N = a.s.N, G = a.s.G, lpr = a.s.lpr;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x / H, h = blockIdx.x - b * H;
    const int g = h / (H / G);
    const int ntok = a.ntok;
    const int lsh = __ffs(lpr) - 1;
    const int rpw = 32 >> lsh, col4 = lane & (lpr - 1), rsub = lane >> lsh;
    const size_t bh = static_cast<size_t>(b) * H + h;
    const size_t copy_elems = static_cast<size_t>(a.s.batch) * H * P * N;

    int src = 0;
    if (VERIFY) {
        src = a.cur[b];
        if (src < 0 || src >= ntok) {
            if (tid == 0) set_error(a.err, RSSM_DEVERR_ACCEPT_RANGE);
            return;
        }
    }
    const uint32_t tb = 4u * P * N;
    const uint32_t bar_a = smem_u32(&bar);
    if (tid == 0) {
        mbar_init(bar_a, 1);
        mbar_expect_tx(bar_a, tb);
        bulk_g2s(smem_u32(smem), a.h + src * copy_elems + bh * P * N, tb, bar_a);
    }
    const TIn* xin = static_cast<const TIn*>(a.x);
    const TIn* Bin = static_cast<const TIn*>(a.B);
    const TIn* Cin = static_cast<const TIn*>(a.C);
    float4 b4[NT], c4[NT];
    float dtj[NT], aj[NT];
    const float Ah = a.A[h];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        const bool on = j < ntok;
        const size_t gi = ((static_cast<size_t>(b) * ntok + j) * G + g) * N + 4 * col4;
        b4[j] = on ? load4(Bin + gi) : make_float4(0.f, 0.f, 0.f, 0.f);
        c4[j] = on ? load4(Cin + gi) : make_float4(0.f, 0.f, 0.f, 0.f);
        dtj[j] = on ? a.dt[(static_cast<size_t>(b) * ntok + j) * H + h] : 0.f;
        aj[j] = expf(dtj[j] * Ah);
    }
    const float Dh = a.D[h];
    // one thread waits for the tile; the barrier publishes it to the CTA
    bool arrived = true;
    if (tid == 0) arrived = mbar_wait_bounded(bar_a, 0, kWaitNs);
    if (__syncthreads_or(!arrived)) {
        if (tid == 0) {
            set_error(a.err, RSSM_DEVERR_TIMEOUT);
            mbar_wait_bounded(bar_a, 0, kWaitNs);
        }
        return;
    }
    const float4* s_tile = reinterpret_cast<const float4*>(smem);
    for (int r0 = warp * rpw; r0 < P; r0 += kWarps * rpw) {
        const int r = r0 + rsub;
        const bool valid = r < P;
        float4 hv = valid ? s_tile[r * (N >> 2) + col4] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            if (j < ntok) {
                const float xr =
                    valid ? to_f32(xin[((static_cast<size_t>(b) * ntok + j) * H + h) * P + r]) : 0.f;
                const float u = dtj[j] * xr;
                hv.x = fmaf(u, b4[j].x, aj[j] * hv.x);
                hv.y = fmaf(u, b4[j].y, aj[j] * hv.y);
                hv.z = fmaf(u, b4[j].z, aj[j] * hv.z);
                hv.w = fmaf(u, b4[j].w, aj[j] * hv.w);
                if (valid) stream_store4(a.h + (VERIFY ? j * copy_elems : 0) + (bh * P + r) * N + 4 * col4, hv);
                const float d = group_sum(dot4(hv, c4[j]), lpr);
                if (valid && col4 == 0)
                    a.y[((static_cast<size_t>(b) * ntok + j) * H + h) * P + r] = fmaf(Dh, xr, d);
            }
        }
    }
}

// accept: pos[b] += n[b] + 1 (replay) or cur[b] = n[b] (conventional)
__global__ void k_accept(int batch, int K, int cap, const int32_t* n, int32_t* pos, int32_t* err, int add_one) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= batch) return;
    const int v = n[b];
    if (v < 0 || v > K) {
        set_error(err, RSSM_DEVERR_ACCEPT_RANGE);
        return;
    }
    if (add_one) {
        const int np = pos[b] + v + 1;
        if (pos[b] < 0 || np > cap) {
            set_error(err, RSSM_DEVERR_CAPACITY);
            return;
        }
        pos[b] = np;
    } else {
        pos[b] = v;
    }
}

// Rounding functions of k_fold, element-wise, for bit-exact tests.
__global__ void k_round_test(int op, int64_t n, const float* v, uint64_t seed, uint32_t c1, uint32_t c2,
                             uint32_t c3, void* out) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (op == 3 || op == 5) {
        // one lane per 4 values; quads of lanes make one 16-value block
        const int64_t q = i;  // group of 4 values
        const bool valid = 4 * q < n;
        const float4 x = valid ? reinterpret_cast<const float4*>(v)[q] : make_float4(0.f, 0.f, 0.f, 0.f);
        uint32_t sc;
        const uint32_t codes = fp4_quant_quad(x, &sc);
        if (valid && op == 3) {
            uint8_t* o = static_cast<uint8_t*>(out);
            *reinterpret_cast<uint16_t*>(o + 2 * q) = static_cast<uint16_t>(codes);
            if ((q & 3) == 0) o[n / 2 + q / 4] = static_cast<uint8_t>(sc);
        }
        if (valid && op == 5) {
            // the decode the FP4-reading kernels use
            reinterpret_cast<float4*>(out)[q] = fp4x4_val(codes, e4m3_val(sc));
        }
        return;
    }
    if (i >= n) return;
    const uint4 rw = philox4x32_10(make_uint4(static_cast<uint32_t>(i >> 2), c1, c2, c3),
                                   make_uint2(static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32)));
    const uint32_t r = (i & 3) == 0 ? rw.x : (i & 3) == 1 ? rw.y : (i & 3) == 2 ? rw.z : rw.w;
    switch (op) {
        case 0: {
            // the packed pair the refresh kernels use: elements i & ~1 and i | 1
            const bool hi = (i & 1) != 0;
            const float v0 = v[i & ~static_cast<int64_t>(1)], v1 = (i | 1) < n ? v[i | 1] : 0.0f;
            const uint32_t r0 = (i & 2) ? rw.z : rw.x, r1 = (i & 2) ? rw.w : rw.y;
            const uint32_t w = sr_bf16x2(v0, v1, r0, r1);
            static_cast<uint16_t*>(out)[i] = static_cast<uint16_t>(hi ? w >> 16 : w & 0xFFFFu);
            break;
        }
        case 1: static_cast<uint8_t*>(out)[i] = static_cast<uint8_t>(sr_e4m3(v[i], r)); break;
        case 2: static_cast<uint8_t*>(out)[i] = static_cast<uint8_t>(e4m3_rn(v[i])); break;
        default: static_cast<uint32_t*>(out)[i] = r; break;
    }
}

// ------------------------------------------------- no-allocation scratch
// Arrival counters for rssm_decode_step_noalloc: one uint32 per request,
// resident on every GPU that loads the library (256 KiB) until exit.
static __device__ __align__(256) uint32_t g_noalloc_arrive[RSSM_NOALLOC_MAX_BATCH];

// Device address of g_noalloc_arrive on the current device, looked up once
// per device (cudaGetSymbolAddress) and cached. nullptr when the lookup
// fails. Host threads may race on the first lookup: each stores the same
// address, and the atomics make that well defined.
uint32_t* noalloc_arrive_scratch() {
    static std::atomic<uint32_t*> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    uint32_t* p = cache[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_arrive) != cudaSuccess) return nullptr;
        p = static_cast<uint32_t*>(ptr);
        cache[dev].store(p, std::memory_order_release);
    }
    return p;
}

// ------------------------------------------------------------------ host

size_t replay_smem_bytes(const Shape& s, int rf, int ntok, int fused) {
    (void)ntok;
    size_t b = align16(tile_bytes(rf, s.P, s.N)) + align16(scale_bytes(rf, s.P, s.N));
    b += 4u * static_cast<size_t>(s.cap) * round_up8(s.P);
    if (fused) b += 4u * static_cast<size_t>(s.L) * s.N;
    return b;
}

size_t fold_smem_bytes(const Shape& s, int uf) {
    size_t b = align16(tile_bytes(uf, s.P, s.N)) + align16(scale_bytes(uf, s.P, s.N));
    if (uf != kF32) b += 4u * static_cast<size_t>(s.P) * s.N;
    b += 4u * static_cast<size_t>(s.cap) * s.N;
    b += 4u * static_cast<size_t>(s.cap) * round_up8(s.P);
    return b;
}

size_t conv_smem_bytes(const Shape& s) { return 4u * static_cast<size_t>(s.P) * s.N; }

template <typename K, typename Args>
static cudaError_t launch_tiles(K kernel, const Args& a, int nblk, size_t smem, cudaStream_t st) {
    if (nblk <= 0) return cudaSuccess;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    // all of the unified L1/shared array as shared memory: the tiles are
    // staged there and the occupancy is bounded by it
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         static_cast<int>(cudaSharedmemCarveoutMaxShared));
    if (e != cudaSuccess) return e;
    kernel<<<nblk, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

// Launch with programmatic stream serialization (see pdl_prologue).
template <typename K, typename A1, typename A2>
static cudaError_t launch_pdl(K kernel, int grid, int threads, size_t smem, cudaStream_t st, const A1& a1,
                              const A2& a2) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, a1, a2);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <typename K, typename... Args>
static cudaError_t launch_grid(K kernel, const ReplayArgs& a, const PipeLayout& L, int grid, int threads,
                               size_t smem, cudaStream_t st) {
    if (grid <= 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             static_cast<int>(cudaSharedmemCarveoutMaxShared));
    if (e != cudaSuccess) return e;
    return launch_pdl(kernel, grid, threads, smem, st, a, L);
}

template <typename TIn, int NT, int W>
static cudaError_t replay_dispatch_fmt(const ReplayArgs& a, int rf, size_t smem, int nblk, cudaStream_t st) {
    switch (rf) {
        case kF32:
            if constexpr (NT == 1) {
                if (a.fused) return launch_tiles(k_replay<TIn, kF32, NT, 1, W>, a, nblk, smem, st);
            }
            return launch_tiles(k_replay<TIn, kF32, NT, 0, W>, a, nblk, smem, st);
        case kBF16: return launch_tiles(k_replay<TIn, kBF16, NT, 0, W>, a, nblk, smem, st);
        case kE4M3: return launch_tiles(k_replay<TIn, kE4M3, NT, 0, W>, a, nblk, smem, st);
        default: return launch_tiles(k_replay<TIn, kFP4, NT, 0, W>, a, nblk, smem, st);
    }
}

template <typename TIn, int NT>
static cudaError_t replay_dispatch_wide(const ReplayArgs& a, int rf, size_t smem, int nblk, cudaStream_t st) {
    const bool wide = a.s.N == 128 && a.s.P % 8 == 0;
    return wide ? replay_dispatch_fmt<TIn, NT, 1>(a, rf, smem, nblk, st)
                : replay_dispatch_fmt<TIn, NT, 0>(a, rf, smem, nblk, st);
}

RecLayout record_layout(const Shape& s, int rf, int in_bytes) {
    RecLayout r;
    r.tile = tile_bytes(rf, s.P, s.N);
    r.scales = rf == kFP4 ? align16(r.tile) : 0u;
    r.dt = align16(align16(r.tile) + scale_bytes(rf, s.P, s.N));
    r.x = r.dt + 4u * static_cast<uint32_t>(s.capr);
    r.bytes = (r.x + static_cast<uint32_t>(s.cap * s.P * in_bytes) + 127u) & ~127u;
    return r;
}

// Stage layout of k_replay_pipe (16-byte aligned pieces, 128-byte aligned
// stages and row buffers); the stages fill what the row buffers leave.
// rows_in_stage: this call's rows travel with the stage (no row buffers).
PipeLayout pipe_layout(const Shape& s, const RecLayout& rec, int ntok, int in_bf16, int groups, int fused,
                       size_t smem_budget, int rows_in_stage) {
    const uint32_t es = in_bf16 ? 2u : 4u;
    PipeLayout L;
    L.brows = align16(rec.x + static_cast<uint32_t>(s.cap * s.P) * es);
    L.meta = L.brows + align16(static_cast<uint32_t>(s.cap * s.N) * es);
    L.nb_off = align16(static_cast<uint32_t>(ntok * s.P) * es);
    L.nc_off = L.nb_off + align16(static_cast<uint32_t>(ntok * s.N) * es);
    L.nd_off = L.nc_off + align16(static_cast<uint32_t>(ntok * s.N) * es);
    if (rows_in_stage) {
        L.rows = L.meta + 64u;
        L.stage_bytes = (L.rows + L.nc_off + static_cast<uint32_t>(ntok * s.N) * es + 127u) & ~127u;
        L.newrows = 0u;
    } else {
        L.rows = 0u;
        L.stage_bytes = (L.meta + 64u + 127u) & ~127u;
        L.newrows = (L.nd_off + 4u * (kMaxTok + 2) + 127u) & ~127u;
    }
    L.xw_bytes = fused ? (4u * static_cast<uint32_t>(s.cap * s.P) + 127u) & ~127u : 0u;
    const size_t rows = static_cast<size_t>(groups) * (2u * L.newrows + L.xw_bytes);
    const size_t n = smem_budget > rows ? (smem_budget - rows) / L.stage_bytes : 0;
    L.stages = static_cast<int>(n < static_cast<size_t>(kPipeStagesMax) ? n : kPipeStagesMax);
    L.budget = smem_budget;
    L.divH = make_fastdiv(static_cast<uint32_t>(s.H));
    L.divHpg = make_fastdiv(static_cast<uint32_t>(s.H / s.G));
    return L;
}

struct DeviceInfo {
    int sms = 0;
    size_t smem_optin = 0;
};

// SM count and opt-in shared memory of the current device, queried once per
// device. The query is idempotent; concurrent first calls store the same
// values (the SM count last, with release order, so a reader that sees it
// also sees the shared-memory size).
static DeviceInfo device_info() {
    static std::atomic<int> sms_cache[64];
    static std::atomic<size_t> smem_cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DeviceInfo{};
    DeviceInfo di;
    di.sms = sms_cache[dev].load(std::memory_order_acquire);
    if (di.sms == 0) {
        int sms = 0, optin = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return DeviceInfo{};
        smem_cache[dev].store(static_cast<size_t>(optin), std::memory_order_relaxed);
        sms_cache[dev].store(sms, std::memory_order_release);
        di.sms = sms;
    }
    di.smem_optin = smem_cache[dev].load(std::memory_order_relaxed);
    return di;
}

template <typename TIn, int NT>
static cudaError_t pipe_dispatch(const ReplayArgs& a, const PipeLayout& L, int rf, int grid, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(L.stages) * L.stage_bytes +
                        static_cast<size_t>(pipe_groups(NT, rf)) * (2u * L.newrows + L.xw_bytes);
    if (smem > L.budget) return cudaErrorInvalidValue;
    if constexpr (NT == 1) {
        if (a.fused) {
            if (rf != kF32) return cudaErrorInvalidValue;
            return launch_grid(k_replay_pipe<TIn, kF32, NT, 1>, a, L, grid, pipe_threads(NT, kF32), smem, st);
        }
    }
    switch (rf) {
        case kF32:
            return launch_grid(k_replay_pipe<TIn, kF32, NT, 0>, a, L, grid, pipe_threads(NT, kF32), smem, st);
        case kBF16:
            return launch_grid(k_replay_pipe<TIn, kBF16, NT, 0>, a, L, grid, pipe_threads(NT, kBF16), smem, st);
        case kE4M3:
            return launch_grid(k_replay_pipe<TIn, kE4M3, NT, 0>, a, L, grid, pipe_threads(NT, kE4M3), smem, st);
        default:
            return launch_grid(k_replay_pipe<TIn, kFP4, NT, 0>, a, L, grid, pipe_threads(NT, kFP4), smem, st);
    }
}

static cudaError_t launch_replay_pipe(const ReplayArgs& a, int in_bf16, int rf, const PipeLayout& L, int grid,
                                      cudaStream_t st) {
    if (a.ntok == 1)
        return in_bf16 ? pipe_dispatch<__nv_bfloat16, 1>(a, L, rf, grid, st) : pipe_dispatch<float, 1>(a, L, rf, grid, st);
    if (a.ntok <= kMidTok)
        return in_bf16 ? pipe_dispatch<__nv_bfloat16, kMidTok>(a, L, rf, grid, st)
                       : pipe_dispatch<float, kMidTok>(a, L, rf, grid, st);
    return in_bf16 ? pipe_dispatch<__nv_bfloat16, kMaxTok>(a, L, rf, grid, st)
                   : pipe_dispatch<float, kMaxTok>(a, L, rf, grid, st);
}

cudaError_t launch_replay(const ReplayArgs& a, int in_bf16, int rf, cudaStream_t st) {
    // the pipelined kernel serves d_state 128 with head_dim a multiple of 8
    if (a.s.N == 128 && a.s.P % 8 == 0 && (!a.fused || (rf == kF32 && a.ntok == 1))) {
        const DeviceInfo di = device_info();
        if (di.sms > 0) {
            const int nt = a.ntok == 1 ? 1 : (a.ntok <= kMidTok ? kMidTok : kMaxTok);  // the kernel's token bound
            const size_t stat = pipe_static_smem(nt, rf);
            const size_t budget = di.smem_optin > stat ? di.smem_optin - stat : 0;
            const int groups = pipe_groups(nt, rf);
            const PipeLayout L = pipe_layout(a.s, a.rec, a.ntok, in_bf16, groups, a.fused, budget,
                                             pipe_rows_in_stage(a.ntok, rf, a.fused));
            if (L.stages >= 2) {
                const int ntiles = a.s.batch * a.s.H;
                const int grid = ntiles < di.sms ? ntiles : di.sms;
                return launch_replay_pipe(a, in_bf16, rf, L, grid, st);
            }
        }
    }
    const size_t smem = replay_smem_bytes(a.s, rf, a.ntok, a.fused);
    const int nblk = a.s.batch * a.s.H;
    if (a.ntok == 1)
        return in_bf16 ? replay_dispatch_wide<__nv_bfloat16, 1>(a, rf, smem, nblk, st)
                       : replay_dispatch_wide<float, 1>(a, rf, smem, nblk, st);
    if (a.ntok <= kMidTok)
        return in_bf16 ? replay_dispatch_wide<__nv_bfloat16, kMidTok>(a, rf, smem, nblk, st)
                       : replay_dispatch_wide<float, kMidTok>(a, rf, smem, nblk, st);
    return in_bf16 ? replay_dispatch_wide<__nv_bfloat16, kMaxTok>(a, rf, smem, nblk, st)
                   : replay_dispatch_wide<float, kMaxTok>(a, rf, smem, nblk, st);
}

template <typename TIn>
static cudaError_t fold_dispatch(const FoldArgs& a, int uf, size_t smem, int nblk, cudaStream_t st) {
    if (a.out_fp4) {
        switch (uf) {
            case kF32: return launch_tiles(k_fold<TIn, kF32, 1>, a, nblk, smem, st);
            case kBF16: return launch_tiles(k_fold<TIn, kBF16, 1>, a, nblk, smem, st);
            case kE4M3: return launch_tiles(k_fold<TIn, kE4M3, 1>, a, nblk, smem, st);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (uf) {
        case kF32: return launch_tiles(k_fold<TIn, kF32, 0>, a, nblk, smem, st);
        case kBF16: return launch_tiles(k_fold<TIn, kBF16, 0>, a, nblk, smem, st);
        case kE4M3: return launch_tiles(k_fold<TIn, kE4M3, 0>, a, nblk, smem, st);
        default: return launch_tiles(k_fold<TIn, kFP4, 0>, a, nblk, smem, st);
    }
}

template <typename TIn>
static cudaError_t fold_pipe_dispatch(const FoldArgs& a, const FoldPipeLayout& L, int uf, int grid, size_t smem,
                                      cudaStream_t st) {
    const int threads = fold_threads(uf);
    auto go = [&](auto kernel) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 static_cast<int>(cudaSharedmemCarveoutMaxShared));
        if (e != cudaSuccess) return e;
        return launch_pdl(kernel, grid, threads, smem, st, a, L);
    };
    if (a.out_fp4) {
        switch (uf) {
            case kF32: return go(k_fold_pipe<TIn, kF32, 1>);
            case kBF16: return go(k_fold_pipe<TIn, kBF16, 1>);
            case kE4M3: return go(k_fold_pipe<TIn, kE4M3, 1>);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (uf) {
        case kF32: return go(k_fold_pipe<TIn, kF32, 0>);
        case kBF16: return go(k_fold_pipe<TIn, kBF16, 0>);
        case kE4M3: return go(k_fold_pipe<TIn, kE4M3, 0>);
        default: return go(k_fold_pipe<TIn, kFP4, 0>);
    }
}

// Stage layout of k_fold_pipe: update copy (+ scales), dt row and x rows
// (at the record's offsets when the update copy is the record's own copy),
// B rows, meta; per consumer group a scratch of fp32 B and w x rows.
static FoldPipeLayout fold_pipe_layout(const FoldArgs& a, int uf, int in_bf16, size_t budget) {
    const Shape& s = a.s;
    const uint32_t es = in_bf16 ? 2u : 4u;
    FoldPipeLayout L;
    if (a.upd == a.record) {
        L.st_dt = a.rec.dt;
        L.st_x = a.rec.x;
    } else {
        L.st_dt = align16(align16(tile_bytes(uf, s.P, s.N)) + scale_bytes(uf, s.P, s.N));
        L.st_x = L.st_dt + (a.rec.x - a.rec.dt);
    }
    L.brows = align16(L.st_x + static_cast<uint32_t>(s.cap * s.P) * es);
    L.meta = L.brows + align16(static_cast<uint32_t>(s.cap * s.N) * es);
    L.stage_bytes = (L.meta + 64u + 127u) & ~127u;
    L.scratch = (4u * static_cast<uint32_t>(s.cap) * (s.N + s.P) + 127u) & ~127u;
    const size_t rows = static_cast<size_t>(fold_groups(uf)) * L.scratch;
    const size_t n = budget > rows ? (budget - rows) / L.stage_bytes : 0;
    L.stages = static_cast<int>(n < static_cast<size_t>(kPipeStagesMax) ? n : kPipeStagesMax);
    L.divH = make_fastdiv(static_cast<uint32_t>(s.H));
    L.divHpg = make_fastdiv(static_cast<uint32_t>(s.H / s.G));
    return L;
}

// The tensor-core refresh (k_fold_umma): bf16 inputs, d_state 128, head_dim
// 64, head pairs inside a group; the low-precision update copies, and an
// fp32 update copy when it also writes the FP4 output copy.
static bool fold_umma_shape(const FoldArgs& a, int in_bf16, int uf) {
    return in_bf16 && a.s.N == kD128 && a.s.P == 64 && a.s.H % 2 == 0 && (a.s.H / a.s.G) % 2 == 0 &&
           a.s.cap <= kMaxCap && (uf != kF32 || a.out_fp4) && !(uf == kFP4 && a.out_fp4);
}

// Stage layout of k_fold_umma: two head blocks (update copy (+ scales), dt
// row, x rows: the record's offsets when the update copy is the record's own
// copy), the group's B rows, meta. The groups' operand areas come first.
static FoldUmmaLayout fold_umma_layout(const FoldArgs& a, int uf, size_t budget) {
    const Shape& s = a.s;
    FoldUmmaLayout L;
    if (a.upd == a.record) {
        L.st_dt = a.rec.dt;
        L.st_x = a.rec.x;
    } else {
        L.st_dt = align16(align16(tile_bytes(uf, s.P, s.N)) + scale_bytes(uf, s.P, s.N));
        L.st_x = L.st_dt + (a.rec.x - a.rec.dt);
    }
    L.hb = (L.st_x + static_cast<uint32_t>(s.cap * s.P) * 2u + 127u) & ~127u;
    L.brows = 2u * L.hb;
    L.meta = L.brows + align16(static_cast<uint32_t>(s.cap * s.N) * 2u);
    L.stage_bytes = (L.meta + 64u + 127u) & ~127u;
    const size_t ops = 1024 + static_cast<size_t>(fu_groups(uf)) * kFuOps;
    const size_t n = budget > ops ? (budget - ops) / L.stage_bytes : 0;
    L.stages = static_cast<int>(n < static_cast<size_t>(kPipeStagesMax) ? n : kPipeStagesMax);
    L.divPr = make_fastdiv(static_cast<uint32_t>(s.H / 2));
    L.divHpg = make_fastdiv(static_cast<uint32_t>(s.H / s.G));
    L.keys = philox_keys(a.seed);
    return L;
}

static cudaError_t fold_umma_dispatch(const FoldArgs& a, const FoldUmmaLayout& L, int uf, int grid, size_t smem,
                                      cudaStream_t st) {
    auto go = [&](auto kernel, int threads) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 static_cast<int>(cudaSharedmemCarveoutMaxShared));
        if (e != cudaSuccess) return e;
        return launch_pdl(kernel, grid, threads, smem, st, a, L);
    };
    if (a.out_fp4) {
        switch (uf) {
            case kF32: return go(k_fold_umma<kF32, 1>, fu_threads(kF32));
            case kBF16: return go(k_fold_umma<kBF16, 1>, fu_threads(kBF16));
            case kE4M3: return go(k_fold_umma<kE4M3, 1>, fu_threads(kE4M3));
            default: return cudaErrorInvalidValue;
        }
    }
    switch (uf) {
        case kBF16: return go(k_fold_umma<kBF16, 0>, fu_threads(kBF16));
        case kE4M3: return go(k_fold_umma<kE4M3, 0>, fu_threads(kE4M3));
        case kFP4: return go(k_fold_umma<kFP4, 0>, fu_threads(kFP4));
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_fold(const FoldArgs& a, int in_bf16, int uf, cudaStream_t st) {
    if (fold_umma_shape(a, in_bf16, uf)) {
        const DeviceInfo di = device_info();
        if (di.sms > 0) {
            const size_t budget = di.smem_optin > 8192 ? di.smem_optin - 8192 : 0;
            const FoldUmmaLayout L = fold_umma_layout(a, uf, budget);
            if (L.stages >= fu_groups(uf)) {
                const int npairs = a.s.batch * (a.s.H / 2);
                if (npairs <= 0) return cudaSuccess;
                const int grid = npairs < di.sms ? npairs : di.sms;
                const size_t smem = 1024 + static_cast<size_t>(fu_groups(uf)) * kFuOps +
                                    static_cast<size_t>(L.stages) * L.stage_bytes;
                return fold_umma_dispatch(a, L, uf, grid, smem, st);
            }
        }
    }
    if (a.s.N == 128 && a.s.P % 8 == 0) {
        const DeviceInfo di = device_info();
        if (di.sms > 0) {
            const size_t budget = di.smem_optin > 8192 ? di.smem_optin - 8192 : 0;
            const FoldPipeLayout L = fold_pipe_layout(a, uf, in_bf16, budget);
            if (L.stages >= 2) {
                const int ntiles = a.s.batch * a.s.H;
                const int grid = ntiles < di.sms ? ntiles : di.sms;
                const size_t smem = static_cast<size_t>(L.stages) * L.stage_bytes +
                                    static_cast<size_t>(fold_groups(uf)) * L.scratch;
                return in_bf16 ? fold_pipe_dispatch<__nv_bfloat16>(a, L, uf, grid, smem, st)
                               : fold_pipe_dispatch<float>(a, L, uf, grid, smem, st);
            }
        }
    }
    const size_t smem = fold_smem_bytes(a.s, uf);
    const int nblk = a.s.batch * a.s.H;
    return in_bf16 ? fold_dispatch<__nv_bfloat16>(a, uf, smem, nblk, st) : fold_dispatch<float>(a, uf, smem, nblk, st);
}

cudaError_t launch_prefill(const PrefillArgs& a, int in_bf16, cudaStream_t st) {
    if (in_bf16 && a.s.N == 128 && a.s.P == 64 && (a.s.H / a.s.G) % 2 == 0) {
        if (a.s.batch * a.s.H <= 0) return cudaSuccess;
        cudaError_t e = cudaFuncSetAttribute(k_prefill_umma, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kUmSmem));
        if (e != cudaSuccess) return e;
        k_prefill_umma<<<a.s.batch * (a.s.H / 2), kUmThreads, kUmSmem, st>>>(a);
        return cudaGetLastError();
    }
    if (in_bf16 && a.s.N == 128 && a.s.P % 16 == 0 && a.s.P <= 64) {
        if (a.s.batch * a.s.H <= 0) return cudaSuccess;
        cudaError_t e = cudaFuncSetAttribute(k_prefill_mma, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kPfSmem));
        if (e != cudaSuccess) return e;
        k_prefill_mma<<<a.s.batch * a.s.H, kPfThreads, kPfSmem, st>>>(a);
        return cudaGetLastError();
    }
    const size_t smem = 4u * (static_cast<size_t>(a.s.P) * a.s.N + static_cast<size_t>(kPrefillChunk) * a.s.N +
                              static_cast<size_t>(kPrefillChunk) * round_up8(a.s.P));
    const int nblk = a.s.batch * a.s.H;
    return in_bf16 ? launch_tiles(k_prefill<__nv_bfloat16>, a, nblk, smem, st)
                   : launch_tiles(k_prefill<float>, a, nblk, smem, st);
}

cudaError_t launch_conv(const ConvArgs& a, int in_bf16, int verify, cudaStream_t st) {
    const size_t smem = conv_smem_bytes(a.s);
    const int nblk = a.s.batch * a.s.H;
    if (!verify)
        return in_bf16 ? launch_tiles(k_conv<__nv_bfloat16, 1, 0>, a, nblk, smem, st)
                       : launch_tiles(k_conv<float, 1, 0>, a, nblk, smem, st);
    if (a.ntok <= kMidTok)
        return in_bf16 ? launch_tiles(k_conv<__nv_bfloat16, kMidTok, 1>, a, nblk, smem, st)
                       : launch_tiles(k_conv<float, kMidTok, 1>, a, nblk, smem, st);
    return in_bf16 ? launch_tiles(k_conv<__nv_bfloat16, kMaxTok, 1>, a, nblk, smem, st)
                   : launch_tiles(k_conv<float, kMaxTok, 1>, a, nblk, smem, st);
}

cudaError_t launch_accept(int batch, int K, int cap, const int32_t* n, int32_t* pos, int32_t* err, int add_one,
                          cudaStream_t st) {
    if (batch <= 0) return cudaSuccess;
    k_accept<<<(batch + 255) / 256, 256, 0, st>>>(batch, K, cap, n, pos, err, add_one);
    return cudaGetLastError();
}

cudaError_t launch_round_test(int op, int64_t n, const float* v, uint64_t seed, uint32_t c1, uint32_t c2,
                              uint32_t c3, void* out, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const int64_t items = (op == 3 || op == 5) ? n / 4 : n;
    const int64_t blocks = (items + 255) / 256;
    k_round_test<<<static_cast<unsigned>(blocks), 256, 0, st>>>(op, n, v, seed, c1, c2, c3, out);
    return cudaGetLastError();
}

}  // namespace rssm
