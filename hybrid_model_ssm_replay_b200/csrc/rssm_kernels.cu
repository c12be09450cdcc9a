// rssm_kernels.cu -- sm_100a kernels of librssm.
//
// Every tile kernel runs one CTA of 256 threads per (request b, head h).
// The CTA's state tile (P x N, one head of one request, contiguous in HBM)
// is brought into shared memory by one bulk copy (cp.async.bulk, completion
// on an mbarrier) issued before anything else, so the HBM stream starts at
// once and overlaps the small per-token work (buffer reads, decay weights,
// B.C dot products). Rows are then read from shared memory by warps: the
// lanes of a row each hold 4 consecutive d_state elements and reduce with
// shuffles. There are no float atomics; every result has a fixed summation
// order, so runs are bit-reproducible.
//
// Method: ReplaySSM article (devotd.net
// "nvidia-replayssm-hybrid-model-ssm-decoding-state-buffer"):
//   s1 "Store recent inputs instead of the full state"     -> k_replay, k_fold
//   s3 "Roll back incorrect predictions using buffer positions" -> k_replay (verify), k_accept
//   s4 "Prevent low-precision errors from accumulating again"   -> k_fold (refresh), FP4 reads
//   conventional scheme of s1/s3 (in-run comparison)            -> k_conv
#include "rssm_device.cuh"
#include "rssm_internal.h"
#include "rssm.h"

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
        const float s = e4m3_val(sc[q >> 2]);
        float4 v = fp4x4_val(reinterpret_cast<const uint16_t*>(t)[q]);
        v.x *= s;
        v.y *= s;
        v.z *= s;
        v.w *= s;
        return v;
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

// The fold of s1: v[r][c] = alpha * tile[r][c] + sum_{s<T} xw[s][r] * B_s[c],
// with xw[s][r] = dt_s exp(A (S_T - S_s)) x_s[r] staged in shared memory and
// the lane's B_s columns held in registers, 16 slots at a time. `s32` is the
// fp32 tile in shared memory (rewritten between chunks); brow(s, c) gives
// B_s columns 4c..4c+3; emit(r, c, v, valid) is called by every lane for
// the final values (valid = row in range).
template <typename BRow, typename Emit>
__device__ __forceinline__ void fold_rows(float* s32, const float* s_xw, int P, int N, int lpr, int T,
                                          float alpha, BRow brow, Emit emit) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int lsh = __ffs(lpr) - 1;
    const int rpw = 32 >> lsh, col4 = lane & (lpr - 1), rsub = lane >> lsh;
    const int nchunk = T > 0 ? (T + 15) >> 4 : 1;
    for (int ch = 0; ch < nchunk; ++ch) {
        float4 br[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int s = ch * 16 + i;
            br[i] = (s < T) ? brow(s, col4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        const bool last = (ch == nchunk - 1);
        for (int r0 = warp * rpw; r0 < P; r0 += kWarps * rpw) {
            const int r = r0 + rsub;
            const bool valid = r < P;
            float4 v = valid ? reinterpret_cast<const float4*>(s32)[r * (N >> 2) + col4]
                             : make_float4(0.f, 0.f, 0.f, 0.f);
            if (ch == 0) {
                v.x *= alpha;
                v.y *= alpha;
                v.z *= alpha;
                v.w *= alpha;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int s = ch * 16 + i;
                if (s < T) {
                    const float xw = valid ? s_xw[s * P + r] : 0.f;
                    v.x = fmaf(xw, br[i].x, v.x);
                    v.y = fmaf(xw, br[i].y, v.y);
                    v.z = fmaf(xw, br[i].z, v.z);
                    v.w = fmaf(xw, br[i].w, v.w);
                }
            }
            if (last)
                emit(r, col4, v, valid);
            else if (valid)
                reinterpret_cast<float4*>(s32)[r * (N >> 2) + col4] = v;
        }
    }
}

// ---------------------------------------------------------------------------
// Replay decode / verify (s1, s3).
//   y_j = exp(A S_t) (h_ckpt C_j) + sum_{s<=t} dt_s exp(A (S_t - S_s)) (B_s . C_j) x_s + D x_t,
//   t = pos + j, for the ntok tokens of this call; S = prefix sum of the
//   buffered dt. The new tokens are appended at slots pos..pos+ntok-1.
//   RF: format of the copy read (fp32 checkpoint, bf16/e4m3 update copy, or
//   FP4 copy). NT: compile-time bound on ntok.
// ---------------------------------------------------------------------------
template <typename TIn, int RF, int NT, int FUSED>
__global__ void __launch_bounds__(kThreads) k_replay(const ReplayArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bar;
    __shared__ float s_w[NT][kMaxCap];
    __shared__ float s_g[NT][kMaxCap];
    __shared__ float s_decay[NT];

    const int H = a.s.H, P = a.s.P, N = a.s.N, G = a.s.G, cap = a.s.cap, lpr = a.s.lpr;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x / H, h = blockIdx.x - b * H;
    const int hpg = H / G, g = h / hpg;
    const int ntok = a.ntok;
    const int lsh = __ffs(lpr) - 1;
    const int rpw = 32 >> lsh, col4 = lane & (lpr - 1), rsub = lane >> lsh;
    const size_t bh = static_cast<size_t>(b) * H + h;

    const uint32_t tb = tile_bytes(RF, P, N), sb = scale_bytes(RF, P, N);
    unsigned char* s_tile = smem;
    unsigned char* s_sc = smem + align16(tb);
    float* s_hc = reinterpret_cast<float*>(smem + align16(tb) + align16(sb));    // [ntok][P]
    float* s_xw = s_hc + ((ntok * P + 3) & ~3);                                   // fused fold: [L][P]
    const uint32_t bar_a = smem_u32(&bar);

    if (tid == 0) {
        mbar_init(bar_a, 1);
        mbar_expect_tx(bar_a, tb + sb);
        bulk_g2s(smem_u32(s_tile), static_cast<const unsigned char*>(a.tile) + bh * tb, tb, bar_a);
        if (RF == kFP4) bulk_g2s(smem_u32(s_sc), a.tile_scales + bh * sb, sb, bar_a);
    }

    const TIn* xin = static_cast<const TIn*>(a.x);
    const TIn* Bin = static_cast<const TIn*>(a.B);
    const TIn* Cin = static_cast<const TIn*>(a.C);
    TIn* xb = static_cast<TIn*>(a.xbuf);
    TIn* bb = static_cast<TIn*>(a.bbuf);

    float4 c4[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j)
        c4[j] = (j < ntok) ? load4(Cin + ((static_cast<size_t>(b) * ntok + j) * G + g) * N + 4 * col4)
                           : make_float4(0.f, 0.f, 0.f, 0.f);

    const int pos = a.pos[b];
    const int T = pos + ntok;
    const bool ok = pos >= 0 && T <= cap;
    if (!ok && tid == 0) set_error(a.err, (pos < 0 || pos > cap) ? RSSM_DEVERR_POS_RANGE : RSSM_DEVERR_CAPACITY);
    __syncthreads();  // barrier initialised before anyone waits on it

    if (ok) {
        const float Ah = a.A[h];
        if (warp == 0) {
            float dts = 0.f;
            if (lane < T)
                dts = (lane < pos) ? a.dtbuf[bh * cap + lane]
                                   : a.dt[(static_cast<size_t>(b) * ntok + (lane - pos)) * H + h];
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
        // g[j][s] = B_s . C_j over the T slots (buffered ones and this call's)
        for (int s0 = warp * rpw; s0 < T; s0 += kWarps * rpw) {
            const int s = s0 + rsub;
            float4 bv = make_float4(0.f, 0.f, 0.f, 0.f);
            if (s < T)
                bv = (s < pos) ? load4(bb + ((static_cast<size_t>(b) * G + g) * cap + s) * N + 4 * col4)
                               : load4(Bin + ((static_cast<size_t>(b) * ntok + (s - pos)) * G + g) * N + 4 * col4);
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                if (j < ntok) {
                    const float d = group_sum(dot4(bv, c4[j]), lpr);
                    if (s < T && col4 == 0) s_g[j][s] = d;
                }
            }
        }
        // append this call's tokens at slots pos..pos+ntok-1
        for (int i = tid; i < ntok * P; i += kThreads) {
            const int j = i / P, p = i - j * P;
            xb[(bh * cap + pos + j) * P + p] = xin[((static_cast<size_t>(b) * ntok + j) * H + h) * P + p];
        }
        if (tid < ntok) a.dtbuf[bh * cap + pos + tid] = a.dt[(static_cast<size_t>(b) * ntok + tid) * H + h];
        if (h == g * hpg) {
            for (int i = tid; i < ntok * N; i += kThreads) {
                const int j = i / N, n = i - j * N;
                bb[((static_cast<size_t>(b) * G + g) * cap + pos + j) * N + n] =
                    Bin[((static_cast<size_t>(b) * ntok + j) * G + g) * N + n];
            }
        }
    }

    const bool arrived = mbar_wait_bounded(bar_a, 0, kWaitNs);
    if (__syncthreads_or(!arrived)) {
        if (tid == 0) set_error(a.err, RSSM_DEVERR_TIMEOUT);
        if (!arrived) mbar_wait_bounded(bar_a, 0, kWaitNs);
        return;
    }
    if (!ok) return;

    // h_ckpt . C_j for every row of the tile
    for (int r0 = warp * rpw; r0 < P; r0 += kWarps * rpw) {
        const int r = r0 + rsub;
        const float4 hv = (r < P) ? tile_load4<RF>(s_tile, s_sc, r, col4, N) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            if (j < ntok) {
                const float d = group_sum(dot4(hv, c4[j]), lpr);
                if (r < P && col4 == 0) s_hc[j * P + r] = d;
            }
        }
    }
    __syncthreads();

    const float Dh = a.D[h];
    for (int i = tid; i < ntok * P; i += kThreads) {
        const int j = i / P, p = i - j * P, t = pos + j;
        float acc = s_decay[j] * s_hc[j * P + p];
        for (int s = 0; s <= t; ++s) {
            const float xs = (s < pos) ? to_f32(xb[(bh * cap + s) * P + p])
                                       : to_f32(xin[((static_cast<size_t>(b) * ntok + (s - pos)) * H + h) * P + p]);
            acc = fmaf(s_w[j][s] * s_g[j][s], xs, acc);
        }
        const float xt = to_f32(xin[((static_cast<size_t>(b) * ntok + j) * H + h) * P + p]);
        a.y[((static_cast<size_t>(b) * ntok + j) * H + h) * P + p] = fmaf(Dh, xt, acc);
    }

    if (!a.advance) return;
    bool fold_now = false;
    if constexpr (RF == kF32 && NT == 1 && FUSED) {
        fold_now = (T == a.s.L);
        if (fold_now) {
            // fused flush: the token that fills the buffer also folds it into
            // the checkpoint, reusing the tile already in shared memory.
            for (int i = tid; i < T * P; i += kThreads) {
                const int s = i / P, p = i - s * P;
                const float xs = (s < pos) ? to_f32(xb[(bh * cap + s) * P + p])
                                           : to_f32(xin[(static_cast<size_t>(b) * H + h) * P + p]);
                s_xw[i] = s_w[0][s] * xs;
            }
            __syncthreads();
            float* dst = a.ckpt_w + bh * P * N;
            auto brow = [&](int s, int c) {
                return (s < pos) ? load4(bb + ((static_cast<size_t>(b) * G + g) * cap + s) * N + 4 * c)
                                 : load4(Bin + (static_cast<size_t>(b) * G + g) * N + 4 * c);
            };
            auto emit = [&](int r, int c, float4 v, bool valid) {
                if (valid) stream_store4(dst + r * N + 4 * c, v);
            };
            fold_rows(reinterpret_cast<float*>(s_tile), s_xw, P, N, lpr, T, s_decay[0], brow, emit);
        }
    }
    __syncthreads();
    if (tid == 0) request_done(a.arrive, b, H, a.pos, fold_now ? 0 : pos + 1, a.flush_count, fold_now);
}

// ---------------------------------------------------------------------------
// Fold of the buffer into the update copy: flush (s1) and precision-split
// refresh (s4). UF: format of the update copy (read and written); OUT4: also
// write the FP4 output copy from the fp32 result.
// ---------------------------------------------------------------------------
template <typename TIn, int UF, int OUT4>
__global__ void __launch_bounds__(kThreads) k_fold(const FoldArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bar;
    __shared__ float s_cw[kMaxCap];
    __shared__ float s_alpha;

    const int H = a.s.H, P = a.s.P, N = a.s.N, G = a.s.G, cap = a.s.cap, lpr = a.s.lpr;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x / H, h = blockIdx.x - b * H;
    const int g = h / (H / G);
    const size_t bh = static_cast<size_t>(b) * H + h;

    const int pos = a.pos[b];
    if (pos < 0 || pos > cap) {
        if (tid == 0) set_error(a.err, RSSM_DEVERR_POS_RANGE);
        return;
    }
    const bool go = (pos >= a.s.L) || (a.mode >= 1 && pos > 0) || (a.mode == 2);
    if (!go) return;
    const int T = pos;
    const uint32_t fc = a.flush_count[b];

    const uint32_t tb = tile_bytes(UF, P, N), sb = scale_bytes(UF, P, N);
    unsigned char* s_in = smem;
    unsigned char* s_insc = smem + align16(tb);
    unsigned char* after_in = smem + align16(tb) + align16(sb);
    float* s32 = (UF == kF32) ? reinterpret_cast<float*>(s_in) : reinterpret_cast<float*>(after_in);
    float* s_xw = reinterpret_cast<float*>(after_in + (UF == kF32 ? 0u : 4u * P * N));  // [T][P]
    const uint32_t bar_a = smem_u32(&bar);

    if (tid == 0) {
        mbar_init(bar_a, 1);
        mbar_expect_tx(bar_a, tb + sb);
        bulk_g2s(smem_u32(s_in), static_cast<const unsigned char*>(a.upd) + bh * tb, tb, bar_a);
        if (UF == kFP4) bulk_g2s(smem_u32(s_insc), a.upd_scales + bh * sb, sb, bar_a);
    }
    const float Ah = a.A[h];
    if (warp == 0) {
        const float dts = (lane < T) ? a.dtbuf[bh * cap + lane] : 0.f;
        const float Sx = warp_prefix(dts);
        const float Stot = T > 0 ? __shfl_sync(0xffffffffu, Sx, T - 1) : 0.f;
        s_cw[lane] = (lane < T) ? dts * expf(Ah * (Stot - Sx)) : 0.f;
        if (lane == 0) s_alpha = expf(Ah * Stot);
    }
    __syncthreads();
    const TIn* xb = static_cast<const TIn*>(a.xbuf);
    const TIn* bb = static_cast<const TIn*>(a.bbuf);
    for (int i = tid; i < T * P; i += kThreads) {
        const int s = i / P, p = i - s * P;
        s_xw[i] = s_cw[s] * to_f32(xb[(bh * cap + s) * P + p]);
    }

    const bool arrived = mbar_wait_bounded(bar_a, 0, kWaitNs);
    if (__syncthreads_or(!arrived)) {
        if (tid == 0) set_error(a.err, RSSM_DEVERR_TIMEOUT);
        if (!arrived) mbar_wait_bounded(bar_a, 0, kWaitNs);
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

    auto brow = [&](int s, int c) { return load4(bb + ((static_cast<size_t>(b) * G + g) * cap + s) * N + 4 * c); };
    auto emit = [&](int r, int c, float4 v, bool valid) {
        const size_t e = (bh * P + r) * N + 4 * c;  // flat element index of v.x
        if constexpr (UF == kF32) {
            if (valid) stream_store4(static_cast<float*>(a.upd) + e, v);
        } else if constexpr (UF == kBF16 || UF == kE4M3) {
            // Philox counter (e/4, head, request, flush_count), e within the head
            const uint32_t e_head = static_cast<uint32_t>(r * N + 4 * c);
            const uint4 rw = philox4x32_10(make_uint4(e_head >> 2, h, b, fc),
                                           make_uint2(static_cast<uint32_t>(a.seed),
                                                      static_cast<uint32_t>(a.seed >> 32)));
            if (valid) {
                if constexpr (UF == kBF16) {
                    const uint2 w = make_uint2(sr_bf16(v.x, rw.x) | (sr_bf16(v.y, rw.y) << 16),
                                               sr_bf16(v.z, rw.z) | (sr_bf16(v.w, rw.w) << 16));
                    *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.upd) + e) = w;
                } else {
                    const uint32_t w = sr_e4m3(v.x, rw.x) | (sr_e4m3(v.y, rw.y) << 8) |
                                       (sr_e4m3(v.z, rw.z) << 16) | (sr_e4m3(v.w, rw.w) << 24);
                    *reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(a.upd) + e) = w;
                }
            }
        } else {
            uint32_t sc;
            const uint32_t codes = fp4_quant_quad(v, &sc);
            if (valid) {
                *reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(a.upd) + e / 2) = static_cast<uint16_t>(codes);
                if ((c & 3) == 0) a.upd_scales[e / 16] = static_cast<uint8_t>(sc);
            }
        }
        if constexpr (OUT4 != 0) {
            uint32_t sc;
            const uint32_t codes = fp4_quant_quad(v, &sc);
            if (valid) {
                *reinterpret_cast<uint16_t*>(a.out_codes + e / 2) = static_cast<uint16_t>(codes);
                if ((c & 3) == 0) a.out_scales[e / 16] = static_cast<uint8_t>(sc);
            }
        }
    };
    fold_rows(s32, s_xw, P, N, lpr, T, s_alpha, brow, emit);
    __syncthreads();
    if (tid == 0) request_done(a.arrive, b, H, a.pos, 0, a.flush_count, true);
}

// ---------------------------------------------------------------------------
// Conventional scheme (in-run comparison, s1/s3): per token
//   h <- exp(dt A) h + dt x B^T, write h, y = h C + D x.
// VERIFY: read copy cur[b], write the state after token j to copy j.
// ---------------------------------------------------------------------------
template <typename TIn, int NT, int VERIFY>
__global__ void __launch_bounds__(kThreads) k_conv(const ConvArgs a) {
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
    __syncthreads();
    const bool arrived = mbar_wait_bounded(bar_a, 0, kWaitNs);
    if (__syncthreads_or(!arrived)) {
        if (tid == 0) set_error(a.err, RSSM_DEVERR_TIMEOUT);
        if (!arrived) mbar_wait_bounded(bar_a, 0, kWaitNs);
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
    if (op == 3) {
        // one lane per 4 values; quads of lanes make one 16-value block
        const int64_t q = i;  // group of 4 values
        const bool valid = 4 * q < n;
        const float4 x = valid ? reinterpret_cast<const float4*>(v)[q] : make_float4(0.f, 0.f, 0.f, 0.f);
        uint32_t sc;
        const uint32_t codes = fp4_quant_quad(x, &sc);
        if (valid) {
            uint8_t* o = static_cast<uint8_t*>(out);
            *reinterpret_cast<uint16_t*>(o + 2 * q) = static_cast<uint16_t>(codes);
            if ((q & 3) == 0) o[n / 2 + q / 4] = static_cast<uint8_t>(sc);
        }
        return;
    }
    if (i >= n) return;
    const uint4 rw = philox4x32_10(make_uint4(static_cast<uint32_t>(i >> 2), c1, c2, c3),
                                   make_uint2(static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32)));
    const uint32_t r = (i & 3) == 0 ? rw.x : (i & 3) == 1 ? rw.y : (i & 3) == 2 ? rw.z : rw.w;
    switch (op) {
        case 0: static_cast<uint16_t*>(out)[i] = static_cast<uint16_t>(sr_bf16(v[i], r)); break;
        case 1: static_cast<uint8_t*>(out)[i] = static_cast<uint8_t>(sr_e4m3(v[i], r)); break;
        case 2: static_cast<uint8_t*>(out)[i] = static_cast<uint8_t>(e4m3_rn(v[i])); break;
        default: static_cast<uint32_t*>(out)[i] = r; break;
    }
}

// ------------------------------------------------------------------ host

size_t replay_smem_bytes(const Shape& s, int rf, int ntok, int fused) {
    size_t b = align16(tile_bytes(rf, s.P, s.N)) + align16(scale_bytes(rf, s.P, s.N));
    b += 4u * static_cast<size_t>((ntok * s.P + 3) & ~3);
    if (fused) b += 4u * static_cast<size_t>(s.L) * s.P;
    return b;
}

size_t fold_smem_bytes(const Shape& s, int uf) {
    size_t b = align16(tile_bytes(uf, s.P, s.N)) + align16(scale_bytes(uf, s.P, s.N));
    if (uf != kF32) b += 4u * static_cast<size_t>(s.P) * s.N;
    b += 4u * static_cast<size_t>(s.cap) * s.P;
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
    kernel<<<nblk, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <typename TIn, int NT>
static cudaError_t replay_dispatch_fmt(const ReplayArgs& a, int rf, size_t smem, int nblk, cudaStream_t st) {
    switch (rf) {
        case kF32:
            if (NT == 1 && a.fused) return launch_tiles(k_replay<TIn, kF32, NT, 1>, a, nblk, smem, st);
            return launch_tiles(k_replay<TIn, kF32, NT, 0>, a, nblk, smem, st);
        case kBF16: return launch_tiles(k_replay<TIn, kBF16, NT, 0>, a, nblk, smem, st);
        case kE4M3: return launch_tiles(k_replay<TIn, kE4M3, NT, 0>, a, nblk, smem, st);
        default: return launch_tiles(k_replay<TIn, kFP4, NT, 0>, a, nblk, smem, st);
    }
}

cudaError_t launch_replay(const ReplayArgs& a, int in_bf16, int rf, cudaStream_t st) {
    const size_t smem = replay_smem_bytes(a.s, rf, a.ntok, a.fused);
    const int nblk = a.s.batch * a.s.H;
    if (a.ntok == 1)
        return in_bf16 ? replay_dispatch_fmt<__nv_bfloat16, 1>(a, rf, smem, nblk, st)
                       : replay_dispatch_fmt<float, 1>(a, rf, smem, nblk, st);
    return in_bf16 ? replay_dispatch_fmt<__nv_bfloat16, kMaxTok>(a, rf, smem, nblk, st)
                   : replay_dispatch_fmt<float, kMaxTok>(a, rf, smem, nblk, st);
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

cudaError_t launch_fold(const FoldArgs& a, int in_bf16, int uf, cudaStream_t st) {
    const size_t smem = fold_smem_bytes(a.s, uf);
    const int nblk = a.s.batch * a.s.H;
    return in_bf16 ? fold_dispatch<__nv_bfloat16>(a, uf, smem, nblk, st) : fold_dispatch<float>(a, uf, smem, nblk, st);
}

cudaError_t launch_conv(const ConvArgs& a, int in_bf16, int verify, cudaStream_t st) {
    const size_t smem = conv_smem_bytes(a.s);
    const int nblk = a.s.batch * a.s.H;
    if (!verify)
        return in_bf16 ? launch_tiles(k_conv<__nv_bfloat16, 1, 0>, a, nblk, smem, st)
                       : launch_tiles(k_conv<float, 1, 0>, a, nblk, smem, st);
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
    const int64_t items = (op == 3) ? n / 4 : n;
    const int64_t blocks = (items + 255) / 256;
    k_round_test<<<static_cast<unsigned>(blocks), 256, 0, st>>>(op, n, v, seed, c1, c2, c3, out);
    return cudaGetLastError();
}

}  // namespace rssm
