// rssm_stage.cu -- the element-wise steps of a Mamba-2 mixer block around
// the replay SSM step (include/rssm_stage.h): the causal conv1d + SiLU of
// the x, B, C channels with the dt softplus, and the gated RMS norm. Both
// are memory-bound passes over a few MB per decode token; one thread per
// channel (conv) and one CTA per (request, norm group) (gate norm).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rssm.h"
#include "rssm_stage.h"

namespace {

constexpr int kTaps = RSSM_STAGE_CONV_WIDTH;  // 4: three past inputs + the current one
constexpr int kConvThreads = 256;
constexpr int kNormThreads = 128;

__device__ __forceinline__ float bf(const __nv_bfloat16 v) { return __bfloat162float(v); }

// x, B, C channels c < din + 2 gn of request blockIdx.y; then the H dt lanes.
__global__ void k_stage_conv(int din, int gn, int H, const __nv_bfloat16* __restrict__ zx,
                             __nv_bfloat16* __restrict__ state, const float* __restrict__ w,
                             const float* __restrict__ bias, const float* __restrict__ dt_bias,
                             __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ Bo,
                             __nv_bfloat16* __restrict__ Co, float* __restrict__ dt) {
    const int chans = din + 2 * gn;
    const size_t b = blockIdx.y;
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    const size_t Dp = 2 * static_cast<size_t>(din) + 2 * gn + H;
    const __nv_bfloat16* row = zx + b * Dp;
    if (c < chans) {
        const __nv_bfloat16 raw = row[din + c];
        __nv_bfloat16* st = state + b * (kTaps - 1) * chans + c;
        const __nv_bfloat16 r0 = st[0], r1 = st[chans], r2 = st[2 * chans];
        const float* wc = w + static_cast<size_t>(kTaps) * c;
        float o = bias[c];
        o = fmaf(wc[0], bf(r0), o);
        o = fmaf(wc[1], bf(r1), o);
        o = fmaf(wc[2], bf(r2), o);
        o = fmaf(wc[3], bf(raw), o);
        st[0] = r1;
        st[chans] = r2;
        st[2 * chans] = raw;
        const __nv_bfloat16 a = __float2bfloat16_rn(o / (1.0f + expf(-o)));
        if (c < din)
            x[b * din + c] = a;
        else if (c < din + gn)
            Bo[b * gn + (c - din)] = a;
        else
            Co[b * gn + (c - din - gn)] = a;
    } else if (c < chans + H) {
        const int h = c - chans;
        const float v = bf(row[2 * din + 2 * gn + h]) + dt_bias[h];
        dt[b * H + h] = v > 20.0f ? v : log1pf(expf(v));
    }
}

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kNormThreads / 32; ++i) s += red[i];
    return s;
}

// group blockIdx.x of request blockIdx.y: gs = din / G channels
__global__ void k_stage_gate_norm(int din, int G, int Dp, const float* __restrict__ y,
                                  const __nv_bfloat16* __restrict__ zx, const float* __restrict__ nw, float eps,
                                  __nv_bfloat16* __restrict__ out) {
    __shared__ float red[kNormThreads / 32];
    const int gs = din / G;
    const size_t b = blockIdx.y;
    const size_t off = static_cast<size_t>(blockIdx.x) * gs;
    const float* yr = y + b * din + off;
    const __nv_bfloat16* zr = zx + b * Dp + off;
    auto gated = [&](int i) {
        const float z = bf(zr[i]);
        return yr[i] * (z / (1.0f + expf(-z)));
    };
    float ss = 0.f;
    for (int i = threadIdx.x; i < gs; i += kNormThreads) {
        const float g = gated(i);
        ss = fmaf(g, g, ss);
    }
    const float inv = rsqrtf(block_sum(ss, red) / static_cast<float>(gs) + eps);
    for (int i = threadIdx.x; i < gs; i += kNormThreads)
        out[b * din + off + i] = __float2bfloat16_rn(gated(i) * inv * nw[off + i]);
}

rssm_status_t stage_shape_ok(const rssm_desc_t* d) {
    if (!d) return RSSM_ERR_INVALID_ARG;
    if (d->batch < 1 || d->nheads < 1 || d->head_dim < 1 || d->d_state < 1 || d->ngroups < 1)
        return RSSM_ERR_SHAPE;
    if (d->nheads % d->ngroups != 0) return RSSM_ERR_SHAPE;
    if (d->in_dtype != RSSM_BF16) return RSSM_ERR_UNSUPPORTED;
    if (static_cast<long long>(d->batch) > 65535) return RSSM_ERR_SHAPE;
    return RSSM_OK;
}

}  // namespace

extern "C" {

rssm_status_t rssm_stage_conv(const rssm_desc_t* d, const void* zxbcdt, void* conv_state, const float* conv_w,
                              const float* conv_b, const float* dt_bias, void* x, void* B, void* C, float* dt,
                              void* stream) {
    rssm_status_t s = stage_shape_ok(d);
    if (s != RSSM_OK) return s;
    if (!zxbcdt || !conv_state || !conv_w || !conv_b || !dt_bias || !x || !B || !C || !dt)
        return RSSM_ERR_INVALID_ARG;
    const int din = d->nheads * d->head_dim, gn = d->ngroups * d->d_state, H = d->nheads;
    const int lanes = din + 2 * gn + H;
    const dim3 grid((lanes + kConvThreads - 1) / kConvThreads, static_cast<unsigned>(d->batch));
    k_stage_conv<<<grid, kConvThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        din, gn, H, static_cast<const __nv_bfloat16*>(zxbcdt), static_cast<__nv_bfloat16*>(conv_state), conv_w,
        conv_b, dt_bias, static_cast<__nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(B),
        static_cast<__nv_bfloat16*>(C), dt);
    return cudaGetLastError() == cudaSuccess ? RSSM_OK : RSSM_ERR_CUDA;
}

rssm_status_t rssm_stage_gate_norm(const rssm_desc_t* d, const float* y, const void* zxbcdt, const float* norm_w,
                                   float eps, void* out, void* stream) {
    rssm_status_t s = stage_shape_ok(d);
    if (s != RSSM_OK) return s;
    if (!y || !zxbcdt || !norm_w || !out) return RSSM_ERR_INVALID_ARG;
    if (!(eps > 0.0f)) return RSSM_ERR_INVALID_ARG;
    const int din = d->nheads * d->head_dim, G = d->ngroups;
    if ((din / G) % 4 != 0) return RSSM_ERR_SHAPE;
    const int Dp = 2 * din + 2 * G * d->d_state + d->nheads;
    const dim3 grid(static_cast<unsigned>(G), static_cast<unsigned>(d->batch));
    k_stage_gate_norm<<<grid, kNormThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        din, G, Dp, y, static_cast<const __nv_bfloat16*>(zxbcdt), norm_w, eps, static_cast<__nv_bfloat16*>(out));
    return cudaGetLastError() == cudaSuccess ? RSSM_OK : RSSM_ERR_CUDA;
}

}  // extern "C"
