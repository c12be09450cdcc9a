/*
 * rssm_stage.h -- C ABI of the two element-wise steps of a Mamba-2 mixer
 * block that sit around the replay SSM step in a hybrid SSM/attention
 * decode stage (librssm.so).
 *
 * The ReplaySSM article (devotd.net "nvidia-replayssm-hybrid-model-ssm-
 * decoding-state-buffer", s2 "Reduce state transfers at large batch sizes")
 * reports the SSM-kernel gain diluted to a smaller decode-stage gain by the
 * rest of each layer. These calls let a synthetic stage be built around
 * rssm_decode_step / rssm_flush (or the conventional rssm_conv_step) with
 * the block's own glue on the GPU; the projections (GEMMs) and the
 * attention layers of such a stage are library calls of the caller. The
 * article gives no formula for the block: the steps follow the Mamba-2
 * mixer (Dao and Gu, "Transformers are SSMs", ICML 2024) -- a depthwise
 * causal conv1d of width 4 with SiLU on the x, B, C channels, dt =
 * softplus(dt_raw + dt_bias), and a gated RMS norm per group,
 * y * silu(z) / rms * w, before the output projection.
 *
 * Conventions are those of rssm.h: device pointers the caller owns, dense
 * row-major layouts, `stream` a cudaStream_t, host checks first (a bad
 * argument returns a status and launches nothing), no allocation, no
 * synchronisation. Shapes come from an rssm_desc_t (batch, nheads H,
 * head_dim P, d_state N, ngroups G); d_inner = H * P.
 *
 * Per request, the input projection's output row is
 *   zxbcdt [Dp] bf16, Dp = 2 d_inner + 2 G N + H:
 *   [ z (d_inner) | x (d_inner) | B (G N) | C (G N) | dt_raw (H) ].
 */
#ifndef RSSM_STAGE_H
#define RSSM_STAGE_H

#include "rssm.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Width of the causal conv1d (taps, including the current token). */
#define RSSM_STAGE_CONV_WIDTH 4

/* Conv step of one decode token: for each of the d_inner + 2 G N channels c
 * of [x | B | C] in zxbcdt (batch rows),
 *   o_c = conv_b[c] + sum_{k<3} conv_w[c][k] state[k][c] + conv_w[c][3] in_c,
 *   state <- (state[1], state[2], in_c),   out_c = silu(o_c) = o_c / (1 + exp(-o_c)),
 * written as bf16 into x [batch][H][P], B [batch][G][N], C [batch][G][N];
 * and dt [batch][H] float = softplus(dt_raw + dt_bias) (log(1 + exp(v)),
 * v itself above 20).
 *   zxbcdt      bf16 [batch][Dp] (read only)
 *   conv_state  bf16 [batch][3][d_inner + 2 G N] (read and updated; start at 0)
 *   conv_w      float [d_inner + 2 G N][4];  conv_b float [d_inner + 2 G N]
 *   dt_bias     float [H]
 * Requires in_dtype BF16. Errors: null pointer -> RSSM_ERR_INVALID_ARG. */
RSSM_API rssm_status_t rssm_stage_conv(const rssm_desc_t *desc, const void *zxbcdt, void *conv_state,
                                       const float *conv_w, const float *conv_b, const float *dt_bias,
                                       void *x, void *B, void *C, float *dt, void *stream);

/* Gated RMS norm per group of d_inner / G channels:
 *   g = y * silu(z),  out = g / sqrt(mean_group(g^2) + eps) * norm_w,
 * out bf16 [batch][d_inner] (the output projection's input).
 *   y       float [batch][d_inner] (the SSM step's output)
 *   zxbcdt  bf16 [batch][Dp] (z = its first d_inner entries)
 *   norm_w  float [d_inner];  eps > 0
 * Requires in_dtype BF16 and d_inner / G a multiple of 4. */
RSSM_API rssm_status_t rssm_stage_gate_norm(const rssm_desc_t *desc, const float *y, const void *zxbcdt,
                                            const float *norm_w, float eps, void *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* RSSM_STAGE_H */
