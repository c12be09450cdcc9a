/*
 * rssm.h -- C ABI of librssm: replay-based decoding of the state-space (SSM)
 * layers of hybrid SSM/attention models on NVIDIA B200 (sm_100a).
 *
 * Method: the ReplaySSM article (devotd.net news page
 * "nvidia-replayssm-hybrid-model-ssm-decoding-state-buffer", English
 * version), sections
 *   s1 "Store recent inputs instead of the full state"
 *   s3 "Roll back incorrect predictions using buffer positions"
 *   s4 "Prevent low-precision errors from accumulating again".
 * The article fixes the idea; the concrete layer is a Mamba-2-style selective
 * SSM with one scalar decay per head h, head_dim P, d_state N, and G groups
 * of H/G consecutive heads sharing B and C:
 *     a_t = exp(dt_t A_h),  h_t = a_t h_{t-1} + dt_t x_t B_t^T,  y_t = h_t C_t + D_h x_t.
 * Per request the library keeps a checkpoint of h taken at the start of an
 * interval of L tokens plus a buffer of the inputs since then (x, B, dt; C
 * is per token and is not kept). Every token reads the checkpoint once and
 * replays the buffer; the checkpoint is rewritten only when the buffer
 * fills (s1):
 *     y_t = exp(A S_t) (h_ckpt C_t) + sum_{s<=t} dt_s exp(A (S_t - S_s)) (B_s . C_t) x_s + D x_t,
 *     S_t = sum_{r<=t} dt_r over the interval.
 *
 * Conventions for every call:
 *  - All array arguments are DEVICE pointers into memory the caller owns
 *    (e.g. allocated through PyTorch). The library never allocates, frees or
 *    synchronises; rssm_get_error is the only call that waits (on its
 *    stream). Sizes come from rssm_state_field_bytes.
 *  - Inputs are read-only; layouts are dense and row-major as documented.
 *    Device pointers must be 16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Work is
 *    enqueued asynchronously; one state must be used from one stream. The
 *    persistent kernels (decode, verify, flush, refresh at d_state 128) are
 *    launched with programmatic stream serialization: they wait for the
 *    previous kernel's writes on entry, and the next kernel on the stream may
 *    begin launching before they finish. Calls can be captured in CUDA graphs.
 *  - Arguments the host can check are checked before anything is launched;
 *    a bad one returns a status and launches nothing.
 *  - Kernels that find bad device state (a buffer position out of range, an
 *    accepted count out of range) write the first error code into
 *    state->err and leave that request untouched. They never trap, assert
 *    or spin without a bound. rssm_get_error reads and clears the word.
 */
#ifndef RSSM_H
#define RSSM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RSSM_ABI_VERSION 2

#if defined(__GNUC__)
#define RSSM_API __attribute__((visibility("default")))
#else
#define RSSM_API
#endif

typedef enum rssm_status {
    RSSM_OK = 0,
    RSSM_ERR_INVALID_ARG = 1,  /* null pointer or bad enum value */
    RSSM_ERR_SHAPE = 2,        /* sizes inconsistent or outside the supported range */
    RSSM_ERR_UNSUPPORTED = 3,  /* valid but not implemented combination */
    RSSM_ERR_CAPACITY = 4,     /* more tokens than the buffer can ever hold */
    RSSM_ERR_CUDA = 5,         /* a CUDA runtime call failed */
    RSSM_ERR_DEVICE = 6        /* rssm_get_error: a kernel reported bad device state */
} rssm_status_t;

/* Element formats. F32/BF16 for inputs and the update copy; E4M3 (OCP fp8)
 * for the update copy; FP4 = e2m1 codes with one e4m3 scale per 16
 * contiguous d_state elements. */
typedef enum rssm_dtype { RSSM_F32 = 0, RSSM_BF16 = 1, RSSM_E4M3 = 2, RSSM_FP4 = 3 } rssm_dtype_t;

typedef enum rssm_outcopy { RSSM_OUTCOPY_NONE = 0, RSSM_OUTCOPY_FP4 = 1 } rssm_outcopy_t;

/* Codes a kernel writes into state->err (first error wins). */
enum {
    RSSM_DEVERR_NONE = 0,
    RSSM_DEVERR_POS_RANGE = 1,    /* pos[b] < 0 or > capacity */
    RSSM_DEVERR_CAPACITY = 2,     /* pos[b] + tokens > capacity */
    RSSM_DEVERR_ACCEPT_RANGE = 3, /* accepted count outside 0..K */
    RSSM_DEVERR_TIMEOUT = 4       /* a bulk copy did not complete within its bound */
};

/* desc.flags */
#define RSSM_FLAG_FUSED_FLUSH 1u  /* rssm_decode_step folds the buffer itself on the
                                     token that fills it (fp32 state only) */

/* Layer description. Supported: batch >= 1; nheads % ngroups == 0;
 * d_state in {16, 32, 64, 128}; 1 <= head_dim <= 256;
 * head_dim * d_state <= 16384; 1 <= interval; capacity = interval +
 * max_draft <= 32; FP4 state or copy needs head_dim * d_state % 256 == 0. */
typedef struct rssm_desc {
    int32_t batch;        /* requests */
    int32_t nheads;       /* H */
    int32_t head_dim;     /* P */
    int32_t d_state;      /* N */
    int32_t ngroups;      /* G */
    int32_t interval;     /* L: tokens per checkpoint interval (16 in the article) */
    int32_t max_draft;    /* K: most draft tokens per verify; buffer capacity L + K */
    int32_t in_dtype;     /* RSSM_F32 or RSSM_BF16: x, B, C and the buffered x, B */
    int32_t update_dtype; /* update copy: F32; BF16 or E4M3 (stochastic rounding);
                             FP4 = one FP4 copy both read and updated (the
                             shared-low-precision control of s4) */
    int32_t out_copy;     /* RSSM_OUTCOPY_FP4: separate FP4 output copy (s4), read by
                             decode/verify; requires update_dtype != FP4 */
    uint32_t flags;       /* RSSM_FLAG_* */
    uint32_t reserved;    /* must be 0 */
    uint64_t seed;        /* Philox key of the stochastic rounding */
} rssm_desc_t;

/* Fields of the per-layer state, for rssm_state_field_bytes. Cap = L + K,
 * CapR = Cap rounded up to a multiple of 4.
 *
 * RECORD: one record of rssm_record_layout().bytes per (request b, head h),
 * record (b, h) at byte b*H*bytes + h*bytes, holding
 *   - at 0: the copy that outputs read, P x N row-major: the fp32 checkpoint;
 *     the bf16 / e4m3 update copy when that is also what decode reads; or FP4
 *     codes (element 2k in the low nibble of byte k) followed, at
 *     .scales_offset, by one e4m3 scale per 16 contiguous d_state elements --
 *     the FP4 output copy (out_copy) or the shared FP4 copy (update FP4);
 *   - at .dt_offset: the buffered dt, CapR floats (slots 0..Cap-1 used);
 *   - at .x_offset: the buffered x, Cap rows of P elements of in_dtype.
 * Keeping a head's tile, dt and x contiguous lets a decode fetch all three
 * with one bulk copy.
 * CKPT: the update copy, only when it is not what decode reads (out_copy
 *   FP4 with update_dtype F32/BF16/E4M3): [batch][H][P][N] of update_dtype.
 * BBUF: buffered B, [batch][G][Cap][N] of in_dtype. */
typedef enum rssm_field {
    RSSM_FIELD_RECORD = 0,
    RSSM_FIELD_CKPT,
    RSSM_FIELD_BBUF,
    RSSM_FIELD_POS,            /* int32 [batch]: valid buffer length */
    RSSM_FIELD_FLUSH_COUNT,    /* uint32 [batch]: refreshes so far (Philox counter word) */
    RSSM_FIELD_ARRIVE,         /* uint32 [batch]: scratch, must be zero before first use;
                                  every call leaves it zero */
    RSSM_FIELD_ERR,            /* int32 [1]: device error word, zero-initialised */
    RSSM_NUM_FIELDS
} rssm_field_t;

/* Byte geometry of one record (see RSSM_FIELD_RECORD). */
typedef struct rssm_record_layout {
    uint64_t bytes;          /* record size, a multiple of 128 */
    uint64_t tile_bytes;     /* bytes of the read copy's values (FP4: codes) */
    uint64_t scales_offset;  /* FP4 scales (0 when the read copy is not FP4) */
    uint64_t dt_offset;      /* buffered dt */
    uint64_t x_offset;       /* buffered x */
} rssm_record_layout_t;

/* Unused fields may be NULL. */
typedef struct rssm_state {
    void *record;
    void *ckpt;
    void *bbuf;
    int32_t *pos;
    uint32_t *flush_count;
    uint32_t *arrive;
    int32_t *err;
} rssm_state_t;

/* ABI version (RSSM_ABI_VERSION). */
RSSM_API int rssm_abi_version(void);

/* Static text for a status. Never NULL. */
RSSM_API const char *rssm_status_string(rssm_status_t s);

/* Validates a description: RSSM_OK, or the status any call would return. */
RSSM_API rssm_status_t rssm_check_desc(const rssm_desc_t *desc);

/* Bytes of one state field for this description; 0 when the field is unused
 * or the description is invalid. Host-only; touches no device. */
RSSM_API size_t rssm_state_field_bytes(const rssm_desc_t *desc, int32_t field);

/* Geometry of one record for this description. Host-only. */
RSSM_API rssm_status_t rssm_record_layout(const rssm_desc_t *desc, rssm_record_layout_t *out);

/* Standard decode of one token per request (s1): appends (x, B, dt) at
 * slot pos[b], writes y, advances pos[b] by one. Reads the record's copy
 * (the checkpoint, or the FP4 output copy) once; writes no state except the
 * buffer slot. The caller calls rssm_flush / rssm_lowprec_refresh once
 * pos reaches the interval, unless RSSM_FLAG_FUSED_FLUSH is set, in which
 * case the token that fills the buffer also folds it and resets pos.
 *   x [batch][H][P], B and C [batch][G][N] (in_dtype); dt [batch][H]
 *   (float, already softplus-ed, > 0); A, D [H] float; y [batch][H][P] float.
 * Device errors: pos[b] + 1 > capacity. */
RSSM_API rssm_status_t rssm_decode_step(const rssm_desc_t *desc, const rssm_state_t *state,
                               const void *x, const void *B, const void *C,
                               const float *dt, const float *A, const float *D,
                               float *y, void *stream);

/* Interval flush of an fp32 state (s1): for every request with
 * pos[b] >= interval (all requests with pos[b] > 0 when force != 0), fold
 * the pos[b] buffered entries into the checkpoint in one read-modify-write
 *     h <- exp(A S) h + sum_s dt_s exp(A (S - S_s)) x_s B_s^T,  S = sum of the pos dt,
 * then pos[b] = 0 and flush_count[b] += 1. Other requests are untouched.
 * A [H] float: the same decay parameters the decode calls received.
 * Requires update_dtype F32 and no output copy (else RSSM_ERR_UNSUPPORTED;
 * use rssm_lowprec_refresh). */
RSSM_API rssm_status_t rssm_flush(const rssm_desc_t *desc, const rssm_state_t *state, const float *A,
                         int32_t force, void *stream);

/* Largest batch rssm_decode_step_noalloc accepts. */
#define RSSM_NOALLOC_MAX_BATCH 65536

/* rssm_decode_step for callers that cannot allocate device memory -- for
 * example an engine that plans all of its device memory ahead and hands each
 * layer only the buffers it planned, or a process whose allocator is owned by
 * another runtime. The article has no counterpart: this is an interface
 * variant of this library, not a step of the method.
 * Same arguments, results and errors as rssm_decode_step, except that
 * state->arrive is not used (it may be NULL): the per-request arrival
 * counters live in a file-scope device array of RSSM_NOALLOC_MAX_BATCH
 * uint32 (256 KiB) that every GPU loading the library holds until the
 * process exits. The call allocates nothing: it clears the counters it uses
 * with cudaMemsetAsync on `stream` and launches the decode kernel.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture. The address is cached per device for the
 *    life of the process: after a device reset, reload the library.
 *  - All calls share the one array: calls whose work overlaps on the GPU
 *    (other streams, concurrent graphs) race on it. Serialise them.
 *  - batch > RSSM_NOALLOC_MAX_BATCH returns RSSM_ERR_CAPACITY and launches
 *    nothing.
 *  - Only the decode step has this variant. rssm_flush, rssm_lowprec_refresh
 *    and rssm_verify still need state->arrive, so a caller that cannot
 *    allocate at all runs allocation-free from start to end only with an
 *    fp32 state (update_dtype F32, no output copy) and RSSM_FLAG_FUSED_FLUSH,
 *    where the decode step itself folds the buffer. */
RSSM_API rssm_status_t rssm_decode_step_noalloc(const rssm_desc_t *desc, const rssm_state_t *state,
                                                const void *x, const void *B, const void *C,
                                                const float *dt, const float *A, const float *D,
                                                float *y, void *stream);

/* Speculative verify (s3): writes the K+1 tokens (the pending token j = 0
 * and K drafts) into slots pos..pos+K and computes their outputs from one
 * read of the checkpoint. pos is NOT advanced and no state is created.
 *   x [batch][K+1][H][P], B and C [batch][K+1][G][N], dt [batch][K+1][H],
 *   y [batch][K+1][H][P].
 * 0 <= K <= max_draft, else RSSM_ERR_CAPACITY. Device error: pos + K + 1 >
 * capacity. */
RSSM_API rssm_status_t rssm_verify(const rssm_desc_t *desc, const rssm_state_t *state, int32_t K,
                          const void *x, const void *B, const void *C, const float *dt,
                          const float *A, const float *D, float *y, void *stream);

/* Accept after verify (s3): pos[b] += n_accepted[b] + 1, which marks the
 * pending token and the first n accepted drafts valid and drops the rest.
 * n_accepted: device int32 [batch], each in 0..max_draft (else device error,
 * request untouched). Follow with rssm_flush / rssm_lowprec_refresh
 * (force = 0), which fold requests whose pos reached the interval. */
RSSM_API rssm_status_t rssm_accept(const rssm_desc_t *desc, const rssm_state_t *state,
                          const int32_t *n_accepted, void *stream);

/* Precision-split refresh (s4): as rssm_flush, on the low-precision state.
 * Widens the update copy to fp32, folds the buffer, then
 *   - BF16/E4M3 update copy: stochastic rounding with Philox4x32-10, key
 *     (lo32(seed), hi32(seed)), counter (e/4, h, b, flush_count[b]), word
 *     e%4, e = p*N + n; up iff r < floor(frac * 2^32);
 *   - F32 update copy: stored as computed;
 *   - FP4 update copy (shared control): re-quantised to nearest;
 *   - FP4 output copy (out_copy): quantised from the fp32 result, before
 *     stochastic rounding: scale = e4m3_rn(amax/6) per 16 elements, codes =
 *     e2m1_rn(v / scale), all zero when the scale is zero.
 * With force != 0 every request is refreshed, including pos[b] == 0, which
 * (re)builds the output copy from the update copy. */
RSSM_API rssm_status_t rssm_lowprec_refresh(const rssm_desc_t *desc, const rssm_state_t *state,
                                   const float *A, int32_t force, void *stream);

/* Prefill of a prompt into the checkpoint -- the step before the decode path,
 * on which the article is silent: for every request, folds T0 prompt tokens
 * into the fp32 checkpoint with an empty buffer, chunk by chunk,
 *     h <- exp(A S) h + sum_{t<T0} dt_t exp(A (S - S_t)) x_t B_t^T,  S = sum of the T0 dt,
 * which is the conventional recurrence over the prompt, started from the
 * current checkpoint (zero it first for a fresh request). pos stays 0,
 * flush_count is unchanged; no outputs are produced.
 *   x [T0][batch][H][P], B [T0][batch][G][N] (in_dtype); dt [T0][batch][H]
 *   float (softplus-ed); A [H] float.
 * Requires an fp32 state (update_dtype F32, no output copy), else
 * RSSM_ERR_UNSUPPORTED; T0 >= 0. Device error: pos[b] != 0 (request untouched). */
RSSM_API rssm_status_t rssm_prefill(const rssm_desc_t *desc, const rssm_state_t *state, int32_t T0,
                                    const void *x, const void *B, const float *dt, const float *A,
                                    void *stream);

/* Conventional decode step, the in-run comparison (s1: read and write the
 * whole state every token): h <- a h + dt x B^T; y = h C + D x.
 * h [batch][H][P][N] float, updated in place; other arguments as in
 * rssm_decode_step. Uses only the shape fields of desc. */
RSSM_API rssm_status_t rssm_conv_step(const rssm_desc_t *desc, float *h, const void *x, const void *B,
                             const void *C, const float *dt, const float *A, const float *D,
                             float *y, void *stream);

/* Conventional speculative verify (s3: one state copy per token for
 * rollback): reads state copy cur[b] of copies [K+1][batch][H][P][N] and
 * writes the state after token j into copy j, for j = 0..K, with outputs
 * y [batch][K+1][H][P]. cur: device int32 [batch], each in 0..K. */
RSSM_API rssm_status_t rssm_conv_verify(const rssm_desc_t *desc, float *copies, const int32_t *cur,
                               int32_t K, const void *x, const void *B, const void *C,
                               const float *dt, const float *A, const float *D, float *y,
                               void *stream);

/* Conventional accept: cur[b] = n_accepted[b] (the copy after the last
 * accepted token becomes the state; nothing is copied). Values outside 0..K
 * leave cur[b] unchanged and set *err (err may be NULL). */
RSSM_API rssm_status_t rssm_conv_accept(const rssm_desc_t *desc, const int32_t *n_accepted, int32_t *cur,
                               int32_t K, int32_t *err, void *stream);

/* Reads and clears the device error word; waits for the stream first.
 * *host_code receives the RSSM_DEVERR_* value. Returns RSSM_ERR_DEVICE when
 * it was non-zero. */
RSSM_API rssm_status_t rssm_get_error(const rssm_desc_t *desc, const rssm_state_t *state,
                             int32_t *host_code, void *stream);

/* Rounding functions of the refresh, exposed for bit-exact testing on the
 * device code the refresh itself runs. For n input floats v:
 *   op 0: SR to bf16      -> uint16 out[n]   (Philox counter (e/4, c1, c2, c3))
 *   op 1: SR to e4m3      -> uint8  out[n]   (same counter)
 *   op 2: e4m3 nearest-even, saturating -> uint8 out[n]
 *   op 3: FP4 block copy  -> uint8 out[n/2] codes, then uint8 out[n/2 + n/16] scales
 *   op 4: Philox word e%4 at (e/4, c1, c2, c3)  -> uint32 out[n]
 *   op 5: FP4 block copy, then decoded the way FP4-reading kernels decode it
 *         -> float out[n]
 * n must be a multiple of 16 for ops 3 and 5. */
RSSM_API rssm_status_t rssm_round_test(int32_t op, int64_t n, const float *v, uint64_t seed, uint32_t c1,
                              uint32_t c2, uint32_t c3, void *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* RSSM_H */
