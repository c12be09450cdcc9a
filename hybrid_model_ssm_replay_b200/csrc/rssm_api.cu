// rssm_api.cu -- the C ABI of librssm (declared in include/rssm.h).
//
// Each entry point validates its arguments on the host first (no CUDA call
// happens before that), then fills an argument block and enqueues kernels
// on the caller's stream. Nothing here allocates, frees or synchronises,
// except rssm_get_error, which waits for its stream.
#include <cuda_runtime.h>

#include "rssm.h"
#include "rssm_internal.h"

using namespace rssm;

namespace {

constexpr int kMaxTokens = 8;  // K + 1 per verify call

bool fmt_ok_input(int d) { return d == RSSM_F32 || d == RSSM_BF16; }
bool fmt_ok_update(int d) { return d >= RSSM_F32 && d <= RSSM_FP4; }

int cap_of(const rssm_desc_t* d) { return d->interval + d->max_draft; }

rssm_status_t check_shape_only(const rssm_desc_t* d) {
    if (!d) return RSSM_ERR_INVALID_ARG;
    if (d->batch < 1 || d->nheads < 1 || d->ngroups < 1 || d->head_dim < 1) return RSSM_ERR_SHAPE;
    if (d->nheads % d->ngroups != 0) return RSSM_ERR_SHAPE;
    const int N = d->d_state;
    if (N != 16 && N != 32 && N != 64 && N != 128) return RSSM_ERR_SHAPE;
    if (d->head_dim > 256 || d->head_dim * N > 16384) return RSSM_ERR_SHAPE;
    if (static_cast<long long>(d->batch) * d->nheads > 0x7fffffffLL) return RSSM_ERR_SHAPE;
    if (!fmt_ok_input(d->in_dtype)) return RSSM_ERR_INVALID_ARG;
    return RSSM_OK;
}

Shape shape_of(const rssm_desc_t* d) {
    Shape s;
    s.batch = d->batch;
    s.H = d->nheads;
    s.P = d->head_dim;
    s.N = d->d_state;
    s.G = d->ngroups;
    s.L = d->interval;
    s.cap = cap_of(d);
    s.lpr = d->d_state / 4;
    s.capr = (s.cap + 3) & ~3;
    return s;
}

rssm_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? RSSM_OK : RSSM_ERR_CUDA; }

// Format of the copy that outputs read (s4: the FP4 output copy when there
// is one, else the update copy itself); it is the copy a record holds.
int read_format(const rssm_desc_t* d) { return d->out_copy == RSSM_OUTCOPY_FP4 ? kFP4 : d->update_dtype; }

RecLayout rec_of(const rssm_desc_t* d) {
    return record_layout(shape_of(d), read_format(d), d->in_dtype == RSSM_BF16 ? 2 : 4);
}

// The update copy lives outside the records only beside an FP4 output copy.
bool separate_ckpt(const rssm_desc_t* d) { return d->out_copy == RSSM_OUTCOPY_FP4; }

rssm_status_t check_state_fields(const rssm_desc_t* d, const rssm_state_t* st, bool need_arrive) {
    if (!st) return RSSM_ERR_INVALID_ARG;
    if (!st->record || !st->bbuf || !st->pos || !st->flush_count || !st->err) return RSSM_ERR_INVALID_ARG;
    if (need_arrive && !st->arrive) return RSSM_ERR_INVALID_ARG;
    if (separate_ckpt(d) && !st->ckpt) return RSSM_ERR_INVALID_ARG;
    return RSSM_OK;
}

rssm_status_t check_state_common(const rssm_desc_t* d, const rssm_state_t* st) {
    return check_state_fields(d, st, true);
}

}  // namespace

extern "C" {

int rssm_abi_version(void) { return RSSM_ABI_VERSION; }

const char* rssm_status_string(rssm_status_t s) {
    switch (s) {
        case RSSM_OK: return "ok";
        case RSSM_ERR_INVALID_ARG: return "invalid argument";
        case RSSM_ERR_SHAPE: return "unsupported or inconsistent shape";
        case RSSM_ERR_UNSUPPORTED: return "unsupported combination";
        case RSSM_ERR_CAPACITY: return "more tokens than the buffer capacity";
        case RSSM_ERR_CUDA: return "CUDA error";
        case RSSM_ERR_DEVICE: return "device-side error reported";
        default: return "unknown status";
    }
}

rssm_status_t rssm_check_desc(const rssm_desc_t* d) {
    rssm_status_t s = check_shape_only(d);
    if (s != RSSM_OK) return s;
    if (d->interval < 1 || d->max_draft < 0) return RSSM_ERR_SHAPE;
    if (cap_of(d) > 32 || d->max_draft + 1 > kMaxTokens) return RSSM_ERR_SHAPE;
    if (!fmt_ok_update(d->update_dtype)) return RSSM_ERR_INVALID_ARG;
    if (d->out_copy != RSSM_OUTCOPY_NONE && d->out_copy != RSSM_OUTCOPY_FP4) return RSSM_ERR_INVALID_ARG;
    if (d->reserved != 0 || (d->flags & ~RSSM_FLAG_FUSED_FLUSH) != 0) return RSSM_ERR_INVALID_ARG;
    if (d->out_copy == RSSM_OUTCOPY_FP4 && d->update_dtype == RSSM_FP4) return RSSM_ERR_UNSUPPORTED;
    const bool fp4 = d->update_dtype == RSSM_FP4 || d->out_copy == RSSM_OUTCOPY_FP4;
    if (fp4 && (d->head_dim * d->d_state) % 256 != 0) return RSSM_ERR_SHAPE;
    if ((d->flags & RSSM_FLAG_FUSED_FLUSH) &&
        (d->update_dtype != RSSM_F32 || d->out_copy != RSSM_OUTCOPY_NONE || d->interval > 16))
        return RSSM_ERR_UNSUPPORTED;
    return RSSM_OK;
}

rssm_status_t rssm_record_layout(const rssm_desc_t* d, rssm_record_layout_t* out) {
    rssm_status_t s = rssm_check_desc(d);
    if (s != RSSM_OK) return s;
    if (!out) return RSSM_ERR_INVALID_ARG;
    const RecLayout r = rec_of(d);
    out->bytes = r.bytes;
    out->tile_bytes = r.tile;
    out->scales_offset = r.scales;
    out->dt_offset = r.dt;
    out->x_offset = r.x;
    return RSSM_OK;
}

size_t rssm_state_field_bytes(const rssm_desc_t* d, int32_t field) {
    if (rssm_check_desc(d) != RSSM_OK) return 0;
    const size_t Bz = d->batch, H = d->nheads, P = d->head_dim, N = d->d_state, G = d->ngroups;
    const size_t cap = cap_of(d);
    const size_t in_el = d->in_dtype == RSSM_BF16 ? 2 : 4;
    const size_t n_state = Bz * H * P * N;
    switch (field) {
        case RSSM_FIELD_RECORD: return Bz * H * rec_of(d).bytes;
        case RSSM_FIELD_CKPT:
            if (!separate_ckpt(d)) return 0;
            switch (d->update_dtype) {
                case RSSM_F32: return 4 * n_state;
                case RSSM_BF16: return 2 * n_state;
                default: return n_state;  // E4M3 (an FP4 update copy has no separate output copy)
            }
        case RSSM_FIELD_BBUF: return Bz * G * cap * N * in_el;
        case RSSM_FIELD_POS: return Bz * 4;
        case RSSM_FIELD_FLUSH_COUNT: return Bz * 4;
        case RSSM_FIELD_ARRIVE: return Bz * 4;
        case RSSM_FIELD_ERR: return 4;
        default: return 0;
    }
}

static rssm_status_t replay_call(const rssm_desc_t* d, const rssm_state_t* st, int ntok, int advance,
                                 const void* x, const void* B, const void* C, const float* dt, const float* A,
                                 const float* D, float* y, void* stream) {
    ReplayArgs a;
    a.s = shape_of(d);
    a.ntok = ntok;
    a.advance = advance;
    a.fused = advance && (d->flags & RSSM_FLAG_FUSED_FLUSH) ? 1 : 0;
    const int rf = read_format(d);
    a.rec = rec_of(d);
    a.record = static_cast<unsigned char*>(st->record);
    a.bbuf = st->bbuf;
    a.pos = st->pos;
    a.flush_count = st->flush_count;
    a.arrive = st->arrive;
    a.err = st->err;
    a.x = x;
    a.B = B;
    a.C = C;
    a.dt = dt;
    a.A = A;
    a.D = D;
    a.y = y;
    return cuda_status(launch_replay(a, d->in_dtype == RSSM_BF16, rf, static_cast<cudaStream_t>(stream)));
}

rssm_status_t rssm_decode_step(const rssm_desc_t* d, const rssm_state_t* st, const void* x, const void* B,
                               const void* C, const float* dt, const float* A, const float* D, float* y,
                               void* stream) {
    rssm_status_t s = rssm_check_desc(d);
    if (s != RSSM_OK) return s;
    if ((s = check_state_common(d, st)) != RSSM_OK) return s;
    if (!x || !B || !C || !dt || !A || !D || !y) return RSSM_ERR_INVALID_ARG;
    return replay_call(d, st, 1, 1, x, B, C, dt, A, D, y, stream);
}

rssm_status_t rssm_decode_step_noalloc(const rssm_desc_t* d, const rssm_state_t* st, const void* x, const void* B,
                                       const void* C, const float* dt, const float* A, const float* D, float* y,
                                       void* stream) {
    rssm_status_t s = rssm_check_desc(d);
    if (s != RSSM_OK) return s;
    if (d->batch > RSSM_NOALLOC_MAX_BATCH) return RSSM_ERR_CAPACITY;
    if ((s = check_state_fields(d, st, false)) != RSSM_OK) return s;
    if (!x || !B || !C || !dt || !A || !D || !y) return RSSM_ERR_INVALID_ARG;
    uint32_t* scratch = noalloc_arrive_scratch();
    if (!scratch) return RSSM_ERR_CUDA;
    // the counters must start at zero; a previous call that stopped on a
    // device error may have left some set
    cudaError_t e = cudaMemsetAsync(scratch, 0, sizeof(uint32_t) * static_cast<size_t>(d->batch),
                                    static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return RSSM_ERR_CUDA;
    rssm_state_t view = *st;
    view.arrive = scratch;
    return replay_call(d, &view, 1, 1, x, B, C, dt, A, D, y, stream);
}

rssm_status_t rssm_verify(const rssm_desc_t* d, const rssm_state_t* st, int32_t K, const void* x, const void* B,
                          const void* C, const float* dt, const float* A, const float* D, float* y,
                          void* stream) {
    rssm_status_t s = rssm_check_desc(d);
    if (s != RSSM_OK) return s;
    if ((s = check_state_common(d, st)) != RSSM_OK) return s;
    if (!x || !B || !C || !dt || !A || !D || !y) return RSSM_ERR_INVALID_ARG;
    if (K < 0 || K > d->max_draft) return RSSM_ERR_CAPACITY;
    return replay_call(d, st, K + 1, 0, x, B, C, dt, A, D, y, stream);
}

rssm_status_t rssm_accept(const rssm_desc_t* d, const rssm_state_t* st, const int32_t* n_accepted,
                          void* stream) {
    rssm_status_t s = rssm_check_desc(d);
    if (s != RSSM_OK) return s;
    if (!st || !st->pos || !st->err || !n_accepted) return RSSM_ERR_INVALID_ARG;
    return cuda_status(launch_accept(d->batch, d->max_draft, cap_of(d), n_accepted, st->pos, st->err, 1,
                                     static_cast<cudaStream_t>(stream)));
}

static rssm_status_t fold_launch(const rssm_desc_t* d, const rssm_state_t* st, int mode, const float* A,
                                 void* stream) {
    FoldArgs a;
    a.s = shape_of(d);
    a.mode = mode;
    a.out_fp4 = d->out_copy == RSSM_OUTCOPY_FP4;
    a.seed = d->seed;
    a.rec = rec_of(d);
    a.record = static_cast<unsigned char*>(st->record);
    if (separate_ckpt(d)) {
        a.upd = static_cast<unsigned char*>(st->ckpt);
        a.upd_stride = static_cast<uint32_t>(d->head_dim) * d->d_state * (d->update_dtype == RSSM_F32 ? 4 : d->update_dtype == RSSM_BF16 ? 2 : 1);
    } else {
        a.upd = a.record;
        a.upd_stride = a.rec.bytes;
    }
    a.bbuf = st->bbuf;
    a.pos = st->pos;
    a.flush_count = st->flush_count;
    a.arrive = st->arrive;
    a.err = st->err;
    a.A = A;
    return cuda_status(
        launch_fold(a, d->in_dtype == RSSM_BF16, d->update_dtype, static_cast<cudaStream_t>(stream)));
}

rssm_status_t rssm_flush(const rssm_desc_t* d, const rssm_state_t* st, const float* A, int32_t force,
                         void* stream) {
    rssm_status_t s = rssm_check_desc(d);
    if (s != RSSM_OK) return s;
    if (d->update_dtype != RSSM_F32 || d->out_copy != RSSM_OUTCOPY_NONE) return RSSM_ERR_UNSUPPORTED;
    if ((s = check_state_common(d, st)) != RSSM_OK) return s;
    if (!A) return RSSM_ERR_INVALID_ARG;
    return fold_launch(d, st, force ? 1 : 0, A, stream);
}

rssm_status_t rssm_lowprec_refresh(const rssm_desc_t* d, const rssm_state_t* st, const float* A, int32_t force,
                                   void* stream) {
    rssm_status_t s = rssm_check_desc(d);
    if (s != RSSM_OK) return s;
    if ((s = check_state_common(d, st)) != RSSM_OK) return s;
    if (!A) return RSSM_ERR_INVALID_ARG;
    return fold_launch(d, st, force ? 2 : 0, A, stream);
}

rssm_status_t rssm_prefill(const rssm_desc_t* d, const rssm_state_t* st, int32_t T0, const void* x, const void* B,
                           const float* dt, const float* A, void* stream) {
    rssm_status_t s = rssm_check_desc(d);
    if (s != RSSM_OK) return s;
    if (d->update_dtype != RSSM_F32 || d->out_copy != RSSM_OUTCOPY_NONE) return RSSM_ERR_UNSUPPORTED;
    if (!st || !st->record || !st->pos || !st->err) return RSSM_ERR_INVALID_ARG;
    if (T0 < 0) return RSSM_ERR_INVALID_ARG;
    if (T0 > 0 && (!x || !B || !dt || !A)) return RSSM_ERR_INVALID_ARG;
    PrefillArgs a;
    a.s = shape_of(d);
    a.T0 = T0;
    a.rec = rec_of(d);
    a.record = static_cast<unsigned char*>(st->record);
    a.pos = st->pos;
    a.err = st->err;
    a.x = x;
    a.B = B;
    a.dt = dt;
    a.A = A;
    return cuda_status(launch_prefill(a, d->in_dtype == RSSM_BF16, static_cast<cudaStream_t>(stream)));
}

static rssm_status_t conv_launch(const rssm_desc_t* d, float* h, const int32_t* cur, int ntok, int32_t* err,
                                 const void* x, const void* B, const void* C, const float* dt, const float* A,
                                 const float* D, float* y, void* stream) {
    ConvArgs a;
    a.s = shape_of(d);
    a.s.L = 1;
    a.s.cap = 1;
    a.s.capr = 4;
    a.ntok = ntok;
    a.h = h;
    a.cur = cur;
    a.err = err;
    a.x = x;
    a.B = B;
    a.C = C;
    a.dt = dt;
    a.A = A;
    a.D = D;
    a.y = y;
    return cuda_status(
        launch_conv(a, d->in_dtype == RSSM_BF16, cur != nullptr, static_cast<cudaStream_t>(stream)));
}

rssm_status_t rssm_conv_step(const rssm_desc_t* d, float* h, const void* x, const void* B, const void* C,
                             const float* dt, const float* A, const float* D, float* y, void* stream) {
    rssm_status_t s = check_shape_only(d);
    if (s != RSSM_OK) return s;
    if (!h || !x || !B || !C || !dt || !A || !D || !y) return RSSM_ERR_INVALID_ARG;
    return conv_launch(d, h, nullptr, 1, nullptr, x, B, C, dt, A, D, y, stream);
}

rssm_status_t rssm_conv_verify(const rssm_desc_t* d, float* copies, const int32_t* cur, int32_t K, const void* x,
                               const void* B, const void* C, const float* dt, const float* A, const float* D,
                               float* y, void* stream) {
    rssm_status_t s = check_shape_only(d);
    if (s != RSSM_OK) return s;
    if (!copies || !cur || !x || !B || !C || !dt || !A || !D || !y) return RSSM_ERR_INVALID_ARG;
    if (K < 0 || K + 1 > kMaxTokens) return RSSM_ERR_CAPACITY;
    return conv_launch(d, copies, cur, K + 1, nullptr, x, B, C, dt, A, D, y, stream);
}

rssm_status_t rssm_conv_accept(const rssm_desc_t* d, const int32_t* n_accepted, int32_t* cur, int32_t K,
                               int32_t* err, void* stream) {
    rssm_status_t s = check_shape_only(d);
    if (s != RSSM_OK) return s;
    if (!n_accepted || !cur) return RSSM_ERR_INVALID_ARG;
    if (K < 0 || K + 1 > kMaxTokens) return RSSM_ERR_CAPACITY;
    return cuda_status(launch_accept(d->batch, K, K, n_accepted, cur, err, 0, static_cast<cudaStream_t>(stream)));
}

rssm_status_t rssm_get_error(const rssm_desc_t* d, const rssm_state_t* st, int32_t* host_code, void* stream) {
    (void)d;
    if (!st || !st->err || !host_code) return RSSM_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, st->err, sizeof(v), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess && v != 0) {
        e = cudaMemsetAsync(st->err, 0, sizeof(int32_t), s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    }
    if (e != cudaSuccess) return RSSM_ERR_CUDA;
    *host_code = v;
    return v != 0 ? RSSM_ERR_DEVICE : RSSM_OK;
}

rssm_status_t rssm_round_test(int32_t op, int64_t n, const float* v, uint64_t seed, uint32_t c1, uint32_t c2,
                              uint32_t c3, void* out, void* stream) {
    if (op < 0 || op > 5 || n < 0) return RSSM_ERR_INVALID_ARG;
    if (op == 5 && n % 16 != 0) return RSSM_ERR_SHAPE;
    if (op == 3 && n % 16 != 0) return RSSM_ERR_SHAPE;
    if (n > 0 && (!v || !out)) return RSSM_ERR_INVALID_ARG;
    return cuda_status(launch_round_test(op, n, v, seed, c1, c2, c3, out, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
