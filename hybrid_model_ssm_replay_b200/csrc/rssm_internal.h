// rssm_internal.h -- argument blocks and launchers shared by the C ABI
// (rssm_api.cu) and the kernels (rssm_kernels.cu). Not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace rssm {

enum Fmt : int { kF32 = 0, kBF16 = 1, kE4M3 = 2, kFP4 = 3 };

// Shapes shared by every kernel. lpr = d_state / 4 lanes per state row;
// capr = cap rounded up to 4 is the row stride of the dt buffer (16-byte rows).
struct Shape {
    int batch, H, P, N, G, L, cap, lpr, capr;
};

// Byte geometry of one (request, head) record (rssm.h, RSSM_FIELD_RECORD):
// [read copy values | FP4 scales | dt, capr floats | x, cap rows of P].
struct RecLayout {
    uint32_t bytes;   // record stride (a multiple of 128)
    uint32_t tile;    // bytes of the read copy's values (FP4: codes)
    uint32_t scales;  // offset of the FP4 scales
    uint32_t dt;      // offset of the buffered dt
    uint32_t x;       // offset of the buffered x
};

// Replay decode / verify (ReplaySSM article s1, s3).
struct ReplayArgs {
    Shape s;
    int ntok;        // tokens per request in this call: 1 (decode) or K+1 (verify)
    int advance;     // decode: pos += 1 by the last CTA of the request
    int fused;       // decode: fold the buffer when this token fills it (fp32 state)
    RecLayout rec;
    unsigned char* record;  // record (b, h) at record + (b*H + h) * rec.bytes
    void* bbuf;
    int32_t* pos;
    uint32_t* flush_count;
    uint32_t* arrive;
    int32_t* err;
    const void* x;
    const void* B;
    const void* C;
    const float* dt;
    const float* A;
    const float* D;
    float* y;
};

// Division by a run-time constant d (1 <= d < 2^31) for 0 <= x < 2^31:
// q = (umulhi(x, mul) + x) >> shr (round-up reciprocal, Granlund-Montgomery).
struct FastDiv {
    uint32_t d, mul, shr;
};

inline FastDiv make_fastdiv(uint32_t d) {
    FastDiv f;
    f.d = d;
    uint32_t s = 0;
    while ((1ull << s) < d) ++s;
    f.shr = s;
    f.mul = static_cast<uint32_t>(((1ull << 32) * ((1ull << s) - d)) / d + 1);
    return f;
}

// Shared-memory stage of the pipelined replay kernel: a mirror of the
// record prefix (same offsets as RecLayout, x rows up to cap), the buffered
// B rows [cap][N] at `brows` and the position and tile index at `meta`;
// `stages` stages. This call's x, B and C rows of a tile ([ntok][P],
// [ntok][N], [ntok][N] at 0, nb_off, nc_off of a row area) come either with
// the stage (rows != 0: the area at `rows`; the FP4-reading decode) or, by
// the consumers, into two buffers per consumer group of `newrows` bytes
// after the stages, with the tile's dt [8], A_h, D_h at nd_off.
struct PipeLayout {
    uint32_t stage_bytes, brows, meta, rows, newrows, nb_off, nc_off, nd_off;
    uint32_t xw_bytes;  // fused fold: per-group fp32 w_s x_s scratch (0 otherwise)
    int stages;
    size_t budget;  // dynamic shared memory the layout may use
    FastDiv divH, divHpg;  // tile -> (request, head), head -> group
};

// Fold of the buffer into the update copy (flush / refresh; s1, s4).
struct FoldArgs {
    Shape s;
    int mode;          // 0: pos >= L only; 1: also any pos > 0; 2: every request
    int out_fp4;       // also write the FP4 output copy (the record's read copy)
    uint64_t seed;
    RecLayout rec;
    unsigned char* record;
    unsigned char* upd;    // update copy of (b, h) at upd + (b*H + h) * upd_stride
    uint32_t upd_stride;   // (FP4 update copy: scales at upd + ... + rec.scales)
    const void* bbuf;
    int32_t* pos;
    uint32_t* flush_count;
    uint32_t* arrive;
    int32_t* err;
    const float* A;
};

// Prefill of T0 prompt tokens into the fp32 checkpoint (empty buffer).
struct PrefillArgs {
    Shape s;
    int T0;
    RecLayout rec;
    unsigned char* record;
    int32_t* pos;
    int32_t* err;
    const void* x;
    const void* B;
    const float* dt;
    const float* A;
};

// Conventional step / verify (s1, s3: the scheme ReplaySSM replaces).
struct ConvArgs {
    Shape s;
    int ntok;
    float* h;              // step: state; verify: copies [ntok][batch][H][P][N]
    const int32_t* cur;    // verify: copy holding the current state
    int32_t* err;
    const void* x;
    const void* B;
    const void* C;
    const float* dt;
    const float* A;
    const float* D;
    float* y;
};

// Launchers return cudaSuccess or the launch error. in_bf16 selects the
// input element type.
cudaError_t launch_replay(const ReplayArgs& a, int in_bf16, int read_fmt, cudaStream_t st);
cudaError_t launch_fold(const FoldArgs& a, int in_bf16, int upd_fmt, cudaStream_t st);
cudaError_t launch_prefill(const PrefillArgs& a, int in_bf16, cudaStream_t st);
cudaError_t launch_conv(const ConvArgs& a, int in_bf16, int verify, cudaStream_t st);
cudaError_t launch_accept(int batch, int K, int cap, const int32_t* n, int32_t* pos, int32_t* err, int add_one,
                          cudaStream_t st);
cudaError_t launch_round_test(int op, int64_t n, const float* v, uint64_t seed, uint32_t c1, uint32_t c2,
                              uint32_t c3, void* out, cudaStream_t st);

// Scratch of the no-allocation decode entry point (see rssm.h).
uint32_t* noalloc_arrive_scratch();

// Dynamic shared memory of one CTA, in bytes.
size_t replay_smem_bytes(const Shape& s, int read_fmt, int ntok, int fused);
size_t fold_smem_bytes(const Shape& s, int upd_fmt);

// Record geometry for the read-copy format and the input element size.
RecLayout record_layout(const Shape& s, int read_fmt, int in_bytes);
size_t conv_smem_bytes(const Shape& s);

}  // namespace rssm
