"""Thin Python binding of librssm (include/rssm.h) over ctypes.

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of librssm.so. Tensors must be CUDA tensors on the current device,
contiguous, of the documented dtype; work is enqueued on torch's current
stream. There is no CPU fallback: without the built library every call
raises.

Functions named rssm_* mirror the C entry points one to one. RssmState
allocates the per-layer state through PyTorch (the library itself never
allocates).
"""
import ctypes as ct
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librssm.so")

RSSM_F32, RSSM_BF16, RSSM_E4M3, RSSM_FP4 = 0, 1, 2, 3
RSSM_OUTCOPY_NONE, RSSM_OUTCOPY_FP4 = 0, 1
RSSM_FLAG_FUSED_FLUSH = 1
DEVERR = {0: "none", 1: "pos out of range", 2: "buffer capacity", 3: "accepted count out of range",
          4: "bulk copy timeout"}

(FIELD_RECORD, FIELD_CKPT, FIELD_BBUF, FIELD_POS, FIELD_FLUSH_COUNT, FIELD_ARRIVE, FIELD_ERR) = range(7)


class Desc(ct.Structure):
    _fields_ = [("batch", ct.c_int32), ("nheads", ct.c_int32), ("head_dim", ct.c_int32),
                ("d_state", ct.c_int32), ("ngroups", ct.c_int32), ("interval", ct.c_int32),
                ("max_draft", ct.c_int32), ("in_dtype", ct.c_int32), ("update_dtype", ct.c_int32),
                ("out_copy", ct.c_int32), ("flags", ct.c_uint32), ("reserved", ct.c_uint32),
                ("seed", ct.c_uint64)]


class StateStruct(ct.Structure):
    _fields_ = [(n, ct.c_void_p) for n in ("record", "ckpt", "bbuf", "pos", "flush_count", "arrive", "err")]


class RecordLayout(ct.Structure):
    _fields_ = [(n, ct.c_uint64) for n in ("bytes", "tile_bytes", "scales_offset", "dt_offset", "x_offset")]


class RssmError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None
_P = ct.POINTER


def lib():
    """The loaded librssm.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with python -m hybrid_model_ssm_replay_b200.build")
    L = ct.CDLL(LIB_PATH)
    vp, i32, u32, u64, i64 = ct.c_void_p, ct.c_int32, ct.c_uint32, ct.c_uint64, ct.c_int64
    D, S = _P(Desc), _P(StateStruct)
    sigs = {
        "rssm_abi_version": ([], ct.c_int),
        "rssm_status_string": ([ct.c_int], ct.c_char_p),
        "rssm_check_desc": ([D], ct.c_int),
        "rssm_state_field_bytes": ([D, i32], ct.c_size_t),
        "rssm_record_layout": ([D, _P(RecordLayout)], ct.c_int),
        "rssm_decode_step": ([D, S, vp, vp, vp, vp, vp, vp, vp, vp], ct.c_int),
        "rssm_decode_step_noalloc": ([D, S, vp, vp, vp, vp, vp, vp, vp, vp], ct.c_int),
        "rssm_flush": ([D, S, vp, i32, vp], ct.c_int),
        "rssm_verify": ([D, S, i32, vp, vp, vp, vp, vp, vp, vp, vp], ct.c_int),
        "rssm_accept": ([D, S, vp, vp], ct.c_int),
        "rssm_lowprec_refresh": ([D, S, vp, i32, vp], ct.c_int),
        "rssm_prefill": ([D, S, i32, vp, vp, vp, vp, vp], ct.c_int),
        "rssm_conv_step": ([D, vp, vp, vp, vp, vp, vp, vp, vp, vp], ct.c_int),
        "rssm_conv_verify": ([D, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp], ct.c_int),
        "rssm_conv_accept": ([D, vp, vp, i32, vp, vp], ct.c_int),
        "rssm_get_error": ([D, S, _P(i32), vp], ct.c_int),
        "rssm_round_test": ([i32, i64, vp, u64, u32, u32, u32, vp, vp], ct.c_int),
    }
    for name, (args, res) in sigs.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def status_string(status):
    return lib().rssm_status_string(int(status)).decode()


def _check(status, what):
    if status != 0:
        raise RssmError(status, what)


def _ptr(t, dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (librssm has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return ct.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ct.c_void_p(s.cuda_stream)


def make_desc(batch, nheads, head_dim, d_state, ngroups, interval=16, max_draft=0, in_dtype=RSSM_BF16,
              update_dtype=RSSM_F32, out_copy=RSSM_OUTCOPY_NONE, flags=0, seed=0):
    return Desc(batch, nheads, head_dim, d_state, ngroups, interval, max_draft, in_dtype, update_dtype,
                out_copy, flags, 0, seed)


def rssm_check_desc(desc):
    return lib().rssm_check_desc(ct.byref(desc))


def rssm_state_field_bytes(desc, field):
    return lib().rssm_state_field_bytes(ct.byref(desc), field)


def rssm_record_layout(desc):
    out = RecordLayout()
    _check(lib().rssm_record_layout(ct.byref(desc), ct.byref(out)), "rssm_record_layout")
    return out


_IN_DT = {RSSM_F32: torch.float32, RSSM_BF16: torch.bfloat16}


class RssmState:
    """Per-layer replay state, allocated through PyTorch on the current device.

    `record` is the uint8 tensor [batch][H][record bytes] of rssm.h; the
    other names are views into it or separate fields:
      ckpt        the update copy [batch][H][P][N] (float32 / bfloat16 /
                  uint8 e4m3; FP4 shared copy: uint8 codes [..][N/2]) --
                  inside the records unless there is an FP4 output copy
      ckpt_scales FP4 shared copy: e4m3 scales [batch][H][P][N/16]
      out_codes, out_scales  FP4 output copy (inside the records)
      xbuf [batch][H][cap][P], dtbuf [batch][H][capr] (views into the records;
      capr = cap rounded up to a multiple of 4), bbuf [batch][G][cap][N],
      pos, flush_count, arrive, err.
    Views into the records are strided (not contiguous). Everything starts at
    zero."""

    def __init__(self, desc, device=None):
        _check(rssm_check_desc(desc), "rssm_check_desc")
        self.desc = desc
        dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        B, H, P, N, G = desc.batch, desc.nheads, desc.head_dim, desc.d_state, desc.ngroups
        cap = desc.interval + desc.max_draft
        self.cap = cap
        capr = (cap + 3) // 4 * 4
        in_dt = _IN_DT[desc.in_dtype]
        self.layout = lay = rssm_record_layout(desc)

        def field(f, shape, dtype):
            nbytes = rssm_state_field_bytes(desc, f)
            if nbytes == 0:
                return None
            t = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
            return t.view(dtype).view(shape)

        self.record = field(FIELD_RECORD, (B, H, lay.bytes), torch.uint8)

        def part(off, nbytes, dtype, shape):
            return self.record[:, :, off:off + nbytes].view(dtype).unflatten(-1, shape)

        upd = {RSSM_F32: (torch.float32, N), RSSM_BF16: (torch.bfloat16, N), RSSM_E4M3: (torch.uint8, N),
               RSSM_FP4: (torch.uint8, N // 2)}[desc.update_dtype]
        fp4_scales = (lay.scales_offset, P * N // 16, torch.uint8, (P, N // 16))
        self.ckpt_scales = self.out_codes = self.out_scales = None
        if desc.out_copy == RSSM_OUTCOPY_FP4:
            self.ckpt = field(FIELD_CKPT, (B, H, P, upd[1]), upd[0])
            self.out_codes = part(0, lay.tile_bytes, torch.uint8, (P, N // 2))
            self.out_scales = part(*fp4_scales)
        else:
            self.ckpt = part(0, lay.tile_bytes, upd[0], (P, upd[1]))
            if desc.update_dtype == RSSM_FP4:
                self.ckpt_scales = part(*fp4_scales)
        es = torch.tensor([], dtype=in_dt).element_size()
        self.xbuf = part(lay.x_offset, cap * P * es, in_dt, (cap, P))
        self.dtbuf = part(lay.dt_offset, 4 * capr, torch.float32, (capr,))
        self.bbuf = field(FIELD_BBUF, (B, G, cap, N), in_dt)
        self.pos = field(FIELD_POS, (B,), torch.int32)
        self.flush_count = field(FIELD_FLUSH_COUNT, (B,), torch.int32)
        self.arrive = field(FIELD_ARRIVE, (B,), torch.int32)
        self.err = field(FIELD_ERR, (1,), torch.int32)
        sep = self.ckpt if desc.out_copy == RSSM_OUTCOPY_FP4 else None
        self.struct = StateStruct(*[None if t is None else t.data_ptr() for t in (
            self.record, sep, self.bbuf, self.pos, self.flush_count, self.arrive, self.err)])


def rssm_decode_step(state, x, B, C, dt, A, D, y, stream=None):
    d = state.desc
    in_dt = _IN_DT[d.in_dtype]
    _check(lib().rssm_decode_step(ct.byref(d), ct.byref(state.struct), _ptr(x, in_dt, "x"), _ptr(B, in_dt, "B"),
                                  _ptr(C, in_dt, "C"), _ptr(dt, torch.float32, "dt"), _ptr(A, torch.float32, "A"),
                                  _ptr(D, torch.float32, "D"), _ptr(y, torch.float32, "y"), _stream(stream)),
           "rssm_decode_step")
    return y


def rssm_decode_step_noalloc(state, x, B, C, dt, A, D, y, stream=None):
    """rssm_decode_step without caller-allocated scratch (state.arrive unused)."""
    d = state.desc
    in_dt = _IN_DT[d.in_dtype]
    _check(lib().rssm_decode_step_noalloc(ct.byref(d), ct.byref(state.struct), _ptr(x, in_dt, "x"),
                                          _ptr(B, in_dt, "B"), _ptr(C, in_dt, "C"), _ptr(dt, torch.float32, "dt"),
                                          _ptr(A, torch.float32, "A"), _ptr(D, torch.float32, "D"),
                                          _ptr(y, torch.float32, "y"), _stream(stream)), "rssm_decode_step_noalloc")
    return y


def rssm_flush(state, A, force=False, stream=None):
    _check(lib().rssm_flush(ct.byref(state.desc), ct.byref(state.struct), _ptr(A, torch.float32, "A"),
                            int(bool(force)), _stream(stream)), "rssm_flush")


def rssm_verify(state, K, x, B, C, dt, A, D, y, stream=None):
    d = state.desc
    in_dt = _IN_DT[d.in_dtype]
    _check(lib().rssm_verify(ct.byref(d), ct.byref(state.struct), int(K), _ptr(x, in_dt, "x"), _ptr(B, in_dt, "B"),
                             _ptr(C, in_dt, "C"), _ptr(dt, torch.float32, "dt"), _ptr(A, torch.float32, "A"),
                             _ptr(D, torch.float32, "D"), _ptr(y, torch.float32, "y"), _stream(stream)),
           "rssm_verify")
    return y


def rssm_accept(state, n_accepted, stream=None):
    _check(lib().rssm_accept(ct.byref(state.desc), ct.byref(state.struct), _ptr(n_accepted, torch.int32, "n"),
                             _stream(stream)), "rssm_accept")


def rssm_lowprec_refresh(state, A, force=False, stream=None):
    _check(lib().rssm_lowprec_refresh(ct.byref(state.desc), ct.byref(state.struct), _ptr(A, torch.float32, "A"),
                                      int(bool(force)), _stream(stream)), "rssm_lowprec_refresh")


def rssm_prefill(state, x, B, dt, A, stream=None):
    """Fold a prompt of T0 = x.shape[0] tokens into the fp32 checkpoint (pos must be 0)."""
    d = state.desc
    in_dt = _IN_DT[d.in_dtype]
    T0 = int(x.shape[0])
    _check(lib().rssm_prefill(ct.byref(d), ct.byref(state.struct), T0, _ptr(x, in_dt, "x"), _ptr(B, in_dt, "B"),
                              _ptr(dt, torch.float32, "dt"), _ptr(A, torch.float32, "A"), _stream(stream)),
           "rssm_prefill")


def rssm_conv_step(desc, h, x, B, C, dt, A, D, y, stream=None):
    in_dt = _IN_DT[desc.in_dtype]
    _check(lib().rssm_conv_step(ct.byref(desc), _ptr(h, torch.float32, "h"), _ptr(x, in_dt, "x"),
                                _ptr(B, in_dt, "B"), _ptr(C, in_dt, "C"), _ptr(dt, torch.float32, "dt"),
                                _ptr(A, torch.float32, "A"), _ptr(D, torch.float32, "D"),
                                _ptr(y, torch.float32, "y"), _stream(stream)), "rssm_conv_step")
    return y


def rssm_conv_verify(desc, copies, cur, K, x, B, C, dt, A, D, y, stream=None):
    in_dt = _IN_DT[desc.in_dtype]
    _check(lib().rssm_conv_verify(ct.byref(desc), _ptr(copies, torch.float32, "copies"),
                                  _ptr(cur, torch.int32, "cur"), int(K), _ptr(x, in_dt, "x"),
                                  _ptr(B, in_dt, "B"), _ptr(C, in_dt, "C"), _ptr(dt, torch.float32, "dt"),
                                  _ptr(A, torch.float32, "A"), _ptr(D, torch.float32, "D"),
                                  _ptr(y, torch.float32, "y"), _stream(stream)), "rssm_conv_verify")
    return y


def rssm_conv_accept(desc, n_accepted, cur, K, err=None, stream=None):
    _check(lib().rssm_conv_accept(ct.byref(desc), _ptr(n_accepted, torch.int32, "n"), _ptr(cur, torch.int32, "cur"),
                                  int(K), _ptr(err, torch.int32, "err"), _stream(stream)), "rssm_conv_accept")


def rssm_get_error(state, stream=None):
    """Device error code (0 = none); reads and clears the word. Synchronises the stream."""
    code = ct.c_int32(0)
    st = lib().rssm_get_error(ct.byref(state.desc), ct.byref(state.struct), ct.byref(code), _stream(stream))
    if st not in (0, 6):
        raise RssmError(st, "rssm_get_error")
    return code.value


def rssm_round_test(op, v, seed=0, c1=0, c2=0, c3=0, stream=None):
    """Device rounding functions on float32 v (see rssm.h); returns the output tensor."""
    n = v.numel()
    if op == 0:
        out = torch.empty(n, dtype=torch.int16, device=v.device)
    elif op in (1, 2):
        out = torch.empty(n, dtype=torch.uint8, device=v.device)
    elif op == 3:
        out = torch.empty(n // 2 + n // 16, dtype=torch.uint8, device=v.device)
    elif op == 5:
        out = torch.empty(n, dtype=torch.float32, device=v.device)
    else:
        out = torch.empty(n, dtype=torch.int32, device=v.device)
    _check(lib().rssm_round_test(int(op), n, _ptr(v, torch.float32, "v"), int(seed), int(c1), int(c2), int(c3),
                                 _ptr(out), _stream(stream)), "rssm_round_test")
    return out
