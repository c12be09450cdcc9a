"""ctypes front end of the fp64 CPU oracle (rssm_oracle.c).

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and the CPU
baseline leg of bench.py may import this module. The GPU library never does.

The per-step arithmetic lives in rssm_oracle.c; this module only marshals
numpy arrays and strings the steps of a run together in the order the
method states (ReplaySSM article, devotd.net
"nvidia-replayssm-hybrid-model-ssm-decoding-state-buffer": s1 for decode and
flush, s3 for verify/accept, s4 for the precision split).

All arrays are per request, C-contiguous:
    ckpt [H][P][N] float64     x [T][H][P]     B, C [T][G][N]     dt [T][H]
    A, D [H]                   y [T][H][P]
"""
import ctypes as ct
import os

import numpy as np

from . import build as _build

_lib = None

F32, BF16, E4M3, FP4 = 0, 1, 2, 3

_dp = ct.POINTER(ct.c_double)
_ip = ct.POINTER(ct.c_int)


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ct.CDLL(path)
        i, d, vp = ct.c_int, _dp, ct.c_void_p
        L.oracle_conv_steps.argtypes = [i, i, i, i, i, d, d, d, d, d, d, d, d]
        L.oracle_replay_decode.argtypes = [i, i, i, i, i, d, d, d, d, _ip, d, d, d, d, d, d, d]
        L.oracle_replay_decode.restype = ct.c_int
        L.oracle_replay_flush.argtypes = [i, i, i, i, d, d, d, d, _ip, d]
        L.oracle_replay_verify.argtypes = [i, i, i, i, i, d, d, d, d, i, i, d, d, d, d, d, d, d]
        L.oracle_replay_verify.restype = ct.c_int
        L.oracle_replay_accept.argtypes = [_ip, i]
        L.oracle_philox4x32_10.argtypes = [vp, vp, vp]
        L.oracle_bf16_value.argtypes = [ct.c_uint16]
        L.oracle_bf16_value.restype = ct.c_double
        L.oracle_e4m3_value.argtypes = [ct.c_uint8]
        L.oracle_e4m3_value.restype = ct.c_double
        L.oracle_e2m1_value.argtypes = [ct.c_uint8]
        L.oracle_e2m1_value.restype = ct.c_double
        L.oracle_e4m3_rne.argtypes = [ct.c_float]
        L.oracle_e4m3_rne.restype = ct.c_uint8
        L.oracle_e2m1_rne.argtypes = [ct.c_float]
        L.oracle_e2m1_rne.restype = ct.c_uint8
        L.oracle_sr_bf16.argtypes = [ct.c_float, ct.c_uint32]
        L.oracle_sr_bf16.restype = ct.c_uint16
        L.oracle_sr_e4m3.argtypes = [ct.c_float, ct.c_uint32]
        L.oracle_sr_e4m3.restype = ct.c_uint8
        L.oracle_fp4_quant16.argtypes = [vp, vp, vp]
        L.oracle_widen.argtypes = [i, ct.c_size_t, vp, vp, d]
        L.oracle_sr_head.argtypes = [i, ct.c_uint64, ct.c_uint32, ct.c_uint32, ct.c_uint32,
                                     ct.c_size_t, vp, vp]
        L.oracle_fp4_quant.argtypes = [ct.c_size_t, vp, vp, vp]
        L.oracle_lowprec_refresh.argtypes = [i, i, i, i, i, i, ct.c_uint64, ct.c_uint32,
                                             ct.POINTER(ct.c_uint32), vp, vp, vp, d, d, d,
                                             _ip, d, vp]
        _lib = L
    return _lib


def _d(a):
    assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"], (a.dtype, a.flags)
    return a.ctypes.data_as(_dp)


def _v(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ct.c_void_p)


def f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


# --------------------------------------------------------------------------
# conventional recurrence
# --------------------------------------------------------------------------

def conv_steps(h, x, B, C, dt, A, D):
    """Run x.shape[0] tokens of the recurrence; h [H][P][N] updated in place."""
    T, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    y = np.zeros((T, H, P), np.float64)
    lib().oracle_conv_steps(H, P, N, G, T, _d(h), _d(x), _d(B), _d(C), _d(dt), _d(A), _d(D), _d(y))
    return y


# --------------------------------------------------------------------------
# replay form
# --------------------------------------------------------------------------

class ReplayRequest:
    """One request's checkpoint + input buffer, in fp64."""

    def __init__(self, ckpt, G, Lcap, A, D):
        self.ckpt = f64(ckpt).copy()
        self.H, self.P, self.N = self.ckpt.shape
        self.G, self.Lcap = G, Lcap
        self.A, self.D = f64(A), f64(D)
        self.xb = np.zeros((Lcap, self.H, self.P))
        self.Bb = np.zeros((Lcap, G, self.N))
        self.dtb = np.zeros((Lcap, self.H))
        self._pos = ct.c_int(0)

    @property
    def pos(self):
        return self._pos.value

    @pos.setter
    def pos(self, v):
        self._pos.value = int(v)

    def decode(self, x, B, C, dt):
        y = np.zeros((self.H, self.P))
        rc = lib().oracle_replay_decode(self.H, self.P, self.N, self.G, self.Lcap, _d(self.ckpt),
                                        _d(self.xb), _d(self.Bb), _d(self.dtb), ct.byref(self._pos),
                                        _d(f64(x)), _d(f64(B)), _d(f64(C)), _d(f64(dt)),
                                        _d(self.A), _d(self.D), _d(y))
        if rc != 0:
            raise ValueError("buffer full")
        return y

    def flush(self):
        lib().oracle_replay_flush(self.H, self.P, self.N, self.G, _d(self.ckpt), _d(self.xb),
                                  _d(self.Bb), _d(self.dtb), ct.byref(self._pos), _d(self.A))

    def verify(self, x, B, C, dt):
        """x [ntok][H][P] ... -> y [ntok][H][P]; pos unchanged."""
        x, B, C, dt = f64(x), f64(B), f64(C), f64(dt)
        ntok = x.shape[0]
        y = np.zeros((ntok, self.H, self.P))
        rc = lib().oracle_replay_verify(self.H, self.P, self.N, self.G, self.Lcap, _d(self.ckpt),
                                        _d(self.xb), _d(self.Bb), _d(self.dtb), self.pos, ntok,
                                        _d(x), _d(B), _d(C), _d(dt), _d(self.A), _d(self.D), _d(y))
        if rc != 0:
            raise ValueError("verify does not fit in the buffer")
        return y

    def accept(self, n):
        lib().oracle_replay_accept(ct.byref(self._pos), int(n))


def run_replay_decode(ckpt0, x, B, C, dt, A, D, L, Lcap=None):
    """Standard decode of T tokens with a flush each time the buffer holds L.

    Returns (y [T][H][P], {step: checkpoint after the flush that followed it})."""
    T = x.shape[0]
    req = ReplayRequest(ckpt0, B.shape[1], Lcap or L, A, D)
    ys = np.zeros(x.shape)
    ckpts = {}
    for t in range(T):
        ys[t] = req.decode(x[t], B[t], C[t], dt[t])
        if req.pos >= L:
            req.flush()
            ckpts[t] = req.ckpt.copy()
    return ys, ckpts


def run_conv(ckpt0, x, B, C, dt, A, D, snap_steps=()):
    """Recurrence over T tokens; returns (y, {step: state after that step})."""
    h = f64(ckpt0).copy()
    ys = np.zeros(x.shape)
    snaps = {}
    snap_steps = sorted(snap_steps)
    t0 = 0
    for s in snap_steps + [x.shape[0] - 1]:
        if s < t0:
            continue
        sl = slice(t0, s + 1)
        ys[sl] = conv_steps(h, f64(x[sl]), f64(B[sl]), f64(C[sl]), f64(dt[sl]), f64(A), f64(D))
        snaps[s] = h.copy()
        t0 = s + 1
    return ys, snaps


def run_spec(ckpt0, x, B, C, dt, A, D, n_acc, L, K):
    """Speculative decode: per step verify K+1 tokens, accept n, flush at L.

    x [S][K+1][H][P] ..., n_acc [S]. Returns (y [S][K+1][H][P],
    {step: checkpoint after the flush that followed it}, pos after each step)."""
    S = x.shape[0]
    req = ReplayRequest(ckpt0, B.shape[2], L + K, A, D)
    ys = np.zeros(x.shape)
    ckpts, poss = {}, []
    for s in range(S):
        ys[s] = req.verify(x[s], B[s], C[s], dt[s])
        req.accept(n_acc[s])
        if req.pos >= L:
            req.flush()
            ckpts[s] = req.ckpt.copy()
        poss.append(req.pos)
    return ys, ckpts, poss


# --------------------------------------------------------------------------
# number formats and rounding
# --------------------------------------------------------------------------

def philox4x32_10(ctr, key):
    c = np.ascontiguousarray(np.asarray(ctr, np.uint32))
    k = np.ascontiguousarray(np.asarray(key, np.uint32))
    out = np.zeros(4, np.uint32)
    lib().oracle_philox4x32_10(_v(c), _v(k), _v(out))
    return out


def bf16_value(bits):
    return lib().oracle_bf16_value(int(bits))


def e4m3_value(c):
    return lib().oracle_e4m3_value(int(c))


def e2m1_value(c):
    return lib().oracle_e2m1_value(int(c))


def e4m3_rne(v):
    return lib().oracle_e4m3_rne(float(np.float32(v)))


def e2m1_rne(v):
    return lib().oracle_e2m1_rne(float(np.float32(v)))


def sr_bf16(v, r):
    return lib().oracle_sr_bf16(float(np.float32(v)), int(r))


def sr_e4m3(v, r):
    return lib().oracle_sr_e4m3(float(np.float32(v)), int(r))


def fp4_quant16(v):
    v = np.ascontiguousarray(np.asarray(v, np.float32))
    assert v.shape == (16,)
    codes = np.zeros(8, np.uint8)
    scale = np.zeros(1, np.uint8)
    lib().oracle_fp4_quant16(_v(v), _v(codes), _v(scale))
    return codes, int(scale[0])


def fp4_quant(v):
    """v float32 [..., multiple of 16] -> (codes uint8 [.../2], scales uint8 [.../16])."""
    v = np.ascontiguousarray(np.asarray(v, np.float32))
    n = v.size
    codes = np.zeros(v.shape[:-1] + (v.shape[-1] // 2,), np.uint8)
    scales = np.zeros(v.shape[:-1] + (v.shape[-1] // 16,), np.uint8)
    lib().oracle_fp4_quant(n, _v(v), _v(codes), _v(scales))
    return codes, scales


def widen(dtype, src, scales=None, shape=None):
    """Values of a state copy (see rssm_oracle.c oracle_widen) as float64."""
    src = np.ascontiguousarray(src)
    n = src.size * (2 if dtype == FP4 else 1)
    out = np.zeros(n, np.float64)
    sc = None if scales is None else np.ascontiguousarray(scales)
    lib().oracle_widen(dtype, n, _v(src), _v(sc), _d(out))
    return out.reshape(shape) if shape is not None else out


def sr_head(dtype, seed, request, head, flush_count, v):
    v = np.ascontiguousarray(np.asarray(v, np.float32))
    out = np.zeros(v.shape, np.uint16 if dtype == BF16 else np.uint8)
    lib().oracle_sr_head(dtype, seed, request, head, flush_count, v.size, _v(v), _v(out))
    return out


class LowPrecRequest:
    """One request in split precision (ReplaySSM article s4).

    upd_dtype F32/BF16/E4M3: update copy `upd` [H][P][N]; out_fp4 adds the
    FP4 output copy that decode reads. upd_dtype FP4: the shared-copy
    control, where the FP4 copy is both read and updated. With neither an
    FP4 copy nor an FP4 update dtype, decode reads the update copy itself."""

    def __init__(self, upd_dtype, out_fp4, upd, codes, scales, G, Lcap, A, D, seed, request):
        self.upd_dtype, self.out_fp4 = upd_dtype, bool(out_fp4)
        self.upd = None if upd is None else np.ascontiguousarray(upd).copy()
        self.codes = None if codes is None else np.ascontiguousarray(codes).copy()
        self.scales = None if scales is None else np.ascontiguousarray(scales).copy()
        H, P, N = self.read_values().shape if self.upd is None else self.upd.shape
        self.H, self.P, self.N, self.G, self.Lcap = H, P, N, G, Lcap
        self.A, self.D = f64(A), f64(D)
        self.seed, self.request = int(seed), int(request)
        self.flush_count = ct.c_uint32(0)
        self.req = ReplayRequest(np.zeros((H, P, N)), G, Lcap, A, D)

    def read_values(self):
        """The copy that outputs read, as float64 [H][P][N]."""
        if self.upd_dtype == FP4 or self.out_fp4:
            shape = self.codes.shape[:-1] + (self.codes.shape[-1] * 2,)
            return widen(FP4, self.codes, self.scales, shape)
        return widen(self.upd_dtype, self.upd, None, self.upd.shape)

    def decode(self, x, B, C, dt):
        self.req.ckpt[...] = self.read_values()
        return self.req.decode(x, B, C, dt)

    def verify(self, x, B, C, dt):
        self.req.ckpt[...] = self.read_values()
        return self.req.verify(x, B, C, dt)

    def accept(self, n):
        self.req.accept(n)

    @property
    def pos(self):
        return self.req.pos

    def refresh(self, want_v32=False):
        H, P, N = self.H, self.P, self.N
        v32 = np.zeros((H, P, N), np.float32) if want_v32 else None
        upd = self.upd if self.upd is not None else np.zeros(1, np.uint8)
        codes = self.codes if self.codes is not None else np.zeros(1, np.uint8)
        scales = self.scales if self.scales is not None else np.zeros(1, np.uint8)
        lib().oracle_lowprec_refresh(H, P, N, self.G, self.upd_dtype, int(self.out_fp4), self.seed,
                                     self.request, ct.byref(self.flush_count), _v(upd), _v(codes),
                                     _v(scales), _d(self.req.xb), _d(self.req.Bb), _d(self.req.dtb),
                                     ct.byref(self.req._pos), _d(self.A), _v(v32))
        return v32
