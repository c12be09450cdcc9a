"""Precision split on the GPU (ReplaySSM article s4): the refresh of a
bf16/e4m3 update copy by Philox stochastic rounding, the FP4 output copy
that decode reads, the shared-low-precision control, and the error of a
whole 512-step run against the fp64 oracle."""
import json
import math
import os

import numpy as np
import pytest
import torch

from hybrid_model_ssm_replay_b200 import rssm
from hybrid_model_ssm_replay_b200.inputs import WORKLOADS, LayerShape, make_inputs
from oracle import oracle as orc

from gpu_helpers import assert_close, desc_for, oracle_map, request_inputs, sample_requests, to_np

pytestmark = pytest.mark.gpu

UPD = {"bf16": (rssm.RSSM_BF16, orc.BF16), "e4m3": (rssm.RSSM_E4M3, orc.E4M3), "f32": (rssm.RSSM_F32, orc.F32)}


@pytest.fixture(scope="module", autouse=True)
def _built():
    from hybrid_model_ssm_replay_b200 import build
    build.build()


def initial_update_copy(ckpt, kind):
    """The update copy a run starts from: the fp32 checkpoint rounded to
    nearest by torch (input preparation), as raw bits."""
    if kind == "bf16":
        return ckpt.to(torch.bfloat16)
    if kind == "e4m3":
        return ckpt.to(torch.float8_e4m3fn).view(torch.uint8)
    return ckpt.clone()


def copy_bits(t):
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    return t.numpy()


def split_state(shape, inp, kind, seed, in_dtype=torch.bfloat16):
    desc = desc_for(shape, in_dtype, update_dtype=UPD[kind][0], out_copy=rssm.RSSM_OUTCOPY_FP4, seed=seed)
    st = rssm.RssmState(desc)
    st.ckpt.copy_(initial_update_copy(inp["ckpt"], kind))
    rssm.rssm_lowprec_refresh(st, inp["A"], force=True)      # builds the FP4 output copy
    return desc, st


def fp4_control_state(shape, inp, seed):
    """Shared FP4 copy: built once from the fp32 checkpoint, then read and updated."""
    d0 = desc_for(shape, update_dtype=rssm.RSSM_F32, out_copy=rssm.RSSM_OUTCOPY_FP4, seed=seed)
    s0 = rssm.RssmState(d0)
    s0.ckpt.copy_(inp["ckpt"])
    rssm.rssm_lowprec_refresh(s0, inp["A"], force=True)
    desc = desc_for(shape, update_dtype=rssm.RSSM_FP4, seed=seed)
    st = rssm.RssmState(desc)
    st.ckpt.copy_(s0.out_codes)
    st.ckpt_scales.copy_(s0.out_scales)
    return desc, st


def widened(kind, st):
    """The values of a state's low-precision update copy, widened exactly to
    fp32 on the device (bf16 / e4m3 casts are exact)."""
    if kind == "bf16":
        return st.ckpt.float()
    if kind == "e4m3":
        return st.ckpt.view(torch.float8_e4m3fn).float()
    raise ValueError(kind)


def f32_twin(shape, values, seed, in_dtype=torch.bfloat16, out_copy=True):
    """An fp32 update copy holding exactly `values` (fp32), with an FP4
    output copy when out_copy. With the output copy, refreshing it runs the
    refresh kernel of the low-precision state it shadows -- same inputs,
    same operation order, the tensor-core fold where the shape takes it --
    and stores the fp32 result unrounded: that result is what the
    low-precision refresh rounds. Without it the refresh is the plain fp32
    flush, whose fold (CUDA cores) may round differently; such a twin
    serves for decode outputs and the fold's accuracy only."""
    desc = desc_for(shape, in_dtype, update_dtype=rssm.RSSM_F32,
                    out_copy=rssm.RSSM_OUTCOPY_FP4 if out_copy else rssm.RSSM_OUTCOPY_NONE, seed=seed)
    st = rssm.RssmState(desc)
    st.ckpt.copy_(values)
    return desc, st


def assert_refresh_bits(kind, seed, st, twin, fc_before, requests, what):
    """Kernel-level bit-exactness of a refresh (s4): for every refreshed
    request the update copy equals the oracle's stochastic rounding, and the
    FP4 copies equal the oracle's FP4 quantisation, of the fp32 values the
    GPU fold produced (read from the fp32 twin). Zero mismatches."""
    for b in requests:
        v32 = twin.ckpt[b].cpu().numpy()                          # [H][P][N] float32
        if kind in ("bf16", "e4m3"):
            got = copy_bits(st.ckpt[b])
            for h in range(v32.shape[0]):
                exp = orc.sr_head(UPD[kind][1], seed, b, h, int(fc_before[b]), v32[h])
                bad = int(np.count_nonzero(got[h].ravel() != exp.ravel()))
                assert bad == 0, f"{what}: request {b} head {h}: {bad} update-copy elements differ"
        codes, scales = orc.fp4_quant(v32)
        for name, t in (("FP4 output copy", st.out_codes if kind != "fp4" else st.ckpt),
                        ("FP4 twin copy", twin.out_codes)):
            if t is None:
                continue
            bad = int(np.count_nonzero(t[b].cpu().numpy() != codes))
            assert bad == 0, f"{what}: request {b}: {bad} codes of the {name} differ"
        for name, t in (("FP4 output scales", st.out_scales if kind != "fp4" else st.ckpt_scales),
                        ("FP4 twin scales", twin.out_scales)):
            if t is None:
                continue
            bad = int(np.count_nonzero(t[b].cpu().numpy() != scales))
            assert bad == 0, f"{what}: request {b}: {bad} scales of the {name} differ"


# d_state 64 runs the one-CTA-per-tile fold, d_state 128 the persistent
# pipelined one; head_dim 64 with head pairs in a group the tensor-core one
SHAPES = [LayerShape(3, 4, 32, 64, 2), LayerShape(3, 4, 32, 128, 2), LayerShape(3, 4, 64, 128, 2)]
SHAPE_IDS = ["dstate64", "dstate128", "tensorcore"]


@pytest.mark.parametrize("shape", SHAPES, ids=SHAPE_IDS)
@pytest.mark.parametrize("kind", ["bf16", "e4m3", "f32"])
def test_refresh_at_empty_buffer_builds_fp4_copy_bit_exact(kind, shape):
    inp = make_inputs(shape, 1, 30, torch.bfloat16, device="cuda")
    desc, st = split_state(shape, inp, kind, 99)
    upd0 = copy_bits(initial_update_copy(inp["ckpt"], kind))
    assert np.array_equal(copy_bits(st.ckpt), upd0)             # SR of representable values is exact
    vals = orc.widen(UPD[kind][1], upd0).astype(np.float32)
    codes, scales = orc.fp4_quant(vals)
    assert np.array_equal(st.out_codes.cpu().numpy().ravel(), codes)
    assert np.array_equal(st.out_scales.cpu().numpy().ravel(), scales)
    assert st.flush_count.cpu().tolist() == [1, 1, 1] and st.pos.cpu().tolist() == [0, 0, 0]
    assert rssm.rssm_get_error(st) == 0


# the pipelined kernels (d_state 128; head_dim 40 leaves a half-empty last
# 16-row group) and the one-CTA-per-tile kernels (d_state 64)
SPLIT_SHAPES = [LayerShape(4, 8, 64, 128, 2), LayerShape(3, 4, 40, 128, 2), LayerShape(3, 4, 32, 64, 2)]
SPLIT_IDS = ["dstate128", "headdim40", "dstate64"]


@pytest.mark.parametrize("shape", SPLIT_SHAPES, ids=SPLIT_IDS)
@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float32], ids=["bf16in", "f32in"])
@pytest.mark.parametrize("kind", ["bf16", "e4m3"])
def test_fp4_decode_and_refresh_match_oracle(kind, in_dtype, shape):
    """One interval from a prepared split state: every output read from the
    FP4 copy matches the oracle (fp32 vs fp64 on exact dequantised values).
    The refresh is pinned at kernel level: an fp32 twin state starting from
    the same (widened) update-copy values runs the same fold, and the
    refreshed update copy and FP4 copy equal, bit for bit, the oracle's
    stochastic rounding and FP4 quantisation of that fp32 result, with zero
    mismatches. The fp32 fold itself matches the oracle's fp64 fold within
    the fp32 tolerance."""
    L = shape.interval
    Bz, H, P = shape.batch, shape.nheads, shape.head_dim
    inp = make_inputs(shape, L, 31, in_dtype, device="cuda")
    seed = 0xBEEF
    desc, st = split_state(shape, inp, kind, seed, in_dtype)
    _, tw = f32_twin(shape, widened(kind, st), seed, in_dtype)
    rssm.rssm_lowprec_refresh(tw, inp["A"], force=True)
    assert np.array_equal(tw.out_codes.cpu().numpy(), st.out_codes.cpu().numpy())
    # the oracle starts from the input recipe and its own FP4 quantiser
    upd0 = copy_bits(initial_update_copy(inp["ckpt"], kind))
    codes0, scales0 = orc.fp4_quant(orc.widen(UPD[kind][1], upd0, None, upd0.shape).astype(np.float32))
    y = torch.empty((L, Bz, H, P), device="cuda")
    y2 = torch.empty_like(y)
    for t in range(L):
        args = (inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"])
        rssm.rssm_decode_step(st, *args, y[t])
        rssm.rssm_decode_step(tw, *args, y2[t])
    fc_before = st.flush_count.cpu().tolist()
    rssm.rssm_lowprec_refresh(st, inp["A"])
    rssm.rssm_lowprec_refresh(tw, inp["A"])
    assert rssm.rssm_get_error(st) == 0 and rssm.rssm_get_error(tw) == 0
    assert torch.equal(y, y2)                       # both read the same FP4 copy
    assert_refresh_bits(kind, seed, st, tw, fc_before, range(Bz), f"{kind} + FP4 refresh")
    for b in range(Bz):
        r = request_inputs(inp, b)
        req = orc.LowPrecRequest(UPD[kind][1], True, upd0[b], codes0[b], scales0[b], shape.ngroups, L, r["A"],
                                 r["D"], seed, b)
        req.flush_count.value = 1
        ys = np.stack([req.decode(r["x"][t], r["B"][t], r["C"][t], r["dt"][t]) for t in range(L)])
        assert_close(to_np(y[:, b]), ys, f"FP4-copy decode, request {b}")
        v64 = req.refresh(want_v32=True).astype(np.float64)
        assert_close(to_np(tw.ckpt[b]), v64, f"fp32 fold of the refresh, request {b}")
    assert st.flush_count.cpu().tolist() == [2] * Bz


@pytest.mark.parametrize("kind", ["bf16", "e4m3"])
def test_split_b256_full_size_sampled(kind):
    """The precision split at the bench's size and launch configuration
    (split_b256: batch 256, 64 heads, head_dim 64, d_state 128; the
    persistent replay and fold kernels over every SM): one interval of 16
    decodes reading the FP4 output copy, then the refresh. For sampled
    requests, the outputs match the oracle replaying the same dequantised
    copy; the refreshed update copy and FP4 copy equal, bit for bit, the
    oracle's stochastic rounding and FP4 quantisation of the fold an fp32
    twin computed; and that fold matches the oracle's fp64 fold."""
    w = WORKLOADS["split_b256"]
    shape = w["shape"]
    L = shape.interval
    Bz, H, P = shape.batch, shape.nheads, shape.head_dim
    inp = make_inputs(shape, L, w["seed"], w["in_dtype"], device="cuda")
    seed = w["seed"]
    desc, st = split_state(shape, inp, kind, seed)
    _, tw = f32_twin(shape, widened(kind, st), seed)
    rssm.rssm_lowprec_refresh(tw, inp["A"], force=True)
    y = torch.empty((L, Bz, H, P), device="cuda")
    y2 = torch.empty_like(y)
    for t in range(L):
        args = (inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"])
        rssm.rssm_decode_step(st, *args, y[t])
        rssm.rssm_decode_step(tw, *args, y2[t])
    fc_before = st.flush_count.cpu().tolist()
    rssm.rssm_lowprec_refresh(st, inp["A"])
    rssm.rssm_lowprec_refresh(tw, inp["A"])
    assert rssm.rssm_get_error(st) == 0 and rssm.rssm_get_error(tw) == 0
    assert torch.equal(y, y2)                       # both read the same FP4 copy
    reqs = sample_requests(Bz, 6)
    assert_refresh_bits(kind, seed, st, tw, fc_before, reqs, f"{kind} + FP4 refresh at split_b256")
    for b in reqs:
        upd0 = copy_bits(initial_update_copy(inp["ckpt"][b], kind))
        codes0, scales0 = orc.fp4_quant(orc.widen(UPD[kind][1], upd0, None, upd0.shape).astype(np.float32))
        r = request_inputs(inp, b)
        req = orc.LowPrecRequest(UPD[kind][1], True, upd0, codes0, scales0, shape.ngroups, L, r["A"], r["D"],
                                 seed, b)
        req.flush_count.value = 1
        ys = np.stack([req.decode(r["x"][t], r["B"][t], r["C"][t], r["dt"][t]) for t in range(L)])
        assert_close(to_np(y[:, b]), ys, f"FP4-copy decode at split_b256, request {b}")
        v64 = req.refresh(want_v32=True).astype(np.float64)
        assert_close(to_np(tw.ckpt[b]), v64, f"fp32 fold of the refresh at split_b256, request {b}")
    assert st.flush_count.cpu().tolist() == [2] * Bz


@pytest.mark.parametrize("T", [1, 15, 17, 32])
@pytest.mark.parametrize("kind", ["bf16", "e4m3"])
def test_tensor_core_refresh_at_each_buffer_fill(kind, T):
    """The tensor-core refresh (head_dim 64, head pairs in a group) folds 16
    buffered tokens per MMA K-step. A forced refresh after T decodes (T = 1
    and 15: one partial step; 17: a full step and a one-token step; 32: two
    full steps, the buffer's capacity) leaves update and FP4 copies equal,
    bit for bit, to the oracle's rounding of the fp32 fold of a twin running
    the same kernel, and that fold matches the oracle's fp64 fold; the
    outputs read from the FP4 copy match the oracle."""
    shape = LayerShape(3, 4, 64, 128, 2, interval=25, max_draft=7)   # capacity 32, the most a buffer holds
    Bz, H, P = shape.batch, shape.nheads, shape.head_dim
    inp = make_inputs(shape, T, 37, torch.bfloat16, device="cuda")
    seed = 0xF00D
    desc, st = split_state(shape, inp, kind, seed)
    _, tw = f32_twin(shape, widened(kind, st), seed)
    rssm.rssm_lowprec_refresh(tw, inp["A"], force=True)
    upd0 = copy_bits(initial_update_copy(inp["ckpt"], kind))
    codes0, scales0 = orc.fp4_quant(orc.widen(UPD[kind][1], upd0, None, upd0.shape).astype(np.float32))
    y = torch.empty((T, Bz, H, P), device="cuda")
    y2 = torch.empty_like(y)
    for t in range(T):
        args = (inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"])
        rssm.rssm_decode_step(st, *args, y[t])
        rssm.rssm_decode_step(tw, *args, y2[t])
    assert torch.equal(y, y2)                       # both read the same FP4 copy
    fc_before = st.flush_count.cpu().tolist()
    rssm.rssm_lowprec_refresh(st, inp["A"], force=True)
    rssm.rssm_lowprec_refresh(tw, inp["A"], force=True)
    assert rssm.rssm_get_error(st) == 0 and rssm.rssm_get_error(tw) == 0
    assert_refresh_bits(kind, seed, st, tw, fc_before, range(Bz), f"{kind} + FP4 refresh of {T} entries")
    for b in range(Bz):
        r = request_inputs(inp, b)
        req = orc.LowPrecRequest(UPD[kind][1], True, upd0[b], codes0[b], scales0[b], shape.ngroups, 32, r["A"],
                                 r["D"], seed, b)
        req.flush_count.value = 1
        ys = np.stack([req.decode(r["x"][t], r["B"][t], r["C"][t], r["dt"][t]) for t in range(T)])
        assert_close(to_np(y[:, b]), ys, f"FP4-copy decode, {T} tokens, request {b}")
        v64 = req.refresh(want_v32=True).astype(np.float64)
        assert_close(to_np(tw.ckpt[b]), v64, f"fp32 fold of {T} entries, request {b}")
    assert st.pos.cpu().tolist() == [0] * Bz and st.flush_count.cpu().tolist() == [2] * Bz


@pytest.mark.parametrize("batch", [1, 5])
def test_tensor_core_refresh_single_pair_requests(batch):
    """Degenerate launches of the tensor-core refresh: requests of one head
    pair (2 heads, 1 group), so the grid is batch CTAs, most consumer groups
    get only their end marker, and each request's arrival count reaches H
    with one pair. One interval: bf16 + FP4 copies bit-exact against the
    oracle's rounding of the fp32 twin's fold, that fold against the oracle's
    fp64 fold, positions reset and flush counts advanced."""
    shape = LayerShape(batch, 2, 64, 128, 1)
    L = shape.interval
    inp = make_inputs(shape, L, 38, torch.bfloat16, device="cuda")
    seed = 0xABBA
    desc, st = split_state(shape, inp, "bf16", seed)
    _, tw = f32_twin(shape, widened("bf16", st), seed)
    rssm.rssm_lowprec_refresh(tw, inp["A"], force=True)
    upd0 = copy_bits(initial_update_copy(inp["ckpt"], "bf16"))
    codes0, scales0 = orc.fp4_quant(orc.widen(orc.BF16, upd0, None, upd0.shape).astype(np.float32))
    y = torch.empty((L, batch, 2, 64), device="cuda")
    for t in range(L):
        args = (inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"])
        rssm.rssm_decode_step(st, *args, y[t])
        rssm.rssm_decode_step(tw, *args, y[t])
    fc_before = st.flush_count.cpu().tolist()
    rssm.rssm_lowprec_refresh(st, inp["A"])
    rssm.rssm_lowprec_refresh(tw, inp["A"])
    assert rssm.rssm_get_error(st) == 0 and rssm.rssm_get_error(tw) == 0
    assert_refresh_bits("bf16", seed, st, tw, fc_before, range(batch), "single-pair refresh")
    for b in range(batch):
        r = request_inputs(inp, b)
        req = orc.LowPrecRequest(orc.BF16, True, upd0[b], codes0[b], scales0[b], 1, L, r["A"], r["D"], seed, b)
        req.flush_count.value = 1
        for t in range(L):
            req.decode(r["x"][t], r["B"][t], r["C"][t], r["dt"][t])
        v64 = req.refresh(want_v32=True).astype(np.float64)
        assert_close(to_np(tw.ckpt[b]), v64, f"fp32 fold, single-pair request {b}")
    assert st.pos.cpu().tolist() == [0] * batch and st.flush_count.cpu().tolist() == [2] * batch


# accepted drafts per step and request (steps x batch) for K = 4 and K = 6:
# three requests reach the interval on the last step, one does not
SPLIT_SPEC = {
    4: np.array([[4, 3, 0, 4], [4, 4, 1, 4], [4, 4, 2, 3], [4, 4, 3, 4]], np.int32),   # pos 20 19 10 19
    6: np.array([[6, 6, 0, 5], [6, 5, 1, 6], [2, 3, 2, 3]], np.int32),                 # pos 17 17 6 17
}


@pytest.mark.parametrize("K", [4, 6])
@pytest.mark.parametrize("kind", ["bf16", "e4m3"])
def test_speculative_verify_on_split_state_matches_oracle(kind, K):
    """Speculative decoding (s3) on a split-precision state (s4): verify of
    the pending token and K drafts (K = 4 and 6: the pipelined kernel's 5-
    and 8-token bounds) reads the FP4 output copy, accept(n) advances pos,
    and the refresh after accept folds the requests whose buffer reached the
    interval (up to 20 buffered entries). No request reaches the interval
    before the last accept, so every verify reads the initial FP4 copy; the
    outputs match the oracle within the fp32 tolerance. An fp32 twin runs
    the same calls: the refreshed requests' update and FP4 copies equal the
    oracle's rounding of the twin's fp32 fold bit for bit (zero mismatches),
    and the untouched request keeps its copies."""
    shape = LayerShape(4, 8, 64, 128, 2, interval=16, max_draft=K)
    n_host = SPLIT_SPEC[K]
    steps, L = n_host.shape[0], 16
    inp = make_inputs(shape, steps, 34, torch.bfloat16, device="cuda", ntok=K + 1)
    n_acc = torch.from_numpy(n_host).cuda()
    seed = 0x5EED
    desc, st = split_state(shape, inp, kind, seed)
    _, tw = f32_twin(shape, widened(kind, st), seed)
    rssm.rssm_lowprec_refresh(tw, inp["A"], force=True)
    upd_start = copy_bits(st.ckpt).copy()
    codes_start = st.out_codes.cpu().numpy().copy()
    upd0 = copy_bits(initial_update_copy(inp["ckpt"], kind))
    codes0, scales0 = orc.fp4_quant(orc.widen(UPD[kind][1], upd0, None, upd0.shape).astype(np.float32))
    y = torch.empty((steps, shape.batch, K + 1, shape.nheads, shape.head_dim), device="cuda")
    y2 = torch.empty_like(y)
    fc_before = st.flush_count.cpu().tolist()
    for s in range(steps):
        args = (inp["x"][s], inp["B"][s], inp["C"][s], inp["dt"][s], inp["A"], inp["D"])
        for state, out in ((st, y), (tw, y2)):
            rssm.rssm_verify(state, K, *args, out[s])
            rssm.rssm_accept(state, n_acc[s])
            rssm.rssm_lowprec_refresh(state, inp["A"])
    assert rssm.rssm_get_error(st) == 0 and rssm.rssm_get_error(tw) == 0
    assert torch.equal(y, y2)
    folded = []
    for b in range(shape.batch):
        r = request_inputs(inp, b)
        req = orc.LowPrecRequest(UPD[kind][1], True, upd0[b], codes0[b], scales0[b], shape.ngroups, L + K,
                                 r["A"], r["D"], seed, b)
        req.flush_count.value = 1
        for s in range(steps):
            ys = req.verify(r["x"][s], r["B"][s], r["C"][s], r["dt"][s])
            assert_close(to_np(y[s, b]), ys, f"verify on the FP4 copy, step {s}, request {b}")
            req.accept(int(n_host[s, b]))
            if req.pos >= L:
                v64 = req.refresh(want_v32=True).astype(np.float64)
                assert_close(to_np(tw.ckpt[b]), v64, f"fp32 fold of the refresh, request {b}")
                folded.append(b)
        assert st.pos[b].item() == req.pos and st.flush_count[b].item() == req.flush_count.value
    assert len(folded) == 3
    assert_refresh_bits(kind, seed, st, tw, fc_before, folded, f"speculative {kind} + FP4 refresh")
    for b in set(range(shape.batch)) - set(folded):
        assert np.array_equal(copy_bits(st.ckpt[b]), upd_start[b])
        assert np.array_equal(st.out_codes[b].cpu().numpy(), codes_start[b])


def refresh_bits_of(kind, seed, b, fc, upd_bits, codes, scales, v32, what):
    """As assert_refresh_bits, for one request's copies taken as arrays."""
    if kind in ("bf16", "e4m3"):
        for h in range(v32.shape[0]):
            exp = orc.sr_head(UPD[kind][1], seed, b, h, int(fc), v32[h])
            bad = int(np.count_nonzero(upd_bits[h].ravel() != exp.ravel()))
            assert bad == 0, f"{what}: request {b} head {h}: {bad} update-copy elements differ"
    c_exp, s_exp = orc.fp4_quant(v32)
    assert int(np.count_nonzero(codes != c_exp)) == 0, f"{what}: request {b}: FP4 codes differ"
    assert int(np.count_nonzero(scales != s_exp)) == 0, f"{what}: request {b}: FP4 scales differ"


def test_spec_b512_k4_on_split_state_sampled():
    """Speculative decoding on a split-precision state at the bench's size
    (spec_b512_k4: batch 512, 128 heads, 64 x 128, K = 4, n ~ U{0..4}, bf16
    update copy + FP4 output copy) and launch configuration: per step verify
    + accept + refresh, with an fp32 twin running the same calls. For
    sampled requests, every verify before the request's first refresh
    matches the oracle; at that refresh the twin's fp32 fold matches the
    oracle's fp64 fold and the refreshed copies equal the oracle's rounding
    of the twin's fold bit for bit."""
    from hybrid_model_ssm_replay_b200.inputs import accept_lengths
    w = WORKLOADS["spec_b512_k4"]
    shape = w["shape"]
    K, L = shape.max_draft, shape.interval
    steps, kind, seed = 6, "bf16", w["seed"]
    inp = make_inputs(shape, steps, w["seed"], w["in_dtype"], device="cuda", ntok=K + 1)
    n_acc = accept_lengths(steps, shape.batch, K, w["seed"], device="cuda")
    n_host = n_acc.cpu().numpy()
    desc, st = split_state(shape, inp, kind, seed)
    _, tw = f32_twin(shape, widened(kind, st), seed)
    rssm.rssm_lowprec_refresh(tw, inp["A"], force=True)
    reqs = sample_requests(shape.batch, 6)
    y = torch.empty((steps, shape.batch, K + 1, shape.nheads, shape.head_dim), device="cuda")
    y2 = torch.empty_like(y)
    snaps = []  # per step, after its refresh: the sampled requests' copies, twin fold and counts
    fc_prev = st.flush_count.cpu().numpy().copy()
    for s in range(steps):
        args = (inp["x"][s], inp["B"][s], inp["C"][s], inp["dt"][s], inp["A"], inp["D"])
        for state, out in ((st, y), (tw, y2)):
            rssm.rssm_verify(state, K, *args, out[s])
            rssm.rssm_accept(state, n_acc[s])
            rssm.rssm_lowprec_refresh(state, inp["A"])
        fc_now = st.flush_count.cpu().numpy().copy()
        snaps.append({b: (copy_bits(st.ckpt[b]), st.out_codes[b].cpu().numpy(), st.out_scales[b].cpu().numpy(),
                          tw.ckpt[b].cpu().numpy(), int(fc_prev[b]), int(fc_now[b])) for b in reqs})
        fc_prev = fc_now
    assert rssm.rssm_get_error(st) == 0 and rssm.rssm_get_error(tw) == 0
    assert torch.equal(y, y2)
    refreshed = 0
    for b in reqs:
        upd0 = copy_bits(initial_update_copy(inp["ckpt"][b], kind))
        codes0, scales0 = orc.fp4_quant(orc.widen(UPD[kind][1], upd0, None, upd0.shape).astype(np.float32))
        r = request_inputs(inp, b)
        req = orc.LowPrecRequest(UPD[kind][1], True, upd0, codes0, scales0, shape.ngroups, L + K, r["A"],
                                 r["D"], seed, b)
        req.flush_count.value = 1
        for s in range(steps):
            ys = req.verify(r["x"][s], r["B"][s], r["C"][s], r["dt"][s])
            assert_close(to_np(y[s, b]), ys, f"verify on the FP4 copy at spec_b512_k4, step {s}, request {b}")
            req.accept(int(n_host[s, b]))
            if req.pos >= L:
                upd, codes, scales, v32, fc_b, fc_a = snaps[s][b]
                assert fc_a == fc_b + 1
                v64 = req.refresh(want_v32=True).astype(np.float64)
                assert_close(v32.astype(np.float64), v64, f"fp32 fold at spec_b512_k4, request {b}")
                refresh_bits_of(kind, seed, b, fc_b, upd, codes, scales, v32,
                                f"speculative {kind} + FP4 refresh at spec_b512_k4")
                refreshed += 1
                break  # later verifies read a copy requantised from the GPU's own fold
    assert refreshed >= 3


@pytest.mark.parametrize("shape", SHAPES, ids=SHAPE_IDS)
def test_shared_fp4_forced_refresh_requantises_bit_exact(shape):
    """A forced refresh of the shared FP4 copy with an empty buffer folds
    nothing (v = h_0, the dequantised copy): the re-quantised codes and
    scales equal the oracle's FP4 quantisation of the dequantised values,
    bit for bit (s4's shared-precision control)."""
    Bz, H, P, N = shape.batch, shape.nheads, shape.head_dim, shape.d_state
    inp = make_inputs(shape, 1, 33, torch.bfloat16, device="cuda")
    desc, st = fp4_control_state(shape, inp, 6)
    c0, s0 = st.ckpt.cpu().numpy(), st.ckpt_scales.cpu().numpy()
    codes, scales = orc.fp4_quant(orc.widen(orc.FP4, c0, s0, (Bz, H, P, N)).astype(np.float32))
    rssm.rssm_lowprec_refresh(st, inp["A"], force=True)
    assert rssm.rssm_get_error(st) == 0
    assert int(np.count_nonzero(st.ckpt.cpu().numpy() != codes.reshape(c0.shape))) == 0
    assert int(np.count_nonzero(st.ckpt_scales.cpu().numpy() != scales.reshape(s0.shape))) == 0
    assert st.flush_count.cpu().tolist() == [1] * Bz and st.pos.cpu().tolist() == [0] * Bz


@pytest.mark.parametrize("shape", SHAPES, ids=SHAPE_IDS)
def test_shared_fp4_control_decode_matches_oracle(shape):
    """The shared FP4 control (s4's ablation): decode reads the one FP4 copy
    and the refresh re-quantises it. Outputs match the oracle; the
    re-quantised codes and scales equal the oracle's FP4 quantisation of the
    fp32 fold that an fp32 twin (same starting values) computes, bit for
    bit, and that fold matches the oracle's fp64 fold."""
    L = shape.interval
    Bz, H, P, N = shape.batch, shape.nheads, shape.head_dim, shape.d_state
    inp = make_inputs(shape, L, 32, torch.bfloat16, device="cuda")
    desc, st = fp4_control_state(shape, inp, 5)
    codes0, scales0 = orc.fp4_quant(inp["ckpt"].cpu().numpy())
    assert np.array_equal(st.ckpt.cpu().numpy(), codes0) and np.array_equal(st.ckpt_scales.cpu().numpy(), scales0)
    vals = orc.widen(orc.FP4, codes0, scales0, (Bz, H, P, N)).astype(np.float32)
    _, tw = f32_twin(shape, torch.from_numpy(vals).cuda(), 5, out_copy=False)
    _, tf = f32_twin(shape, torch.from_numpy(vals).cuda(), 5)   # the refresh kernel's fp32 fold
    y = torch.empty((L, Bz, H, P), device="cuda")
    y2 = torch.empty_like(y)
    y3 = torch.empty_like(y)
    for t in range(L):
        args = (inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"])
        rssm.rssm_decode_step(st, *args, y[t])
        rssm.rssm_decode_step(tw, *args, y2[t])
        rssm.rssm_decode_step(tf, *args, y3[t])
    rssm.rssm_lowprec_refresh(st, inp["A"])
    rssm.rssm_lowprec_refresh(tw, inp["A"])
    rssm.rssm_lowprec_refresh(tf, inp["A"])
    assert rssm.rssm_get_error(st) == 0 and rssm.rssm_get_error(tw) == 0 and rssm.rssm_get_error(tf) == 0
    assert_refresh_bits("fp4", 5, st, tf, None, range(Bz), "shared FP4 refresh")
    for b in range(Bz):
        r = request_inputs(inp, b)
        req = orc.LowPrecRequest(orc.FP4, False, None, codes0[b], scales0[b], shape.ngroups, L, r["A"], r["D"], 5, b)
        ys = np.stack([req.decode(r["x"][t], r["B"][t], r["C"][t], r["dt"][t]) for t in range(L)])
        assert_close(to_np(y[:, b]), ys, f"shared FP4 decode, request {b}")
        assert_close(to_np(y2[:, b]), ys, f"fp32 twin decode, request {b}")
        v64 = req.refresh(want_v32=True).astype(np.float64)
        assert_close(to_np(tw.ckpt[b]), v64, f"fp32 fold of the shared FP4 refresh, request {b}")
        assert_close(to_np(tf.ckpt[b]), v64, f"fp32 fold of the refresh kernel, request {b}")


def test_shared_fp4_control_split_b256_sampled():
    """The shared FP4 control at the bench's size (split_b256) and launch
    configuration: one interval of decodes reading the FP4 copy and its
    re-quantising refresh, with an fp32 twin from the same dequantised
    values. For sampled requests the outputs match the oracle, the twin's
    fold matches the fp64 fold, and the re-quantised codes and scales equal
    the oracle's FP4 quantisation of the twin's fold bit for bit."""
    w = WORKLOADS["split_b256"]
    shape = w["shape"]
    L = shape.interval
    Bz, H, P, N = shape.batch, shape.nheads, shape.head_dim, shape.d_state
    inp = make_inputs(shape, L, w["seed"], w["in_dtype"], device="cuda")
    seed = w["seed"]
    desc, st = fp4_control_state(shape, inp, seed)
    vals = torch.empty((Bz, H, P, N), dtype=torch.float32, device="cuda")
    reqs = sample_requests(Bz, 6)
    codes0, scales0 = {}, {}
    for b in range(Bz):  # dequantised starting values, request by request
        c, sc = st.ckpt[b].cpu().numpy(), st.ckpt_scales[b].cpu().numpy()
        vals[b].copy_(torch.from_numpy(orc.widen(orc.FP4, c, sc, (H, P, N)).astype(np.float32)))
        if b in reqs:
            codes0[b], scales0[b] = c, sc
    _, tw = f32_twin(shape, vals, seed, out_copy=False)
    _, tf = f32_twin(shape, vals, seed)   # the refresh kernel's fp32 fold
    del vals
    y = torch.empty((L, Bz, H, P), device="cuda")
    y2 = torch.empty_like(y)
    y3 = torch.empty_like(y)
    for t in range(L):
        args = (inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"])
        rssm.rssm_decode_step(st, *args, y[t])
        rssm.rssm_decode_step(tw, *args, y2[t])
        rssm.rssm_decode_step(tf, *args, y3[t])
    rssm.rssm_lowprec_refresh(st, inp["A"])
    rssm.rssm_lowprec_refresh(tw, inp["A"])
    rssm.rssm_lowprec_refresh(tf, inp["A"])
    assert rssm.rssm_get_error(st) == 0 and rssm.rssm_get_error(tw) == 0 and rssm.rssm_get_error(tf) == 0
    assert_refresh_bits("fp4", seed, st, tf, None, reqs, "shared FP4 refresh at split_b256")
    for b in reqs:
        r = request_inputs(inp, b)
        req = orc.LowPrecRequest(orc.FP4, False, None, codes0[b], scales0[b], shape.ngroups, L, r["A"], r["D"],
                                 seed, b)
        ys = np.stack([req.decode(r["x"][t], r["B"][t], r["C"][t], r["dt"][t]) for t in range(L)])
        assert_close(to_np(y[:, b]), ys, f"shared FP4 decode at split_b256, request {b}")
        v64 = req.refresh(want_v32=True).astype(np.float64)
        assert_close(to_np(tw.ckpt[b]), v64, f"fp32 fold of the shared FP4 refresh at split_b256, request {b}")
        assert_close(to_np(tf.ckpt[b]), v64, f"fp32 fold of the refresh kernel at split_b256, request {b}")


@pytest.mark.parametrize("shape", SPLIT_SHAPES, ids=SPLIT_IDS)
@pytest.mark.parametrize("kind", ["bf16", "e4m3"])
def test_shared_copy_decode_and_refresh_match_oracle(kind, shape):
    """One bf16 or e4m3 copy both read by decode and updated by the refresh
    (the secondary shared-precision control of s4): the outputs match the
    oracle reading the same values, and the stochastically rounded copy
    equals the oracle's rounding of the fp32 fold (from an fp32 twin with the
    same starting values) bit for bit."""
    L = shape.interval
    Bz, H, P = shape.batch, shape.nheads, shape.head_dim
    inp = make_inputs(shape, L, 36, torch.bfloat16, device="cuda")
    seed = 0xC0FFEE
    desc = desc_for(shape, update_dtype=UPD[kind][0], seed=seed)
    st = rssm.RssmState(desc)
    st.ckpt.copy_(initial_update_copy(inp["ckpt"], kind))
    _, tw = f32_twin(shape, widened(kind, st), seed, out_copy=False)
    _, tf = f32_twin(shape, widened(kind, st), seed)   # the refresh kernel's fp32 fold
    upd0 = copy_bits(initial_update_copy(inp["ckpt"], kind))
    y = torch.empty((L, Bz, H, P), device="cuda")
    y2 = torch.empty_like(y)
    y3 = torch.empty_like(y)
    for t in range(L):
        args = (inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"])
        rssm.rssm_decode_step(st, *args, y[t])
        rssm.rssm_decode_step(tw, *args, y2[t])
        rssm.rssm_decode_step(tf, *args, y3[t])
    fc_before = st.flush_count.cpu().tolist()
    rssm.rssm_lowprec_refresh(st, inp["A"])
    rssm.rssm_lowprec_refresh(tw, inp["A"])
    rssm.rssm_lowprec_refresh(tf, inp["A"])
    assert rssm.rssm_get_error(st) == 0 and rssm.rssm_get_error(tw) == 0 and rssm.rssm_get_error(tf) == 0
    assert_refresh_bits(kind, seed, st, tf, fc_before, range(Bz), f"shared {kind} refresh")
    for b in range(Bz):
        r = request_inputs(inp, b)
        req = orc.LowPrecRequest(UPD[kind][1], False, upd0[b], None, None, shape.ngroups, L, r["A"], r["D"], seed, b)
        ys = np.stack([req.decode(r["x"][t], r["B"][t], r["C"][t], r["dt"][t]) for t in range(L)])
        assert_close(to_np(y[:, b]), ys, f"shared {kind} decode, request {b}")
        v64 = req.refresh(want_v32=True).astype(np.float64)
        assert_close(to_np(tw.ckpt[b]), v64, f"fp32 fold of the shared {kind} refresh, request {b}")
        assert_close(to_np(tf.ckpt[b]), v64, f"fp32 fold of the refresh kernel, request {b}")
    assert st.flush_count.cpu().tolist() == [1] * Bz and st.pos.cpu().tolist() == [0] * Bz


def test_shared_bf16_control_split_b256_sampled():
    """The shared bf16 control (one bf16 copy read by decode and updated
    with stochastic rounding) at the bench's size (split_b256) and launch
    configuration: one interval of decodes, then the refresh, beside an
    fp32 twin with an FP4 output copy that runs the same refresh kernel.
    For sampled requests the outputs match the oracle reading the same
    copy, the twin's fold matches the oracle's fp64 fold, and the refreshed
    copy equals the oracle's rounding of that fold bit for bit."""
    w = WORKLOADS["split_b256"]
    shape = w["shape"]
    L = shape.interval
    Bz, H, P = shape.batch, shape.nheads, shape.head_dim
    inp = make_inputs(shape, L, w["seed"], w["in_dtype"], device="cuda")
    seed = w["seed"]
    st = rssm.RssmState(desc_for(shape, update_dtype=rssm.RSSM_BF16, seed=seed))
    st.ckpt.copy_(initial_update_copy(inp["ckpt"], "bf16"))
    _, tf = f32_twin(shape, widened("bf16", st), seed)   # the refresh kernel's fp32 fold
    y = torch.empty((L, Bz, H, P), device="cuda")
    y2 = torch.empty_like(y)
    for t in range(L):
        args = (inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"])
        rssm.rssm_decode_step(st, *args, y[t])
        rssm.rssm_decode_step(tf, *args, y2[t])
    fc_before = st.flush_count.cpu().tolist()
    rssm.rssm_lowprec_refresh(st, inp["A"])
    rssm.rssm_lowprec_refresh(tf, inp["A"])
    assert rssm.rssm_get_error(st) == 0 and rssm.rssm_get_error(tf) == 0
    reqs = sample_requests(Bz, 6)
    assert_refresh_bits("bf16", seed, st, tf, fc_before, reqs, "shared bf16 refresh at split_b256")
    for b in reqs:
        upd0 = copy_bits(initial_update_copy(inp["ckpt"][b], "bf16"))
        r = request_inputs(inp, b)
        req = orc.LowPrecRequest(orc.BF16, False, upd0, None, None, shape.ngroups, L, r["A"], r["D"], seed, b)
        ys = np.stack([req.decode(r["x"][t], r["B"][t], r["C"][t], r["dt"][t]) for t in range(L)])
        assert_close(to_np(y[:, b]), ys, f"shared bf16 decode at split_b256, request {b}")
        v64 = req.refresh(want_v32=True).astype(np.float64)
        assert_close(to_np(tf.ckpt[b]), v64, f"fp32 fold of the shared bf16 refresh at split_b256, request {b}")
    assert st.flush_count.cpu().tolist() == [1] * Bz and st.pos.cpu().tolist() == [0] * Bz


@pytest.mark.parametrize("K", [4, 6])
@pytest.mark.parametrize("kind", ["bf16", "e4m3"])
def test_speculative_verify_on_shared_copy_matches_oracle(kind, K):
    """Verify (s3) reading a bf16 or e4m3 copy that is also the update copy
    (the secondary shared-precision control of s4): the K+1 outputs of every
    step match the oracle reading the same copy values, and the refresh
    after accept equals the oracle's rounding of the fp32 twin's fold."""
    shape = LayerShape(4, 8, 64, 128, 2, interval=16, max_draft=K)
    n_host = SPLIT_SPEC[K]
    steps, L = n_host.shape[0], 16
    inp = make_inputs(shape, steps, 35, torch.bfloat16, device="cuda", ntok=K + 1)
    n_acc = torch.from_numpy(n_host).cuda()
    seed = 0xACE
    desc = desc_for(shape, update_dtype=UPD[kind][0], seed=seed)
    st = rssm.RssmState(desc)
    st.ckpt.copy_(initial_update_copy(inp["ckpt"], kind))
    _, tw = f32_twin(shape, widened(kind, st), seed, out_copy=False)
    _, tf = f32_twin(shape, widened(kind, st), seed)   # the refresh kernel's fp32 fold
    upd0 = copy_bits(initial_update_copy(inp["ckpt"], kind))
    y = torch.empty((steps, shape.batch, K + 1, shape.nheads, shape.head_dim), device="cuda")
    y2 = torch.empty_like(y)
    y3 = torch.empty_like(y)
    fc_before = st.flush_count.cpu().tolist()
    for s in range(steps):
        args = (inp["x"][s], inp["B"][s], inp["C"][s], inp["dt"][s], inp["A"], inp["D"])
        for state, out in ((st, y), (tw, y2), (tf, y3)):
            rssm.rssm_verify(state, K, *args, out[s])
            rssm.rssm_accept(state, n_acc[s])
            rssm.rssm_lowprec_refresh(state, inp["A"])
    assert rssm.rssm_get_error(st) == 0 and rssm.rssm_get_error(tw) == 0 and rssm.rssm_get_error(tf) == 0
    folded = []
    for b in range(shape.batch):
        r = request_inputs(inp, b)
        req = orc.LowPrecRequest(UPD[kind][1], False, upd0[b], None, None, shape.ngroups, L + K, r["A"], r["D"],
                                 seed, b)
        for s in range(steps):
            ys = req.verify(r["x"][s], r["B"][s], r["C"][s], r["dt"][s])
            assert_close(to_np(y[s, b]), ys, f"verify on the shared {kind} copy, step {s}, request {b}")
            assert_close(to_np(y2[s, b]), ys, f"verify on the fp32 twin, step {s}, request {b}")
            req.accept(int(n_host[s, b]))
            if req.pos >= L:
                req.refresh()
                folded.append(b)
        assert st.pos[b].item() == req.pos
    assert len(folded) == 3
    assert_refresh_bits(kind, seed, st, tf, fc_before, folded, f"speculative shared {kind} refresh")


def run_lowprec(desc, st, inp, steps):
    y = torch.empty((steps,) + tuple(inp["x"].shape[1:]), device="cuda")
    for t in range(steps):
        rssm.rssm_decode_step(st, inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"], y[t])
        if (t + 1) % desc.interval == 0:
            rssm.rssm_lowprec_refresh(st, inp["A"])
    return y


def rel_rms(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return math.sqrt(float(np.mean((a - b) ** 2)) / float(np.mean(b * b)))


def test_split_b256_error_report():
    """batch 256, 64 heads, 64 x 128, 512 steps: output error of the precision
    split (bf16 or e4m3 stochastic-rounded update copy + FP4 output copy)
    and of the shared-copy controls, against the fp64 oracle and against the
    fp32-state GPU run. The split keeps the error below the shared FP4 copy's
    (s4: errors of the output copy do not feed later updates)."""
    w = WORKLOADS["split_b256"]
    shape, steps = w["shape"], w["steps"]
    inp = make_inputs(shape, steps, w["seed"], w["in_dtype"], device="cuda")
    seed = w["seed"]
    from gpu_helpers import gpu_replay_decode
    y32, _, _ = gpu_replay_decode(desc_for(shape), inp, steps)
    runs = {}
    for kind in ("bf16", "e4m3"):
        d, st = split_state(shape, inp, kind, seed)
        runs[f"split_{kind}_sr+fp4"] = run_lowprec(d, st, inp, steps)
    d, st = fp4_control_state(shape, inp, seed)
    runs["shared_fp4"] = run_lowprec(d, st, inp, steps)
    d = desc_for(shape, update_dtype=rssm.RSSM_BF16, seed=seed)
    st = rssm.RssmState(d)
    st.ckpt.copy_(inp["ckpt"].to(torch.bfloat16))
    runs["shared_bf16_sr"] = run_lowprec(d, st, inp, steps)
    reqs = sample_requests(shape.batch, 4)
    refs = oracle_map([("conv", request_inputs(inp, b), []) for b in reqs])
    report = {"workload": "split_b256", "steps": steps, "metric": "rel rms of y"}
    y32s = np.stack([to_np(y32[:, b]) for b in reqs])
    yref = np.stack([r[0] for r in refs])
    report["fp32_state_vs_oracle"] = rel_rms(y32s, yref)
    for name, y in runs.items():
        ys = np.stack([to_np(y[:, b]) for b in reqs])
        report[name] = {"vs_oracle": rel_rms(ys, yref),
                        "vs_fp32_gpu_all_requests": rel_rms(to_np(y), to_np(y32))}
    out_dir = os.environ.get("RSSM_REPORT_DIR")
    if out_dir:
        os.makedirs(out_dir, exist_ok=True)
        with open(os.path.join(out_dir, "precision_split_b256.json"), "w") as f:
            json.dump(report, f, indent=1)
    print(json.dumps(report, indent=1))
    assert report["fp32_state_vs_oracle"] < 1e-5
    ctrl = report["shared_fp4"]["vs_oracle"]
    assert report["split_bf16_sr+fp4"]["vs_oracle"] < ctrl
    assert report["split_e4m3_sr+fp4"]["vs_oracle"] < ctrl
