"""GPU parity of the replay decode, flush, verify/accept and conventional
kernels against the fp64 oracle (ReplaySSM article s1 and s3), through the
C ABI. Tolerance: max |dy| <= 1e-4 * rms(y_ref) per request, and the same
bound on every flushed checkpoint against the oracle's recurrent state."""
import numpy as np
import pytest
import torch

from hybrid_model_ssm_replay_b200 import rssm
from hybrid_model_ssm_replay_b200.inputs import WORKLOADS, LayerShape, accept_lengths, make_inputs

from gpu_helpers import (assert_close, desc_for, gpu_conv_decode, gpu_conv_spec, gpu_replay_decode, gpu_spec,
                         oracle_map, request_inputs, sample_requests, to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from hybrid_model_ssm_replay_b200 import build
    build.build()
    torch.cuda.init()


def check_decode_case(shape, steps, seed, in_dtype, fused, reqs=None, conv=True):
    inp = make_inputs(shape, steps, seed, in_dtype, device="cuda")
    desc = desc_for(shape, in_dtype, flags=rssm.RSSM_FLAG_FUSED_FLUSH if fused else 0)
    reqs = reqs if reqs is not None else sample_requests(shape.batch)
    idx = torch.tensor(reqs, device="cuda")
    y, snaps, st = gpu_replay_decode(desc, inp, steps, fused, snap=idx)
    flush_steps = sorted(snaps)
    assert len(flush_steps) == steps // shape.interval
    yc = None
    if conv:
        yc, csnaps, _ = gpu_conv_decode(desc, inp, steps, snap=idx, snap_steps=set(flush_steps))
    res = oracle_map([("conv", request_inputs(inp, b), flush_steps) for b in reqs])
    for i, (b, (y_ref, s_ref)) in enumerate(zip(reqs, res)):
        assert_close(to_np(y[:, b]), y_ref, f"replay y, request {b}")
        for t in flush_steps:
            assert_close(snaps[t][i], s_ref[t], f"checkpoint after step {t}, request {b}")
        if conv:
            assert_close(to_np(yc[:, b]), y_ref, f"conventional y, request {b}")
            for t in flush_steps:
                assert_close(csnaps[t][i], s_ref[t], f"conventional state after step {t}, request {b}")
    rem = steps % shape.interval
    assert set(st.pos.cpu().tolist()) == {rem}
    assert set(st.flush_count.cpu().tolist()) == {steps // shape.interval}
    assert set(st.arrive.cpu().tolist()) == {0}
    assert rssm.rssm_get_error(st) == 0
    return y


@pytest.mark.parametrize("fused", [False, True])
def test_tiny_workload_all_requests(fused):
    w = WORKLOADS["tiny"]
    check_decode_case(w["shape"], w["steps"], w["seed"], w["in_dtype"], fused, reqs=list(range(4)))


@pytest.mark.parametrize("in_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [LayerShape(5, 6, 40, 32, 3, interval=5),
                                   LayerShape(3, 4, 17, 64, 1, interval=7),
                                   LayerShape(2, 8, 8, 128, 4, interval=16),
                                   LayerShape(7, 2, 33, 16, 2, interval=1)])
def test_ragged_shapes(shape, in_dtype):
    """Tails: head_dim not a multiple of the rows a CTA pass covers, odd
    intervals, interval 1, every supported d_state, a partial last interval."""
    steps = 3 * shape.interval + 2
    check_decode_case(shape, steps, 11, in_dtype, False, reqs=list(range(shape.batch)))
    if shape.interval <= 16:
        check_decode_case(shape, steps, 12, in_dtype, True, reqs=list(range(shape.batch)), conv=False)


def test_small_b256_full_run_sampled():
    """batch 256, 64 heads, 64 x 128, 8 groups, bf16, 512 steps (32 flushes):
    8 sampled requests x all heads x all steps + every flushed checkpoint."""
    w = WORKLOADS["small_b256"]
    check_decode_case(w["shape"], w["steps"], w["seed"], w["in_dtype"], False)


def test_small_b256_fused_flush_sampled():
    w = WORKLOADS["small_b256"]
    check_decode_case(w["shape"], 64, w["seed"], w["in_dtype"], True, conv=False)


def test_large_b512_full_run_sampled():
    w = WORKLOADS["large_b512"]
    check_decode_case(w["shape"], w["steps"], w["seed"], w["in_dtype"], False, conv=False)


@pytest.mark.parametrize("batch", [1, 32, 128])
def test_large_shape_batch_sweep(batch):
    w = WORKLOADS["large_b512"]
    s = w["shape"]
    shape = LayerShape(batch, s.nheads, s.head_dim, s.d_state, s.ngroups, s.interval)
    check_decode_case(shape, 48, w["seed"], w["in_dtype"], False)


# ----------------------------------------------------------- speculative

def check_spec_case(shape, steps, seed, reqs, conv=True, in_dtype=torch.bfloat16):
    K = shape.max_draft
    inp = make_inputs(shape, steps, seed, in_dtype, device="cuda", ntok=K + 1)
    n_acc = accept_lengths(steps, shape.batch, K, seed, device="cuda")
    desc = desc_for(shape, in_dtype)
    y, st = gpu_spec(desc, inp, n_acc, steps)
    n_np = n_acc.cpu().numpy()
    res = oracle_map([("spec", request_inputs(inp, b), (n_np[:, b], shape.interval, K)) for b in reqs])
    for b, (y_ref, _ck, poss) in zip(reqs, res):
        assert_close(to_np(y[:, b]), y_ref, f"verify outputs (all K+1 per step), request {b}")
        assert int(st.pos[b]) == poss[-1]
    assert rssm.rssm_get_error(st) == 0
    if conv:
        yc, copies, cur = gpu_conv_spec(desc, inp, n_acc, steps)
        for b, (y_ref, _ck, _p) in zip(reqs, res):
            # accepted tokens (j <= n) agree with the oracle; rejected drafts of
            # the conventional scheme continue from the same state too
            assert_close(to_np(yc[:, b]), y_ref, f"conventional verify outputs, request {b}")
        # accepted lengths are the same input for both schemes
        assert torch.equal(cur, n_acc[-1])


def test_spec_small_all_requests():
    shape = LayerShape(6, 4, 16, 32, 2, interval=16, max_draft=4)
    check_spec_case(shape, 60, 5, list(range(6)))


def test_spec_b512_k4_sampled():
    w = WORKLOADS["spec_b512_k4"]
    check_spec_case(w["shape"], w["steps"], w["seed"], sample_requests(w["shape"].batch, 4), conv=True)


@pytest.mark.parametrize("shape", [LayerShape(5, 4, 32, 128, 2, interval=16, max_draft=1),
                                   LayerShape(5, 4, 32, 128, 2, interval=16, max_draft=6),
                                   LayerShape(3, 4, 32, 128, 2, interval=27, max_draft=5),
                                   LayerShape(4, 6, 40, 128, 3, interval=16, max_draft=4)],
                         ids=["k1", "k6", "cap32", "headdim40"])
def test_spec_pipelined_drafts_and_capacity(shape):
    """The pipelined verify at other draft counts (2 and 7 tokens per call,
    under the kernel's 5- and 8-token bounds), with the largest buffer
    (interval 27 + 5 drafts = 32 slots: two 16-slot B.C products, four
    8-slot replay steps), and with head_dim 40 (a last 16-row group that is
    half empty), every request against the oracle, the conventional verify
    beside it."""
    check_spec_case(shape, 40, 13, list(range(shape.batch)))


@pytest.mark.parametrize("K", [4, 6])
def test_spec_pipelined_fp32_inputs(K):
    """The pipelined verify with fp32 x/B/C (its float-input instantiations)."""
    shape = LayerShape(4, 4, 32, 128, 2, interval=16, max_draft=K)
    check_spec_case(shape, 30, 17, list(range(shape.batch)), in_dtype=torch.float32)


def test_spec_rollback_leaves_no_trace():
    """verify K+1 then accept(n) gives the same later outputs and checkpoint as
    decoding only the n+1 accepted tokens (s3), on the GPU itself."""
    shape = LayerShape(4, 4, 32, 64, 2, interval=16, max_draft=4)
    K = 4
    inp = make_inputs(shape, 6, 21, torch.bfloat16, device="cuda", ntok=K + 1)
    tail = make_inputs(shape, 20, 22, torch.bfloat16, device="cuda")
    n = torch.tensor([0, 1, 3, 4], dtype=torch.int32, device="cuda")
    da = desc_for(shape)
    sa = rssm.RssmState(da)
    sa.ckpt.copy_(inp["ckpt"])
    sb = rssm.RssmState(da)
    sb.ckpt.copy_(inp["ckpt"])
    ya = torch.empty((shape.batch, K + 1, 4, 32), device="cuda")
    rssm.rssm_verify(sa, K, inp["x"][0], inp["B"][0], inp["C"][0], inp["dt"][0], inp["A"], inp["D"], ya)
    rssm.rssm_accept(sa, n)
    # plain decode of the accepted tokens, request by request: token j goes to the requests with n >= j
    for j in range(K + 1):
        yb = torch.empty((shape.batch, 4, 32), device="cuda")
        xs, Bs, Cs, dts = (inp[k][0][:, j].contiguous() for k in ("x", "B", "C", "dt"))
        live = (n >= j)
        snap_pos = sb.pos.clone()
        rssm.rssm_decode_step(sb, xs, Bs, Cs, dts, inp["A"], inp["D"], yb)
        # requests that should not take token j: undo by restoring pos (their slot is rewritten later)
        sb.pos.copy_(torch.where(live, sb.pos, snap_pos))
        for b in range(shape.batch):
            if live[b]:
                assert torch.allclose(yb[b], ya[b, j], rtol=0, atol=1e-5 * float(ya.abs().max()))
    assert torch.equal(sa.pos, sb.pos)
    for t in range(20):
        y1 = torch.empty((shape.batch, 4, 32), device="cuda")
        y2 = torch.empty_like(y1)
        for st, yy in ((sa, y1), (sb, y2)):
            rssm.rssm_decode_step(st, tail["x"][t], tail["B"][t], tail["C"][t], tail["dt"][t], inp["A"], inp["D"], yy)
            rssm.rssm_flush(st, inp["A"])
        assert torch.equal(y1, y2)
    assert torch.equal(sa.ckpt, sb.ckpt)


# ------------------------------------------------ errors, determinism, resume

def small_state(shape=LayerShape(4, 4, 32, 64, 2, interval=16, max_draft=2)):
    inp = make_inputs(shape, 4, 3, torch.bfloat16, device="cuda", ntok=0)
    desc = desc_for(shape)
    st = rssm.RssmState(desc)
    st.ckpt.copy_(inp["ckpt"])
    return shape, inp, desc, st


@pytest.mark.parametrize("d_state", [64, 128])
def test_device_error_bad_pos_is_reported_and_contained(d_state):
    """d_state 128 runs the pipelined kernel, 64 the per-tile kernel."""
    shape, inp, desc, st = small_state(LayerShape(4, 4, 32, d_state, 2, interval=16, max_draft=2))
    y = torch.full((4, 4, 32), 7.0, device="cuda")
    st.pos[2] = 99
    rssm.rssm_decode_step(st, inp["x"][0], inp["B"][0], inp["C"][0], inp["dt"][0], inp["A"], inp["D"], y)
    assert rssm.rssm_get_error(st) == 1
    assert rssm.rssm_get_error(st) == 0          # read-and-clear
    assert torch.all(y[2] == 7.0)                 # bad request untouched
    assert not torch.any(y[0] == 7.0)
    assert st.pos.cpu().tolist() == [1, 1, 99, 1]
    assert set(st.arrive.cpu().tolist()) == {0}


@pytest.mark.parametrize("d_state", [64, 128])
def test_device_error_capacity_and_accept_range(d_state):
    shape, inp, desc, st = small_state(LayerShape(4, 4, 32, d_state, 2, interval=16, max_draft=2))
    K = 2
    vi = make_inputs(shape, 1, 4, torch.bfloat16, device="cuda", ntok=K + 1)
    y = torch.empty((4, K + 1, 4, 32), device="cuda")
    st.pos.fill_(16)                               # 16 + 3 > capacity 18
    rssm.rssm_verify(st, K, vi["x"][0], vi["B"][0], vi["C"][0], vi["dt"][0], vi["A"], vi["D"], y)
    assert rssm.rssm_get_error(st) == 2
    st.pos.zero_()
    rssm.rssm_accept(st, torch.tensor([0, 3, 1, -1], dtype=torch.int32, device="cuda"))
    assert rssm.rssm_get_error(st) == 3
    assert st.pos.cpu().tolist() == [1, 0, 2, 0]
    with pytest.raises(rssm.RssmError):
        rssm.rssm_verify(st, K + 1, vi["x"][0], vi["B"][0], vi["C"][0], vi["dt"][0], vi["A"], vi["D"], y)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    cur = torch.zeros(4, dtype=torch.int32, device="cuda")
    rssm.rssm_conv_accept(desc, torch.tensor([0, 1, 5, 2], dtype=torch.int32, device="cuda"), cur, K, err)
    assert int(err[0]) == 3 and cur.cpu().tolist() == [0, 1, 0, 2]


def test_bit_reproducible():
    w = WORKLOADS["small_b256"]
    s = w["shape"]
    shape = LayerShape(16, s.nheads, s.head_dim, s.d_state, s.ngroups)
    inp = make_inputs(shape, 40, 9, torch.bfloat16, device="cuda")
    desc = desc_for(shape)
    y1, _, st1 = gpu_replay_decode(desc, inp, 40)
    y2, _, st2 = gpu_replay_decode(desc, inp, 40)
    assert torch.equal(y1, y2) and torch.equal(st1.ckpt, st2.ckpt)


def test_resume_from_host_copy_is_bit_identical():
    """The replay state (checkpoint, buffer, pos, flush count) is the whole
    decode state: copied to the host mid-interval and restored into fresh
    buffers, the run continues bit for bit."""
    shape = LayerShape(8, 8, 64, 128, 2)
    inp = make_inputs(shape, 45, 10, torch.bfloat16, device="cuda")
    desc = desc_for(shape)
    y_ref, _, _ = gpu_replay_decode(desc, inp, 45)
    st = rssm.RssmState(desc)
    st.ckpt.copy_(inp["ckpt"])
    y = torch.empty_like(y_ref)
    names = ("ckpt", "xbuf", "bbuf", "dtbuf", "pos", "flush_count")
    for t in range(45):
        if t == 21:
            saved = {k: getattr(st, k).cpu() for k in names}
            st = rssm.RssmState(desc)
            for k in names:
                getattr(st, k).copy_(saved[k])
        rssm.rssm_decode_step(st, inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"], y[t])
        if (t + 1) % 16 == 0:
            rssm.rssm_flush(st, inp["A"])
    assert torch.equal(y, y_ref)
