"""Prefill of a prompt into the checkpoint (the step before the decode path;
the article is silent on it): the checkpoint after rssm_prefill equals the
fp64 recurrence over the prompt, and decoding on from it equals the
recurrence over prompt + decoded tokens. bf16 inputs at d_state 128 and
head_dim 16/32/48/64 run the tensor-core contraction over 64-token chunks
(whole and partial chunks are covered); other shapes the chunked CUDA-core
fold."""
import numpy as np
import pytest
import torch

from hybrid_model_ssm_replay_b200 import rssm
from hybrid_model_ssm_replay_b200.inputs import WORKLOADS, LayerShape, make_inputs

from gpu_helpers import assert_close, desc_for, oracle_map, request_inputs, sample_requests, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from hybrid_model_ssm_replay_b200 import build
    build.build()


def split(inp, T0):
    """The first T0 tokens (prompt) and the rest (decode) of a run's inputs."""
    pre = {k: (v[:T0].contiguous() if k in ("x", "B", "C", "dt") else v) for k, v in inp.items()}
    dec = {k: (v[T0:].contiguous() if k in ("x", "B", "C", "dt") else v) for k, v in inp.items()}
    return pre, dec


@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("shape,T0", [(LayerShape(4, 4, 40, 128, 2), 50), (LayerShape(3, 4, 17, 64, 1), 33),
                                      (LayerShape(2, 2, 8, 16, 1), 16), (LayerShape(3, 4, 64, 128, 2), 150),
                                      (LayerShape(2, 4, 32, 128, 2), 64), (LayerShape(2, 2, 48, 128, 1), 200)],
                         ids=["d128", "ragged", "one-chunk", "umma-5chunks", "mma-1chunk", "mma-headdim48"])
def test_prefill_then_decode_matches_recurrence(shape, T0, in_dtype):
    steps = T0 + 24
    inp = make_inputs(shape, steps, 41, in_dtype, device="cuda")
    pre, dec = split(inp, T0)
    desc = desc_for(shape, in_dtype)
    st = rssm.RssmState(desc)
    st.ckpt.copy_(inp["ckpt"])
    rssm.rssm_prefill(st, pre["x"], pre["B"], pre["dt"], inp["A"])
    ck = st.ckpt.double().cpu().numpy()
    L = shape.interval
    y = torch.empty((steps - T0,) + tuple(inp["x"].shape[1:]), device="cuda")
    for t in range(steps - T0):
        rssm.rssm_decode_step(st, dec["x"][t], dec["B"][t], dec["C"][t], dec["dt"][t], inp["A"], inp["D"], y[t])
        if (t + 1) % L == 0:
            rssm.rssm_flush(st, inp["A"])
    assert rssm.rssm_get_error(st) == 0
    reqs = list(range(shape.batch))
    res = oracle_map([("conv", request_inputs(inp, b), [T0 - 1]) for b in reqs])
    for b, (y_ref, snaps) in zip(reqs, res):
        assert_close(ck[b], snaps[T0 - 1], f"checkpoint after a {T0}-token prefill, request {b}")
        assert_close(to_np(y[:, b]), y_ref[T0:], f"decode after the prefill, request {b}")
    assert set(st.flush_count.cpu().tolist()) == {(steps - T0) // L}


@pytest.mark.parametrize("T0", [1, 31, 32, 33, 65])
def test_prefill_tensor_memory_chunk_edges(T0):
    """The tcgen05 prefill (head_dim 64, two heads per group) at prompt
    lengths around its 32-token chunks: one token, a chunk minus one, one
    chunk, a chunk plus one, two chunks plus one; every request's checkpoint
    against the recurrence."""
    shape = LayerShape(3, 8, 64, 128, 2)
    inp = make_inputs(shape, T0, 44 + T0, torch.bfloat16, device="cuda")
    st = rssm.RssmState(desc_for(shape))
    st.ckpt.copy_(inp["ckpt"])
    rssm.rssm_prefill(st, inp["x"], inp["B"], inp["dt"], inp["A"])
    assert rssm.rssm_get_error(st) == 0
    res = oracle_map([("conv", request_inputs(inp, b), [T0 - 1]) for b in range(shape.batch)])
    for b, (_, snaps) in enumerate(res):
        assert_close(st.ckpt[b].double().cpu().numpy(), snaps[T0 - 1], f"checkpoint after a {T0}-token prefill, "
                                                                        f"request {b}")


def test_prefill_b256_t512_sampled():
    """The bench's prefill: small_b256 shapes (batch 256, 64 heads, head_dim
    64, d_state 128, bf16 inputs), 512-token prompts, the tensor-core kernel
    at its launch configuration; the checkpoint of sampled requests against
    the fp64 recurrence."""
    w = WORKLOADS["small_b256"]
    shape, T0 = w["shape"], 512
    inp = make_inputs(shape, T0, 43, torch.bfloat16, device="cuda")
    st = rssm.RssmState(desc_for(shape))
    st.ckpt.copy_(inp["ckpt"])
    rssm.rssm_prefill(st, inp["x"], inp["B"], inp["dt"], inp["A"])
    assert rssm.rssm_get_error(st) == 0
    assert st.pos.cpu().tolist() == [0] * shape.batch
    reqs = sample_requests(shape.batch, 6)
    res = oracle_map([("conv", request_inputs(inp, b), [T0 - 1]) for b in reqs])
    for b, (_, snaps) in zip(reqs, res):
        assert_close(st.ckpt[b].double().cpu().numpy(), snaps[T0 - 1], f"checkpoint after a {T0}-token prefill, "
                                                                        f"request {b}")


def test_prefill_needs_an_empty_buffer_and_zero_tokens_change_nothing():
    shape = LayerShape(3, 2, 16, 128, 1)
    inp = make_inputs(shape, 20, 42, torch.bfloat16, device="cuda")
    desc = desc_for(shape)
    st = rssm.RssmState(desc)
    st.ckpt.copy_(inp["ckpt"])
    before = st.ckpt.clone()
    rssm.rssm_prefill(st, inp["x"][:0], inp["B"][:0], inp["dt"][:0], inp["A"])
    assert torch.equal(st.ckpt, before) and rssm.rssm_get_error(st) == 0
    st.pos[1] = 3
    rssm.rssm_prefill(st, inp["x"], inp["B"], inp["dt"], inp["A"])
    assert rssm.rssm_get_error(st) == 1  # RSSM_DEVERR_POS_RANGE
    assert torch.equal(st.ckpt[1], before[1])  # the request with buffered tokens is untouched
    assert not torch.equal(st.ckpt[0], before[0]) and not torch.equal(st.ckpt[2], before[2])
    assert st.pos.cpu().tolist() == [0, 3, 0]
