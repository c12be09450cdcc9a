"""rssm_decode_step_noalloc: the decode step for callers that cannot
allocate device memory, such as an engine that plans all of its device
memory ahead and hands each layer only its planned buffers. Its arrival
counters live in a device array inside the library instead of in a
caller-allocated scratch buffer.

Checked through the C ABI against rssm_decode_step on two calls in a row:
same outputs (within the parity tolerance of the other tests), same
positions and buffers; and over two whole intervals plus one token with the
fused fold (the one way to run an interval without any caller scratch),
against rssm_decode_step and against the fp64 recurrence. The file is named
to be collected last; it also passes on its own in a fresh process.
"""
import ctypes as ct

import pytest
import torch

from hybrid_model_ssm_replay_b200 import rssm
from hybrid_model_ssm_replay_b200.inputs import LayerShape, make_inputs

from gpu_helpers import assert_close, desc_for, request_inputs, to_np
from oracle import oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from hybrid_model_ssm_replay_b200 import build
    build.build()


@pytest.mark.parametrize("shape", [LayerShape(8, 16, 64, 128, 4), LayerShape(5, 4, 24, 64, 2)],
                         ids=["dstate128", "dstate64"])
def test_noalloc_decode_matches_decode_step(shape):
    inp = make_inputs(shape, 2, 41, torch.bfloat16, device="cuda")
    desc = desc_for(shape)
    ref = rssm.RssmState(desc)
    ref.ckpt.copy_(inp["ckpt"])
    na = rssm.RssmState(desc)
    na.ckpt.copy_(inp["ckpt"])
    na.struct.arrive = None  # the entry point must not need the scratch field
    for t in range(2):
        y_ref = torch.empty((shape.batch, shape.nheads, shape.head_dim), device="cuda")
        y_na = torch.full_like(y_ref, float("nan"))
        rssm.rssm_decode_step(ref, inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"], y_ref)
        rssm.rssm_decode_step_noalloc(na, inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"],
                                      y_na)
        torch.cuda.synchronize()
        assert_close(to_np(y_na), to_np(y_ref), f"noalloc decode, call {t}")
        assert torch.equal(na.pos, ref.pos) and set(na.pos.cpu().tolist()) == {t + 1}
        assert torch.equal(na.xbuf, ref.xbuf) and torch.equal(na.dtbuf, ref.dtbuf)
    assert rssm.rssm_get_error(na) == 0 and rssm.rssm_get_error(ref) == 0


@pytest.mark.parametrize("shape", [LayerShape(6, 16, 64, 128, 4), LayerShape(5, 4, 24, 64, 2)],
                         ids=["dstate128", "dstate64"])
def test_noalloc_fused_intervals_match_decode_step_and_oracle(shape):
    """2 intervals + 1 token with RSSM_FLAG_FUSED_FLUSH and no arrival field:
    the token that fills the buffer folds it (the last arrival, counted in
    the library's array, resets pos and bumps flush_count). Outputs, pos,
    flush_count and the checkpoint after each fold match rssm_decode_step
    with a caller-allocated scratch, and the outputs and folded checkpoints
    match the fp64 recurrence."""
    L = shape.interval
    steps = 2 * L + 1
    inp = make_inputs(shape, steps, 43, torch.bfloat16, device="cuda")
    desc = desc_for(shape, flags=rssm.RSSM_FLAG_FUSED_FLUSH)
    ref = rssm.RssmState(desc)
    ref.ckpt.copy_(inp["ckpt"])
    na = rssm.RssmState(desc)
    na.ckpt.copy_(inp["ckpt"])
    na.struct.arrive = None
    y_ref = torch.empty((steps, shape.batch, shape.nheads, shape.head_dim), device="cuda")
    y_na = torch.full_like(y_ref, float("nan"))
    ck = {}
    for t in range(steps):
        args = (inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"])
        rssm.rssm_decode_step(ref, *args, y_ref[t])
        rssm.rssm_decode_step_noalloc(na, *args, y_na[t])
        if (t + 1) % L == 0:
            assert torch.equal(na.ckpt, ref.ckpt), f"folded checkpoint after token {t}"
            ck[t] = na.ckpt.double().cpu().numpy()
    torch.cuda.synchronize()
    assert torch.equal(y_na, y_ref)
    assert na.pos.cpu().tolist() == [1] * shape.batch and torch.equal(na.pos, ref.pos)
    assert na.flush_count.cpu().tolist() == [2] * shape.batch and torch.equal(na.flush_count, ref.flush_count)
    assert rssm.rssm_get_error(na) == 0 and rssm.rssm_get_error(ref) == 0
    for b in (0, shape.batch - 1):
        r = request_inputs(inp, b)
        ys, snaps = orc.run_conv(r["ckpt"], r["x"], r["B"], r["C"], r["dt"], r["A"], r["D"],
                                 snap_steps=sorted(ck))
        assert_close(to_np(y_na[:, b]), ys, f"noalloc fused decode, request {b}")
        for t, h in ck.items():
            assert_close(h[b], snaps[t], f"noalloc fused checkpoint after token {t}, request {b}")


def test_noalloc_rejects_batch_above_its_maximum():
    d = rssm.make_desc(65537, 2, 8, 128, 1)
    st = rssm.StateStruct(*([0x1000] * 7))
    p = ct.c_void_p(0x1000)
    status = rssm.lib().rssm_decode_step_noalloc(ct.byref(d), ct.byref(st), p, p, p, p, p, p, p, None)
    assert status == 4  # RSSM_ERR_CAPACITY, nothing launched
