"""Pins for the oracle's precision split (ReplaySSM article s4): refresh of
the update copy, the FP4 output copy, and decode reading that copy.

The references are the conventional recurrence started from the same
values (an independent form), the neighbour property of stochastic
rounding, and the hand-checked FP4 block rule."""
import math

import numpy as np

from oracle import oracle as orc


def rand_state(rng, H, P, N, G, T):
    return dict(
        ckpt=rng.normal(0, 0.1, (H, P, N)).astype(np.float32),
        x=rng.normal(size=(T, H, P)), B=rng.normal(size=(T, G, N)), C=rng.normal(size=(T, G, N)),
        dt=np.log1p(np.exp(rng.normal(-3, 1, (T, H)))),
        A=-np.exp(rng.uniform(0, math.log(16), H)), D=rng.normal(size=H))


def ulp32(v):
    v = np.abs(np.asarray(v, np.float32))
    return np.nextafter(v, np.float32(np.inf)) - v


def test_refresh_at_empty_buffer_copies_and_quantises():
    rng = np.random.default_rng(0)
    s = rand_state(rng, 2, 4, 32, 1, 1)
    codes = np.zeros((2, 4, 16), np.uint8)
    scales = np.zeros((2, 4, 2), np.uint8)
    req = orc.LowPrecRequest(orc.F32, True, s["ckpt"], codes, scales, 1, 16, s["A"], s["D"], 5, 0)
    v32 = req.refresh(want_v32=True)
    assert np.array_equal(v32, s["ckpt"]) and np.array_equal(req.upd, s["ckpt"])
    c_ref, s_ref = orc.fp4_quant(s["ckpt"])
    assert np.array_equal(req.codes, c_ref) and np.array_equal(req.scales, s_ref)
    assert req.pos == 0 and req.flush_count.value == 1


def test_refresh_f32_equals_recurrence_state():
    rng = np.random.default_rng(1)
    H, P, N, G, L = 4, 3, 16, 2, 16
    s = rand_state(rng, H, P, N, G, L)
    req = orc.LowPrecRequest(orc.F32, False, s["ckpt"], None, None, G, L, s["A"], s["D"], 1, 0)
    for t in range(L):
        req.decode(s["x"][t], s["B"][t], s["C"][t], s["dt"][t])
    req.refresh()
    _, snaps = orc.run_conv(s["ckpt"].astype(np.float64), s["x"], s["B"], s["C"], s["dt"], s["A"], s["D"],
                            snap_steps=[L - 1])
    ref = snaps[L - 1].astype(np.float32)
    assert np.all(np.abs(req.upd - ref) <= ulp32(ref))


def test_refresh_bf16_rounds_to_a_neighbour_of_the_recurrence_state():
    rng = np.random.default_rng(2)
    H, P, N, G, L = 4, 4, 32, 2, 16
    s = rand_state(rng, H, P, N, G, L)
    upd0 = (s["ckpt"].view(np.uint32) >> 16).astype(np.uint16)        # truncated start copy
    start = (upd0.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    reqs = [orc.LowPrecRequest(orc.BF16, True, upd0, np.zeros((H, P, N // 2), np.uint8),
                               np.zeros((H, P, N // 16), np.uint8), G, L, s["A"], s["D"], 77, r)
            for r in (0, 1)]
    for req in reqs:
        for t in range(L):
            req.decode(s["x"][t], s["B"][t], s["C"][t], s["dt"][t])
        v32 = req.refresh(want_v32=True)
        assert req.flush_count.value == 1 and req.pos == 0
        c_ref, s_ref = orc.fp4_quant(v32)
        assert np.array_equal(req.codes, c_ref) and np.array_equal(req.scales, s_ref)
    _, snaps = orc.run_conv(start, s["x"], s["B"], s["C"], s["dt"], s["A"], s["D"], snap_steps=[L - 1])
    ref = snaps[L - 1]
    got = (reqs[0].upd.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    # bf16 neighbours of the exact state (a few fp32 ulps of slack for its rounding)
    spacing = np.abs(ref) * 2.0 ** -7
    assert np.all(np.abs(got - ref) <= spacing * (1 + 1e-5))
    # different request id -> different random words -> different roundings somewhere
    assert not np.array_equal(reqs[0].upd, reqs[1].upd)


def test_decode_reads_fp4_copy_as_recurrence_from_dequantised_state():
    rng = np.random.default_rng(3)
    H, P, N, G, L = 2, 4, 32, 1, 16
    s = rand_state(rng, H, P, N, G, 6)
    codes, scales = orc.fp4_quant(s["ckpt"])
    req = orc.LowPrecRequest(orc.FP4, False, None, codes, scales, G, L, s["A"], s["D"], 3, 0)
    deq = orc.widen(orc.FP4, codes, scales, (H, P, N))
    ys = np.stack([req.decode(s["x"][t], s["B"][t], s["C"][t], s["dt"][t]) for t in range(6)])
    y_ref, _ = orc.run_conv(deq, s["x"], s["B"], s["C"], s["dt"], s["A"], s["D"])
    assert np.max(np.abs(ys - y_ref)) < 1e-12 * np.sqrt(np.mean(y_ref ** 2))
    # the shared-copy control re-quantises the folded state with nearest rounding
    req.refresh()
    _, snaps = orc.run_conv(deq, s["x"], s["B"], s["C"], s["dt"], s["A"], s["D"], snap_steps=[5])
    c2, s2 = orc.fp4_quant(snaps[5].astype(np.float32))
    assert np.mean(req.codes == c2) > 0.99 and np.mean(req.scales == s2) > 0.99
