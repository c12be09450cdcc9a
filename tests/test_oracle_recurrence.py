"""Pins for the oracle's recurrence, replay, flush and verify/accept.

Each check comes from mathematics that does not reuse the oracle's code:
closed forms of special cases, one-hot probes of operand orientation,
linearity, and identities between the two independently written forms
(ReplaySSM article s1: replay outputs equal the conventional ones up to
rounding; s3: verify-then-accept equals decoding the accepted tokens).
"""
import math

import numpy as np
import pytest

from oracle import oracle as orc


def rel_err(a, b):
    b = np.asarray(b)
    scale = math.sqrt(float(np.mean(b * b))) or 1.0
    return float(np.max(np.abs(np.asarray(a) - b))) / scale


def rand_problem(rng, T, H, P, N, G, ntok=0):
    tok = (ntok,) if ntok else ()
    return dict(
        ckpt=rng.normal(0, 0.1, (H, P, N)),
        x=rng.normal(size=(T,) + tok + (H, P)),
        B=rng.normal(size=(T,) + tok + (G, N)),
        C=rng.normal(size=(T,) + tok + (G, N)),
        dt=np.log1p(np.exp(rng.normal(-3, 1, (T,) + tok + (H,)))),
        A=-np.exp(rng.uniform(0, math.log(16), H)),
        D=rng.normal(size=H),
    )


# ---------------------------------------------------------------- closed forms

def test_geometric_series_closed_form():
    """P = N = H = G = 1 with constant inputs: h_t is a geometric series."""
    T, h0, dt, A, x, Bv, Cv, D = 40, 0.3, 0.07, -2.5, 1.3, -0.8, 0.6, 0.9
    a = math.exp(dt * A)
    x_ = np.full((T, 1, 1), x)
    B_ = np.full((T, 1, 1), Bv)
    C_ = np.full((T, 1, 1), Cv)
    dt_ = np.full((T, 1), dt)
    A_, D_ = np.array([A]), np.array([D])
    t = np.arange(T)
    h_exact = a ** (t + 1) * h0 + dt * x * Bv * (1 - a ** (t + 1)) / (1 - a)
    y_exact = (h_exact * Cv + D * x).reshape(T, 1, 1)
    y_conv, snaps = orc.run_conv(np.full((1, 1, 1), h0), x_, B_, C_, dt_, A_, D_, snap_steps=[15, 31])
    assert rel_err(y_conv, y_exact) < 1e-13
    assert abs(snaps[15][0, 0, 0] - h_exact[15]) < 1e-14
    y_rep, ck = orc.run_replay_decode(np.full((1, 1, 1), h0), x_, B_, C_, dt_, A_, D_, L=16)
    assert rel_err(y_rep, y_exact) < 1e-13
    assert abs(ck[31][0, 0, 0] - h_exact[31]) < 1e-14


@pytest.mark.parametrize("form", ["conv", "replay"])
def test_dt_zero_keeps_state(form):
    """dt = 0 gives a = 1 and no input: h stays h0 and y = h0 . C + D x."""
    rng = np.random.default_rng(1)
    pr = rand_problem(rng, 20, 4, 3, 5, 2)
    pr["dt"][:] = 0.0
    if form == "conv":
        y, _ = orc.run_conv(pr["ckpt"], pr["x"], pr["B"], pr["C"], pr["dt"], pr["A"], pr["D"])
    else:
        y, _ = orc.run_replay_decode(pr["ckpt"], pr["x"], pr["B"], pr["C"], pr["dt"], pr["A"], pr["D"], L=8)
    g = np.arange(4) // 2
    expect = np.einsum("hpn,thn->thp", pr["ckpt"], pr["C"][:, g, :]) + pr["D"][None, :, None] * pr["x"]
    assert rel_err(y, expect) < 1e-13


@pytest.mark.parametrize("form", ["conv", "replay"])
def test_full_forgetting(form):
    """A = -inf gives a = 0: h_t = dt_t x_t (outer) B_t, whatever came before."""
    rng = np.random.default_rng(2)
    pr = rand_problem(rng, 20, 4, 3, 5, 2)
    pr["A"][:] = -np.inf
    if form == "conv":
        y, _ = orc.run_conv(pr["ckpt"], pr["x"], pr["B"], pr["C"], pr["dt"], pr["A"], pr["D"])
    else:
        y, _ = orc.run_replay_decode(pr["ckpt"], pr["x"], pr["B"], pr["C"], pr["dt"], pr["A"], pr["D"], L=8)
    g = np.arange(4) // 2
    bc = np.einsum("thn,thn->th", pr["B"][:, g, :], pr["C"][:, g, :])
    expect = pr["dt"][..., None] * pr["x"] * bc[..., None] + pr["D"][None, :, None] * pr["x"]
    assert rel_err(y, expect) < 1e-13


@pytest.mark.parametrize("form", ["conv", "replay"])
def test_operand_orientation_one_hot(form):
    """From h0 = 0, one token with x = e_i (head_dim) and B = e_j (d_state)
    puts dt at h[i, j] only, so y[i] = dt C[j] + D and y[p != i] = 0; heads
    read the B and C of their own group (groups of H/G consecutive heads)."""
    H, P, N, G = 4, 3, 5, 2
    dt = np.array([[0.25, 0.5, 0.75, 1.0]])
    x = np.zeros((1, H, P))
    Bm = np.zeros((1, G, N))
    C = np.arange(1.0, 1.0 + G * N).reshape(1, G, N)
    i_of = [0, 2, 1, 2]
    j_of = [4, 1]
    for h in range(H):
        x[0, h, i_of[h]] = 1.0
    for g in range(G):
        Bm[0, g, j_of[g]] = 1.0
    A = np.full(H, -1.0)
    D = np.array([0.5, -0.5, 2.0, 3.0])
    h0 = np.zeros((H, P, N))
    if form == "conv":
        y, snaps = orc.run_conv(h0, x, Bm, C, dt, A, D, snap_steps=[0])
        state = snaps[0]
    else:
        req = orc.ReplayRequest(h0, G, 16, A, D)
        y = req.decode(x[0], Bm[0], C[0], dt[0])[None]
        req.flush()
        state = req.ckpt
    for h in range(H):
        g = h // (H // G)
        for p in range(P):
            want = dt[0, h] * C[0, g, j_of[g]] + D[h] if p == i_of[h] else 0.0
            assert y[0, h, p] == pytest.approx(want, rel=1e-14, abs=1e-14)
        expect_state = np.zeros((P, N))
        expect_state[i_of[h], j_of[g]] = dt[0, h]
        assert np.array_equal(state[h], expect_state)


def test_linearity():
    """For fixed dt, B, C the map (h0, x) -> y is linear."""
    rng = np.random.default_rng(3)
    p1 = rand_problem(rng, 24, 4, 6, 8, 2)
    p2 = rand_problem(rng, 24, 4, 6, 8, 2)
    args = lambda h0, x: (h0, x, p1["B"], p1["C"], p1["dt"], p1["A"], p1["D"])
    y1, _ = orc.run_replay_decode(*args(p1["ckpt"], p1["x"]), L=16)
    y2, _ = orc.run_replay_decode(*args(p2["ckpt"], p2["x"]), L=16)
    y12, _ = orc.run_replay_decode(*args(p1["ckpt"] + p2["ckpt"], p1["x"] + p2["x"]), L=16)
    # D x is linear too, so the sum carries over exactly up to rounding
    assert rel_err(y12, y1 + y2) < 1e-12
    y1c, _ = orc.run_conv(*args(p1["ckpt"], p1["x"]))
    y2c, _ = orc.run_conv(*args(p2["ckpt"], p2["x"]))
    y12c, _ = orc.run_conv(*args(p1["ckpt"] + p2["ckpt"], p1["x"] + p2["x"]))
    assert rel_err(y12c, y1c + y2c) < 1e-12


# ---------------------------------------------------------- form identities

@pytest.mark.parametrize("L", [1, 2, 5, 16])
@pytest.mark.parametrize("seed", [0, 1])
def test_replay_equals_recurrence(L, seed):
    """Replay outputs and every flushed checkpoint equal the recurrence."""
    rng = np.random.default_rng(10 + seed)
    H, P, N, G = (4, 5, 7, 2) if seed == 0 else (6, 3, 4, 3)
    T = 3 * L + 3
    pr = rand_problem(rng, T, H, P, N, G)
    y_rep, ck = orc.run_replay_decode(pr["ckpt"], pr["x"], pr["B"], pr["C"], pr["dt"], pr["A"], pr["D"], L=L)
    y_conv, snaps = orc.run_conv(pr["ckpt"], pr["x"], pr["B"], pr["C"], pr["dt"], pr["A"], pr["D"],
                                 snap_steps=list(ck.keys()))
    assert sorted(ck.keys()) == [L * k - 1 for k in range(1, T // L + 1)]
    assert rel_err(y_rep, y_conv) < 1e-12
    for s, c in ck.items():
        assert rel_err(c, snaps[s]) < 1e-12


def test_interval_one_matches_conventional_tightly():
    """With interval 1 the replay scheme flushes after every token."""
    rng = np.random.default_rng(4)
    pr = rand_problem(rng, 30, 2, 4, 4, 1)
    y_rep, ck = orc.run_replay_decode(pr["ckpt"], pr["x"], pr["B"], pr["C"], pr["dt"], pr["A"], pr["D"], L=1)
    y_conv, snaps = orc.run_conv(pr["ckpt"], pr["x"], pr["B"], pr["C"], pr["dt"], pr["A"], pr["D"],
                                 snap_steps=list(range(30)))
    assert rel_err(y_rep, y_conv) < 1e-13
    assert all(rel_err(ck[t], snaps[t]) < 1e-13 for t in range(30))


def test_tiny_workload_replay_equals_recurrence():
    """The tiny workload (batch 4, 2 heads, 16 x 16, 1 group, interval 16,
    64 steps, seed 0) through both forms."""
    import torch
    from hybrid_model_ssm_replay_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["tiny"]
    inp = make_inputs(w["shape"], w["steps"], w["seed"], w["in_dtype"])
    f = {k: v.double().numpy() for k, v in inp.items()}
    for b in range(w["shape"].batch):
        args = (f["ckpt"][b], f["x"][:, b], f["B"][:, b], f["C"][:, b], f["dt"][:, b], f["A"], f["D"])
        y_rep, ck = orc.run_replay_decode(*args, L=16)
        y_conv, snaps = orc.run_conv(*args, snap_steps=list(ck.keys()))
        assert len(ck) == 4
        assert rel_err(y_rep, y_conv) < 1e-12
        for s in ck:
            assert rel_err(ck[s], snaps[s]) < 1e-12
    assert torch.is_tensor(inp["x"])


@pytest.mark.parametrize("K", [1, 4, 6, 7])
def test_verify_then_accept_equals_decoding_accepted(K):
    """For every n in 0..K: verify of K+1 tokens then accept(n) gives, for
    tokens 0..n, the outputs of plain decode, and leaves the same state."""
    rng = np.random.default_rng(5 + K)
    H, P, N, G, L = 4, 3, 6, 2, 8
    pre = rand_problem(rng, 5, H, P, N, G)
    spec = rand_problem(rng, 1, H, P, N, G, ntok=K + 1)
    after = rand_problem(rng, L, H, P, N, G)
    for n in range(K + 1):
        ra = orc.ReplayRequest(pre["ckpt"], G, L + K, pre["A"], pre["D"])
        rb = orc.ReplayRequest(pre["ckpt"], G, L + K, pre["A"], pre["D"])
        for t in range(5):
            ra.decode(pre["x"][t], pre["B"][t], pre["C"][t], pre["dt"][t])
            rb.decode(pre["x"][t], pre["B"][t], pre["C"][t], pre["dt"][t])
        ys = ra.verify(spec["x"][0], spec["B"][0], spec["C"][0], spec["dt"][0])
        assert ra.pos == 5
        ra.accept(n)
        for j in range(n + 1):
            yb = rb.decode(spec["x"][0, j], spec["B"][0, j], spec["C"][0, j], spec["dt"][0, j])
            assert rel_err(ys[j], yb) < 1e-13
        assert ra.pos == rb.pos == 5 + n + 1
        # later tokens see the same history: rejected drafts left no trace
        for t in range(2):
            ya = ra.decode(after["x"][t], after["B"][t], after["C"][t], after["dt"][t])
            yb = rb.decode(after["x"][t], after["B"][t], after["C"][t], after["dt"][t])
            assert rel_err(ya, yb) < 1e-13
        ra.flush()
        rb.flush()
        assert rel_err(ra.ckpt, rb.ckpt) < 1e-13


def test_verify_rejects_overflow():
    rng = np.random.default_rng(6)
    pr = rand_problem(rng, 1, 2, 2, 4, 1, ntok=5)
    req = orc.ReplayRequest(pr["ckpt"], 1, 20, pr["A"], pr["D"])
    req.pos = 16
    with pytest.raises(ValueError):
        req.verify(pr["x"][0], pr["B"][0], pr["C"][0], pr["dt"][0])
    req.pos = 15
    req.verify(pr["x"][0], pr["B"][0], pr["C"][0], pr["dt"][0])


@pytest.mark.parametrize("L,K", [(16, 4), (16, 1), (16, 6), (27, 5)])
def test_spec_run_equals_recurrence_on_accepted_stream(L, K):
    """A whole speculative run (verify K+1, accept n, flush at L) gives, for
    the accepted tokens, the outputs of the recurrence over those tokens --
    including the largest buffer (27 + 5 = 32 slots)."""
    rng = np.random.default_rng(7 + K + L)
    H, P, N, G, S = 4, 3, 5, 2, 30
    pr = rand_problem(rng, S, H, P, N, G, ntok=K + 1)
    n_acc = rng.integers(0, K + 1, S)
    ys, ck, poss = orc.run_spec(pr["ckpt"], pr["x"], pr["B"], pr["C"], pr["dt"], pr["A"], pr["D"],
                                n_acc, L, K)
    assert len(ck) >= 1 and max(poss) < L
    sel = [(s, j) for s in range(S) for j in range(n_acc[s] + 1)]
    xs = np.stack([pr["x"][s, j] for s, j in sel])
    Bs = np.stack([pr["B"][s, j] for s, j in sel])
    Cs = np.stack([pr["C"][s, j] for s, j in sel])
    dts = np.stack([pr["dt"][s, j] for s, j in sel])
    y_conv, _ = orc.run_conv(pr["ckpt"], xs, Bs, Cs, dts, pr["A"], pr["D"])
    y_spec = np.stack([ys[s, j] for s, j in sel])
    assert rel_err(y_spec, y_conv) < 1e-12
