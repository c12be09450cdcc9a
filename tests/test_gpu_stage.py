"""The synthetic hybrid decode stage (hybrid_model_ssm_replay_b200.stage):
its element-wise kernels against fp64 references, and whole stage steps --
replay and conventional SSM step -- against an fp64 chain that rounds to
bf16 where the stage does (GEMM outputs, norms, conv outputs, residual
stream) and takes the SSM step from the oracle.

Tolerances come from the bf16 boundaries: a bf16 result is within half a
spacing (2^-8 relative) of its fp32 value, so a kernel's bf16 output is
compared with the fp64 value at 2^-8 relative plus the fp32 error; across
whole steps the GPU and the fp64 chain can round an element to neighbouring
bf16 values, so the residual stream is compared in aggregate (rms of the
difference <= 1% of rms, max <= 5%)."""
import math

import numpy as np
import pytest
import torch

from hybrid_model_ssm_replay_b200 import rssm
from hybrid_model_ssm_replay_b200.stage import (HybridStage, StageShape, make_weights, rssm_stage_conv,
                                                rssm_stage_gate_norm)
from oracle import oracle as orc

from gpu_helpers import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from hybrid_model_ssm_replay_b200 import build
    build.build()


def bf16(a):
    """fp64 values rounded to bf16 (nearest even), back as fp64."""
    return torch.from_numpy(np.asarray(a, np.float64)).to(torch.bfloat16).double().numpy()


def f64(t):
    return t.detach().double().cpu().numpy()


def silu(v):
    return v / (1.0 + np.exp(-v))


def check_bf16(got, ref, what):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    bad = np.abs(got - ref) > (2.0 ** -8 + 1e-6) * np.abs(ref) + 1e-30
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} beyond half a bf16 spacing"


TINY = StageShape(batch=3, d_model=64, nheads=4, head_dim=32, d_state=64, ngroups=2, interval=16, n_ssm=2,
                  n_attn=1, attn_heads=2, kv_heads=1, attn_head_dim=32, ctx=8)


def test_stage_conv_matches_reference():
    s = TINY
    g = torch.Generator().manual_seed(3)
    desc = rssm.make_desc(s.batch, s.nheads, s.head_dim, s.d_state, s.ngroups)
    chans = s.d_inner + 2 * s.ngroups * s.d_state
    w = torch.randn(chans, 4, generator=g).float().cuda()
    b = torch.randn(chans, generator=g).float().cuda()
    dtb = torch.randn(s.nheads, generator=g).float().cuda()
    state = torch.randn(s.batch, 3, chans, generator=g).to(torch.bfloat16).cuda()
    ref_state = f64(state)
    x = torch.empty(s.batch, s.nheads, s.head_dim, dtype=torch.bfloat16, device="cuda")
    B = torch.empty(s.batch, s.ngroups, s.d_state, dtype=torch.bfloat16, device="cuda")
    C = torch.empty_like(B)
    dt = torch.empty(s.batch, s.nheads, device="cuda")
    wn, bn, dtbn = f64(w), f64(b), f64(dtb)
    for step in range(5):
        zx = (torch.randn(s.batch, s.d_proj, generator=g) * 3).to(torch.bfloat16).cuda()
        rssm_stage_conv(desc, zx, state, w, b, dtb, x, B, C, dt)
        torch.cuda.synchronize()
        z = f64(zx)
        inp = z[:, s.d_inner:s.d_inner + chans]
        o = bn + wn[:, 0] * ref_state[:, 0] + wn[:, 1] * ref_state[:, 1] + wn[:, 2] * ref_state[:, 2] + wn[:, 3] * inp
        ref_state = np.stack([ref_state[:, 1], ref_state[:, 2], inp], axis=1)
        a = silu(o)
        din, gn = s.d_inner, s.ngroups * s.d_state
        check_bf16(f64(x).reshape(s.batch, -1), a[:, :din], f"conv x, step {step}")
        check_bf16(f64(B).reshape(s.batch, -1), a[:, din:din + gn], f"conv B, step {step}")
        check_bf16(f64(C).reshape(s.batch, -1), a[:, din + gn:], f"conv C, step {step}")
        v = z[:, -s.nheads:] + dtbn
        sp = np.where(v > 20, v, np.log1p(np.exp(v)))
        assert np.max(np.abs(f64(dt) - sp) / sp) < 1e-5
        assert np.array_equal(f64(state), ref_state), "conv state shift"


def test_stage_gate_norm_matches_reference():
    s = TINY
    g = torch.Generator().manual_seed(4)
    desc = rssm.make_desc(s.batch, s.nheads, s.head_dim, s.d_state, s.ngroups)
    y = torch.randn(s.batch, s.d_inner, generator=g).float().cuda()
    zx = (torch.randn(s.batch, s.d_proj, generator=g) * 2).to(torch.bfloat16).cuda()
    nw = (1 + 0.1 * torch.randn(s.d_inner, generator=g)).float().cuda()
    out = torch.empty(s.batch, s.d_inner, dtype=torch.bfloat16, device="cuda")
    rssm_stage_gate_norm(desc, y, zx, nw, 1e-5, out)
    torch.cuda.synchronize()
    gg = f64(y) * silu(f64(zx)[:, :s.d_inner])
    gs = s.d_inner // s.ngroups
    gg = gg.reshape(s.batch, s.ngroups, gs)
    ref = (gg / np.sqrt(np.mean(gg * gg, axis=-1, keepdims=True) + 1e-5)).reshape(s.batch, -1) * f64(nw)
    check_bf16(f64(out), ref, "gated norm")


def test_stage_rejects_bad_arguments():
    s = TINY
    d = rssm.make_desc(s.batch, s.nheads, s.head_dim, s.d_state, s.ngroups, in_dtype=rssm.RSSM_F32)
    t = torch.zeros(16, device="cuda")
    with pytest.raises(rssm.RssmError):
        rssm_stage_gate_norm(d, t, t.to(torch.bfloat16), t, 1e-5, t.to(torch.bfloat16))


def reference_chain(shape, weights, stage, u0, steps):
    """The stage in fp64 with bf16 rounding at the stage's boundaries and the
    oracle's recurrence for the SSM step. Initial SSM and conv states and KV
    caches are read from `stage` before it runs."""
    s = shape
    blocks, attn = weights
    W = [{k: f64(v) for k, v in b.items()} for b in blocks]
    Wa = [{k: f64(v) for k, v in a.items()} for a in attn]
    h = [f64(st["state"].ckpt if stage.scheme == "replay" else st["state"]).copy() for st in stage.ssm]
    conv = [f64(st["conv"]).copy() for st in stage.ssm]
    kv = [{"k": f64(c["k"]).copy(), "v": f64(c["v"]).copy()} for c in stage.kv]
    din, gn, chans = s.d_inner, s.ngroups * s.d_state, s.d_inner + 2 * s.ngroups * s.d_state

    def rms(u, w):
        return bf16(u / np.sqrt(np.mean(u * u, axis=-1, keepdims=True) + s.eps) * w)

    u = f64(u0)
    outs = []
    for t in range(steps):
        for i, b in enumerate(W):
            zx = bf16(rms(u, b["norm"]) @ b["w_in"])
            inp = zx[:, din:din + chans]
            c = conv[i]
            o = b["conv_b"] + sum(b["conv_w"][:, k] * c[:, k] for k in range(3)) + b["conv_w"][:, 3] * inp
            conv[i] = np.stack([c[:, 1], c[:, 2], inp], axis=1)
            a = bf16(silu(o))
            x = a[:, :din].reshape(s.batch, s.nheads, s.head_dim)
            Bv = a[:, din:din + gn].reshape(s.batch, s.ngroups, s.d_state)
            Cv = a[:, din + gn:].reshape(s.batch, s.ngroups, s.d_state)
            v = zx[:, -s.nheads:] + b["dt_bias"]
            dt = np.where(v > 20, v, np.log1p(np.exp(v)))
            y = np.zeros((s.batch, din))
            for r in range(s.batch):
                hh = np.ascontiguousarray(h[i][r])
                cc = np.ascontiguousarray
                y[r] = orc.conv_steps(hh, cc(x[r][None]), cc(Bv[r][None]), cc(Cv[r][None]), cc(dt[r][None]),
                                      cc(b["A"]), cc(b["D"])).ravel()
                h[i][r] = hh
            gg = (y * silu(zx[:, :din])).reshape(s.batch, s.ngroups, din // s.ngroups)
            vn = bf16((gg / np.sqrt(np.mean(gg * gg, axis=-1, keepdims=True) + s.eps)).reshape(s.batch, -1)
                      * b["gnorm"])
            u = bf16(u + bf16(vn @ b["w_out"]))
        for i, a in enumerate(Wa):
            hq, hk, hd = s.attn_heads, s.kv_heads, s.attn_head_dim
            qkv = bf16(rms(u, a["norm"]) @ a["w_qkv"])
            q = qkv[:, :hq * hd].reshape(s.batch, hq, hd)
            kv[i]["k"][:, :, t % s.ctx] = qkv[:, hq * hd:(hq + hk) * hd].reshape(s.batch, hk, hd)
            kv[i]["v"][:, :, t % s.ctx] = qkv[:, (hq + hk) * hd:].reshape(s.batch, hk, hd)
            rep = hq // hk
            K = np.repeat(kv[i]["k"], rep, axis=1)
            V = np.repeat(kv[i]["v"], rep, axis=1)
            sc = np.einsum("bhd,bhcd->bhc", q, K) / math.sqrt(hd)
            p = np.exp(sc - sc.max(-1, keepdims=True))
            p /= p.sum(-1, keepdims=True)
            o = bf16(np.einsum("bhc,bhcd->bhd", p, V)).reshape(s.batch, hq * hd)
            u = bf16(u + bf16(o @ a["w_o"]))
        outs.append(u.copy())
    return outs


@pytest.mark.parametrize("scheme", ["replay", "conventional"])
def test_stage_steps_match_fp64_chain(scheme):
    """20 decode tokens (one interval flush inside) of a 2-Mamba + 1-attention
    stage, against the fp64 chain with the oracle's SSM step."""
    s = TINY
    weights = make_weights(s, 11)
    stage = HybridStage(s, weights, scheme=scheme, seed=5)
    g = torch.Generator().manual_seed(9)
    u0 = torch.randn(s.batch, s.d_model, generator=g).to(torch.bfloat16).cuda()
    steps = 20
    refs = reference_chain(s, weights, stage, u0, steps)
    u = u0
    for t in range(steps):
        u = stage.step(u)
        got, ref = f64(u), refs[t]
        scale = math.sqrt(float(np.mean(ref * ref)))
        d = got - ref
        assert math.sqrt(float(np.mean(d * d))) <= 0.01 * scale, f"{scheme} step {t}: rms diff"
        assert float(np.max(np.abs(d))) <= 0.05 * scale, f"{scheme} step {t}: max diff"
    if scheme == "replay":
        for st in stage.ssm:
            assert rssm.rssm_get_error(st["state"]) == 0


def test_stage_ssm_step_matches_oracle_on_stage_inputs():
    """Inside a stage, the SSM step's outputs (replay, with the flush after 16
    tokens) equal the oracle's recurrence on the x, B, C, dt the stage's conv
    kernel produced, within the SSM tolerance (1e-4 rms)."""
    s = TINY
    weights = make_weights(s, 12)
    stage = HybridStage(s, weights, scheme="replay", seed=6)
    h0 = f64(stage.ssm[0]["state"].ckpt).copy()
    g = torch.Generator().manual_seed(10)
    u = torch.randn(s.batch, s.d_model, generator=g).to(torch.bfloat16).cuda()
    xs, Bs, Cs, dts, ys = [], [], [], [], []
    b0 = stage.blocks[0]
    for t in range(20):
        # block 0 by hand, recording the SSM inputs and outputs
        u1 = stage.ssm_block(0, u)
        xs.append(f64(stage.x)), Bs.append(f64(stage.Bv)), Cs.append(f64(stage.Cv))
        dts.append(f64(stage.dt)), ys.append(f64(stage.y))
        for i in range(1, s.n_ssm):
            u1 = stage.ssm_block(i, u1)
        for i in range(s.n_attn):
            u1 = stage.attn_block(i, u1)
        stage.t += 1
        u = u1
    X, Bv, Cv, DT, Y = (np.stack(a) for a in (xs, Bs, Cs, dts, ys))
    for r in range(s.batch):
        yr, _ = orc.run_conv(h0[r], X[:, r], Bv[:, r], Cv[:, r], DT[:, r], f64(b0["A"]), f64(b0["D"]))
        assert_close(Y[:, r], yr, f"stage SSM step, request {r}")
