"""Helpers shared by the GPU tests: drive librssm through whole runs and
compute the oracle's answer for sampled requests (in a spawn process pool,
started before any work is forked)."""
import math
import multiprocessing as mp
import os

import numpy as np
import torch

from hybrid_model_ssm_replay_b200 import rssm
from hybrid_model_ssm_replay_b200.inputs import LayerShape, accept_lengths, make_inputs

TOL = 1e-4  # max |dy| <= TOL * rms(y_ref) per compared tensor (fp32 state vs fp64 oracle)


def rel_err(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = math.sqrt(float(np.mean(ref * ref))) or 1.0
    return float(np.max(np.abs(got - ref))) / rms


def assert_close(got, ref, what, tol=TOL):
    e = rel_err(got, ref)
    assert e <= tol, f"{what}: max|d|/rms = {e:.3e} > {tol:.0e}"
    return e


def to_np(t):
    return t.detach().double().cpu().numpy()


def desc_for(shape: LayerShape, in_dtype=torch.bfloat16, **kw):
    return rssm.make_desc(shape.batch, shape.nheads, shape.head_dim, shape.d_state, shape.ngroups,
                          interval=shape.interval, max_draft=shape.max_draft,
                          in_dtype=rssm.RSSM_BF16 if in_dtype == torch.bfloat16 else rssm.RSSM_F32, **kw)


def sample_requests(batch, k=8):
    if batch <= k:
        return list(range(batch))
    rng = np.random.default_rng(batch)
    mid = sorted(rng.choice(np.arange(1, batch - 1), k - 2, replace=False).tolist())
    return [0] + mid + [batch - 1]


# ------------------------------------------------------------------ GPU runs

def gpu_replay_decode(desc, inp, steps, fused=False, snap=None):
    """Standard decode of `steps` tokens; flush after every interval (or fused).
    Returns (y [steps][B][H][P] on GPU, {step: ckpt[snap] after the flush}, state)."""
    st = rssm.RssmState(desc)
    st.ckpt.copy_(inp["ckpt"])
    L = desc.interval
    y = torch.empty((steps,) + tuple(inp["x"].shape[1:]), dtype=torch.float32, device="cuda")
    snaps = {}
    for t in range(steps):
        rssm.rssm_decode_step(st, inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"], y[t])
        if (t + 1) % L == 0:
            if not fused:
                rssm.rssm_flush(st, inp["A"])
            if snap is not None:
                snaps[t] = st.ckpt[snap].double().cpu().numpy()
    return y, snaps, st


def gpu_conv_decode(desc, inp, steps, snap=None, snap_steps=()):
    h = inp["ckpt"].clone()
    y = torch.empty((steps,) + tuple(inp["x"].shape[1:]), dtype=torch.float32, device="cuda")
    snaps = {}
    for t in range(steps):
        rssm.rssm_conv_step(desc, h, inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"], y[t])
        if t in snap_steps and snap is not None:
            snaps[t] = h[snap].double().cpu().numpy()
    return y, snaps, h


def gpu_spec(desc, inp, n_acc, steps):
    st = rssm.RssmState(desc)
    st.ckpt.copy_(inp["ckpt"])
    K = desc.max_draft
    y = torch.empty((steps,) + tuple(inp["x"].shape[1:]), dtype=torch.float32, device="cuda")
    for s in range(steps):
        rssm.rssm_verify(st, K, inp["x"][s], inp["B"][s], inp["C"][s], inp["dt"][s], inp["A"], inp["D"], y[s])
        rssm.rssm_accept(st, n_acc[s])
        rssm.rssm_flush(st, inp["A"])
    return y, st


def gpu_conv_spec(desc, inp, n_acc, steps):
    K = desc.max_draft
    copies = torch.zeros((K + 1,) + tuple(inp["ckpt"].shape), dtype=torch.float32, device="cuda")
    copies[0].copy_(inp["ckpt"])
    cur = torch.zeros(desc.batch, dtype=torch.int32, device="cuda")
    y = torch.empty((steps,) + tuple(inp["x"].shape[1:]), dtype=torch.float32, device="cuda")
    for s in range(steps):
        rssm.rssm_conv_verify(desc, copies, cur, K, inp["x"][s], inp["B"][s], inp["C"][s], inp["dt"][s],
                              inp["A"], inp["D"], y[s])
        rssm.rssm_conv_accept(desc, n_acc[s], cur, K)
    return y, copies, cur


# ------------------------------------------------------------ oracle side

def request_inputs(inp, b):
    """fp64 numpy inputs of request b (exact copies of the bf16/fp32 values)."""
    return dict(ckpt=to_np(inp["ckpt"][b]), x=to_np(inp["x"][:, b]), B=to_np(inp["B"][:, b]),
                C=to_np(inp["C"][:, b]), dt=to_np(inp["dt"][:, b]), A=to_np(inp["A"]), D=to_np(inp["D"]))


def _oracle_job(job):
    kind, r, extra = job
    from oracle import oracle as orc
    if kind == "conv":
        return orc.run_conv(r["ckpt"], r["x"], r["B"], r["C"], r["dt"], r["A"], r["D"], snap_steps=extra)
    if kind == "spec":
        n_acc, L, K = extra
        return orc.run_spec(r["ckpt"], r["x"], r["B"], r["C"], r["dt"], r["A"], r["D"], n_acc, L, K)
    raise ValueError(kind)


_POOL = None


def oracle_pool():
    global _POOL
    if _POOL is None:
        _POOL = mp.get_context("spawn").Pool(max(1, min(8, os.cpu_count() or 1)))
    return _POOL


def oracle_map(jobs):
    if len(jobs) == 1:
        return [_oracle_job(jobs[0])]
    return oracle_pool().map(_oracle_job, jobs)
