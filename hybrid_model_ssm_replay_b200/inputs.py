"""Seeded synthetic inputs for the SSM decode layer.

This module holds only the input recipe (random draws and their
distributions); it contains none of the method's arithmetic. Tests, the
benchmark and the smoke check feed the same tensors to the GPU library and
to the CPU oracle.

Recipe (one torch.Generator seeded with `seed`, drawn in this order):
    ckpt ~ N(0, 0.1^2)            [batch][H][P][N] fp32
    A_h  = -exp(U(0, ln 16))      [H] fp32, in [-16, -1]
    D_h  ~ N(0, 1)                [H] fp32
    x    ~ N(0, 1)                [steps][batch][(ntok)][H][P], rounded once to in_dtype
    B    ~ N(0, 1)                [steps][batch][(ntok)][G][N], rounded once to in_dtype
    C    ~ N(0, 1)                same shape as B
    dt   = softplus(N(-3, 1))     [steps][batch][(ntok)][H] fp32, > 0
Accepted draft counts for speculative decoding come from a second generator
(seed + 7919): n ~ U{0..K} per request and step.
"""
import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class LayerShape:
    batch: int
    nheads: int
    head_dim: int
    d_state: int
    ngroups: int
    interval: int = 16
    max_draft: int = 0


# Named workloads: shapes of the decode layers the benchmark and the tests run.
WORKLOADS = {
    # tiny replay-vs-recurrence check, fp32 inputs, 64 steps
    "tiny": dict(shape=LayerShape(4, 2, 16, 16, 1), steps=64, seed=0, in_dtype=torch.float32),
    # small-model-like layer: batch 256, 64 heads, 2 MiB fp32 state per request
    "small_b256": dict(shape=LayerShape(256, 64, 64, 128, 8), steps=512, seed=1,
                       in_dtype=torch.bfloat16),
    # large-model-like layer: batch 512, 128 heads, 4 MiB fp32 state per request
    "large_b512": dict(shape=LayerShape(512, 128, 64, 128, 8), steps=512, seed=2,
                       in_dtype=torch.bfloat16),
    # speculative verify: large-layer shapes, 4 drafts per step, 256 steps
    "spec_b512_k4": dict(shape=LayerShape(512, 128, 64, 128, 8, 16, 4), steps=256, seed=3,
                         in_dtype=torch.bfloat16),
    # precision split: small-layer shapes, 512 steps
    "split_b256": dict(shape=LayerShape(256, 64, 64, 128, 8), steps=512, seed=4,
                       in_dtype=torch.bfloat16),
}


def make_inputs(shape: LayerShape, steps: int, seed: int, in_dtype=torch.bfloat16,
                device="cpu", ntok: int = 0):
    """Draw one layer's initial checkpoint, parameters and per-step inputs.

    ntok = 0: decode layout (no token axis); ntok >= 1: verify layout with
    a [ntok] axis after the batch axis."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    Bsz, H, P, N, G = shape.batch, shape.nheads, shape.head_dim, shape.d_state, shape.ngroups
    tok = (ntok,) if ntok else ()
    kw = dict(generator=g, device=device, dtype=torch.float32)
    ckpt = torch.randn(Bsz, H, P, N, **kw) * 0.1
    A = -torch.exp(torch.rand(H, **kw) * math.log(16.0))
    D = torch.randn(H, **kw)
    x = torch.randn((steps, Bsz) + tok + (H, P), **kw).to(in_dtype)
    Bm = torch.randn((steps, Bsz) + tok + (G, N), **kw).to(in_dtype)
    C = torch.randn((steps, Bsz) + tok + (G, N), **kw).to(in_dtype)
    dt = torch.nn.functional.softplus(torch.randn((steps, Bsz) + tok + (H,), **kw) - 3.0)
    return dict(ckpt=ckpt, A=A, D=D, x=x, B=Bm, C=C, dt=dt)


def accept_lengths(steps: int, batch: int, max_draft: int, seed: int, device="cpu"):
    """Accepted draft counts n ~ U{0..max_draft}, int32 [steps][batch]."""
    g = torch.Generator(device=device)
    g.manual_seed(seed + 7919)
    return torch.randint(0, max_draft + 1, (steps, batch), generator=g, device=device,
                         dtype=torch.int32)
