"""A synthetic hybrid SSM/attention decode stage around librssm.

The ReplaySSM article (devotd.net "nvidia-replayssm-hybrid-model-ssm-
decoding-state-buffer", s2 "Reduce state transfers at large batch sizes")
reports the SSM-kernel speed-up diluted by the rest of each decode step: a
decode-stage gain smaller than the kernel gain, and none at batch 1. This
module builds such a stage with random weights so the dilution can be
measured: n_ssm Mamba-2 mixer blocks and n_attn attention blocks, one decode
token per request per step.

Mamba-2 mixer block (Dao and Gu, "Transformers are SSMs", ICML 2024), per
request, u the residual stream [d_model]:
    zxbcdt = W_in^T rmsnorm(u)                      (GEMM, bf16, cuBLAS via torch)
    x, B, C, dt = conv1d+SiLU, softplus             (rssm_stage_conv)
    y = SSM step                                    (rssm_decode_step [+ rssm_flush], or rssm_conv_step)
    v = gated RMS norm(y, z)                        (rssm_stage_gate_norm)
    u += W_out^T v                                  (GEMM)
Attention block (the stand-in for a hybrid model's attention layers):
    q, k, v = W_qkv^T rmsnorm(u); k, v overwrite the oldest slot of a KV
    cache of ctx tokens; o = softmax(q K^T / sqrt(d)) V (torch SDPA, GQA);
    u += W_o^T o.
The projections and the attention are library calls; the SSM step and the
block's element-wise glue run in librssm's kernels. scheme="replay" uses the
replay decode (flush every interval tokens); scheme="conventional" the
per-token read + write kernel on the same inputs and weights.
"""
import ctypes as ct
import math
from dataclasses import dataclass

import torch

from . import rssm


@dataclass(frozen=True)
class StageShape:
    batch: int
    d_model: int
    nheads: int          # SSM heads H
    head_dim: int        # P
    d_state: int         # N
    ngroups: int         # G
    interval: int = 16
    n_ssm: int = 4       # Mamba-2 blocks per stage
    n_attn: int = 1      # attention blocks per stage
    attn_heads: int = 16
    kv_heads: int = 4
    attn_head_dim: int = 128
    ctx: int = 1024      # KV-cache length each attention block attends over
    eps: float = 1e-5

    @property
    def d_inner(self):
        return self.nheads * self.head_dim

    @property
    def d_proj(self):
        return 2 * self.d_inner + 2 * self.ngroups * self.d_state + self.nheads


def _lib():
    L = rssm.lib()
    if not hasattr(L, "_stage_sigs"):
        vp, D = ct.c_void_p, ct.POINTER(rssm.Desc)
        L.rssm_stage_conv.argtypes = [D, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.rssm_stage_conv.restype = ct.c_int
        L.rssm_stage_gate_norm.argtypes = [D, vp, vp, vp, ct.c_float, vp, vp]
        L.rssm_stage_gate_norm.restype = ct.c_int
        L._stage_sigs = True
    return L


def rssm_stage_conv(desc, zxbcdt, conv_state, conv_w, conv_b, dt_bias, x, B, C, dt, stream=None):
    p = rssm._ptr
    rssm._check(_lib().rssm_stage_conv(ct.byref(desc), p(zxbcdt, torch.bfloat16, "zxbcdt"),
                                       p(conv_state, torch.bfloat16, "conv_state"),
                                       p(conv_w, torch.float32, "conv_w"), p(conv_b, torch.float32, "conv_b"),
                                       p(dt_bias, torch.float32, "dt_bias"), p(x, torch.bfloat16, "x"),
                                       p(B, torch.bfloat16, "B"), p(C, torch.bfloat16, "C"),
                                       p(dt, torch.float32, "dt"), rssm._stream(stream)), "rssm_stage_conv")


def rssm_stage_gate_norm(desc, y, zxbcdt, norm_w, eps, out, stream=None):
    p = rssm._ptr
    rssm._check(_lib().rssm_stage_gate_norm(ct.byref(desc), p(y, torch.float32, "y"),
                                            p(zxbcdt, torch.bfloat16, "zxbcdt"),
                                            p(norm_w, torch.float32, "norm_w"), float(eps),
                                            p(out, torch.bfloat16, "out"), rssm._stream(stream)),
                "rssm_stage_gate_norm")


def rmsnorm(u, w, eps):
    """Pre-norm of a block (fp32 arithmetic, bf16 result)."""
    uf = u.float()
    return (uf * torch.rsqrt(uf.pow(2).mean(-1, keepdim=True) + eps) * w).to(torch.bfloat16)


def make_weights(shape: StageShape, seed: int, device="cuda"):
    """Random weights of the stage (seeded; scaled so activations stay O(1))."""
    g = torch.Generator(device="cpu").manual_seed(seed)

    def rn(*size, std=1.0):
        return (torch.randn(*size, generator=g) * std)

    s = shape
    chans = s.d_inner + 2 * s.ngroups * s.d_state
    blocks = []
    for _ in range(s.n_ssm):
        blocks.append({
            "norm": (1.0 + 0.1 * rn(s.d_model)).float(),
            "w_in": rn(s.d_model, s.d_proj, std=1.0 / math.sqrt(s.d_model)).to(torch.bfloat16),
            "conv_w": rn(chans, 4, std=0.5).float(),
            "conv_b": rn(chans, std=0.1).float(),
            "dt_bias": (torch.rand(s.nheads, generator=g) * 2.0 - 4.0).float(),
            "A": (-torch.exp(torch.rand(s.nheads, generator=g) * math.log(16.0))).float(),
            "D": rn(s.nheads).float(),
            "gnorm": (1.0 + 0.1 * rn(s.d_inner)).float(),
            "w_out": rn(s.d_inner, s.d_model, std=1.0 / math.sqrt(s.d_inner)).to(torch.bfloat16),
        })
    attn = []
    qkv = (s.attn_heads + 2 * s.kv_heads) * s.attn_head_dim
    for _ in range(s.n_attn):
        attn.append({
            "norm": (1.0 + 0.1 * rn(s.d_model)).float(),
            "w_qkv": rn(s.d_model, qkv, std=1.0 / math.sqrt(s.d_model)).to(torch.bfloat16),
            "w_o": rn(s.attn_heads * s.attn_head_dim, s.d_model,
                      std=1.0 / math.sqrt(s.attn_heads * s.attn_head_dim)).to(torch.bfloat16),
        })
    mv = lambda d: {k: v.to(device) for k, v in d.items()}
    return [mv(b) for b in blocks], [mv(a) for a in attn]


class HybridStage:
    """n_ssm Mamba-2 blocks then n_attn attention blocks, one decode token per
    request per step(); scheme "replay" or "conventional" for the SSM step."""

    def __init__(self, shape: StageShape, weights, scheme="replay", seed=0, device="cuda"):
        assert scheme in ("replay", "conventional")
        s = self.shape = shape
        self.scheme = scheme
        self.blocks, self.attn = weights
        self.desc = rssm.make_desc(s.batch, s.nheads, s.head_dim, s.d_state, s.ngroups, interval=s.interval)
        g = torch.Generator(device="cpu").manual_seed(seed + 1)
        chans = s.d_inner + 2 * s.ngroups * s.d_state
        self.ssm = []
        for _ in range(s.n_ssm):
            ck = (torch.randn(s.batch, s.nheads, s.head_dim, s.d_state, generator=g) * 0.1).to(device)
            if scheme == "replay":
                st = rssm.RssmState(self.desc, device)
                st.ckpt.copy_(ck)
            else:
                st = ck
            self.ssm.append({"state": st,
                             "conv": torch.zeros(s.batch, 3, chans, dtype=torch.bfloat16, device=device)})
        self.kv = []
        for _ in range(s.n_attn):
            kc = (torch.randn(s.batch, s.kv_heads, s.ctx, s.attn_head_dim, generator=g)).to(torch.bfloat16)
            vc = (torch.randn(s.batch, s.kv_heads, s.ctx, s.attn_head_dim, generator=g)).to(torch.bfloat16)
            self.kv.append({"k": kc.to(device), "v": vc.to(device)})
        self.t = 0
        B_, din, gn = s.batch, s.d_inner, s.ngroups * s.d_state
        self.zx = torch.empty(B_, s.d_proj, dtype=torch.bfloat16, device=device)
        self.x = torch.empty(B_, s.nheads, s.head_dim, dtype=torch.bfloat16, device=device)
        self.Bv = torch.empty(B_, s.ngroups, s.d_state, dtype=torch.bfloat16, device=device)
        self.Cv = torch.empty_like(self.Bv)
        self.dt = torch.empty(B_, s.nheads, dtype=torch.float32, device=device)
        self.y = torch.empty(B_, s.nheads, s.head_dim, dtype=torch.float32, device=device)
        self.v = torch.empty(B_, din, dtype=torch.bfloat16, device=device)

    def ssm_block(self, i, u):
        s, b = self.shape, self.blocks[i]
        st = self.ssm[i]
        torch.matmul(rmsnorm(u, b["norm"], s.eps), b["w_in"], out=self.zx)
        rssm_stage_conv(self.desc, self.zx, st["conv"], b["conv_w"], b["conv_b"], b["dt_bias"],
                        self.x, self.Bv, self.Cv, self.dt)
        if self.scheme == "replay":
            rssm.rssm_decode_step(st["state"], self.x, self.Bv, self.Cv, self.dt, b["A"], b["D"], self.y)
            if (self.t + 1) % s.interval == 0:
                rssm.rssm_flush(st["state"], b["A"])
        else:
            rssm.rssm_conv_step(self.desc, st["state"], self.x, self.Bv, self.Cv, self.dt, b["A"], b["D"], self.y)
        rssm_stage_gate_norm(self.desc, self.y, self.zx, b["gnorm"], s.eps, self.v)
        return u + torch.matmul(self.v, b["w_out"])

    def attn_block(self, i, u):
        s, a, kv = self.shape, self.attn[i], self.kv[i]
        hq, hk, hd = s.attn_heads, s.kv_heads, s.attn_head_dim
        qkv = torch.matmul(rmsnorm(u, a["norm"], s.eps), a["w_qkv"])
        q = qkv[:, :hq * hd].view(s.batch, hq, 1, hd)
        k = qkv[:, hq * hd:(hq + hk) * hd].view(s.batch, hk, hd)
        v = qkv[:, (hq + hk) * hd:].view(s.batch, hk, hd)
        slot = self.t % s.ctx
        kv["k"][:, :, slot].copy_(k)
        kv["v"][:, :, slot].copy_(v)
        o = torch.nn.functional.scaled_dot_product_attention(q, kv["k"], kv["v"], enable_gqa=True)
        return u + torch.matmul(o.reshape(s.batch, hq * hd), a["w_o"])

    def step(self, u):
        """One decode token per request: u [batch][d_model] bf16 -> same."""
        for i in range(self.shape.n_ssm):
            u = self.ssm_block(i, u)
        for i in range(self.shape.n_attn):
            u = self.attn_block(i, u)
        self.t += 1
        return u
