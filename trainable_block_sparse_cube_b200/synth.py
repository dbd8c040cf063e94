"""Seeded synthetic video-latent inputs for the VSA forward pass.

This module only draws random tensors. It holds none of the attention
method's arithmetic (no cube reordering, pooling, attention or selection):
both the CUDA path and the fp64 CPU checker consume its output unchanged.

Layout of every tensor it returns: ``[B, heads, N, D]`` (q, k, v; bf16) and
``[B, heads, N]`` (gate_c, gate_f; fp32), with ``N = T*H*W`` tokens in raster
order ``n = (t*H + h)*W + w``.

Each (b, head) slice has its own torch CPU generator seeded with
``seed*1_000_003 + b*1009 + h``, so one head can be regenerated on its own
(used when checking sampled heads of the large workloads).

Workload recipes (sizes follow the pages' long-video shapes: 61,440 tokens
with K=16 / K=32 in "Faster Video Diffusion with Trainable Sparse Attention",
"Surprising findings"; 87.5% sparsity in its "Key results"):

``iid``       q, k, v ~ N(0, 1) per element.
``cube``      N(0, 1) per element plus an offset ~ N(0, 0.5^2) per channel that
              is constant over each 4x4x4 block of the (t, h, w) grid, drawn
              independently for q, k and v, so block-level scores are
              structured.
``cube_sin``  ``cube`` plus, for q and k, 0.5*sin(2*pi*(ft*t/T + fh*h/H +
              fw*w/W) + phi_d) with per-channel integer frequencies in {0,1,2}
              (not all zero) and a phase phi_d ~ U[0, 2*pi), shared by q and k.
``cluster``   8 centres per head ~ N(0, I_D) shared by q and k, 8 separate
              centres for v, mixing weights ~ Dirichlet(1,...,1); every 4x4x4
              block draws one centre id and all its tokens are
              centre + N(0, 0.3^2) noise (fresh noise for q, k and v).

Gates: gate_c, gate_f = sigmoid(N(0, 1)) per token and head, fp32.
All draws are made in fp32 and rounded to bf16 (round to nearest even).
"""
from __future__ import annotations

import dataclasses
import math

import torch

__all__ = ["Workload", "WORKLOADS", "head_inputs", "make_inputs", "head_dout", "make_dout"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: int
    D: int
    T: int
    H: int
    W: int
    topk: int            # > 0: fixed top-K; 0: top-p mode
    top_p: float = 0.0
    kmin: int = 0
    kmax: int = 0
    gen: str = "iid"
    seed: int = 0

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def C(self) -> int:
        return self.N // 64

    @property
    def kcap(self) -> int:
        return self.topk if self.topk > 0 else self.kmax

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 1, 2, 64, 8, 8, 8, topk=2, gen="iid", seed=0),
        Workload("pretrain16k", 1, 12, 128, 16, 32, 32, topk=32, gen="cube", seed=1),
        Workload("long61k_k32", 1, 12, 128, 16, 48, 80, topk=32, gen="cube", seed=2),
        Workload("long61k_k16", 1, 12, 128, 16, 48, 80, topk=16, gen="cube", seed=2),
        Workload("large77k", 1, 40, 128, 20, 48, 80, topk=150, gen="cube_sin", seed=3),
        Workload("dynamic61k", 1, 12, 128, 16, 48, 80, topk=0, top_p=0.9, kmin=4, kmax=128,
                 gen="cluster", seed=4),
    ]
}


def _block_field(g: torch.Generator, T: int, H: int, W: int, D: int, std: float) -> torch.Tensor:
    """A [T*H*W, D] field that is constant over each 4x4x4 block of the grid."""
    f = torch.randn(T // 4, H // 4, W // 4, D, generator=g) * std
    f = f.repeat_interleave(4, 0).repeat_interleave(4, 1).repeat_interleave(4, 2)
    return f.reshape(T * H * W, D)


def head_inputs(wl: Workload, b: int, h: int):
    """Inputs of one (b, head): q, k, v as [N, D] bf16; gate_c, gate_f as [N] fp32."""
    T, H, W, D, N = wl.T, wl.H, wl.W, wl.D, wl.N
    if T % 4 or H % 4 or W % 4:
        raise ValueError("grid dimensions must be multiples of 4")
    g = torch.Generator().manual_seed(wl.seed * 1_000_003 + b * 1009 + h)
    if wl.gen == "iid":
        q, k, v = (torch.randn(N, D, generator=g) for _ in range(3))
    elif wl.gen in ("cube", "cube_sin"):
        xs = []
        for _ in range(3):
            tok = torch.randn(N, D, generator=g)
            xs.append(tok + _block_field(g, T, H, W, D, 0.5))
        q, k, v = xs
        if wl.gen == "cube_sin":
            freq = torch.randint(0, 3, (D, 3), generator=g)
            for d in range(D):  # redraw the all-zero frequency rows, in channel order
                while int(freq[d].abs().sum()) == 0:
                    freq[d] = torch.randint(0, 3, (3,), generator=g)
            phase = torch.rand(D, generator=g) * (2 * math.pi)
            t = torch.arange(T, dtype=torch.float32).view(T, 1, 1, 1) / T
            hh = torch.arange(H, dtype=torch.float32).view(1, H, 1, 1) / H
            ww = torch.arange(W, dtype=torch.float32).view(1, 1, W, 1) / W
            f = freq.to(torch.float32)
            arg = 2 * math.pi * (f[:, 0] * t + f[:, 1] * hh + f[:, 2] * ww) + phase
            s = (0.5 * torch.sin(arg)).reshape(N, D)
            q = q + s
            k = k + s
    elif wl.gen == "cluster":
        n_cent = 8
        mu_qk = torch.randn(n_cent, D, generator=g)
        mu_v = torch.randn(n_cent, D, generator=g)
        e = -torch.log(torch.rand(n_cent, generator=g).clamp_min(1e-12))
        mix = e / e.sum()
        nb = (T // 4) * (H // 4) * (W // 4)
        ids = torch.multinomial(mix, nb, replacement=True, generator=g)
        ids = ids.view(T // 4, H // 4, W // 4)
        ids = ids.repeat_interleave(4, 0).repeat_interleave(4, 1).repeat_interleave(4, 2).reshape(N)
        q = mu_qk[ids] + 0.3 * torch.randn(N, D, generator=g)
        k = mu_qk[ids] + 0.3 * torch.randn(N, D, generator=g)
        v = mu_v[ids] + 0.3 * torch.randn(N, D, generator=g)
    else:
        raise ValueError(f"unknown generator {wl.gen!r}")
    gate_c = torch.sigmoid(torch.randn(N, generator=g))
    gate_f = torch.sigmoid(torch.randn(N, generator=g))
    bf = torch.bfloat16
    return q.to(bf), k.to(bf), v.to(bf), gate_c, gate_f


def head_dout(wl: Workload, b: int, h: int) -> torch.Tensor:
    """Upstream gradient of the gated output for one (b, head): [N, D] bf16,
    N(0, 1) per element, from its own generator (seed offset so that it is
    independent of the forward inputs)."""
    g = torch.Generator().manual_seed(wl.seed * 1_000_003 + b * 1009 + h + 7_777_777)
    return torch.randn(wl.N, wl.D, generator=g).to(torch.bfloat16)


def make_dout(wl: Workload) -> torch.Tensor:
    """Upstream gradients [B, heads, N, D] bf16 (see head_dout)."""
    return torch.stack([torch.stack([head_dout(wl, b, h) for h in range(wl.heads)]) for b in range(wl.B)])


def make_inputs(wl: Workload, heads=None):
    """Full inputs [B, heads, N, D] (bf16) and gates [B, heads, N] (fp32) on the CPU.

    ``heads`` optionally restricts generation to a subset of head indices
    (the returned tensors then have len(heads) heads, in that order)."""
    hs = list(range(wl.heads)) if heads is None else list(heads)
    per_b = []
    for b in range(wl.B):
        per_b.append([head_inputs(wl, b, h) for h in hs])
    out = []
    for j in range(5):
        out.append(torch.stack([torch.stack([per_b[b][i][j] for i in range(len(hs))]) for b in range(wl.B)]))
    return tuple(out)
