"""Seeded synthetic Q/K/V for the rf_v2 workloads.

This module only makes inputs: it holds none of the method's arithmetic and
is the one piece shared by the CUDA path's tests/benchmark and the CPU
oracle.  Every tensor comes from a ``torch.Generator`` seeded per workload,
on the device asked for, rounded to bf16.

Workloads (shapes of the pages' use cases; the activations themselves are
synthetic, no model weights or data are involved):

* ``tiny``     1 x 2 heads, latent (4, 32, 32), no text, sparsity 0.5, N(0, 1).
* ``text``     1 x 12 heads, 512 text tokens + latent (8, 48, 64), sparsity 0.8.
               N(0, 1) plus a per-head rank-8 component shared by the tokens of
               each 8x8 tile (per token for text) added to Q and K, so block
               scores are not uniform.
* ``wan``      1 x 40 heads, latent (21, 45, 80) (a 720p 5 s clip), no text,
               sparsity 0.8.  N(0, 1) plus a spatially smooth field (white noise
               blurred by a separable Gaussian, sigma (1, 2, 2) tokens over
               (t, y, x), renormalised) shared by Q and K per head.
* ``minimax``  1 x 56 heads, 256 text tokens + latent (62, 24, 42) (1344x768),
               sparsity 0.8.  Q and K are RMS-normalised per head (eps 1e-5,
               weight 1) and rotated on channel pairs (d, d + 48), d < 48, with
               positions split 16/16/16 over (t, y, x), theta_i = 10000^(-i/16);
               text tokens sit at position 0; channels 96..127 pass through.
               V ~ N(0, 1).  This follows the pre-attention recipe of the
               FlashInfer ``minimax_h3_fp8_pre_attention`` page.
"""

from __future__ import annotations

from dataclasses import dataclass, replace
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int
    D: int
    txt_len: int
    latent: tuple
    sparsity: float
    layout: str = "BSND"
    kind: str = "normal"
    seed: int = 0

    @property
    def S(self) -> int:
        t, h, w = self.latent
        return self.txt_len + t * h * w


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 128, 0, (4, 32, 32), 0.5, kind="normal", seed=1),
    "text": Workload("text", 1, 12, 128, 512, (8, 48, 64), 0.8, kind="lowrank", seed=2),
    "wan": Workload("wan", 1, 40, 128, 0, (21, 45, 80), 0.8, kind="smooth", seed=3),
    "minimax": Workload("minimax", 1, 56, 128, 256, (62, 24, 42), 0.8, kind="rope", seed=4),
}


def workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return replace(w, **overrides) if overrides else w


def _randn(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _video_coords(T, H, W, device):
    t = torch.arange(T, device=device).view(T, 1, 1).expand(T, H, W).reshape(-1)
    y = torch.arange(H, device=device).view(1, H, 1).expand(T, H, W).reshape(-1)
    x = torch.arange(W, device=device).view(1, 1, W).expand(T, H, W).reshape(-1)
    return t, y, x


def _lowrank(w: Workload, gen, device):
    """Per-head rank-8 component, constant over each 8x8 tile."""
    T, H, W = w.latent
    S, N = w.S, w.N
    nty, ntx = -(-H // 8), -(-W // 8)
    ztile = _randn((T, nty, ntx, 8), gen, device)
    t, y, x = _video_coords(T, H, W, device)
    zvid = ztile[t, y // 8, x // 8]                         # [T*H*W, 8]
    ztxt = _randn((w.txt_len, 8), gen, device)
    z = torch.cat([ztxt, zvid], 0)                          # [S, 8]
    aq = _randn((N, 8, w.D), gen, device) / math.sqrt(8.0)
    ak = _randn((N, 8, w.D), gen, device) / math.sqrt(8.0)
    return torch.einsum("sr,nrd->snd", z, aq), torch.einsum("sr,nrd->snd", z, ak)


def _gauss_kernel(sigma, device):
    r = max(1, int(math.ceil(3 * sigma)))
    xs = torch.arange(-r, r + 1, device=device, dtype=torch.float32)
    k = torch.exp(-0.5 * (xs / sigma) ** 2)
    return k / k.sum()


def _smooth(w: Workload, gen, device):
    """Gaussian-blurred white noise over (t, y, x), unit variance, per head/channel."""
    T, H, W = w.latent
    N, D = w.N, w.D
    g = _randn((N * D, 1, T, H, W), gen, device)
    for axis, sigma in ((2, 1.0), (3, 2.0), (4, 2.0)):
        k = _gauss_kernel(sigma, device)
        shape = [1, 1, 1, 1, 1]
        shape[axis] = k.numel()
        pad = [0, 0, 0]
        pad[axis - 2] = k.numel() // 2
        g = torch.nn.functional.conv3d(g, k.view(shape), padding=tuple(pad))
    g = g.view(N, D, T * H * W)
    g = g / g.std(dim=2, keepdim=True)
    g = g.permute(2, 0, 1)                                   # [THW, N, D]
    return torch.cat([torch.zeros(w.txt_len, N, D, device=device), g], 0)


def _rope(w: Workload, x, device):
    """RMSNorm (weight 1) then rotation of channel pairs (d, d + 48), d < 48."""
    x = x * torch.rsqrt(x.pow(2).mean(dim=-1, keepdim=True) + 1e-5)
    T, H, W = w.latent
    t, y, xx = _video_coords(T, H, W, device)
    zeros = torch.zeros(w.txt_len, device=device, dtype=torch.long)
    pos = torch.stack([torch.cat([zeros, t]), torch.cat([zeros, y]), torch.cat([zeros, xx])], 1).float()  # [S, 3]
    i = torch.arange(48, device=device)
    theta = torch.pow(torch.tensor(10000.0, device=device), -(i % 16).float() / 16.0)
    ang = pos[:, (i // 16)] * theta                          # [S, 48]
    c, s = torch.cos(ang)[:, None, :], torch.sin(ang)[:, None, :]
    a, b = x[..., :48], x[..., 48:96]
    return torch.cat([a * c - b * s, a * s + b * c, x[..., 96:]], dim=-1)


def make_inputs(w: Workload, device="cpu", dtype=torch.bfloat16):
    """Seeded q, k, v in ``w.layout`` ([B,S,N,D] or [B,N,S,D]), rounded to
    ``dtype`` (bfloat16 or float16) from the same fp32 draws."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(1000 + w.seed)
    B, S, N, D = w.B, w.S, w.N, w.D
    outs = []
    for b in range(B):
        q = _randn((S, N, D), gen, device)
        k = _randn((S, N, D), gen, device)
        v = _randn((S, N, D), gen, device)
        if w.kind == "lowrank":
            dq, dk = _lowrank(w, gen, device)
            q, k = q + dq, k + dk
        elif w.kind == "smooth":
            sm = _smooth(w, gen, device)
            q, k = q + sm, k + sm
        elif w.kind == "rope":
            q, k = _rope(w, q, device), _rope(w, k, device)
        outs.append((q.to(dtype), k.to(dtype), v.to(dtype)))
        del q, k, v
    q, k, v = (torch.stack([o[i] for o in outs], 0) for i in range(3))   # [B,S,N,D]
    if w.layout == "BNSD":
        q, k, v = (t.transpose(1, 2).contiguous() for t in (q, k, v))
    elif w.layout != "BSND":
        raise ValueError("layout must be BSND or BNSD")
    return q, k, v
