"""Seeded synthetic Q/K/V for the video-latent attention workloads.

This module only draws inputs. It holds none of the attention method's
arithmetic (no tiling, pooling, scoring, selection, quantisation or
softmax), so both the CUDA path and the fp64 oracle can take their inputs
from it without sharing any of the computation under test.

Two recipes:

* ``iid``: Q, K, V drawn i.i.d. N(0, 1) and rounded to bf16.
* ``field``: per (tensor, batch, head, channel) an i.i.d. N(0, 1) field over
  the unpadded T x H x W latent grid, blurred by a separable Gaussian
  (sigma = 2 tokens, 13 taps, normalised weights, zero boundary), rescaled to
  unit standard deviation, plus N(0, 0.5^2) noise, rounded to bf16. The blur
  makes neighbouring tokens alike, so tile-pooled scores have the spatial
  structure that real video latents show.

Optionally Q of head h is multiplied by 1/tau_h with tau_h log-uniform in
[tau_lo, tau_hi]: a per-head sharpness of the block scores.

All tensors come back in the natural token layout [B, L, heads, D] with
L = T*H*W flattened (t, h, w) row-major.
"""

from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and input recipe of one attention layer."""

    name: str
    B: int
    heads: int
    head_dim: int
    T: int
    H: int
    W: int
    rule: str  # "topk" | "topp" | "window"
    k: int = 0
    p: float = 0.0
    win: tuple = (0, 0, 0)  # half-widths in tiles along (t, h, w)
    qk_fp8: bool = False
    recipe: str = "field"  # "iid" | "field"
    seed: int = 0
    temperature: tuple | None = None  # (tau_lo, tau_hi) or None
    tile: tuple = (4, 4, 4)

    @property
    def L(self) -> int:
        return self.T * self.H * self.W


# The five video-latent workloads: a tiny i.i.d. case, Wan2.1-1.3B and -14B
# shaped top-k layers, a fixed (3,3,1) tile window with e4m3 Q/K, and
# adaptive top-p routing with a top-k floor and per-head temperature.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 64, 8, 16, 16, "topk", k=8, recipe="iid", seed=0),
    "wan1.3b": Workload("wan1.3b", 1, 12, 128, 16, 28, 52, "topk", k=46, seed=1),
    "wan14b": Workload("wan14b", 1, 40, 128, 21, 45, 80, "topk", k=144, seed=2),
    "window_fp8": Workload("window_fp8", 1, 12, 128, 21, 30, 52, "window",
                           win=(1, 1, 0), qk_fp8=True, seed=3),
    "topp": Workload("topp", 1, 40, 128, 21, 45, 80, "topp", k=16, p=0.9, seed=4,
                     temperature=(0.3, 3.0)),
    # The hardware-friendly (6, 8, 8) tile of 384 tokens: the Wan-14B layer at
    # the same 10% density (24 of 240 tiles), and the e4m3 tile window.
    "wan14b_t688": Workload("wan14b_t688", 1, 40, 128, 21, 45, 80, "topk", k=24, seed=2,
                            tile=(6, 8, 8)),
    "window_fp8_t688": Workload("window_fp8_t688", 1, 12, 128, 21, 30, 52, "window",
                                win=(1, 1, 0), qk_fp8=True, seed=3, tile=(6, 8, 8)),
}


def gaussian_taps(sigma: float = 2.0, radius: int = 6) -> torch.Tensor:
    """Normalised 1-D Gaussian weights, 2*radius+1 taps, float64."""
    x = torch.arange(-radius, radius + 1, dtype=torch.float64)
    w = torch.exp(-0.5 * (x / sigma) ** 2)
    return w / w.sum()


def _blur_axis(f: torch.Tensor, taps: torch.Tensor, axis: int) -> torch.Tensor:
    """Convolve the last three axes' `axis` (0,1,2 -> T,H,W) with zero boundary."""
    n = f.shape[0]
    dims = list(f.shape[1:])
    perm = [0] + [1 + a for a in range(3) if a != axis] + [1 + axis]
    g = f.permute(*perm).contiguous()
    lead = g.shape[:-1]
    g = g.reshape(-1, 1, g.shape[-1])
    r = (taps.numel() - 1) // 2
    out = torch.nn.functional.conv1d(g, taps.to(g).view(1, 1, -1), padding=r)
    out = out.reshape(*lead, dims[axis])
    inv = [0] * 4
    for i, p in enumerate(perm):
        inv[p] = i
    return out.permute(*inv).contiguous().reshape(n, *dims)


def _field(gen: torch.Generator, n: int, T: int, H: int, W: int, device) -> torch.Tensor:
    """n independent blurred, standardised fields plus noise, float32 [n,T,H,W]."""
    taps = gaussian_taps().to(device=device, dtype=torch.float32)
    f = torch.randn((n, T, H, W), generator=gen, device=device, dtype=torch.float32)
    for axis in range(3):
        f = _blur_axis(f, taps, axis)
    std = f.reshape(n, -1).std(dim=1, unbiased=False).clamp_min(1e-12)
    f = f / std.view(n, 1, 1, 1)
    f += 0.5 * torch.randn((n, T, H, W), generator=gen, device=device, dtype=torch.float32)
    return f


def head_temperatures(wl: Workload) -> torch.Tensor | None:
    """tau_h, log-uniform in [tau_lo, tau_hi], drawn from its own seeded stream."""
    if wl.temperature is None:
        return None
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed * 1_000_003 + 1)
    lo, hi = (math.log(x) for x in wl.temperature)
    u = torch.rand((wl.heads,), generator=g, dtype=torch.float64)
    return torch.exp(lo + (hi - lo) * u)


def make_qkv(wl: Workload, device="cpu", batch_offset: int = 0):
    """Return (q, k, v) bf16 tensors [B, L, heads, D] on `device`.

    The draw is a pure function of (workload, device type, batch_offset);
    `batch_offset` lets independent replicas draw distinct layers.
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed * 7919 + 104729 * batch_offset)
    out = []
    for _tensor in range(3):
        if wl.recipe == "iid":
            x = torch.randn((wl.B, wl.L, wl.heads, wl.head_dim), generator=gen,
                            device=device, dtype=torch.float32)
        else:
            n = wl.B * wl.heads * wl.head_dim
            f = _field(gen, n, wl.T, wl.H, wl.W, device)
            x = f.reshape(wl.B, wl.heads, wl.head_dim, wl.L).permute(0, 3, 1, 2)
        out.append(x.contiguous())
    tau = head_temperatures(wl)
    if tau is not None:
        out[0] = out[0] / tau.to(device=device, dtype=torch.float32).view(1, 1, -1, 1)
    return tuple(t.to(torch.bfloat16).contiguous() for t in out)


def random_scores(rows: int, n: int, seed: int, ties: bool = True,
                  dtype=torch.float32) -> torch.Tensor:
    """A seeded [rows, n] block-score-like matrix with planted exact ties.

    Used to feed the same score matrix to the selection kernels and to the
    oracle's selection. With `ties`, about a quarter of the entries are
    copied from another entry of the same row, and a few are +0.0 / -0.0.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    s = torch.randn((rows, n), generator=g, dtype=torch.float64).to(dtype)
    if ties and n > 1:
        src = torch.randint(0, n, (rows, n), generator=g)
        pick = torch.rand((rows, n), generator=g) < 0.25
        s = torch.where(pick, torch.gather(s, 1, src), s)
        z = torch.rand((rows, n), generator=g)
        s = torch.where(z < 0.02, torch.zeros_like(s), s)
        s = torch.where(z > 0.98, -torch.zeros_like(s), s)
    return s.contiguous()
