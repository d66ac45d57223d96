"""Seeded synthetic inputs for the NABLA hot path (video-latent-shaped Q, K, V, dO).

This module holds no arithmetic of the method itself: it only draws random tensors.
Both the CUDA path and the CPU oracle are fed from here; neither is imported here.

Recipe (stand-in for video-DiT latents at 720p, which are not available):
  * per (b, h): white noise Z ~ N(0, 1) of shape (T, Hg, W, D), fp32;
  * a separable Gaussian filter along T, Hg and W with standard deviation ``sigma``
    tokens, mirror-reflected at the edges, truncated at 4 sigma;
  * every channel of the smoothed field rescaled to unit standard deviation over the
    head's tokens, then multiplied by ``field_scale`` (2.0): the field F;
  * Q = 0.5 N1 + F, K = 0.5 N2 + F, V = 0.5 N3 + F with N1, N2, N3 iid N(0, 1);
  * tensors are laid out [B, H, S, D] in natural token order, S = T*Hg*W with index
    (t*Hg + h)*W + w, and rounded to bf16 (round to nearest even);
  * dO ~ N(0, 1), bf16, drawn in the reordered order.
The per-head sigma is drawn from a CPU generator (uniform in [lo, hi]) so that it does
not depend on the device.  The noise is drawn on the target device from a generator
seeded with ``seed``; CPU and CUDA streams of numbers differ, so a comparison always
copies one generated tensor to both sides.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    """One synthetic NABLA workload (shape, thresholds, window, recipe parameters)."""

    name: str
    B: int
    H: int
    T: int
    Hg: int
    W: int
    D: int
    P: int = 8
    thrs: tuple = (0.8,)
    window: tuple = (0, 0, 0)
    sigma: tuple = (2.0, 2.0)          # per-head sigma ~ U[lo, hi] (lo == hi: fixed)
    backward: bool = False
    seed: int = 1000
    field_scale: float = 2.0
    noise_scale: float = 0.5
    notes: str = field(default="", compare=False)

    @property
    def S(self) -> int:
        return self.T * self.Hg * self.W

    @property
    def N(self) -> int:
        return self.P * self.P

    @property
    def nb(self) -> int:
        return self.S // self.N

    @property
    def block_grid(self):
        return (self.T, self.Hg // self.P, self.W // self.P)


# The five workloads of the benchmark plan (video-latent shapes, bf16).
WORKLOADS = {
    "tiny": Workload("tiny", B=1, H=2, T=2, Hg=16, W=16, D=64, thrs=(0.8,),
                     sigma=(2.0, 2.0), seed=1000),
    "small": Workload("small", B=1, H=8, T=4, Hg=32, W=32, D=128, thrs=(0.5, 0.8, 0.95),
                      sigma=(1.0, 4.0), seed=1001),
    "wan720p": Workload("wan720p", B=1, H=40, T=21, Hg=48, W=80, D=128, thrs=(0.8,),
                        sigma=(1.0, 6.0), seed=1002),
    "wan720p_sta": Workload("wan720p_sta", B=1, H=40, T=21, Hg=48, W=80, D=128,
                            thrs=(0.7,), window=(3, 3, 5), sigma=(1.0, 6.0), seed=1002),
    # heads 0-7 of the 720p-like workload (identical draws: streams are seeded per head),
    # a smaller case for profiler captures
    "wan720p_h8": Workload("wan720p_h8", B=1, H=8, T=21, Hg=48, W=80, D=128, thrs=(0.8,),
                           sigma=(1.0, 6.0), seed=1002),
    "train_mid": Workload("train_mid", B=2, H=24, T=11, Hg=32, W=56, D=128, thrs=(0.8,),
                          window=(3, 3, 3), sigma=(2.0, 2.0), backward=True, seed=1004),
    # heads 0-11 of batch 0 of the training-like workload (identical draws), a smaller
    # case for profiler captures of the backward
    "train_mid_h12": Workload("train_mid_h12", B=1, H=12, T=11, Hg=32, W=56, D=128, thrs=(0.8,),
                              window=(3, 3, 3), sigma=(2.0, 2.0), backward=True, seed=1004),
}


def smoothing_matrix(L: int, sigma: float) -> np.ndarray:
    """L x L matrix of a 1-D Gaussian filter (sigma in samples), mirror-reflected edges.

    Out-of-range taps are folded back with period 2L (index -1 -> 0, L -> L-1), so any
    radius works even when 4 sigma exceeds L.
    """
    r = int(math.ceil(4.0 * sigma))
    offs = np.arange(-r, r + 1)
    w = np.exp(-0.5 * (offs / sigma) ** 2)
    w /= w.sum()
    M = np.zeros((L, L), dtype=np.float64)
    for i in range(L):
        j = (i + offs) % (2 * L)
        j = np.where(j >= L, 2 * L - 1 - j, j)
        np.add.at(M[i], j, w)
    return M


def head_sigmas(wl: Workload) -> np.ndarray:
    g = torch.Generator().manual_seed(wl.seed + 7919)
    lo, hi = wl.sigma
    u = torch.rand(wl.B * wl.H, generator=g, dtype=torch.float64).numpy()
    return lo + (hi - lo) * u


def make_qkv(wl: Workload, device="cpu", heads=None):
    """Draw Q, K, V (bf16, natural order, [B, H, S, D]) for a workload.

    ``heads`` (optional) restricts generation to a list of flat head indices b*H + h;
    the other heads are left zero.  The per-head stream is seeded from (seed, b*H + h)
    so any subset of heads reproduces the full draw.
    """
    device = torch.device(device)
    B, H, D = wl.B, wl.H, wl.D
    T, Hg, W = wl.T, wl.Hg, wl.W
    q = torch.zeros(B, H, wl.S, D, dtype=torch.bfloat16, device=device)
    k = torch.zeros_like(q)
    v = torch.zeros_like(q)
    sig = head_sigmas(wl)
    todo = range(B * H) if heads is None else heads
    for bh in todo:
        b, h = divmod(bh, H)
        g = torch.Generator(device=device).manual_seed(wl.seed * 100003 + bh)
        z = torch.randn(T, Hg, W, D, generator=g, device=device, dtype=torch.float32)
        mt, mh, mw = (torch.tensor(smoothing_matrix(L, float(sig[bh])), device=device,
                                   dtype=torch.float32) for L in (T, Hg, W))
        f = torch.einsum("at,thwd->ahwd", mt, z)
        f = torch.einsum("bh,ahwd->abwd", mh, f)
        f = torch.einsum("cw,abwd->abcd", mw, f)
        f = f.reshape(wl.S, D)
        f = f / f.std(dim=0, unbiased=False, keepdim=True) * wl.field_scale
        for dst in (q, k, v):
            n = torch.randn(wl.S, D, generator=g, device=device, dtype=torch.float32)
            dst[b, h] = (wl.noise_scale * n + f).to(torch.bfloat16)
    return q, k, v


def make_dout(wl: Workload, device="cpu"):
    """Upstream gradient dO ~ N(0, 1), bf16, [B, H, S, D] in reordered token order."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(wl.seed * 100003 + 99991)
    return torch.randn(wl.B, wl.H, wl.S, wl.D, generator=g, device=device,
                       dtype=torch.float32).to(torch.bfloat16)


def random_bf16(shape, seed: int, device="cpu", scale: float = 1.0):
    """Plain N(0, scale^2) bf16 tensor (edge-case tests)."""
    g = torch.Generator(device=device).manual_seed(seed)
    return (torch.randn(*shape, generator=g, device=device) * scale).to(torch.bfloat16)
