"""Seeded synthetic inputs shaped like the video-diffusion self-attention calls.

This module only draws random numbers: it contains none of the selection or
attention arithmetic, so the CPU oracle and the CUDA path can both consume its
tensors without sharing any of the method's code.

Workload shapes follow the video models that the SpargeAttention documentation
lists as supported ("SpargeAttention Documentation", supported models:
Wan2.1-T2V-1.3B/14B, HunyuanVideo, CogVideoX-2B) and the 720p settings table of
the AB-Attention README ("Paper settings, timing, and pipeline integration":
1280x720, 81 frames for Wan2.1, 129 frames for HunyuanVideo).  No video data
exists here, so q/k are a smooth random field over the (t, h, w) token grid plus
noise, which gives the spatially coherent block scores a real video model shows.

Recipe (fixed; every tensor is drawn on the CPU with ``torch.Generator``):

* positions: video token m on a T x Hg x Wg grid in raster order maps to
  t = m // (Hg*Wg), y = (m // Wg) % Hg, x = m % Wg and u = (t/T, y/Hg, x/Wg);
* per head h and feature j = 1..4: omega_hj ~ N(0, (4 pi)^2 I_3),
  phi_hj ~ U[0, 2 pi), a_hj ~ N(0, I_d), shared by q and k and by every batch
  entry;
* q = 1.5 d^(-1/4) sum_j cos(omega_hj . u + phi_hj) a_hj + 0.3 eps_q, and k the
  same with its own eps_k; eps ~ N(0, 1); v ~ N(0, 1);
* text tokens (CogVideoX) come first and are plain N(0, 1) in q, k and v;
* draw order: features (h-major), then q, k, v, each slice (b, h) in order;
* every value is drawn in fp32 and rounded to bf16 (round to nearest even).

The caller-supplied random block mask draws ``torch.rand(B, H, Qb, Kb) < p``
from a generator seeded with 1.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BLOCK_Q = 128  # query rows per mask block
BLOCK_K = 64   # key rows per mask block


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    grid: tuple  # (T, Hg, Wg) video token grid
    text: int = 0  # text tokens placed before the video tokens
    topk: tuple = (0.5,)
    mask_density: tuple = ()
    seed: int = 0
    mask_seed: int = 1
    note: str = ""

    @property
    def N(self) -> int:
        T, Hg, Wg = self.grid
        return self.text + T * Hg * Wg

    @property
    def Qb(self) -> int:
        return -(-self.N // BLOCK_Q)

    @property
    def Kb(self) -> int:
        return -(-self.N // BLOCK_K)

    def dense_flops(self) -> float:
        """4*B*H*N^2*d: the FLOPs of dense attention (QK^T plus PV)."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * self.d


WORKLOADS = {
    "tiny": Workload("tiny", B=1, H=2, d=64, grid=(4, 16, 16), topk=(0.5,),
                     note="4x16x16 grid, parity case the oracle finishes in seconds"),
    "cogvideox2b": Workload("cogvideox2b", B=2, H=30, d=64, grid=(13, 30, 45), text=226,
                            topk=(0.5,), note="CogVideoX-2B-shaped, B=2 for CFG, 226 text tokens first"),
    "wan13b": Workload("wan13b", B=1, H=12, d=128, grid=(21, 45, 80),
                       topk=(1.0, 0.5, 0.3, 0.1), note="Wan2.1-1.3B-shaped 720p 81 frames"),
    "wan14b": Workload("wan14b", B=1, H=40, d=128, grid=(21, 45, 80), topk=(0.5,),
                       mask_density=(0.5, 0.1), note="Wan2.1-14B-shaped 720p 81 frames"),
    "hunyuan13b": Workload("hunyuan13b", B=1, H=24, d=128, grid=(33, 45, 80), topk=(0.1,),
                           note="HunyuanVideo-13B-shaped 720p 129 frames"),
}


def custom(name: str, B: int, H: int, d: int, N: int, seed: int = 0) -> Workload:
    """A workload of arbitrary length: a 1 x 1 x N video grid (used for ragged-edge cases)."""
    return Workload(name, B=B, H=H, d=d, grid=(1, 1, N), seed=seed)


def _positions(wl: Workload) -> torch.Tensor:
    T, Hg, Wg = wl.grid
    m = torch.arange(T * Hg * Wg, dtype=torch.int64)
    t = torch.div(m, Hg * Wg, rounding_mode="floor")
    y = torch.div(m, Wg, rounding_mode="floor") % Hg
    x = m % Wg
    return torch.stack([t.float() / T, y.float() / Hg, x.float() / Wg], dim=1)  # [Nv, 3]


def make_qkv(wl: Workload, device: str = "cpu"):
    """Draw q, k, v as contiguous bf16 tensors of shape [B, H, N, d]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed)
    B, H, N, d = wl.B, wl.H, wl.N, wl.d
    nv = N - wl.text
    u = _positions(wl)
    omega = torch.randn(H, 4, 3, generator=g) * (4.0 * math.pi)
    phi = torch.rand(H, 4, generator=g) * (2.0 * math.pi)
    amp = torch.randn(H, 4, d, generator=g)
    field_ = []
    for h in range(H):
        c = torch.cos(u @ omega[h].T + phi[h])  # [Nv, 4]
        field_.append((1.5 * d ** -0.25) * (c @ amp[h]))  # [Nv, d]
    out = []
    for which in ("q", "k", "v"):
        t = torch.empty(B, H, N, d, dtype=torch.bfloat16)
        for b in range(B):
            for h in range(H):
                noise = torch.randn(N, d, generator=g)
                if which == "v":
                    t[b, h] = noise.to(torch.bfloat16)
                else:
                    x = noise.clone()
                    x[wl.text:] = field_[h] + 0.3 * noise[wl.text:]
                    t[b, h] = x.to(torch.bfloat16)
        out.append(t if device == "cpu" else t.to(device))
    return tuple(out)


def make_random_mask(wl: Workload, density: float) -> torch.Tensor:
    """Caller-supplied block mask: uint8 [B, H, Qb, Kb], 1 with probability `density`."""
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.mask_seed)
    r = torch.rand(wl.B, wl.H, wl.Qb, wl.Kb, generator=g)
    return (r < density).to(torch.uint8)


def make_uniform(shape, seed: int, dtype=torch.bfloat16, scale: float = 1.0) -> torch.Tensor:
    """Plain N(0, scale^2) draws, for small hand-made cases."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(dtype)
