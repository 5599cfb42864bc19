"""Seeded synthetic inputs and the named workloads.

This module only draws inputs; it holds none of the method's arithmetic, so
both the CUDA path and the oracle can read what it produces.

Inputs stand in for VAE latents of 2K-Bench clips (not available here), at
the grid sizes of 720p- and 2K-like latents:

* Q, K, V: per (tensor, head, channel) a smooth 3D field, the sum of four
  unit-amplitude sinusoids sin(2*pi*(f_t t/T + f_h h/H + f_w w/W) + phi) with
  f ~ U(0,3) cycles per grid and phi ~ U(0, 2*pi), plus N(0, 0.5^2) noise,
  rounded to bf16.
* planted zones (V only): a few 8x8x8 zones, each with one random axis, get
  slice-constant offsets along that axis, drawn N(0, planted_amp^2) per
  (channel, slice); this raises the zone's directional variation along that
  axis well above the other zones'.
* a (audio-to-video cross-attention norms): a sum of isotropic Gaussian
  blobs exp(-|x-c|^2 / (2 sigma^2)) with uniform centres, plus U(0, 0.05).
* dO ~ N(0, 1) in bf16 (training step only).

Parameters come from numpy's PCG64 (identical on every machine); the bulk
noise comes from torch's generator on the target device.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Tuple

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    W: int
    heads: int
    head_dim: int
    top_k: int
    top_p: float
    max_frac: float = 0.0            # 0 = no per-row cap
    fixed_shape: Tuple[int, int, int] = (0, 0, 0)
    planted: int = 0                 # number of planted high-variance zones
    blobs: int = 1
    blob_sigma: float = 3.0
    backward: bool = False
    batch: int = 1
    planted_amp: float = 2.0

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def zones(self) -> int:
        return self.N // 512


WORKLOADS = {
    w.name: w
    for w in [
        # 4 zones, fixed 4x4x4 blocks (32 blocks), forward only.
        Workload("tiny_8x16x16", 8, 16, 16, 2, 64, top_k=2, top_p=0.9,
                 fixed_shape=(4, 4, 4), planted=0, blobs=1, blob_sigma=3.0),
        # 32 zones, full dynamic shape selection, forward only.
        Workload("dynamic_16x32x32", 16, 32, 32, 8, 128, top_k=8, top_p=0.9,
                 planted=8, blobs=3, blob_sigma=4.0),
        # 720p-like latent: 180 zones, 5% planted, cap 12.5% of key blocks.
        Workload("latent720p_24x48x80", 24, 48, 80, 24, 128, top_k=16, top_p=0.95,
                 max_frac=0.125, planted=9, blobs=4, blob_sigma=4.0),
        # 2K-like latent: 720 zones, 5% planted, cap 6.25% of key blocks.
        Workload("latent2k_24x96x160", 24, 96, 160, 24, 128, top_k=32, top_p=0.95,
                 max_frac=0.0625, planted=36, blobs=8, blob_sigma=4.0),
        # 2K-like training step: the 2K latent plus dO, forward then backward.
        Workload("latent2k_train_24x96x160", 24, 96, 160, 24, 128, top_k=32, top_p=0.95,
                 max_frac=0.0625, planted=36, blobs=8, blob_sigma=4.0, backward=True),
    ]
}


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (small test cases)."""
    d = dict(w.__dict__)
    d.update(kw)
    return Workload(**d)


@dataclass
class Inputs:
    Q: torch.Tensor        # [B, N, heads, D] bf16
    K: torch.Tensor
    V: torch.Tensor
    a: torch.Tensor        # [B, T, H, W] fp32
    dO: Optional[torch.Tensor] = None
    planted_zones: list = field(default_factory=list)   # per sample: [(zone, axis)]


def _smooth_field(rs: np.random.Generator, T, H, W, C, device) -> torch.Tensor:
    f = rs.uniform(0.0, 3.0, size=(4, 3, C))
    phi = rs.uniform(0.0, 2.0 * math.pi, size=(4, C))
    out = torch.zeros(T, H, W, C, dtype=torch.float32, device=device)
    tt = torch.arange(T, dtype=torch.float64, device=device)[:, None] / T
    hh = torch.arange(H, dtype=torch.float64, device=device)[:, None] / H
    ww = torch.arange(W, dtype=torch.float64, device=device)[:, None] / W
    for s in range(4):
        ft = torch.as_tensor(f[s, 0], device=device)[None, :]
        fh = torch.as_tensor(f[s, 1], device=device)[None, :]
        fw = torch.as_tensor(f[s, 2], device=device)[None, :]
        ph = torch.as_tensor(phi[s], device=device)[None, :]
        at = (2.0 * math.pi * ft * tt + ph).float()          # [T, C]
        ah = (2.0 * math.pi * fh * hh).float()               # [H, C]
        aw = (2.0 * math.pi * fw * ww).float()               # [W, C]
        out += torch.sin(at[:, None, None, :] + ah[None, :, None, :] + aw[None, None, :, :])
    return out


def make_inputs(w: Workload, seed: int = 0, device="cpu", with_grad_output: Optional[bool] = None) -> Inputs:
    """Draw one batch of inputs for workload w on `device`."""
    device = torch.device(device)
    T, H, W, hN, D = w.T, w.H, w.W, w.heads, w.head_dim
    C = hN * D
    N = T * H * W
    MT, MH, MW = T // 8, H // 8, W // 8
    with_dO = w.backward if with_grad_output is None else with_grad_output
    Qs, Ks, Vs, As, dOs, planted_all = [], [], [], [], [], []
    for b in range(w.batch):
        rs = np.random.Generator(np.random.PCG64(seed + 7919 * b))
        gen = torch.Generator(device=device)
        gen.manual_seed(seed * 1000003 + 17 * b)
        tens = []
        for x in range(3):
            fld = _smooth_field(rs, T, H, W, C, device)
            fld += 0.5 * torch.randn(fld.shape, generator=gen, device=device, dtype=torch.float32)
            tens.append(fld)
        Qf, Kf, Vf = tens
        planted = []
        if w.planted > 0:
            zones = rs.choice(MT * MH * MW, size=w.planted, replace=False)
            axes = rs.integers(0, 3, size=w.planted)
            offs = rs.normal(0.0, w.planted_amp, size=(w.planted, 8, C)).astype(np.float32)
            for z, ax, off in zip(zones, axes, offs):
                zt, zh, zw = z // (MH * MW), (z // MW) % MH, z % MW
                o = torch.as_tensor(off, device=device)            # [8, C]
                view = Vf[zt * 8:(zt + 1) * 8, zh * 8:(zh + 1) * 8, zw * 8:(zw + 1) * 8, :]
                if ax == 0:
                    view += o[:, None, None, :]
                elif ax == 1:
                    view += o[None, :, None, :]
                else:
                    view += o[None, None, :, :]
                planted.append((int(z), int(ax)))
        centres = rs.uniform(0.0, 1.0, size=(w.blobs, 3)) * np.array([T, H, W])
        base = rs.uniform(0.0, 0.05, size=(T, H, W)).astype(np.float32)
        a = torch.as_tensor(base, device=device)
        tt = torch.arange(T, device=device, dtype=torch.float32)[:, None, None]
        hh = torch.arange(H, device=device, dtype=torch.float32)[None, :, None]
        ww = torch.arange(W, device=device, dtype=torch.float32)[None, None, :]
        for c in centres:
            d2 = (tt - float(c[0])) ** 2 + (hh - float(c[1])) ** 2 + (ww - float(c[2])) ** 2
            a += torch.exp(-d2 / (2.0 * w.blob_sigma ** 2))
        Qs.append(Qf.reshape(N, hN, D).to(torch.bfloat16))
        Ks.append(Kf.reshape(N, hN, D).to(torch.bfloat16))
        Vs.append(Vf.reshape(N, hN, D).to(torch.bfloat16))
        del Qf, Kf, Vf, tens
        As.append(a)
        planted_all.append(planted)
        if with_dO:
            g2 = torch.Generator(device=device)
            g2.manual_seed(seed * 1000003 + 17 * b + 1)
            dOs.append(torch.randn((N, hN, D), generator=g2, device=device,
                                   dtype=torch.float32).to(torch.bfloat16))
    return Inputs(torch.stack(Qs), torch.stack(Ks), torch.stack(Vs), torch.stack(As),
                  torch.stack(dOs) if with_dO else None, planted_all)


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a tensor as a host numpy uint16 array."""
    return x.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
