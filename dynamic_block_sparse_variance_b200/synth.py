"""Seeded synthetic workloads: token grids, Q/K/V fields, audio norms, dO.

This module only draws inputs.  It holds none of the method's arithmetic (no
pooling, variance, shapes, selection or attention), so both the CUDA path and
the fp64 oracle can be fed from it.  It uses torch and runs on any device; a
given seed gives the same tensors on the CPU every time (the GPU's random
stream differs from the CPU's, so parity tests draw on the CPU and upload).

Field recipe (per tensor X in {Q, K, V}, head h, channel c):
  X(t, y, x) = gain_X * sum_axis A[zone, axis] * f_{X,h,c,axis}(coord_axis) + 0.1 N(0,1)
  f(u) = sum of 3 cosines, frequency U[1/64, 1/16] cycles/token, phase U[0, 2pi),
         weight N(0, 1/3)                     -- a per-axis low-frequency field
  A[zone, axis] ~ U[0.1, 2] per zone and axis -- anisotropic per-zone amplitude
With ``mix`` the zones are dealt into thirds: static (A = 0.1 on every axis),
temporal (A_T ~ U[1,2], A_H = A_W = 0.1) and spatial (A_T = 0.1,
A_H, A_W ~ U[1,2]), so all three block volumes occur.
Audio norms: a sum of Gaussian bumps exp(-1/2 sum_axis ((coord - c)/s)^2),
divided by its maximum so that max a = 1.
"""

from __future__ import annotations

import dataclasses
import math

import torch

SEED_Q, SEED_K, SEED_V, SEED_AUDIO, SEED_DOUT, SEED_ZONES = 1, 2, 3, 4, 5, 6


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    W: int
    heads: int
    head_dim: int
    dtype: str            # "f32" or "bf16": storage type of Q/K/V/dO
    top_k: int
    top_p: float
    bumps: int            # audio bumps
    bump_width: float     # bump std as a fraction of each axis length
    mix: bool             # static / temporal / spatial zone thirds
    qk_gain: float        # gain on Q and K (sets how peaked the block scores are)
    index: int            # seed offset: seeds are base + 100 * index
    backward: bool = True

    @property
    def N(self):
        return self.T * self.H * self.W

    @property
    def zones(self):
        return self.N // 512


# The five workloads: token grid, heads x head_dim, storage type and the
# selection knobs k / p of each.  The Q/K gain sets how peaked the block
# scores are; it is calibrated once per grid so that the achieved block
# sparsity lands in the stated band (Small about 85%, 2K 90-95%) and the
# others near 90%.
WORKLOADS = {
    "tiny": Workload("tiny", 8, 16, 16, 2, 64, "f32", 2, 0.9, 2, 0.25, False, 1.0, 0),
    "small": Workload("small", 16, 48, 80, 24, 128, "bf16", 8, 0.9, 6, 0.08, False, 1.2, 1,
                      backward=False),
    "720p": Workload("720p", 24, 48, 80, 24, 128, "bf16", 16, 0.9, 6, 0.06, False, 1.4, 2),
    "1080p": Workload("1080p", 24, 72, 120, 24, 128, "bf16", 16, 0.95, 8, 0.05, True, 3.9, 3),
    "2k": Workload("2k", 64, 96, 160, 24, 128, "bf16", 32, 0.9, 12, 0.04, True, 3.7, 4),
}

# Smaller grids used only by the parity tests: several tiles per head, every
# block volume present, sizes the oracle finishes in seconds.
TEST_WORKLOADS = {
    "mix16": Workload("mix16", 16, 32, 32, 3, 128, "bf16", 4, 0.9, 3, 0.15, True, 1.0, 11),
    "aniso8": Workload("aniso8", 8, 24, 40, 2, 64, "bf16", 3, 0.8, 2, 0.2, False, 1.0, 12),
    # six zones, head_dim 128 (the tensor-core kernels), all three block volumes
    "smoke128": Workload("smoke128", 8, 16, 24, 2, 128, "bf16", 2, 0.9, 2, 0.2, True, 1.0, 13),
}


# The 720p grid with a third of the heads: inputs still larger than L2 (0.19 GB
# per tensor) but a whole layer's buffers within a few GB, the size used for
# profiler captures that replay each kernel many times.
PROFILE_WORKLOADS = {
    "720p-8h": Workload("720p-8h", 24, 48, 80, 8, 128, "bf16", 16, 0.9, 6, 0.06, False, 1.4, 2),
    # the 1080p grid with 4 heads and the 2K grid with 2 heads: the same
    # generator and knobs, so each head's selection density and working set
    # match the full grids' in distribution (heads are independent and the
    # attention kernels take them one after another), at a few GB per layer
    "1080p-4h": Workload("1080p-4h", 24, 72, 120, 4, 128, "bf16", 16, 0.95, 8, 0.05, True, 3.9, 3),
    "2k-2h": Workload("2k-2h", 64, 96, 160, 2, 128, "bf16", 32, 0.9, 12, 0.04, True, 3.7, 4),
}


def get_workload(name):
    for table in (WORKLOADS, TEST_WORKLOADS, PROFILE_WORKLOADS):
        if name in table:
            return table[name]
    raise KeyError(name)


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def zone_amplitudes(wl: Workload, device="cpu"):
    """A[zone, axis] in float32, [Z, 3]."""
    g = _gen(SEED_ZONES + 100 * wl.index, device)
    Z = wl.zones
    if not wl.mix:
        return 0.1 + 1.9 * torch.rand(Z, 3, generator=g, device=device)
    cls = torch.randperm(Z, generator=g, device=device) % 3
    hi = 1.0 + torch.rand(Z, 3, generator=g, device=device)
    A = torch.full((Z, 3), 0.1, device=device)
    A[cls == 1, 0] = hi[cls == 1, 0]
    A[cls == 2, 1] = hi[cls == 2, 1]
    A[cls == 2, 2] = hi[cls == 2, 2]
    return A


def _axis_fields(g, L, C, device):
    """f(u) for u in [0, L): [L, C] float32, sum of three random cosines."""
    freq = 1.0 / 64 + (1.0 / 16 - 1.0 / 64) * torch.rand(3, C, generator=g, device=device)
    phase = 2 * math.pi * torch.rand(3, C, generator=g, device=device)
    weight = torch.randn(3, C, generator=g, device=device) * math.sqrt(1.0 / 3.0)
    u = torch.arange(L, device=device, dtype=torch.float32)[:, None, None]
    return (weight * torch.cos(2 * math.pi * freq * u + phase)).sum(dim=1)


def field(wl: Workload, seed, gain, device="cpu", out_dtype=None):
    """One Q/K/V-like tensor [N, heads, head_dim] in the workload's storage type."""
    dtype = out_dtype or (torch.float32 if wl.dtype == "f32" else torch.bfloat16)
    g = _gen(seed + 100 * wl.index, device)
    C = wl.heads * wl.head_dim
    FT = _axis_fields(g, wl.T, C, device)
    FH = _axis_fields(g, wl.H, C, device)
    FW = _axis_fields(g, wl.W, C, device)
    A = zone_amplitudes(wl, device)
    ZY, ZX = wl.H // 8, wl.W // 8
    zy = torch.arange(wl.H, device=device) // 8
    zx = torch.arange(wl.W, device=device) // 8
    out = torch.empty(wl.N, C, dtype=dtype, device=device)
    plane = wl.H * wl.W
    for t in range(wl.T):
        zone = ((t // 8) * ZY + zy[:, None]) * ZX + zx[None, :]          # [H, W]
        a = A[zone.reshape(-1)]                                           # [HW, 3]
        x = (a[:, 0:1] * FT[t][None, :]
             + (a[:, 1:2] * FH.repeat_interleave(wl.W, dim=0))
             + (a[:, 2:3] * FW.repeat(wl.H, 1)))
        x = gain * x + 0.1 * torch.randn(plane, C, generator=g, device=device)
        out[t * plane:(t + 1) * plane] = x.to(dtype)
    return out.view(wl.N, wl.heads, wl.head_dim)


def audio_norms(wl: Workload, device="cpu"):
    """Cached audio-to-video norms a[N] in float32 with max 1 (None if no bumps)."""
    if wl.bumps == 0:
        return None
    g = _gen(SEED_AUDIO + 100 * wl.index, device)
    lens = torch.tensor([wl.T, wl.H, wl.W], dtype=torch.float32, device=device)
    centres = torch.rand(wl.bumps, 3, generator=g, device=device) * lens
    widths = wl.bump_width * lens * (0.5 + torch.rand(wl.bumps, 3, generator=g, device=device))
    t = torch.arange(wl.T, device=device, dtype=torch.float32)
    y = torch.arange(wl.H, device=device, dtype=torch.float32)
    x = torch.arange(wl.W, device=device, dtype=torch.float32)
    a = torch.zeros(wl.T, wl.H, wl.W, device=device)
    for b in range(wl.bumps):
        et = torch.exp(-0.5 * ((t - centres[b, 0]) / widths[b, 0]) ** 2)
        ey = torch.exp(-0.5 * ((y - centres[b, 1]) / widths[b, 1]) ** 2)
        ex = torch.exp(-0.5 * ((x - centres[b, 2]) / widths[b, 2]) ** 2)
        a += et[:, None, None] * ey[None, :, None] * ex[None, None, :]
    a = a / a.max()
    return a.reshape(-1).contiguous()


def make_inputs(wl: Workload, device="cpu", with_dout=None):
    """Q, K, V (natural layout [N, heads, d]), audio [N] and optionally dO."""
    out = dict(
        q=field(wl, SEED_Q, wl.qk_gain, device),
        k=field(wl, SEED_K, wl.qk_gain, device),
        v=field(wl, SEED_V, 1.0, device),
        audio=audio_norms(wl, device),
    )
    if with_dout if with_dout is not None else wl.backward:
        g = _gen(SEED_DOUT + 100 * wl.index, device)
        dt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
        out["dout"] = torch.randn(wl.N, wl.heads, wl.head_dim, generator=g, device=device).to(dt)
    return out
