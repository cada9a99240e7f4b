"""Spatially correlated synthetic Q/K/V standing in for video-DiT activations.

The pages measure on real Wan2.1 / CogVideoX activations (JourneyDB prompts,
VBench suites) that are not available; these seeded fields stand in for them.
Recipe:

  F[t, y, x] = sum_m a_m cos(2 pi (f_t t / T + f_y y / H + f_x x / W) + phi_m)
      a_m ~ N(0, 1/M_m) in R^d, integer frequencies f uniform in [0, 3],
      phi_m ~ U[0, 2 pi), independent modes for each (batch, head);
  Q = s (F + sigma eps_q),  K = s (F + sigma eps_k),  eps ~ N(0, 1);
  s chosen so that q.k / sqrt(d) over 65,536 random (b, h, i, j) pairs has the
  target standard deviation (logits scale as s^2);
  V ~ N(0, 1) and dO ~ N(0, 1).
Every tensor is drawn in float32/float64 with NumPy PCG64 streams spawned from the
workload seed, then rounded to bf16 (round-to-nearest-even).  Layout is the
model's raster layout [B, N, H, d] with token n = (t * H + y) * W + x.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int          # attention heads
    d: int          # head dim
    T: int          # latent frames
    Hg: int         # latent height
    W: int          # latent width
    tau: float
    modes: int
    noise: float
    logit_std: float
    seed: int
    global_window: int = 0
    backward: bool = False

    @property
    def N(self) -> int:
        return self.T * self.Hg * self.W

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads of the ASA benchmark (shapes of the models the pages use).
WORKLOADS = {
    "tiny": Workload("tiny-4x16x16", 1, 2, 64, 4, 16, 16, 0.90, 8, 0.3, 3.0, 1235),
    "wan2.1-1.3b": Workload("wan2.1-1.3b-21x30x52", 1, 12, 128, 21, 30, 52, 0.95, 16, 0.3, 3.0, 1236),
    "cogvideox-5b": Workload("cogvideox-5b-13x30x45", 1, 48, 64, 13, 30, 45, 0.90, 12, 0.5, 2.5, 1237),
    "wan2.1-1.3b-asag": Workload("wan2.1-1.3b-asag-21x30x52", 1, 12, 128, 21, 30, 52, 0.90, 8, 0.3, 3.0,
                                 1238, global_window=64),
    "wan-14b-720p": Workload("wan-14b-720p-21x45x80", 1, 40, 128, 21, 45, 80, 0.95, 16, 0.3, 3.0, 1239,
                             backward=True),
}


def _fields(wl: Workload, rng: np.random.Generator) -> np.ndarray:
    """F as float32 [B, N, H, d]."""
    B, H, d, Mm = wl.B, wl.H, wl.d, wl.modes
    amp = rng.normal(0.0, 1.0 / math.sqrt(Mm), size=(B, H, Mm, d))
    freq = rng.integers(0, 4, size=(B, H, Mm, 3))
    phase = rng.uniform(0.0, 2.0 * math.pi, size=(B, H, Mm))
    t = np.arange(wl.T, dtype=np.float64)[:, None, None] / wl.T
    y = np.arange(wl.Hg, dtype=np.float64)[None, :, None] / wl.Hg
    x = np.arange(wl.W, dtype=np.float64)[None, None, :] / wl.W
    F = np.empty((B, wl.N, H, d), dtype=np.float32)
    for b in range(B):
        for h in range(H):
            arg = np.empty((wl.N, Mm), dtype=np.float64)
            for m in range(Mm):
                ft, fy, fx = freq[b, h, m]
                arg[:, m] = (2.0 * math.pi * (ft * t + fy * y + fx * x) + phase[b, h, m]).reshape(-1)
            F[b, :, h, :] = np.cos(arg) @ amp[b, h]
    return F


def to_bf16_tensor(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def make_inputs(wl: Workload, with_dout: bool | None = None) -> dict:
    """Seeded bf16 CPU tensors q, k, v (and dout) in raster layout [B, N, H, d]."""
    if with_dout is None:
        with_dout = wl.backward
    seqs = np.random.SeedSequence(wl.seed).spawn(6)
    rng = [np.random.Generator(np.random.PCG64(s)) for s in seqs]
    F = _fields(wl, rng[0])
    shape = F.shape
    qn = F + np.float32(wl.noise) * rng[1].standard_normal(shape, dtype=np.float32)
    kn = F + np.float32(wl.noise) * rng[2].standard_normal(shape, dtype=np.float32)
    del F
    # scale so that the unit-scale logits q.k/sqrt(d) reach the target std
    npairs = 65536
    bi = rng[5].integers(0, wl.B, npairs)
    hi = rng[5].integers(0, wl.H, npairs)
    ii = rng[5].integers(0, wl.N, npairs)
    jj = rng[5].integers(0, wl.N, npairs)
    logits = np.einsum("pc,pc->p", qn[bi, ii, hi].astype(np.float64),
                       kn[bi, jj, hi].astype(np.float64)) / math.sqrt(wl.d)
    s = math.sqrt(wl.logit_std / float(logits.std()))
    out = {
        "q": to_bf16_tensor(qn * np.float32(s)),
        "k": to_bf16_tensor(kn * np.float32(s)),
    }
    del qn, kn
    out["v"] = to_bf16_tensor(rng[3].standard_normal(shape, dtype=np.float32))
    if with_dout:
        out["dout"] = to_bf16_tensor(rng[4].standard_normal(shape, dtype=np.float32))
    out["scale"] = s
    return out
