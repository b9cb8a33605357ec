"""Seeded synthetic inputs for the Lighthouse Attention layer.

This module only draws random numbers; it holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle may take their inputs
from it.

Recipe (the pages' single-layer benchmark shape, "Long Context Pre-Training
with Lighthouse Attention", Sec. 6.2: bf16, B=1, H=8, d=128, L=3, p=4; the
pages do not describe the data, so the values are synthetic):

* Q, K, V ~ N(0, 1) i.i.d., drawn with numpy's PCG64 from ``seed``.
* Every (b, t) token row of each tensor (all H*d values) is multiplied by its
  own lognormal(mean 0, sigma 0.5) draw, so per-token norms spread over a
  few octaves the way projected activations do.
* ``n_heavy`` token positions per batch row (drawn without replacement and
  shared by Q, K and V) are multiplied by ``heavy_scale``.
* The result is rounded to bf16 (round-to-nearest-even).
* The output gradient dO ~ N(0, 1) comes from ``seed + 100``.
"""
from __future__ import annotations

import numpy as np
import torch

__all__ = ["make_qkv", "make_dout", "WORKLOADS", "Workload"]


class Workload(dict):
    """Shape of one layer call: B, N, H, d, L, p, k (a plain dict)."""

    @property
    def name(self) -> str:
        return self["name"]


def _w(name, B, H, d, N, L, p, k, **extra):
    return Workload(name=name, B=B, H=H, d=d, N=N, L=L, p=p, k=k, **extra)


# Workloads with the pages' benchmark shapes.  Index = seed.
WORKLOADS = [
    _w("tiny_n4k_l3_p4_k64_d64", 1, 2, 64, 4096, 3, 4, 64, dtype="f32"),
    _w("n64k_l3_p4_k1024", 1, 8, 128, 65536, 3, 4, 1024),
    _w("b2_n128k_l3_p4_k2048", 2, 8, 128, 131072, 3, 4, 2048),
    _w("n512k_l3_p4_k4096", 1, 8, 128, 524288, 3, 4, 4096),
    _w("n1m_l4_p4_k4096", 1, 8, 128, 1048576, 4, 4, 4096),
]


def _draw(rng: np.random.Generator, B: int, N: int, H: int, d: int,
          heavy: np.ndarray, heavy_scale: float) -> np.ndarray:
    x = rng.standard_normal((B, N, H * d), dtype=np.float32)
    tok = rng.lognormal(0.0, 0.5, size=(B, N, 1)).astype(np.float32)
    x *= tok
    for b in range(B):
        x[b, heavy[b]] *= np.float32(heavy_scale)
    return x.reshape(B, N, H, d)


def make_qkv(B: int, N: int, H: int, d: int, seed: int, n_heavy: int = 64,
             heavy_scale: float = 4.0, as_fp32: bool = False):
    """Return (q, k, v) as CPU torch tensors of shape [B, N, H, d].

    bf16 by default; ``as_fp32=True`` returns the float32 draws before the
    bf16 rounding (used by the oracle's own self-checks).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    n_heavy = min(n_heavy, N)
    heavy = np.stack([rng.choice(N, size=n_heavy, replace=False) for _ in range(B)])
    out = []
    for _ in range(3):
        x = torch.from_numpy(_draw(rng, B, N, H, d, heavy, heavy_scale))
        out.append(x if as_fp32 else x.to(torch.bfloat16))
    return tuple(out)


def make_dout(B: int, N: int, H: int, d: int, seed: int) -> torch.Tensor:
    """dO ~ N(0, 1) as a bf16 CPU tensor [B, N, H, d], drawn from seed + 100."""
    rng = np.random.Generator(np.random.PCG64(seed + 100))
    x = rng.standard_normal((B, N, H, d), dtype=np.float32)
    return torch.from_numpy(x).to(torch.bfloat16)
