"""Seeded synthetic inputs shaped like SANA latents.

This module only draws random numbers and rounds them to the storage dtype; it
holds none of the attention arithmetic.  The tests hand the very same tensors to
the CUDA library and to the fp64 oracle.

Token counts follow the DC-AE F32 autoencoder (32x spatial compression): an
image of side ``res`` gives N = (res / 32)^2 latent tokens, so 512px -> 256,
1024px -> 1024, 2048px -> 4096, 4096px -> 16384 ("Sana: Efficient
High-Resolution Image Synthesis with Linear Diffusion Transformers", section 1,
AE-F32C32P1).  The channel width C = 2240 is SANA-1.6B / 4.8B's ("SANA 1.5 ...",
section "Model architecture"), split here into H = 70 heads of D = 32.

Recipes (numpy ``default_rng(seed)``; draws happen in the order listed, in
float32, then are rounded once to the storage dtype, round-to-nearest-even):

* ``gaussian``     q, k, v ~ N(0, 1); gains g_q, g_k as ``gains`` says.
* ``lognormal``    q = z_q * s_q, k = z_k * s_k with z ~ N(0, 1) and a per-token
                   scale s ~ LogNormal(0, 1), drawn independently for q and k and
                   shared by all C channels of a token; v ~ N(0, 1).
* ``overflow``     q, v ~ N(0, 1); k ~ 100 * N(0, 1); the norm is off (no gains).
* ``fused``        x ~ N(0, 1) of shape (B, N, C); Wqkv ~ N(0, 0.02^2) of shape
                   (C, 3C); gains 1 + 0.1 * N(0, 1).

``gains``: ``"ones"`` (g = 1), ``"random"`` (g = 1 + 0.1 * N(0, 1) per channel,
length C, independent for q and k) or ``"off"`` (no norm: both gains None).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One named input configuration."""
    name: str
    B: int
    N: int
    C: int
    H: int
    dtype: str          # "bf16" or "f32": storage and output dtype
    recipe: str         # gaussian | lognormal | overflow | fused
    gains: str          # ones | random | off
    eps: float
    seed: int

    @property
    def D(self) -> int:
        return self.C // self.H

    @property
    def tokens(self) -> int:
        return self.B * self.N

    def scaled(self, **kw) -> "Workload":
        """Same recipe with some sizes changed (for small parity cases)."""
        return dataclasses.replace(self, **kw)


# The workloads: a tiny Eq. (1) check, then SANA latents at 1024px, a 2048px
# batch, a 4K overflow stress with the norm off, the fused path, and the fused
# path with a W8A8 prologue (same recipe; x and Wqkv are quantised by the op).
CONFIGS = (
    Workload("tiny-512px-f32", B=1, N=256, C=64, H=2, dtype="f32", recipe="gaussian",
             gains="ones", eps=1e-6, seed=0),
    Workload("1024px-b1", B=1, N=1024, C=2240, H=70, dtype="bf16", recipe="gaussian",
             gains="random", eps=1e-6, seed=1),
    Workload("2048px-b8-lognormal", B=8, N=4096, C=2240, H=70, dtype="bf16",
             recipe="lognormal", gains="ones", eps=1e-6, seed=2),
    Workload("4096px-b2-overflow", B=2, N=16384, C=2240, H=70, dtype="bf16",
             recipe="overflow", gains="off", eps=1e-6, seed=3),
    Workload("fused-2048px-b4", B=4, N=4096, C=2240, H=70, dtype="bf16", recipe="fused",
             gains="random", eps=1e-6, seed=4),
    Workload("w8a8-2048px-b4", B=4, N=4096, C=2240, H=70, dtype="bf16", recipe="fused",
             gains="random", eps=1e-6, seed=5),
)


def _store(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(f"unknown dtype {dtype}")


def _gains(rng: np.random.Generator, C: int, mode: str):
    if mode == "off":
        return None, None
    if mode == "ones":
        return (torch.ones(C, dtype=torch.float32), torch.ones(C, dtype=torch.float32))
    if mode == "random":
        gq = 1.0 + 0.1 * rng.standard_normal(C, dtype=np.float32)
        gk = 1.0 + 0.1 * rng.standard_normal(C, dtype=np.float32)
        return torch.from_numpy(gq.astype(np.float32)), torch.from_numpy(gk.astype(np.float32))
    raise ValueError(f"unknown gains mode {mode}")


def make_inputs(w: Workload) -> dict:
    """CPU tensors for one workload.

    Unfused recipes return q, k, v (B, N, C) in the storage dtype and gq, gk
    (float32 [C] or None).  The fused recipe returns x (B, N, C), W (C, 3C) and
    gq, gk.  ``eps`` is included for convenience."""
    rng = np.random.default_rng(w.seed)
    shape = (w.B, w.N, w.C)
    if w.recipe == "fused":
        x = rng.standard_normal(shape, dtype=np.float32)
        W = 0.02 * rng.standard_normal((w.C, 3 * w.C), dtype=np.float32)
        gq, gk = _gains(rng, w.C, w.gains)
        return dict(x=_store(x, w.dtype), W=_store(W, w.dtype), gq=gq, gk=gk, eps=w.eps)
    if w.recipe == "gaussian":
        q = rng.standard_normal(shape, dtype=np.float32)
        k = rng.standard_normal(shape, dtype=np.float32)
        v = rng.standard_normal(shape, dtype=np.float32)
    elif w.recipe == "lognormal":
        zq = rng.standard_normal(shape, dtype=np.float32)
        sq = rng.lognormal(0.0, 1.0, size=(w.B, w.N)).astype(np.float32)
        zk = rng.standard_normal(shape, dtype=np.float32)
        sk = rng.lognormal(0.0, 1.0, size=(w.B, w.N)).astype(np.float32)
        v = rng.standard_normal(shape, dtype=np.float32)
        q = zq * sq[:, :, None]
        k = zk * sk[:, :, None]
    elif w.recipe == "overflow":
        q = rng.standard_normal(shape, dtype=np.float32)
        k = 100.0 * rng.standard_normal(shape, dtype=np.float32)
        v = rng.standard_normal(shape, dtype=np.float32)
    else:
        raise ValueError(f"unknown recipe {w.recipe}")
    gq, gk = _gains(rng, w.C, w.gains)
    return dict(q=_store(q, w.dtype), k=_store(k, w.dtype), v=_store(v, w.dtype),
                gq=gq, gk=gk, eps=w.eps)


def make_output_grad(w: Workload, seed_offset: int = 100) -> torch.Tensor:
    """dL/dO for backward tests and timing: N(0, 1) of shape (B, N, C) in the
    workload's storage dtype, from default_rng(w.seed + seed_offset)."""
    rng = np.random.default_rng(w.seed + seed_offset)
    return _store(rng.standard_normal((w.B, w.N, w.C), dtype=np.float32), w.dtype)

