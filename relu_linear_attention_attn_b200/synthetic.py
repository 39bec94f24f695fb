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
WORKLOAD_LIST = (
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
WORKLOADS = {w.name: w for w in WORKLOAD_LIST}


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



# ----------------------------------------------------------------------------- Mix-FFN
@dataclasses.dataclass(frozen=True)
class MixFFNWorkload:
    """One Mix-FFN input configuration: tokens on a row-major (Hs, Ws) latent grid.

    Recipe (numpy ``default_rng(seed)``, float32 draws in this order, then the
    storage rounding): x ~ N(0, 1) (B, Hs*Ws, C) bf16; W1 ~ N(0, 1/C) (C, 2F) bf16;
    b1 ~ 0.1 N(0, 1) [2F]; wdw ~ N(0, 1/9) (2F, 3, 3); bdw ~ 0.1 N(0, 1) [2F];
    W2 ~ N(0, 1/F) (F, C) bf16; b2 ~ 0.1 N(0, 1) [C] (fp32 biases and depthwise
    weights; the biases are None when ``bias`` is False, after being drawn)."""
    name: str
    B: int
    Hs: int
    Ws: int
    C: int
    F: int
    gate: str           # sigmoid | silu
    bias: bool
    seed: int

    @property
    def N(self) -> int:
        return self.Hs * self.Ws

    @property
    def tokens(self) -> int:
        return self.B * self.N

    def scaled(self, **kw) -> "MixFFNWorkload":
        return dataclasses.replace(self, **kw)


# A tiny grid, SANA-1.6B's widths (C = 2240, F = 5600) on the 1024px latent grid
# (32 x 32 tokens), and a 2048px batch of 4 (64 x 64 tokens).
MIXFFN_WORKLOAD_LIST = (
    MixFFNWorkload("mixffn-tiny", B=1, Hs=8, Ws=8, C=64, F=96, gate="sigmoid", bias=True,
                   seed=31),
    MixFFNWorkload("mixffn-1024px-b1", B=1, Hs=32, Ws=32, C=2240, F=5600, gate="sigmoid",
                   bias=True, seed=32),
    MixFFNWorkload("mixffn-2048px-b4", B=4, Hs=64, Ws=64, C=2240, F=5600, gate="sigmoid",
                   bias=True, seed=33),
)
MIXFFN_WORKLOADS = {w.name: w for w in MIXFFN_WORKLOAD_LIST}


def make_mixffn_inputs(w: MixFFNWorkload) -> dict:
    """CPU tensors x, W1, b1, wdw, bdw, W2, b2 of one Mix-FFN workload."""
    rng = np.random.default_rng(w.seed)
    x = rng.standard_normal((w.B, w.N, w.C), dtype=np.float32)
    W1 = rng.standard_normal((w.C, 2 * w.F), dtype=np.float32) / np.float32(np.sqrt(w.C))
    b1 = 0.1 * rng.standard_normal(2 * w.F, dtype=np.float32)
    wdw = rng.standard_normal((2 * w.F, 3, 3), dtype=np.float32) / np.float32(3.0)
    bdw = 0.1 * rng.standard_normal(2 * w.F, dtype=np.float32)
    W2 = rng.standard_normal((w.F, w.C), dtype=np.float32) / np.float32(np.sqrt(w.F))
    b2 = 0.1 * rng.standard_normal(w.C, dtype=np.float32)
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return dict(x=_store(x, "bf16"), W1=_store(W1, "bf16"), W2=_store(W2, "bf16"),
                wdw=f32(wdw), b1=f32(b1) if w.bias else None, bdw=f32(bdw) if w.bias else None,
                b2=f32(b2) if w.bias else None)


def make_gemm_inputs(M: int, K: int, Nc: int, seed: int, bias: bool = True) -> dict:
    """A ~ N(0, 1) (M, K) bf16, W ~ N(0, 1/K) (K, Nc) bf16, bias ~ 0.1 N(0, 1) fp32."""
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((M, K), dtype=np.float32)
    W = rng.standard_normal((K, Nc), dtype=np.float32) / np.float32(np.sqrt(K))
    b = 0.1 * rng.standard_normal(Nc, dtype=np.float32)
    return dict(A=_store(A, "bf16"), W=_store(W, "bf16"),
                bias=torch.from_numpy(b) if bias else None)


def make_dwconv_inputs(B: int, Hs: int, Ws: int, F: int, seed: int, bias: bool = True) -> dict:
    """u ~ N(0, 1) (B, Hs*Ws, 2F) bf16, wdw ~ N(0, 1/9) (2F, 3, 3), bdw ~ 0.1 N(0, 1)."""
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((B, Hs * Ws, 2 * F), dtype=np.float32)
    wdw = rng.standard_normal((2 * F, 3, 3), dtype=np.float32) / np.float32(3.0)
    bdw = 0.1 * rng.standard_normal(2 * F, dtype=np.float32)
    return dict(u=_store(u, "bf16"), wdw=torch.from_numpy(wdw),
                bdw=torch.from_numpy(bdw) if bias else None)
