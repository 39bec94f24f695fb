"""Parity of the Mix-FFN kernels (through the C ABI) with the fp64 oracle
("Sana: Efficient High-Resolution Image Synthesis with Linear Diffusion
Transformers", sections 2.2-2.3).

Tolerances, from the arithmetic:
* gemm_bias and dwconv_glu write bf16 results of fp32 sums, so each element is
  the exact value rounded once to bf16 (relative error <= 2^-8, the unit
  roundoff of its 8 significant bits) plus fp32
  summation error: |got - ref| <= 2^-8 |ref| + 1e-5 max|ref| + 1e-6.
* mixffn_forward stores U and Hg in bf16 between the kernels (the oracle keeps
  fp64 throughout); each rounding is <= 2^-8 relative and the project sums F
  terms of random sign, so the normwise error is about 2^-8: rel-L2 <=
  1.5e-2, max |got - ref| <= 0.1 max|ref|.  Its stages are also checked to chain
  exactly: the one-call forward equals the three stage calls bit for bit."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from parity import to_np
from relu_linear_attention_attn_b200.synthetic import (MIXFFN_WORKLOADS, make_dwconv_inputs,
                                                       make_gemm_inputs, make_mixffn_inputs)

pytestmark = pytest.mark.gpu

U8 = 2.0 ** -8                      # unit roundoff of bf16 (8 significant bits)


def _elementwise(got, ref, what):
    g = to_np(got).astype(np.float64)
    assert np.isfinite(g).all(), f"{what}: non-finite"
    tol = U8 * np.abs(ref) + 1e-5 * np.abs(ref).max() + 1e-6
    bad = np.abs(g - ref) > tol
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} elements out of tolerance, "
                           f"worst {np.abs(g - ref).max():.3e}")


def _normwise(got, ref, what):
    g = to_np(got).astype(np.float64).reshape(ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite"
    rel = np.linalg.norm(g - ref) / np.linalg.norm(ref)
    mx = np.abs(g - ref).max() / np.abs(ref).max()
    assert rel <= 1.5e-2 and mx <= 0.1, f"{what}: rel-L2 {rel:.3e}, max {mx:.3e}"


@pytest.mark.parametrize("M,K,Nc,bias", [(100, 64, 192, True), (300, 200, 520, True),
                                         (257, 72, 256, False), (1024, 2240, 11200, True),
                                         (1024, 5600, 2240, True), (4100, 256, 1032, True)],
                         ids=lambda v: str(v))
def test_gemm_bias_parity(cuda_lib, M, K, Nc, bias):
    x = make_gemm_inputs(M, K, Nc, seed=M + K + Nc, bias=bias)
    got = cuda_lib.gemm_bias(x["A"].cuda(), x["W"].cuda(),
                             None if x["bias"] is None else x["bias"].cuda())
    torch.cuda.synchronize()
    ref = O.linear(x["A"].float().numpy(), x["W"].float().numpy(),
                   None if x["bias"] is None else x["bias"].numpy())
    _elementwise(got, ref, f"gemm {M}x{K}x{Nc}")


@pytest.mark.parametrize("B,Hs,Ws,F,gate,bias", [
    (1, 8, 8, 96, "sigmoid", True),
    (2, 5, 37, 40, "sigmoid", True),          # ragged strip and channel chunk
    (1, 1, 9, 32, "silu", True),              # one grid row
    (1, 11, 1, 48, "sigmoid", False),         # one grid column
    (1, 20, 33, 64, "silu", False),           # the row ring wraps twice
    (1, 32, 32, 5600, "sigmoid", True),       # SANA width on the 1024px grid
    (2, 32, 32, 5600, "silu", True),
], ids=lambda v: str(v))
def test_dwconv_glu_parity(cuda_lib, B, Hs, Ws, F, gate, bias):
    x = make_dwconv_inputs(B, Hs, Ws, F, seed=7 * Hs + Ws + F, bias=bias)
    got = cuda_lib.mixffn_dwconv_glu(x["u"].cuda(), x["wdw"].cuda(),
                                     None if x["bdw"] is None else x["bdw"].cuda(), Hs, Ws, gate)
    torch.cuda.synchronize()
    ref = O.dwconv_glu(x["u"].float().numpy(), x["wdw"].numpy(),
                       None if x["bdw"] is None else x["bdw"].numpy(), Hs, Ws, gate)
    _elementwise(got, ref, f"dwconv+glu B{B} {Hs}x{Ws} F{F} {gate}")


def _dev(x):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def _oracle_args(x):
    f = lambda t: None if t is None else t.float().numpy()
    return (f(x["x"]), f(x["W1"]), f(x["b1"]), f(x["wdw"]), f(x["bdw"]), f(x["W2"]), f(x["b2"]))


@pytest.mark.parametrize("w", [MIXFFN_WORKLOADS["mixffn-tiny"], MIXFFN_WORKLOADS["mixffn-tiny"].scaled(Hs=7, Ws=13, gate="silu",
                                                                           bias=False, seed=40),
                               MIXFFN_WORKLOADS["mixffn-1024px-b1"]], ids=lambda w: f"{w.name}-{w.Hs}x{w.Ws}-{w.gate}")
def test_mixffn_forward_parity(cuda_lib, w):
    x = make_mixffn_inputs(w)
    d = _dev(x)
    got = cuda_lib.mixffn_forward(d["x"], d["W1"], d["b1"], d["wdw"], d["bdw"], d["W2"], d["b2"],
                                  w.Hs, w.Ws, w.gate)
    # the same three stages called one by one
    u = cuda_lib.gemm_bias(d["x"], d["W1"], d["b1"])
    h = cuda_lib.mixffn_dwconv_glu(u, d["wdw"], d["bdw"], w.Hs, w.Ws, w.gate)
    y = cuda_lib.gemm_bias(h, d["W2"], d["b2"])
    torch.cuda.synchronize()
    assert torch.equal(got, y), "one-call forward differs from its stages"
    ref = O.mixffn_forward(*_oracle_args(x), w.Hs, w.Ws, w.gate)
    _normwise(got, ref, w.name)


def test_mixffn_full_size_sampled(cuda_lib):
    """The 2048px batch of 4, in the launch configuration the benchmark times,
    on tokens at the grid's corners, edges and interior of every batch."""
    w = MIXFFN_WORKLOADS["mixffn-2048px-b4"]
    x = make_mixffn_inputs(w)
    d = _dev(x)
    got = cuda_lib.mixffn_forward(d["x"], d["W1"], d["b1"], d["wdw"], d["bdw"], d["W2"], d["b2"],
                                  w.Hs, w.Ws, w.gate)
    torch.cuda.synchronize()
    cells = [(0, 0), (0, w.Ws - 1), (w.Hs - 1, 0), (w.Hs - 1, w.Ws - 1), (0, 17), (31, 0),
             (w.Hs - 1, 40), (33, 31), (32, 32)]
    tok = [b * w.N + yy * w.Ws + xx for b in range(w.B) for yy, xx in cells]
    ref = O.mixffn_forward(*_oracle_args(x), w.Hs, w.Ws, w.gate, tokens=tok)
    _normwise(got.reshape(-1, w.C)[tok].cpu(), ref, f"{w.name} sampled")


def test_mixffn_is_deterministic(cuda_lib):
    w = MIXFFN_WORKLOADS["mixffn-1024px-b1"]
    d = _dev(make_mixffn_inputs(w))
    a = cuda_lib.mixffn_forward(d["x"], d["W1"], d["b1"], d["wdw"], d["bdw"], d["W2"], d["b2"],
                                w.Hs, w.Ws, w.gate)
    b = cuda_lib.mixffn_forward(d["x"], d["W1"], d["b1"], d["wdw"], d["bdw"], d["W2"], d["b2"],
                                w.Hs, w.Ws, w.gate)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_row_shards_reassemble_the_unsharded_forward(cuda_lib):
    """Three row shards of the 1024px grid (the halo rows copied between them as the
    ranks' exchange would) give the one-call forward bit for bit."""
    from relu_linear_attention_attn_b200 import sharding
    w = MIXFFN_WORKLOADS["mixffn-1024px-b1"].scaled(Hs=17, seed=41)            # ragged: 5, 6, 6 rows
    d = _dev(make_mixffn_inputs(w))
    ref = cuda_lib.mixffn_forward(d["x"], d["W1"], d["b1"], d["wdw"], d["bdw"], d["W2"], d["b2"],
                                  w.Hs, w.Ws, w.gate)
    world = 3
    shards = [sharding.row_shard(w.Hs, r, world) for r in range(world)]
    Us = [sharding.mixffn_shard_expand(d["x"][:, y0 * w.Ws:(y0 + c) * w.Ws].contiguous(), d["W1"],
                                       d["b1"], w.Ws) for y0, c in shards]
    parts = []
    for r, (y0, c) in enumerate(shards):
        zero = torch.zeros_like(Us[r][:, 0])
        top = Us[r - 1][:, -2] if r > 0 else zero              # the neighbour's last own row
        bottom = Us[r + 1][:, 1] if r < world - 1 else zero    # and its first
        parts.append(sharding.mixffn_shard_finish(Us[r], top, bottom, d["wdw"], d["bdw"], d["W2"],
                                                  d["b2"], w.Ws, w.gate))
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts, dim=1), ref)
