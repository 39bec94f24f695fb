"""Parity of the prefix (causal) form (through the C ABI) with the fp64 oracle.

Small cases compare every element; the 2048px and 4096px workloads compare the
oracle's full result.  The last token's output must also agree with the
non-causal path, whose prefix is the whole sequence."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from parity import assert_close, to_dev
from relu_linear_attention_attn_b200.synthetic import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def run(lib, d, w):
    out = lib.forward_causal(d["q"], d["k"], d["v"], d["gq"], d["gk"], w.H, w.eps)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("w", [WORKLOADS["tiny-512px-f32"], WORKLOADS["tiny-512px-f32"].scaled(N=300, seed=90),
                               WORKLOADS["1024px-b1"].scaled(N=1, seed=91),
                               WORKLOADS["1024px-b1"].scaled(N=333, seed=92),
                               WORKLOADS["1024px-b1"].scaled(B=2, N=129, gains="off", seed=93),
                               WORKLOADS["2048px-b8-lognormal"].scaled(B=1, N=1000, seed=94),
                               WORKLOADS["1024px-b1"].scaled(N=129, C=160, H=5, seed=96),
                               WORKLOADS["4096px-b2-overflow"].scaled(B=3, N=640, seed=97),
                               WORKLOADS["1024px-b1"].scaled(B=2, N=2049, seed=98),
                               # chunk edges of the tensor-core form (128-token chunks):
                               # one chunk exactly, one short of it, two and a token,
                               # one head, and more rows than CTAs
                               WORKLOADS["1024px-b1"].scaled(N=128, C=64, H=2, seed=100),
                               WORKLOADS["1024px-b1"].scaled(N=127, C=96, H=3, seed=101),
                               WORKLOADS["1024px-b1"].scaled(B=2, N=257, C=32, H=1, seed=102),
                               WORKLOADS["1024px-b1"].scaled(B=5, N=512, C=448, H=14, seed=103)],
                         ids=lambda w: f"{w.dtype}-B{w.B}-N{w.N}-{w.gains}")
def test_causal_small_full_parity(cuda_lib, w):
    x = make_inputs(w)
    out = run(cuda_lib, to_dev(x), w)
    ref = O.causal_forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps)
    assert_close(out, ref, w.dtype, w.name)


@pytest.mark.parametrize("name", ["2048px-b8-lognormal", "4096px-b2-overflow"])
def test_causal_full_size_parity(cuda_lib, name):
    w = WORKLOADS[name]
    x = make_inputs(w)
    out = run(cuda_lib, to_dev(x), w)
    ref = O.causal_forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps)
    assert_close(out, ref, w.dtype, w.name)


def test_causal_last_token_matches_noncausal_and_is_deterministic(cuda_lib):
    w = WORKLOADS["1024px-b1"].scaled(B=2, N=777, seed=95)
    d = to_dev(make_inputs(w))
    a = run(cuda_lib, d, w)
    b = run(cuda_lib, d, w)
    assert torch.equal(a, b)
    full = cuda_lib.forward(d["q"], d["k"], d["v"], d["gq"], d["gk"], w.H, w.eps)
    torch.cuda.synchronize()
    diff = (a[:, -1].float() - full[:, -1].float()).abs().max().item()
    assert diff < 2e-2, diff


def test_causal_gains_without_16_byte_alignment(cuda_lib):
    """Gains that are 4- but not 16-byte aligned take the CUDA-core kernels (the
    tensor-core path reads them as 16-byte vectors); the result is the same."""
    w = WORKLOADS["1024px-b1"].scaled(N=300, seed=99)
    x = make_inputs(w)
    d = to_dev(x)
    gq = torch.empty(w.C + 1, dtype=torch.float32, device="cuda")[1:]
    gk = torch.empty(w.C + 1, dtype=torch.float32, device="cuda")[1:]
    gq.copy_(d["gq"])
    gk.copy_(d["gk"])
    assert gq.data_ptr() % 16 != 0
    out = cuda_lib.forward_causal(d["q"], d["k"], d["v"], gq, gk, w.H, w.eps)
    torch.cuda.synchronize()
    ref = O.causal_forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps)
    assert_close(out, ref, w.dtype, "causal, unaligned gains")
