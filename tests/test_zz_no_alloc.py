"""sana_linattn_forward_noalloc: the forward pass for callers that cannot
allocate device memory (inside a graph capture, in allocator or framework hooks,
under a fixed memory budget).  It runs the same kernels as sana_linattn_forward
with the library's static device scratch in place of a workspace.

Collected last (file name) so that a stop-at-first-failure run has already run
every other test; it also passes alone in a fresh process."""
import pytest
import torch

from oracle import oracle as O
from parity import assert_close, to_dev
from relu_linear_attention_attn_b200.synthetic import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

ESCRATCH = -6


def _noalloc(lib, d, w, out):
    """Call the entry point through the C ABI."""
    s = torch.cuda.current_stream().cuda_stream
    gq = d["gq"].data_ptr() if d["gq"] is not None else None
    gk = d["gk"].data_ptr() if d["gk"] is not None else None
    dt = 0 if w.dtype == "bf16" else 1
    return lib.sana_linattn_forward_noalloc(d["q"].data_ptr(), d["k"].data_ptr(),
                                            d["v"].data_ptr(), gq, gk, out.data_ptr(), w.B, w.N,
                                            w.C, w.H, w.eps, dt, s)


def test_noalloc_matches_forward_on_two_calls_in_a_row(cuda_lib):
    """Calls in a row on different shapes, so each one meets the one before's
    leftovers in the shared scratch: the bf16 tensor-core path twice, then the
    fp32 CUDA-core path (which also uses the scratch's state region and a
    different split plan), then the one-launch short-sequence path (which needs
    no scratch).  The no-allocation call runs the same kernels with the same fixed
    plan as sana_linattn_forward, so the two agree bit for bit; each is also
    checked against the fp64 oracle."""
    lib = cuda_lib.load()
    cases = (WORKLOADS["2048px-b8-lognormal"].scaled(B=2, N=3000, seed=61),
             WORKLOADS["4096px-b2-overflow"].scaled(B=1, N=5000, seed=62),
             WORKLOADS["tiny-512px-f32"].scaled(seed=63),
             WORKLOADS["1024px-b1"].scaled(seed=64))
    for w in cases:
        x = make_inputs(w)
        d = to_dev(x)
        ref = cuda_lib.forward(d["q"], d["k"], d["v"], d["gq"], d["gk"], w.H, w.eps)
        out = torch.empty_like(d["q"])
        assert _noalloc(lib, d, w, out) == 0
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"noalloc differs from forward on {w.name}"
        assert_close(out, O.forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps),
                     w.dtype, f"noalloc vs oracle {w.name}")


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_lib):
    lib = cuda_lib.load()
    w = WORKLOADS["4096px-b2-overflow"].scaled(B=64, N=16384)            # needs far more than 16 MiB
    assert cuda_lib.workspace_bytes(w.B, w.N, w.C, w.H) > (16 << 20)
    small = WORKLOADS["1024px-b1"].scaled(N=8)
    d = to_dev(make_inputs(small))
    out = torch.empty_like(d["q"])
    assert _noalloc(lib, d, w, out) == ESCRATCH      # rejected before anything is launched
    assert b"16 MiB" in lib.sana_linattn_strerror(ESCRATCH)
