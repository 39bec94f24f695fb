"""sana_linattn_forward_noalloc: the forward pass for callers that cannot
allocate device memory (inside a graph capture, in allocator or framework hooks,
under a fixed memory budget).  It runs the same kernels as sana_linattn_forward
with the library's static device scratch in place of a workspace.

Collected last (file name) so that a stop-at-first-failure run has already run
every other test; it also passes alone in a fresh process."""
import pytest
import torch

from parity import assert_close, to_dev
from relu_linear_attention_attn_b200.synthetic import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

ESCRATCH = -6


def _noalloc(lib, d, w, out):
    """Call the entry point through the C ABI."""
    s = torch.cuda.current_stream().cuda_stream
    gq = d["gq"].data_ptr() if d["gq"] is not None else None
    gk = d["gk"].data_ptr() if d["gk"] is not None else None
    return lib.sana_linattn_forward_noalloc(d["q"].data_ptr(), d["k"].data_ptr(),
                                            d["v"].data_ptr(), gq, gk, out.data_ptr(), w.B, w.N,
                                            w.C, w.H, w.eps, 0, s)


def test_noalloc_matches_forward_on_two_calls_in_a_row(cuda_lib):
    lib = cuda_lib.load()
    # two calls in a row, different shapes, so the second one meets the first
    # one's leftovers in the shared scratch
    for w in (WORKLOADS["2048px-b8-lognormal"].scaled(B=2, N=3000, seed=61), WORKLOADS["4096px-b2-overflow"].scaled(B=1, N=5000, seed=62)):
        d = to_dev(make_inputs(w))
        ref = cuda_lib.forward(d["q"], d["k"], d["v"], d["gq"], d["gk"], w.H, w.eps)
        out = torch.empty_like(d["q"])
        assert _noalloc(lib, d, w, out) == 0
        torch.cuda.synchronize()
        assert_close(out, ref, "bf16", f"noalloc vs forward {w.name}")


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_lib):
    lib = cuda_lib.load()
    w = WORKLOADS["4096px-b2-overflow"].scaled(B=64, N=16384)            # needs far more than 16 MiB
    assert cuda_lib.workspace_bytes(w.B, w.N, w.C, w.H) > (16 << 20)
    small = WORKLOADS["1024px-b1"].scaled(N=8)
    d = to_dev(make_inputs(small))
    out = torch.empty_like(d["q"])
    assert _noalloc(lib, d, w, out) == ESCRATCH      # rejected before anything is launched
    assert b"16 MiB" in lib.sana_linattn_strerror(ESCRATCH)
