"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Small cases compare every output element; the full-size workloads compare the
oracle's exact result on sampled tokens (the oracle forms the whole state, then
applies it to the sampled queries one by one).  All inputs are seeded and
synthetic (relu_linear_attention_attn_b200.synthetic)."""
import numpy as np
import pytest
import torch

import relu_linear_attention_attn_b200 as sla
from oracle import oracle as O
from parity import assert_close, errors, sample_tokens, to_dev, to_np
from relu_linear_attention_attn_b200.synthetic import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu


def run_forward(lib, d, w):
    return lib.forward(d["q"], d["k"], d["v"], d["gq"], d["gk"], w.H, w.eps)


@pytest.mark.parametrize("name", ["tiny-512px-f32", "1024px-b1"])
def test_workload_full_parity(cuda_lib, name):
    w = WORKLOADS[name]
    x = make_inputs(w)
    out = run_forward(cuda_lib, to_dev(x), w)
    torch.cuda.synchronize()
    ref = O.forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps)
    assert_close(out, ref, w.dtype, w.name)


@pytest.mark.parametrize("name", ["2048px-b8-lognormal", "4096px-b2-overflow"])
def test_workload_full_size_sampled_parity(cuda_lib, name):
    w = WORKLOADS[name]
    x = make_inputs(w)
    d = to_dev(x)
    out = run_forward(cuda_lib, d, w)
    torch.cuda.synchronize()
    tok = sample_tokens(w.B, w.N)
    S = O.kv_state(x["k"], x["v"], x["gk"], w.H, w.eps)
    ref = O.apply(x["q"], x["gq"], S, w.H, w.eps, tokens=tok)
    got = out.reshape(w.B * w.N, w.C)[torch.from_numpy(tok).cuda()]
    assert_close(got, ref, w.dtype, w.name)
    # the state the library reduces over the whole sequence agrees too
    kv = cuda_lib.kv_state(d["k"], d["v"], d["gk"], w.H, w.eps)
    e = errors(kv, S)
    assert e["normwise"] < 1e-2, e


def test_gains_reading_random_on_lognormal_recipe(cuda_lib):
    """The 2048px recipe under the other reading of its gains (1 + 0.1 N(0,1))."""
    w = WORKLOADS["2048px-b8-lognormal"].scaled(B=2, N=1500, gains="random", seed=12)
    x = make_inputs(w)
    out = run_forward(cuda_lib, to_dev(x), w)
    torch.cuda.synchronize()
    assert_close(out, O.forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps), w.dtype)


RAGGED = [(1, 1), (1, 2), (1, 127), (1, 129), (3, 777), (2, 1000), (1, 4097)]


@pytest.mark.parametrize("recipe,gains", [("gaussian", "random"), ("lognormal", "ones"),
                                          ("overflow", "off")])
@pytest.mark.parametrize("B,N", RAGGED)
def test_ragged_shapes_full_parity(cuda_lib, recipe, gains, B, N):
    w = Workload(f"{recipe}-{B}x{N}", B=B, N=N, C=2240, H=70, dtype="bf16", recipe=recipe,
                 gains=gains, eps=1e-6, seed=100 + B * 7 + N)
    x = make_inputs(w)
    out = run_forward(cuda_lib, to_dev(x), w)
    torch.cuda.synchronize()
    assert_close(out, O.forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps), w.dtype,
                 w.name)


@pytest.mark.parametrize("B,N,H,recipe,gains", [
    (1, 1, 70, "gaussian", "random"), (1, 64, 70, "lognormal", "ones"),
    (1, 129, 70, "overflow", "off"), (1, 1000, 70, "gaussian", "random"),
    (1, 1024, 70, "overflow", "off"), (2, 384, 6, "gaussian", "random"),
    (1, 500, 5, "lognormal", "random"), (3, 256, 70, "gaussian", "ones"),
    (2, 300, 1, "gaussian", "random"), (2, 1024, 70, "lognormal", "random"),
    (1, 896, 3, "overflow", "off"), (4, 128, 70, "gaussian", "random"),
    (1, 1023, 70, "lognormal", "ones"), (1, 640, 4, "gaussian", "random")])
def test_short_sequences_full_parity(cuda_lib, B, N, H, recipe, gains):
    """Short sequences: ragged token counts (clusters of 1 to 8 CTAs, a partly
    empty last CTA) and head counts that leave a head group or a head pair partly
    or wholly empty; the one-call forward (one cluster launch at these sizes) and
    the split kv_state + apply (the persistent passes) both match the oracle, and
    the forward is reproducible bit for bit."""
    w = Workload(f"short-{B}x{N}-h{H}", B=B, N=N, C=32 * H, H=H, dtype="bf16", recipe=recipe,
                 gains=gains, eps=1e-6, seed=300 + 7 * B + N + H)
    x = make_inputs(w)
    d = to_dev(x)
    out = run_forward(cuda_lib, d, w)
    kv = cuda_lib.kv_state(d["k"], d["v"], d["gk"], w.H, w.eps)
    two_pass = cuda_lib.apply(d["q"], d["gq"], kv, w.H, w.eps)
    torch.cuda.synchronize()
    ref = O.forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps)
    assert_close(out, ref, "bf16", w.name)
    assert_close(two_pass, ref, "bf16", w.name + " two-pass")
    again = run_forward(cuda_lib, d, w)
    torch.cuda.synchronize()
    assert torch.equal(out, again), "short-sequence path is not reproducible"


@pytest.mark.parametrize("B,N,H", [(1, 1, 2), (2, 300, 2), (1, 1000, 5), (1, 4096, 70)])
def test_fp32_path(cuda_lib, B, N, H):
    w = Workload("f32", B=B, N=N, C=32 * H, H=H, dtype="f32", recipe="gaussian", gains="random",
                 eps=1e-6, seed=7 + N)
    x = make_inputs(w)
    out = run_forward(cuda_lib, to_dev(x), w)
    torch.cuda.synchronize()
    assert_close(out, O.forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps), "f32")


def test_fused_full_size_sampled_parity(cuda_lib):
    w = WORKLOADS["fused-2048px-b4"]
    x = make_inputs(w)
    d = to_dev(x)
    out = cuda_lib.qkv_fused(d["x"], d["W"], d["gq"], d["gk"], w.H, w.eps)
    torch.cuda.synchronize()
    tok = sample_tokens(w.B, w.N, n=256)
    ref = O.fused_forward(x["x"], x["W"], x["gq"], x["gk"], w.H, w.eps, tokens=tok)
    got = out.reshape(w.B * w.N, w.C)[torch.from_numpy(tok).cuda()]
    assert_close(got, ref, "bf16", w.name)


@pytest.mark.parametrize("B,N,gains", [(1, 1, "random"), (1, 300, "random"), (2, 129, "off"),
                                       (1, 1000, "ones"), (2, 800, "random"), (3, 333, "off")])
def test_fused_small_full_parity(cuda_lib, B, N, gains):
    """Small shapes: one to eight token splits per head group, a last split with
    fewer tiles than the others (2 x 800: 7 tiles in splits of 2), the norm on and
    off."""
    w = WORKLOADS["fused-2048px-b4"].scaled(B=B, N=N, gains=gains, seed=40 + N)
    x = make_inputs(w)
    d = to_dev(x)
    out = cuda_lib.qkv_fused(d["x"], d["W"], d["gq"], d["gk"], w.H, w.eps)
    torch.cuda.synchronize()
    ref = O.fused_forward(x["x"], x["W"], x["gq"], x["gk"], w.H, w.eps)
    assert_close(out, ref, "bf16", f"fused {B}x{N} {gains}")


def test_apply_with_oracle_state(cuda_lib):
    w = WORKLOADS["1024px-b1"]
    x = make_inputs(w)
    S = O.kv_state(x["k"], x["v"], x["gk"], w.H, w.eps)
    kv = torch.from_numpy(S).float().cuda()
    out = cuda_lib.apply(x["q"].cuda(), x["gq"].cuda(), kv, w.H, w.eps)
    torch.cuda.synchronize()
    assert_close(out, O.apply(x["q"], x["gq"], S, w.H, w.eps), "bf16")


def test_sequence_shards_sum_to_the_whole_state(cuda_lib):
    """States of disjoint token ranges add up to the state of the whole sequence,
    so a sequence-sharded run needs one sum all-reduce of the state."""
    w = WORKLOADS["2048px-b8-lognormal"].scaled(B=2, N=2000, seed=21)
    x = to_dev(make_inputs(w))
    full = cuda_lib.kv_state(x["k"], x["v"], x["gk"], w.H, w.eps)
    a = cuda_lib.kv_state(x["k"][:, :700].contiguous(), x["v"][:, :700].contiguous(), x["gk"],
                          w.H, w.eps)
    b = cuda_lib.kv_state(x["k"][:, 700:].contiguous(), x["v"][:, 700:].contiguous(), x["gk"],
                          w.H, w.eps)
    torch.cuda.synchronize()
    e = errors(a + b, full)
    assert e["normwise"] < 1e-5, e


def test_bitwise_determinism(cuda_lib):
    w = WORKLOADS["2048px-b8-lognormal"].scaled(B=2, N=3000, seed=22)
    d = to_dev(make_inputs(w))
    o1 = run_forward(cuda_lib, d, w)
    o2 = run_forward(cuda_lib, d, w)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


def test_zero_denominator_row_gives_zero(cuda_lib):
    w = WORKLOADS["1024px-b1"].scaled(N=300, seed=23)
    x = make_inputs(w)
    x["q"][0, 17] = -x["q"][0, 17].abs() - 0.25     # every head of token 17 is negative
    out = run_forward(cuda_lib, to_dev(x), w)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out[0, 17]).item() == 0
    assert_close(out, O.forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps), "bf16")


def test_overflow_stress_is_finite_and_exceeds_fp16(cuda_lib):
    w = WORKLOADS["4096px-b2-overflow"].scaled(B=1, N=16384, seed=24)
    d = to_dev(make_inputs(w))
    kv = cuda_lib.kv_state(d["k"], d["v"], None, w.H, w.eps)
    out = run_forward(cuda_lib, d, w)
    torch.cuda.synchronize()
    assert kv[..., 32].max().item() > 65504.0
    assert torch.isfinite(out.float()).all()


def test_empty_problems(cuda_lib):
    z = torch.empty((0, 5, 2240), dtype=torch.bfloat16, device="cuda")
    assert run_forward(cuda_lib, dict(q=z, k=z, v=z, gq=None, gk=None),
                       WORKLOADS["4096px-b2-overflow"]).numel() == 0
    e = torch.empty((2, 0, 2240), dtype=torch.bfloat16, device="cuda")
    kv = torch.full((2, 70, 32, 33), 7.0, device="cuda")
    cuda_lib.kv_state(e, e, None, 70, 1e-6, kv=kv)
    torch.cuda.synchronize()
    assert torch.count_nonzero(kv).item() == 0


def test_validation_with_real_buffers(cuda_lib):
    lib = cuda_lib.load()
    w = WORKLOADS["1024px-b1"]
    d = to_dev(make_inputs(w))
    q = d["q"]
    out = torch.empty_like(q)
    nbytes = cuda_lib.workspace_bytes(w.B, w.N, w.C, w.H)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    base = dict(q=q.data_ptr(), k=d["k"].data_ptr(), v=d["v"].data_ptr(), gq=d["gq"].data_ptr(),
                gk=d["gk"].data_ptr(), out=out.data_ptr(), ws=ws.data_ptr(), wsb=nbytes)

    def call(**kw):
        a = dict(base, **kw)
        return lib.sana_linattn_forward(a["q"], a["k"], a["v"], a["gq"], a["gk"], a["out"], w.B,
                                        w.N, w.C, w.H, w.eps, 0, a["ws"], a["wsb"], s)
    assert call(q=q.data_ptr() + 2) == -2
    assert call(wsb=nbytes - 1) == -4
    assert call(out=q.data_ptr()) == -1
    assert call(gk=None) == -1
    assert call() == 0
    torch.cuda.synchronize()
    kv = cuda_lib.kv_state(d["k"], d["v"], d["gk"], w.H, w.eps)
    with pytest.raises(ValueError):
        cuda_lib.apply(q[:, ::2], d["gq"], kv, w.H, w.eps)      # non-contiguous


def test_no_device_error_after_the_suite_so_far(cuda_lib):
    torch.cuda.synchronize()
    assert cuda_lib.device_error(clear=True) == (0, 0)


def test_bounded_wait_gives_up_and_reports(cuda_lib):
    """A wait that nothing satisfies gives up after its limit, records the error,
    and leaves the context usable (no trap, no hang)."""
    cuda_lib.device_error(clear=True)
    cuda_lib.selftest_wait_timeout(limit_us=20000)
    torch.cuda.synchronize()
    assert cuda_lib.device_error(clear=True) == (1, 999)
    w = WORKLOADS["1024px-b1"].scaled(N=200, seed=31)
    x = make_inputs(w)
    out = run_forward(cuda_lib, to_dev(x), w)
    torch.cuda.synchronize()
    assert_close(out, O.forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps), "bf16")
    assert cuda_lib.device_error(clear=True) == (0, 0)


def test_wide_head_count_runs_the_cuda_core_path(cuda_lib):
    """H = 130 (C = 4160) is past the tensor-core kernels' gain cache; the library
    runs its CUDA-core kernels for bf16 there, with the same results."""
    w = Workload("wide", B=1, N=300, C=32 * 130, H=130, dtype="bf16", recipe="gaussian",
                 gains="random", eps=1e-6, seed=77)
    x = make_inputs(w)
    out = run_forward(cuda_lib, to_dev(x), w)
    torch.cuda.synchronize()
    assert_close(out, O.forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps), "bf16")


@pytest.mark.parametrize("name", ["2048px-b8-lognormal", "4096px-b2-overflow"])
def test_state_reduction_is_reproducible_at_full_size(cuda_lib, name):
    """Pass 1 at full size, twice: the combine order is fixed, so the states are
    bitwise equal (a race in the ring or the combine would show up here)."""
    w = WORKLOADS[name]
    d = to_dev(make_inputs(w))
    a = cuda_lib.kv_state(d["k"], d["v"], d["gk"], w.H, w.eps)
    b = cuda_lib.kv_state(d["k"], d["v"], d["gk"], w.H, w.eps)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_independent_problems_on_concurrent_streams(cuda_lib):
    """Forward calls on different streams share the GPU (the persistent passes of
    one fill SMs another leaves idle); each result equals the same call run alone,
    bit for bit."""
    cases = [WORKLOADS["1024px-b1"].scaled(N=700, seed=111),
             WORKLOADS["2048px-b8-lognormal"].scaled(B=2, N=2500, seed=112),
             WORKLOADS["4096px-b2-overflow"].scaled(B=1, N=6000, seed=113)]
    data = [to_dev(make_inputs(w)) for w in cases]
    alone = []
    for w, d in zip(cases, data):
        alone.append(run_forward(cuda_lib, d, w))
        torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in cases]
    outs = [torch.empty_like(d["q"]) for d in data]
    for _ in range(3):
        for s in streams:
            s.wait_stream(torch.cuda.current_stream())
        for s, w, d, o in zip(streams, cases, data, outs):
            with torch.cuda.stream(s):
                cuda_lib.forward(d["q"], d["k"], d["v"], d["gq"], d["gk"], w.H, w.eps, out=o)
        for s in streams:
            torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for w, a, o in zip(cases, alone, outs):
        assert torch.equal(a, o), w.name


@pytest.mark.parametrize("B,N", [(2, 3000), (3, 1500), (1, 16384)])
def test_forward_passes_called_separately_equal_forward(cuda_lib, B, N):
    """sana_linattn_forward_pass1 then _pass2 on one stream are the forward (for
    sequences the forward runs as the two persistent passes): the same kernels and
    plan, so the output is bit-identical, also with unrelated work enqueued between
    the two calls."""
    w = WORKLOADS["4096px-b2-overflow"].scaled(B=B, N=N, seed=120 + N)
    d = to_dev(make_inputs(w))
    ref = run_forward(cuda_lib, d, w)
    ws = torch.empty(cuda_lib.workspace_bytes(B, N, w.C, w.H), dtype=torch.uint8, device="cuda")
    cuda_lib.forward_pass1(d["k"], d["v"], d["gk"], w.H, w.eps, ws)
    scratch = torch.randn(1 << 20, device="cuda").sum()        # unrelated work in between
    out = cuda_lib.forward_pass2(d["q"], d["gq"], w.H, w.eps, ws)
    torch.cuda.synchronize()
    assert torch.isfinite(scratch)
    assert torch.equal(out, ref)
