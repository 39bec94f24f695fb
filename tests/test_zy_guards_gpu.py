"""Every entry point writes only inside the buffers it is given: outputs and
workspaces are carved out of larger buffers whose guard bands hold a canary, and
the bands must be intact after the call (the plan's guard-band canaries; the
library's bounds checks replace a sanitizer, which is closed here).  Also: a
launch the runtime rejects surfaces as SANA_ECUDA and leaves the context usable."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from parity import Guarded, assert_close, to_dev
from relu_linear_attention_attn_b200.synthetic import (MIXFFN_WORKLOADS, WORKLOADS,
                                                       make_dwconv_inputs, make_gemm_inputs,
                                                       make_inputs, make_mixffn_inputs,
                                                       make_output_grad)

pytestmark = pytest.mark.gpu

DEV = "cuda"
BF, F32 = torch.bfloat16, torch.float32


def _ok(*guards):
    torch.cuda.synchronize()
    for g in guards:
        assert g.intact(), "a write landed outside its buffer"


@pytest.mark.parametrize("name,kw", [("1024px-b1", dict(B=2, N=333, seed=61)),
                                     ("1024px-b1", dict(N=1, seed=62)),
                                     ("1024px-b1", dict(N=1500, seed=65)),
                                     ("4096px-b2-overflow", dict(B=1, N=1024, seed=66)),
                                     ("tiny-512px-f32", dict(N=77, seed=63))])
def test_forward_and_causal_stay_in_bounds(cuda_lib, name, kw):
    w = WORKLOADS[name].scaled(**kw)
    d = to_dev(make_inputs(w))
    dt = d["q"].dtype
    esz = d["q"].element_size()
    shape = (w.B, w.N, w.C)
    out = Guarded(w.B * w.N * w.C * esz, DEV)
    ws = Guarded(cuda_lib.workspace_bytes(w.B, w.N, w.C, w.H), DEV)
    cuda_lib.forward(d["q"], d["k"], d["v"], d["gq"], d["gk"], w.H, w.eps,
                     out=out.view(dt, shape), workspace=ws.region)
    _ok(out, ws)
    out2 = Guarded(w.B * w.N * w.C * esz, DEV)
    ws2 = Guarded(int(cuda_lib.load().sana_linattn_workspace_bytes(w.B, w.N, w.C, w.H, 2)), DEV)
    cuda_lib.forward_causal(d["q"], d["k"], d["v"], d["gq"], d["gk"], w.H, w.eps,
                            out=out2.view(dt, shape), workspace=ws2.region)
    _ok(out2, ws2)
    assert torch.isfinite(out.view(dt, shape).float()).all()
    assert torch.isfinite(out2.view(dt, shape).float()).all()


def test_fused_and_w8a8_stay_in_bounds(cuda_lib):
    w = WORKLOADS["fused-2048px-b4"].scaled(B=1, N=200, seed=64)
    d = to_dev(make_inputs(w))
    shape = (w.B, w.N, w.C)
    out = Guarded(w.B * w.N * w.C * 2, DEV)
    ws = Guarded(cuda_lib.workspace_bytes(w.B, w.N, w.C, w.H, fused=True), DEV)
    cuda_lib.qkv_fused(d["x"], d["W"], d["gq"], d["gk"], w.H, w.eps, out=out.view(BF, shape),
                       workspace=ws.region)
    _ok(out, ws)
    xq = Guarded(w.B * w.N * w.C, DEV)
    sx = Guarded(w.B * w.N * 4, DEV)
    cuda_lib.quantize_rows_i8(d["x"], out=xq.view(torch.int8, shape),
                              scales=sx.view(F32, (w.B, w.N)))
    Wq = Guarded(w.C * 3 * w.C, DEV)
    sw = Guarded(3 * w.C * 4, DEV)
    cuda_lib.quantize_cols_i8(d["W"], out=Wq.view(torch.int8, (w.C, 3 * w.C)),
                              scales=sw.view(F32, (3 * w.C,)))
    _ok(xq, sx, Wq, sw)
    out8 = Guarded(w.B * w.N * w.C * 2, DEV)
    ws8 = Guarded(cuda_lib.workspace_bytes(w.B, w.N, w.C, w.H, fused=True), DEV)
    cuda_lib.qkv_fused_w8a8(xq.view(torch.int8, shape), sx.view(F32, (w.B, w.N)),
                            Wq.view(torch.int8, (w.C, 3 * w.C)), sw.view(F32, (3 * w.C,)),
                            d["gq"], d["gk"], w.H, w.eps, out=out8.view(BF, shape),
                            workspace=ws8.region)
    _ok(out8, ws8)


def test_backward_stays_in_bounds(cuda_lib):
    w = WORKLOADS["1024px-b1"].scaled(B=2, N=129, gains="random", seed=65)
    d = to_dev(make_inputs(w))
    do = make_output_grad(w).cuda()
    shape = (w.B, w.N, w.C)
    gs = [Guarded(w.B * w.N * w.C * 2, DEV) for _ in range(3)] + \
         [Guarded(w.C * 4, DEV) for _ in range(2)]
    ws = Guarded(int(cuda_lib.load().sana_linattn_backward_workspace_bytes(w.B, w.N, w.C, w.H)),
                 DEV)
    grads = tuple(g.view(BF, shape) for g in gs[:3]) + tuple(g.view(F32, (w.C,)) for g in gs[3:])
    cuda_lib.backward(d["q"], d["k"], d["v"], d["gq"], d["gk"], do, w.H, w.eps, grads=grads,
                      workspace=ws.region)
    _ok(*gs, ws)


def test_mixffn_kernels_stay_in_bounds(cuda_lib):
    w = MIXFFN_WORKLOADS["mixffn-tiny"].scaled(B=2, Hs=5, Ws=37, C=64, F=40, seed=66)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in
         make_mixffn_inputs(w).items()}
    shape = (w.B, w.N, w.C)
    out = Guarded(w.B * w.N * w.C * 2, DEV)
    ws = Guarded(cuda_lib.mixffn_workspace_bytes(w.B, w.Hs, w.Ws, w.C, w.F), DEV)
    cuda_lib.mixffn_forward(d["x"], d["W1"], d["b1"], d["wdw"], d["bdw"], d["W2"], d["b2"], w.Hs,
                            w.Ws, w.gate, out=out.view(BF, shape), workspace=ws.region)
    _ok(out, ws)
    g = make_gemm_inputs(300, 200, 520, seed=67)
    o = Guarded(300 * 520 * 2, DEV)
    cuda_lib.gemm_bias(g["A"].cuda(), g["W"].cuda(), g["bias"].cuda(), out=o.view(BF, (300, 520)))
    _ok(o)
    c = make_dwconv_inputs(2, 5, 37, 40, seed=68)
    h = Guarded(2 * 5 * 37 * 40 * 2, DEV)
    cuda_lib.mixffn_dwconv_glu(c["u"].cuda(), c["wdw"].cuda(), c["bdw"].cuda(), 5, 37, "silu",
                               out=h.view(BF, (2, 5 * 37, 40)))
    _ok(h)


def test_rejected_launch_is_reported_and_not_sticky(cuda_lib):
    assert cuda_lib.selftest_launch_failure() == -5           # SANA_ECUDA
    torch.cuda.synchronize()
    w = WORKLOADS["1024px-b1"].scaled(N=100, seed=69)
    x = make_inputs(w)
    out = cuda_lib.forward(*(to_dev(x)[n] for n in ("q", "k", "v", "gq", "gk")), w.H, w.eps)
    torch.cuda.synchronize()
    assert_close(out, O.forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps), "bf16")
    assert cuda_lib.device_error(clear=True) == (0, 0)
