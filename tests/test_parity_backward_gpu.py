"""Parity of the backward (through the C ABI) with the fp64 oracle's hand-derived
gradients (themselves pinned against autograd and finite differences).

Tolerances (gradients have no fixed scale, so they are normwise against a scale
s = max(max|g_ref|, max|dV_ref|)): bf16 outputs max|g - g_ref| <= 2e-2 * s and
||g - g_ref||_2 <= 2e-2 * max(||g_ref||_2, s * sqrt(size) * 1e-2); fp32 outputs
max|g - g_ref| <= 1e-4 * s (the backward chains more roundings than the forward:
the RMS term of the feature-map gradient cancels).  dV sets the floor of the
scale because dQ, dK and the gain gradients vanish where the output barely
depends on them (N = 1: O = V den / (den + eps)), and their relative error is then
ill-posed; with the normalised features of unit RMS, one token's share of a gain
gradient is of the order of its dQ, so the same floor serves the gains.  That
floor is for N = 1 only: with two or more tokens each gradient must also be within
a relative L2 error of its own norm (2e-2 for bf16, 1e-3 for fp32)."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from parity import to_dev, to_np
from relu_linear_attention_attn_b200.synthetic import WORKLOADS, make_inputs, make_output_grad

pytestmark = pytest.mark.gpu


def _close(got, ref, dtype, what, scale, own_l2):
    g, r = to_np(got), to_np(ref)
    assert np.isfinite(g).all(), f"{what}: non-finite"
    s = max(float(np.abs(r).max()), scale)
    err = float(np.abs(g - r).max())
    l2 = float(np.linalg.norm(g - r))
    if dtype == "f32":
        assert err <= 1e-4 * s, f"{what}: max err {err:.3e}, scale {s:.3e}"
    else:
        ref_l2 = max(float(np.linalg.norm(r)), s * np.sqrt(r.size) * 1e-2)
        assert err <= 2e-2 * s and l2 <= 2e-2 * ref_l2, \
            f"{what}: max err {err:.3e} (scale {s:.3e}), l2 {l2:.3e} vs {ref_l2:.3e}"
    if own_l2:
        # With two or more tokens every gradient is of the order of dV (no O(eps)
        # cancellation), so each must also meet a relative L2 bound of its own.
        own = float(np.linalg.norm(r))
        bound = (1e-3 if dtype == "f32" else 2e-2) * own
        assert own > 0 and l2 <= bound, f"{what}: l2 {l2:.3e} vs own-norm bound {bound:.3e}"


def _check(cuda_lib, w):
    x = make_inputs(w)
    do = make_output_grad(w)
    d = to_dev(x)
    got = cuda_lib.backward(d["q"], d["k"], d["v"], d["gq"], d["gk"], do.cuda(), w.H, w.eps)
    torch.cuda.synchronize()
    ref = O.backward(x["q"], x["k"], x["v"], x["gq"], x["gk"], do, w.H, w.eps)
    dv_scale = float(np.abs(ref[2]).max())
    for name, g, r in zip(("dq", "dk", "dv", "dgq", "dgk"), got, ref):
        if r is None:
            assert g is None
            continue
        # gain gradients are fp32 outputs whatever the dtype
        _close(g, r, "f32" if name.startswith("dg") and w.dtype == "f32" else w.dtype,
               f"{w.name} {name}", dv_scale, own_l2=w.N >= 2)


@pytest.mark.parametrize("w", [WORKLOADS["tiny-512px-f32"], WORKLOADS["tiny-512px-f32"].scaled(N=300, gains="random", seed=80),
                               WORKLOADS["1024px-b1"].scaled(N=1, seed=81),
                               WORKLOADS["1024px-b1"].scaled(N=333, seed=82),
                               WORKLOADS["1024px-b1"].scaled(B=2, N=129, gains="off", seed=83),
                               WORKLOADS["1024px-b1"],
                               WORKLOADS["2048px-b8-lognormal"].scaled(B=2, seed=84)],
                         ids=lambda w: f"{w.dtype}-B{w.B}-N{w.N}-{w.gains}")
def test_backward_parity(cuda_lib, w):
    _check(cuda_lib, w)


def test_backward_is_deterministic(cuda_lib):
    w = WORKLOADS["1024px-b1"].scaled(B=2, N=1000, seed=85)
    d = to_dev(make_inputs(w))
    do = make_output_grad(w).cuda()
    a = cuda_lib.backward(d["q"], d["k"], d["v"], d["gq"], d["gk"], do, w.H, w.eps)
    b = cuda_lib.backward(d["q"], d["k"], d["v"], d["gq"], d["gk"], do, w.H, w.eps)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("w", [WORKLOADS["1024px-b1"].scaled(B=2, N=1000, seed=90),
                               WORKLOADS["1024px-b1"].scaled(N=64, seed=91),
                               WORKLOADS["4096px-b2-overflow"].scaled(B=1, N=700, seed=92),
                               WORKLOADS["tiny-512px-f32"].scaled(N=300, gains="random", seed=93)],
                         ids=lambda w: f"{w.dtype}-B{w.B}-N{w.N}-{w.gains}")
def test_backward_with_the_forward_state_equals_backward(cuda_lib, w):
    """sana_linattn_backward_with_state given kv_state()'s state: the same gradients
    bit for bit (the backward forms its state exactly as kv_state does), on the
    tensor-core path, the short-sequence and fp32 CUDA-core paths and with the norm
    off."""
    d = to_dev(make_inputs(w))
    do = make_output_grad(w).cuda()
    kv = cuda_lib.kv_state(d["k"], d["v"], d["gk"], w.H, w.eps)
    a = cuda_lib.backward(d["q"], d["k"], d["v"], d["gq"], d["gk"], do, w.H, w.eps)
    b = cuda_lib.backward(d["q"], d["k"], d["v"], d["gq"], d["gk"], do, w.H, w.eps, kv=kv)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert (x is None and y is None) or torch.equal(x, y)


def test_backward_gains_without_16_byte_alignment(cuda_lib):
    """Gains 4-byte but not 16-byte aligned: the backward takes its CUDA-core path
    and still matches the oracle (the tensor-core kernels read gains as 16-byte
    vectors)."""
    w = WORKLOADS["1024px-b1"].scaled(N=300, seed=88)
    x = make_inputs(w)
    do = make_output_grad(w)
    d = to_dev(x)
    gq = torch.empty(w.C + 1, dtype=torch.float32, device="cuda")[1:]
    gk = torch.empty(w.C + 1, dtype=torch.float32, device="cuda")[1:]
    gq.copy_(d["gq"])
    gk.copy_(d["gk"])
    assert gq.data_ptr() % 16 != 0 and gk.data_ptr() % 16 != 0
    got = cuda_lib.backward(d["q"], d["k"], d["v"], gq, gk, do.cuda(), w.H, w.eps)
    torch.cuda.synchronize()
    ref = O.backward(x["q"], x["k"], x["v"], x["gq"], x["gk"], do, w.H, w.eps)
    dv_scale = float(np.abs(ref[2]).max())
    for name, g, r in zip(("dq", "dk", "dv", "dgq", "dgk"), got, ref):
        _close(g, r, w.dtype, f"unaligned gains {name}", dv_scale, own_l2=True)
