"""Pins for the fp64 oracle (CPU only).

Each test ties the oracle to something other than itself: hand-derived worked
examples of Eq. (1), the quadratic (brute-force) form of Eq. (1), closed forms,
invariants that follow from the formula, and torch's library rms_norm.
Eq. (1): "Sana: Efficient High-Resolution Image Synthesis with Linear
Diffusion Transformers", section 2.1.  QK-Norm: "SANA 1.5 ...", section
"Model architecture", QK Norm bullet.
"""
import numpy as np
import pytest

from oracle import oracle as O
from oracle_checks import (battery, golden_case_inputs, load_golden, phi_lib, quadratic_form,
                           rel_err)


def test_battery_passes_on_the_oracle():
    assert battery(O) == []


@pytest.mark.parametrize("case", load_golden()["cases"], ids=lambda c: c["name"])
def test_golden_worked_examples(case):
    q, k, v, gq, gk = golden_case_inputs(case)
    got = O.forward(q, k, v, gq, gk, case["H"], case["eps"])[0]
    np.testing.assert_allclose(got, np.asarray(case["expected"]), rtol=1e-13, atol=1e-13)


def test_golden_per_head_norm_differs_from_full_channel_norm():
    case = [c for c in load_golden()["cases"] if c["name"] == "two_heads_per_head_norm"][0]
    q, k, v, gq, gk = golden_case_inputs(case)
    full = O.forward(q, k, v, gq, gk, case["H"], case["eps"], scope="full")[0]
    assert np.abs(full - np.asarray(case["expected"])).max() > 1e-3


@pytest.mark.parametrize("B,N,H,D", [(1, 1, 1, 32), (1, 2, 2, 4), (1, 3, 1, 1), (2, 17, 2, 32),
                                     (1, 256, 2, 32), (1, 64, 3, 5)])
@pytest.mark.parametrize("norm", [True, False])
def test_quadratic_form(B, N, H, D, norm):
    rng = np.random.default_rng(B * 1000 + N * 10 + H + D)
    C = H * D
    q, k, v = (rng.standard_normal((B, N, C)) for _ in range(3))
    gq = 1 + 0.1 * rng.standard_normal(C) if norm else None
    gk = 1 + 0.1 * rng.standard_normal(C) if norm else None
    eps = 1e-6
    assert rel_err(O.forward(q, k, v, gq, gk, H, eps), quadratic_form(q, k, v, gq, gk, H, eps)) \
        < 1e-11


def test_tiny_config_matches_quadratic_form():
    """The whole tiny configuration (B=1, H=2, D=32, N=256, fp32 inputs, g=1)."""
    from relu_linear_attention_attn_b200.synthetic import WORKLOADS, make_inputs
    w = WORKLOADS["tiny-512px-f32"]
    x = make_inputs(w)
    got = O.forward(x["q"], x["k"], x["v"], x["gq"], x["gk"], w.H, w.eps)
    ref = quadratic_form(x["q"].double().numpy(), x["k"].double().numpy(),
                         x["v"].double().numpy(), x["gq"].double().numpy(),
                         x["gk"].double().numpy(), w.H, w.eps)
    assert rel_err(got, ref) < 1e-12


def test_phi_against_torch_rms_norm():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((9, 3, 64)) * rng.lognormal(size=(9, 3, 1))
    g = 1 + 0.1 * rng.standard_normal(64)
    for scope in ("head", "full"):
        np.testing.assert_allclose(O.phi(x, g, 2, 1e-6, scope=scope),
                                   phi_lib(x, g, 2, 1e-6, scope), rtol=1e-13, atol=1e-15)
    np.testing.assert_array_equal(O.phi(x, None, 2, 1e-6), np.maximum(x, 0))


def test_rmsnorm_mean_square_is_one():
    """With g = 1 and positive inputs (so ReLU is the identity) the normalised head
    vector has mean square ms / (ms + eps)."""
    rng = np.random.default_rng(8)
    x = np.abs(rng.standard_normal((4, 96))) + 0.05
    eps = 1e-3
    p = O.phi(x, np.ones(96), 3, eps).reshape(4, 3, 32)
    ms = (x.reshape(4, 3, 32) ** 2).mean(-1)
    np.testing.assert_allclose((p ** 2).mean(-1), ms / (ms + eps), rtol=1e-13)


def test_closed_form_single_token():
    rng = np.random.default_rng(9)
    C, H, D = 64, 2, 32
    q, k, v = (rng.standard_normal((1, 1, C)) for _ in range(3))
    g = 1 + 0.1 * rng.standard_normal(C)
    eps = 0.25
    got = O.forward(q, k, v, g, g, H, eps)
    pq, pk = phi_lib(q, g, H, eps), phi_lib(k, g, H, eps)
    for h in range(H):
        sl = slice(h * D, (h + 1) * D)
        den = float(pq[0, 0, sl] @ pk[0, 0, sl])
        np.testing.assert_allclose(got[0, 0, sl], v[0, 0, sl] * den / (den + eps), rtol=1e-13)


def test_closed_form_one_hot_keys():
    """Norm off, K_j = e_{c(j)}, Q = e_d: O = mean of the V_j whose key is e_d,
    times den / (den + eps) with den = their count."""
    rng = np.random.default_rng(10)
    N, D = 40, 4
    cls = rng.integers(0, D, size=N)
    k = np.zeros((1, N, D))
    k[0, np.arange(N), cls] = 1.0
    v = rng.standard_normal((1, N, D))
    q = np.eye(D)[None]
    eps = 1e-3
    # D query rows against N key rows: state, then apply
    got = O.apply(q, None, O.kv_state(k, v, None, 1, eps), 1, eps)[0]
    for d in range(D):
        sel = v[0, cls == d]
        cnt = len(sel)
        want = sel.sum(0) / (cnt + eps) if cnt else np.zeros(D)
        np.testing.assert_allclose(got[d], want, rtol=1e-13, atol=1e-15)


def test_closed_form_head_dim_one():
    """D = 1, norm off: O_i = sum_j relu(k_j) v_j / (sum_j relu(k_j) + eps / relu(q_i))."""
    rng = np.random.default_rng(11)
    N = 25
    q, k, v = (rng.standard_normal((1, N, 1)) for _ in range(3))
    q = np.abs(q) + 0.1
    eps = 1e-2
    got = O.forward(q, k, v, None, None, 1, eps)[0, :, 0]
    rk = np.maximum(k[0, :, 0], 0)
    want = (rk @ v[0, :, 0]) / (rk.sum() + eps / q[0, :, 0])
    np.testing.assert_allclose(got, want, rtol=1e-13)


def test_constant_values():
    rng = np.random.default_rng(12)
    B, N, H, D = 2, 50, 2, 8
    C = H * D
    q, k = rng.standard_normal((B, N, C)), rng.standard_normal((B, N, C))
    g = np.ones(C)
    v = np.full((B, N, C), 3.5)
    eps = 1e-6
    out = O.forward(q, k, v, g, g, H, eps)
    S = O.kv_state(k, v, g, H, eps)
    pq = phi_lib(q, g, H, eps).reshape(B, N, H, D)
    den = np.einsum("bnhd,bhd->bnh", pq, S[..., D])
    want = 3.5 * den / (den + eps)
    np.testing.assert_allclose(out.reshape(B, N, H, D), np.repeat(want[..., None], D, -1),
                               rtol=1e-12)
    assert np.abs(out - 3.5).max() < 1e-4


def test_linearity_in_values():
    rng = np.random.default_rng(13)
    B, N, H, D = 1, 60, 2, 16
    C = H * D
    q, k, v1, v2 = (rng.standard_normal((B, N, C)) for _ in range(4))
    g = 1 + 0.1 * rng.standard_normal(C)
    f = lambda v: O.forward(q, k, v, g, g, H, 1e-6)  # noqa: E731
    np.testing.assert_allclose(f(2.5 * v1), 2.5 * f(v1), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(f(v1 + v2), f(v1) + f(v2), rtol=1e-10, atol=1e-12)


def test_permutations():
    rng = np.random.default_rng(14)
    B, N, H, D = 1, 31, 2, 8
    C = H * D
    q, k, v = (rng.standard_normal((B, N, C)) for _ in range(3))
    g = 1 + 0.1 * rng.standard_normal(C)
    base = O.forward(q, k, v, g, g, H, 1e-6)
    p = rng.permutation(N)
    # permuting (K, V) together leaves O unchanged
    np.testing.assert_allclose(O.forward(q, k[:, p], v[:, p], g, g, H, 1e-6), base, rtol=1e-11)
    # permuting Q rows permutes O rows
    np.testing.assert_allclose(O.forward(q[:, p], k, v, g, g, H, 1e-6), base[:, p], rtol=1e-11)
    # permuting K alone (not V) changes O
    assert np.abs(O.forward(q, k[:, p], v, g, g, H, 1e-6) - base).max() > 1e-3


def test_heads_and_batches_are_independent():
    rng = np.random.default_rng(15)
    B, N, H, D = 2, 20, 3, 8
    C = H * D
    q, k, v = (rng.standard_normal((B, N, C)) for _ in range(3))
    g = 1 + 0.1 * rng.standard_normal(C)
    base = O.forward(q, k, v, g, g, H, 1e-6)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[1] += 1.0
    k2[:, :, D:2 * D] *= -1.3
    v2[:, :, 2 * D:] += 2.0
    out = O.forward(q2, k2, v2, g, g, H, 1e-6)
    np.testing.assert_array_equal(out[0, :, :D], base[0, :, :D])   # head 0, batch 0 untouched
    assert np.abs(out[1] - base[1]).max() > 1e-3
    assert np.abs(out[0, :, D:2 * D] - base[0, :, D:2 * D]).max() > 1e-3


def test_convex_combination_bounds():
    rng = np.random.default_rng(16)
    B, N, H, D = 1, 80, 2, 8
    C = H * D
    q, k, v = (rng.standard_normal((B, N, C)) for _ in range(3))
    g = np.ones(C)
    out = O.forward(q, k, v, g, g, H, 1e-12)
    assert (out <= v.max(axis=1, keepdims=True) + 1e-9).all()
    assert (out >= v.min(axis=1, keepdims=True) - 1e-9).all()


def test_scale_invariance():
    rng = np.random.default_rng(17)
    B, N, H, D = 1, 40, 2, 8
    C = H * D
    q, k, v = (rng.standard_normal((B, N, C)) for _ in range(3))
    # norm off: O(Q, aK, V) = O(Q, K, V) as eps -> 0; scaling one Q row leaves it unchanged
    base = O.forward(q, k, v, None, None, H, 0.0)
    np.testing.assert_allclose(O.forward(q, 7.0 * k, v, None, None, H, 0.0), base, rtol=1e-11)
    q2 = q.copy()
    q2[0, 5] *= 3.0
    np.testing.assert_allclose(O.forward(q2, k, v, None, None, H, 0.0), base, rtol=1e-11)
    # norm on: a positive per-token scale of Q or K is removed (up to the RMSNorm eps)
    g = 1 + 0.1 * rng.standard_normal(C)
    s_q = rng.lognormal(size=(B, N, 1))
    s_k = rng.lognormal(size=(B, N, 1))
    a = O.forward(q, k, v, g, g, H, 1e-12)
    b = O.forward(q * s_q, k * s_k, v, g, g, H, 1e-12)
    np.testing.assert_allclose(a, b, rtol=1e-8, atol=1e-10)


def test_state_is_additive_over_token_splits():
    """S over all tokens = sum of S over disjoint token ranges (the split-N and
    sequence-shard reduction rests on this)."""
    rng = np.random.default_rng(18)
    B, N, H, D = 2, 70, 2, 8
    C = H * D
    k, v = rng.standard_normal((B, N, C)), rng.standard_normal((B, N, C))
    g = 1 + 0.1 * rng.standard_normal(C)
    S = O.kv_state(k, v, g, H, 1e-6)
    parts = [O.kv_state(k[:, a:b], v[:, a:b], g, H, 1e-6) for a, b in [(0, 13), (13, 50), (50, 70)]]
    np.testing.assert_allclose(sum(parts), S, rtol=1e-12, atol=1e-12)


def test_apply_subset_matches_full():
    rng = np.random.default_rng(19)
    B, N, H, D = 2, 30, 2, 8
    C = H * D
    q, k, v = (rng.standard_normal((B, N, C)) for _ in range(3))
    g = 1 + 0.1 * rng.standard_normal(C)
    full = O.forward(q, k, v, g, g, H, 1e-6)
    S = O.kv_state(k, v, g, H, 1e-6)
    tok = np.array([0, 5, 29, 30, 59])
    sub = O.apply(q, g, S, H, 1e-6, tokens=tok)
    np.testing.assert_array_equal(sub, full.reshape(B * N, C)[tok])


def test_zero_denominator_row():
    """A query whose normalised head vector is all <= 0 gives num = den = 0 and
    O = 0 / eps = 0 for eps > 0."""
    rng = np.random.default_rng(20)
    N, H, D = 10, 1, 8
    q, k, v = (rng.standard_normal((1, N, D)) for _ in range(3))
    q[0, 3] = -np.abs(q[0, 3]) - 0.1
    g = np.ones(D)
    out = O.forward(q, k, v, g, g, H, 1e-6)
    np.testing.assert_array_equal(out[0, 3], np.zeros(D))


def test_overflow_stress_stays_finite_and_exceeds_fp16():
    """Unnormalised keys with scale 100: per-channel sums of phi(K) pass the fp16
    maximum, and the oracle still matches the quadratic form."""
    rng = np.random.default_rng(21)
    N, H, D = 2048, 1, 32
    q, v = rng.standard_normal((1, N, D)), rng.standard_normal((1, N, D))
    k = 100 * rng.standard_normal((1, N, D))
    S = O.kv_state(k, v, None, H, 1e-6)
    assert S[..., D].max() > 65504.0
    out = O.forward(q, k, v, None, None, H, 1e-6)
    assert np.isfinite(out).all()
    assert rel_err(out, quadratic_form(q, k, v, None, None, H, 1e-6)) < 1e-11


def test_fused_projection_column_order():
    """W = [I | 2I | 3I] gives Q = x, K = 2x, V = 3x, so the fused oracle equals the
    unfused one on those inputs."""
    rng = np.random.default_rng(22)
    B, N, H, D = 1, 12, 2, 4
    C = H * D
    x = rng.standard_normal((B, N, C))
    I = np.eye(C)
    W = np.concatenate([I, 2 * I, 3 * I], axis=1)
    g = 1 + 0.1 * rng.standard_normal(C)
    got = O.fused_forward(x, W, g, g, H, 1e-6)
    want = O.forward(x, 2 * x, 3 * x, g, g, H, 1e-6)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-15)


def test_fused_projection_matches_brute_force_and_subset():
    rng = np.random.default_rng(23)
    B, N, H, D = 2, 9, 2, 4
    C = H * D
    x = rng.standard_normal((B, N, C))
    W = 0.3 * rng.standard_normal((C, 3 * C))
    qkv = np.zeros((B, N, 3 * C))
    for b in range(B):
        for n in range(N):
            for j in range(3 * C):
                qkv[b, n, j] = sum(x[b, n, c] * W[c, j] for c in range(C))
    g = 1 + 0.1 * rng.standard_normal(C)
    ref = quadratic_form(qkv[..., :C], qkv[..., C:2 * C], qkv[..., 2 * C:], g, g, H, 1e-6)
    got = O.fused_forward(x, W, g, g, H, 1e-6)
    assert rel_err(got, ref) < 1e-11
    tok = np.array([1, 8, 9, 17])
    np.testing.assert_allclose(O.fused_forward(x, W, g, g, H, 1e-6, tokens=tok),
                               got.reshape(B * N, C)[tok], rtol=1e-12)


@pytest.mark.parametrize("gains", ["ones", "random", "off"])
def test_oracle_quadratic_forward_is_eq1(gains):
    """The oracle's O(N^2) form agrees with its linear form (associativity) and with
    the tests' independent quadratic form (torch's rms_norm feature map)."""
    from relu_linear_attention_attn_b200.synthetic import WORKLOADS, make_inputs
    w = WORKLOADS["tiny-512px-f32"].scaled(N=97, gains=gains, seed=44)
    x = make_inputs(w)
    q, k, v = (x[n].double().numpy() for n in ("q", "k", "v"))
    got = O.quadratic_forward(q, k, v, x["gq"], x["gk"], w.H, w.eps)
    assert rel_err(got, O.forward(q, k, v, x["gq"], x["gk"], w.H, w.eps)) < 1e-12
    assert rel_err(got, quadratic_form(q, k, v, x["gq"], x["gk"], w.H, w.eps)) < 1e-12
