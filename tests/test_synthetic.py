"""The seeded input generators that feed both the CUDA path and the oracle: each
named workload is reproducible, has the documented shapes and storage dtype, and
its values have the documented structure (latent token counts of the DC-AE F32
autoencoder, log-normal per-token scales, x100 keys of the overflow stress, gain
modes, fused-projection and Mix-FFN weight scales)."""
import numpy as np
import pytest
import torch

from relu_linear_attention_attn_b200.synthetic import (MIXFFN_WORKLOADS, WORKLOADS,
                                                       make_dwconv_inputs, make_gemm_inputs,
                                                       make_inputs, make_mixffn_inputs,
                                                       make_output_grad)


def _small(name, **kw):
    return WORKLOADS[name].scaled(**({"B": 1, "N": 512} | kw))


def test_latent_token_counts_follow_the_32x_autoencoder():
    for name, res in (("1024px-b1", 1024), ("2048px-b8-lognormal", 2048),
                      ("4096px-b2-overflow", 4096), ("fused-2048px-b4", 2048)):
        assert WORKLOADS[name].N == (res // 32) ** 2
    for name, res in (("mixffn-1024px-b1", 1024), ("mixffn-2048px-b4", 2048)):
        w = MIXFFN_WORKLOADS[name]
        assert w.Hs == w.Ws == res // 32 and w.N == (res // 32) ** 2
    for w in WORKLOADS.values():
        assert w.C == w.H * 32
    assert WORKLOADS["1024px-b1"].C == 2240 and MIXFFN_WORKLOADS["mixffn-2048px-b4"].F == 5600


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_inputs_are_reproducible_and_shaped(name):
    w = _small(name)
    a, b = make_inputs(w), make_inputs(w)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    keys = ("x", "W") if w.recipe == "fused" else ("q", "k", "v")
    for k in keys:
        assert torch.equal(a[k], b[k]) and a[k].dtype == dt
    if w.recipe == "fused":
        assert a["x"].shape == (w.B, w.N, w.C) and a["W"].shape == (w.C, 3 * w.C)
    else:
        assert all(a[k].shape == (w.B, w.N, w.C) for k in keys)
    assert (a["gq"] is None) == (w.gains == "off") == (a["gk"] is None)
    other = make_inputs(w.scaled(seed=w.seed + 1))
    assert not torch.equal(a[keys[0]], other[keys[0]])


def test_storage_rounding_is_exact_bf16():
    x = make_inputs(_small("1024px-b1"))
    q = x["q"].float()
    assert torch.equal(q.to(torch.bfloat16).float(), q)


def test_lognormal_recipe_scales_whole_tokens():
    w = _small("2048px-b8-lognormal", N=2048)
    x = make_inputs(w)
    rms = x["q"].float().pow(2).mean(-1).sqrt().log().numpy().ravel()
    # log of the per-token scale ~ N(0, 1): spread about 1; a plain Gaussian's is ~0.02
    assert 0.8 < rms.std() < 1.2
    g = make_inputs(_small("1024px-b1", N=2048))
    assert g["q"].float().pow(2).mean(-1).sqrt().log().std() < 0.05
    assert x["gq"] is not None and torch.equal(x["gq"], torch.ones(w.C))


def test_overflow_recipe_has_hundredfold_keys_and_no_norm():
    x = make_inputs(_small("4096px-b2-overflow"))
    k_rms = float(x["k"].float().pow(2).mean().sqrt())
    q_rms = float(x["q"].float().pow(2).mean().sqrt())
    assert 95 < k_rms < 105 and 0.95 < q_rms < 1.05
    assert x["gq"] is None and x["gk"] is None


def test_random_gains_and_fused_weights():
    x = make_inputs(_small("1024px-b1"))
    for g in (x["gq"], x["gk"]):
        assert g.dtype == torch.float32 and abs(float(g.mean()) - 1) < 0.01
        assert 0.09 < float(g.std()) < 0.11
    assert not torch.equal(x["gq"], x["gk"])
    f = make_inputs(_small("fused-2048px-b4", N=256))
    assert 0.019 < float(f["W"].float().std()) < 0.021


def test_output_gradient_is_seeded_unit_gaussian():
    w = _small("1024px-b1")
    a, b = make_output_grad(w), make_output_grad(w)
    assert torch.equal(a, b) and a.shape == (w.B, w.N, w.C) and a.dtype == torch.bfloat16
    assert abs(float(a.float().std()) - 1) < 0.01
    assert not torch.equal(a, make_output_grad(w, seed_offset=101))


def test_mixffn_recipes():
    w = MIXFFN_WORKLOADS["mixffn-tiny"].scaled(C=256, F=512)
    a, b = make_mixffn_inputs(w), make_mixffn_inputs(w)
    for k in ("x", "W1", "W2", "wdw", "b1", "bdw", "b2"):
        assert torch.equal(a[k], b[k])
    assert a["x"].shape == (w.B, w.N, w.C) and a["W1"].shape == (w.C, 2 * w.F)
    assert a["W2"].shape == (w.F, w.C) and a["wdw"].shape == (2 * w.F, 3, 3)
    assert abs(float(a["W1"].float().std()) * np.sqrt(w.C) - 1) < 0.03
    assert abs(float(a["W2"].float().std()) * np.sqrt(w.F) - 1) < 0.03
    assert abs(float(a["wdw"].std()) * 3 - 1) < 0.05
    n = make_mixffn_inputs(w.scaled(bias=False))
    assert n["b1"] is None and n["bdw"] is None and n["b2"] is None
    g = make_gemm_inputs(64, 128, 96, seed=1, bias=False)
    assert g["bias"] is None and g["A"].shape == (64, 128) and g["W"].shape == (128, 96)
    d = make_dwconv_inputs(2, 3, 5, 16, seed=2)
    assert d["u"].shape == (2, 15, 32) and d["wdw"].shape == (32, 3, 3) and d["bdw"].shape == (32,)
