"""Pins of the oracle's prefix (causal) form (CPU only).

Checked against hand-derived worked examples (tests/golden/causal_worked_examples.json),
a masked quadratic form brute-forced in numpy with a textbook RMSNorm, the last
token (whose prefix is the whole sequence) against the non-causal forward, the
first token's closed form, and causality itself; plausible mistakes planted in a
copy of the C oracle must fail the battery."""
import ctypes
import json
import os
import subprocess

import numpy as np
import pytest

from oracle import oracle as O

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                   "causal_worked_examples.json")))


def _phi_textbook(x, g, H, eps):
    """ReLU(g * x / sqrt(mean_d x^2 + eps)) per head, straight from the definition."""
    B, N, C = x.shape
    D = C // H
    xh = x.reshape(B, N, H, D)
    r = 1.0 / np.sqrt((xh ** 2).mean(-1, keepdims=True) + eps)
    y = xh * r * (g.reshape(H, D) if g is not None else 1.0)
    return np.maximum(y, 0.0).reshape(B, N, C)


def _masked_quadratic(q, k, v, gq, gk, H, eps):
    B, N, C = q.shape
    D = C // H
    pq = _phi_textbook(q, gq, H, eps) if gq is not None else np.maximum(q, 0)
    pk = _phi_textbook(k, gk, H, eps) if gk is not None else np.maximum(k, 0)
    out = np.empty_like(q)
    mask = np.tril(np.ones((N, N)))
    for b in range(B):
        for h in range(H):
            s = slice(h * D, (h + 1) * D)
            A = (pq[b, :, s] @ pk[b, :, s].T) * mask
            out[b, :, s] = (A @ v[b, :, s]) / (A.sum(1, keepdims=True) + eps)
    return out


def causal_battery(M) -> list:
    bad = []
    for c in GOLD["cases"]:
        q, k, v = (np.array([c[n]], float) for n in ("q", "k", "v"))
        o = M.causal_forward(q, k, v, None, None, c["H"], c["eps"])
        if not np.allclose(o[0], np.array(c["out"]), rtol=1e-14, atol=1e-14):
            bad.append(f"golden {c['name']}: {o[0].tolist()}")
    rng = np.random.default_rng(11)
    B, N, C, H, eps = 2, 37, 64, 2, 1e-6
    q, k, v = (rng.standard_normal((B, N, C)) for _ in range(3))
    gq, gk = 1 + 0.1 * rng.standard_normal(C), 1 + 0.1 * rng.standard_normal(C)
    o = M.causal_forward(q, k, v, gq, gk, H, eps)
    ref = _masked_quadratic(q, k, v, gq, gk, H, eps)
    if not np.allclose(o, ref, rtol=1e-10, atol=1e-12):
        bad.append(f"masked quadratic form: max diff {np.abs(o - ref).max():.3e}")
    full = O.forward(q, k, v, gq, gk, H, eps)
    if not np.allclose(o[:, -1], full[:, -1], rtol=1e-12, atol=1e-13):
        bad.append("last token differs from the non-causal forward")
    # first token: one key, O_0 = V_0 * den / (den + eps)
    o1 = M.causal_forward(q, k, v, None, None, H, 0.5)
    pq, pk = np.maximum(q, 0), np.maximum(k, 0)
    for h in range(H):
        s = slice(h * 32, (h + 1) * 32)
        den = (pq[:, 0, s] * pk[:, 0, s]).sum(-1, keepdims=True)
        if not np.allclose(o1[:, 0, s], v[:, 0, s] * den / (den + 0.5), rtol=1e-12, atol=1e-14):
            bad.append("first-token closed form")
    # causality: later tokens do not change earlier outputs
    k2, v2 = k.copy(), v.copy()
    k2[:, 20:] = rng.standard_normal(k2[:, 20:].shape)
    v2[:, 20:] *= -3.0
    o2 = M.causal_forward(q, k2, v2, gq, gk, H, eps)
    if not np.array_equal(o2[:, :20], o[:, :20]):
        bad.append("outputs before token 20 depend on later tokens")
    return bad


def test_causal_pins_hold():
    assert causal_battery(O) == []


SRC = os.path.join(os.path.dirname(O.__file__), "sana_oracle.c")
MUTATIONS = {
    "state_updated_after_apply": (
        "        /* O_n = phi(Q_n) S_n[:, :D] / (phi(Q_n) S_n[:, D] + eps) */",
        "        for (int i = 0; i < D; ++i) { for (int j = 0; j < D; ++j) run[i * (D + 1) + j] -= fk[i] * vn[j];"
        " run[i * (D + 1) + D] -= fk[i]; }"),
    "causal_normaliser_counts_tokens": ("            run[i * (D + 1) + D] += fk[i];",
                                        "            run[i * (D + 1) + D] += 1.0;"),
    "causal_eps_dropped": ("            on[j] = nm / (dn + c->eps);", "            on[j] = nm / dn;"),
    "causal_value_head_offset_lost": ("        const double* vn = c->v + at + (size_t)h * D;",
                                      "        const double* vn = c->v + at;"),
    "causal_state_transposed": ("            for (int j = 0; j < D; ++j) run[i * (D + 1) + j] += fk[i] * vn[j];",
                                "            for (int j = 0; j < D; ++j) run[i * (D + 1) + j] += fk[j] * vn[i];"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_causal_battery_catches_planted_mistake(name, tmp_path, monkeypatch):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    mutated = tmp_path / f"oracle_{name}.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / f"oracle_{name}.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", "-o",
                    str(so), str(mutated), "-lpthread", "-lm"], check=True)
    lib = O._bind(ctypes.CDLL(str(so)))
    monkeypatch.setattr(O, "_lib", lib)
    assert causal_battery(O), f"planted mistake {name} went unnoticed"
