"""Independent checks that pin the fp64 oracle to facts outside itself.

None of these re-types the oracle's own loops.  The brute force below evaluates
Eq. (1) in its quadratic form, sum_j (phi(Q_i).phi(K_j)) V_j / (sum_j
phi(Q_i).phi(K_j) + eps), which the linear form equals only by associativity,
and builds phi from torch's library ``rms_norm``.  The battery is shared by the
pin tests and by the mutation test, which plants mistakes in a copy of the
oracle and expects this battery to notice each one.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "eq1_worked_examples.json")


def phi_lib(x, g, H: int, eps: float, scope: str = "head") -> np.ndarray:
    """Feature map from library routines: ReLU(torch rms_norm(x) * g); g None -> ReLU(x)."""
    x = torch.as_tensor(np.asarray(x, dtype=np.float64))
    if g is None:
        return torch.relu(x).numpy()
    g = torch.as_tensor(np.asarray(g, dtype=np.float64))
    C = x.shape[-1]
    if scope == "full":
        return torch.relu(F.rms_norm(x, (C,), weight=g, eps=eps)).numpy()
    D = C // H
    xh = x.reshape(*x.shape[:-1], H, D)
    gh = g.reshape(H, D)
    parts = [F.rms_norm(xh[..., h, :], (D,), weight=gh[h], eps=eps) for h in range(H)]
    return torch.relu(torch.stack(parts, dim=-2)).reshape(x.shape).numpy()


def quadratic_form(q, k, v, gq, gk, H: int, eps: float, scope: str = "head") -> np.ndarray:
    """Brute-force O(N^2) evaluation: explicit N x N weights A_ij = phi(Q_i).phi(K_j),
    O_i = sum_j A_ij V_j / (sum_j A_ij + eps)."""
    pq = phi_lib(q, gq, H, eps, scope)
    pk = phi_lib(k, gk, H, eps, scope)
    v = np.asarray(v, dtype=np.float64)
    B, N, C = pq.shape
    D = C // H
    out = np.empty_like(v)
    for b in range(B):
        for h in range(H):
            sl = slice(h * D, (h + 1) * D)
            A = pq[b, :, sl] @ pk[b, :, sl].T
            out[b, :, sl] = (A @ v[b, :, sl]) / (A.sum(axis=1, keepdims=True) + eps)
    return out


def rel_err(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = max(np.abs(b).max(), 1e-300)
    return float(np.abs(a - b).max() / den)


def load_golden():
    with open(GOLDEN) as f:
        return json.load(f)


def golden_case_inputs(case):
    q = np.asarray(case["q"], dtype=np.float64)[None]
    k = np.asarray(case["k"], dtype=np.float64)[None]
    v = np.asarray(case["v"], dtype=np.float64)[None]
    gq = np.asarray(case["gq"], dtype=np.float64) if case["norm"] else None
    gk = np.asarray(case["gk"], dtype=np.float64) if case["norm"] else None
    return q, k, v, gq, gk


def _rand(rng, shape, scale=1.0):
    return scale * rng.standard_normal(shape)


def battery(O) -> list[str]:
    """Run the pin battery against oracle module ``O``; return the names of failed pins."""
    failed = []

    # 1. Hand-derived worked examples of Eq. (1) (tests/golden).
    for case in load_golden()["cases"]:
        q, k, v, gq, gk = golden_case_inputs(case)
        got = O.forward(q, k, v, gq, gk, case["H"], case["eps"])[0]
        if not np.allclose(got, np.asarray(case["expected"]), rtol=1e-12, atol=1e-12):
            failed.append("golden:" + case["name"])

    # 2. Quadratic form, brute force, several shapes and both norm modes.
    rng = np.random.default_rng(1234)
    for (B, N, H, D, norm, kscale) in [(1, 1, 1, 4, True, 1.0), (2, 3, 2, 4, True, 1.0),
                                      (1, 17, 2, 32, True, 1.0), (1, 17, 1, 1, True, 1.0),
                                      (2, 9, 3, 5, False, 1.0), (1, 33, 2, 32, False, 100.0)]:
        C = H * D
        q, k, v = _rand(rng, (B, N, C)), _rand(rng, (B, N, C), kscale), _rand(rng, (B, N, C))
        gq = 1 + 0.1 * rng.standard_normal(C) if norm else None
        gk = 1 + 0.1 * rng.standard_normal(C) if norm else None
        eps = 1e-3
        ref = quadratic_form(q, k, v, gq, gk, H, eps)
        got = O.forward(q, k, v, gq, gk, H, eps)
        if rel_err(got, ref) > 1e-11:
            failed.append(f"quadratic:B{B}N{N}H{H}D{D}norm{norm}")

    # 3. Closed form N = 1: O = V * den / (den + eps), den = phi(q).phi(k).
    C, H = 8, 2
    q, k, v = np.abs(_rand(rng, (1, 1, C))) + 0.1, np.abs(_rand(rng, (1, 1, C))) + 0.1, \
        _rand(rng, (1, 1, C))
    eps = 0.5
    got = O.forward(q, k, v, None, None, H, eps)
    want = np.empty_like(v)
    for h in range(H):
        sl = slice(h * 4, (h + 1) * 4)
        den = float(q[0, 0, sl] @ k[0, 0, sl])
        want[0, 0, sl] = v[0, 0, sl] * den / (den + eps)
    if rel_err(got, want) > 1e-13:
        failed.append("closed:N1")

    # 4. The feature map alone against torch's rms_norm (per head and full-C).
    x = _rand(rng, (5, 12))
    g = 1 + 0.1 * rng.standard_normal(12)
    for scope in ("head", "full"):
        if rel_err(O.phi(x, g, 3, 1e-6, scope=scope), phi_lib(x, g, 3, 1e-6, scope)) > 1e-13:
            failed.append("phi:" + scope)
    return failed
