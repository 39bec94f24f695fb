"""Pins of the oracle's backward (CPU only).

The hand-derived gradients are checked against automatic differentiation of an
independently written fp64 torch forward (norm on and off), central finite
differences of the oracle's own forward, and the closed form of dV (O is linear
in V); plausible mistakes planted in a copy of the oracle's backward must fail."""
import types

import numpy as np
import pytest
import torch

from oracle import oracle as O


def _autograd(q, k, v, gq, gk, do, H, eps):
    B, N, C = q.shape
    D = C // H
    T = lambda a: None if a is None else torch.tensor(a, dtype=torch.float64, requires_grad=True)
    tq, tk, tv, tgq, tgk = T(q), T(k), T(v), T(gq), T(gk)

    def phi(x, g):
        xh = x.reshape(B, N, H, D)
        if g is None:
            return torch.relu(xh)
        r = torch.rsqrt((xh * xh).mean(-1, keepdim=True) + eps)
        return torch.relu(g.reshape(H, D) * xh * r)
    pq, pk = phi(tq, tgq), phi(tk, tgk)
    vh = tv.reshape(B, N, H, D)
    S = torch.einsum("bnhd,bnhe->bhde", pk, vh)
    z = pk.sum(1)
    o = torch.einsum("bnhd,bhde->bnhe", pq, S) / (torch.einsum("bnhd,bhd->bnh", pq, z)[..., None] + eps)
    (o.reshape(B, N, C) * torch.tensor(do)).sum().backward()
    g = lambda t: None if t is None else t.grad.numpy()
    return g(tq), g(tk), g(tv), g(tgq), g(tgk)


def backward_battery(M) -> list:
    bad = []
    rng = np.random.default_rng(5)
    B, N, C, H = 2, 19, 64, 2
    for norm in (True, False):
        q, k, v, do = (rng.standard_normal((B, N, C)) for _ in range(4))
        gq = 1 + 0.1 * rng.standard_normal(C) if norm else None
        gk = 1 + 0.1 * rng.standard_normal(C) if norm else None
        got = M.backward(q, k, v, gq, gk, do, H, 1e-6)
        ref = _autograd(q, k, v, gq, gk, do, H, 1e-6)
        for name, a, b in zip(("dq", "dk", "dv", "dgq", "dgk"), got, ref):
            if (a is None) != (b is None) or (a is not None and not np.allclose(a, b, rtol=1e-9, atol=1e-12)):
                bad.append(f"{name} vs autograd (norm {norm})")
    # central differences of the forward on a tiny case
    B, N, C, H, eps, h = 1, 6, 64, 2, 1e-3, 1e-6
    q, k, v, do = (rng.standard_normal((B, N, C)) for _ in range(4))
    gq, gk = 1 + 0.1 * rng.standard_normal(C), 1 + 0.1 * rng.standard_normal(C)
    dq, dk, dv, dgq, dgk = M.backward(q, k, v, gq, gk, do, H, eps)
    loss = lambda q_, k_, v_, gq_, gk_: float((O.forward(q_, k_, v_, gq_, gk_, H, eps) * do).sum())
    for (name, grad, which) in (("dq", dq, 0), ("dk", dk, 1), ("dv", dv, 2), ("dgq", dgq, 3),
                                ("dgk", dgk, 4)):
        args = [q, k, v, gq, gk]
        flat = args[which].reshape(-1)
        for idx in (0, 17, 33, flat.size - 1):
            p, m = [a.copy() for a in args], [a.copy() for a in args]
            p[which].reshape(-1)[idx] += h
            m[which].reshape(-1)[idx] -= h
            fd = (loss(*p) - loss(*m)) / (2 * h)
            if abs(fd - grad.reshape(-1)[idx]) > 1e-6 * max(1.0, abs(fd)):
                bad.append(f"{name}[{idx}] vs central difference: {grad.reshape(-1)[idx]} {fd}")
    # dV closed form with the norm off: dV_j = sum_i (phi(Q_i).phi(K_j)) / den_i * dO_i
    B, N, C, H, eps = 1, 9, 32, 1, 0.25
    q, k, v, do = (rng.standard_normal((B, N, C)) for _ in range(4))
    _, _, dv, _, _ = M.backward(q, k, v, None, None, do, H, eps)
    pq, pk = np.maximum(q[0], 0), np.maximum(k[0], 0)
    A = pq @ pk.T
    den = A.sum(1) + eps
    if not np.allclose(dv[0], (A / den[:, None]).T @ do[0], rtol=1e-12, atol=1e-13):
        bad.append("dV closed form")
    return bad


def test_backward_pins_hold():
    assert backward_battery(O) == []


MUTATIONS = {
    "dden_sign": ("dden = -(do * o).sum(-1, keepdims=True) / den",
                  "dden = (do * o).sum(-1, keepdims=True) / den"),
    "dden_not_divided": ("dden = -(do * o).sum(-1, keepdims=True) / den",
                         "dden = -(do * o).sum(-1, keepdims=True)"),
    "dphiq_state_not_transposed": ('dpq = np.einsum("bnhe,bhde->bnhd", dnum, S)',
                                   'dpq = np.einsum("bnhe,bhed->bnhd", dnum, S)'),
    "dz_dropped_from_dk": ('dpk = np.einsum("bhde,bnhe->bnhd", dS, vh) + dz[:, None]',
                           'dpk = np.einsum("bhde,bnhe->bnhd", dS, vh)'),
    "relu_mask_missing": ("du = np.where(u > 0.0, dphi, 0.0)", "du = dphi"),
    "rms_term_dropped": ("dx = gh * r * du - (r ** 3) * xh * t / D", "dx = gh * r * du"),
    "gain_grad_without_r": ("dg = (du * xh * r).sum(axis=(0, 1)).reshape(C)",
                            "dg = (du * xh).sum(axis=(0, 1)).reshape(C)"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_backward_battery_catches_planted_mistake(name):
    old, new = MUTATIONS[name]
    src = open(O.__file__).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    mod = types.ModuleType(f"oracle_{name}")
    mod.__file__ = O.__file__
    exec(compile(src.replace(old, new), O.__file__, "exec"), mod.__dict__)
    assert backward_battery(mod), f"planted mistake {name} went unnoticed"
