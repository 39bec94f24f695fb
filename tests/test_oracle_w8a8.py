"""Pins of the oracle's W8A8 prologue (CPU only).

The quantisation rule and the dequantised projection are checked against
hand-derived values (tests/golden/w8a8_quantize.json), a pure-Python integer
brute force, the rounding-error bound of the rule, and the linearity of the
projection in its scales; plausible mistakes planted in a copy of the oracle's
W8A8 code must fail the battery."""
import json
import os
import types

import numpy as np
import pytest

from oracle import oracle as O

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "w8a8_quantize.json")))


def w8a8_battery(M) -> list:
    """Failures of the W8A8 pins for an oracle-like module M (empty = all pass)."""
    bad = []
    for c in GOLD["cases"]:
        q, s = M.quantize_i8(np.array([c["x"]], dtype=np.float32))
        if list(q[0].astype(int)) != c["codes"] or float(s[0]) != c["scale"]:
            bad.append(f"golden {c['name']}: {list(q[0])} scale {float(s[0])}")
    p = GOLD["projection_case"]
    out = M.w8a8_project(np.array(p["xq"], np.int8), np.array(p["sx"], np.float32),
                         np.array(p["Wq"], np.int8), np.array(p["sw"], np.float32))
    if not np.array_equal(out, np.array(p["out"])):
        bad.append(f"golden projection {out.tolist()}")
    # column scales: per output channel of W (axis 0 reduced)
    rng = np.random.default_rng(7)
    W = rng.standard_normal((24, 9)).astype(np.float32)
    qw, sw = M.quantize_i8(W, axis=0)
    if sw.shape != (9,) or not np.all(np.abs(qw).max(axis=0) == 127):
        bad.append("column quantisation does not reach +-127 per column")
    # rounding error bound and range on random rows
    x = (rng.standard_normal((64, 100)) * rng.lognormal(size=(64, 1))).astype(np.float32)
    q, s = M.quantize_i8(x)
    err = np.abs(x - q.astype(np.float32) * s[:, None])
    if np.any(err > s[:, None] * 0.5000005):
        bad.append("rounding error above half a step")
    if np.any(np.abs(q).max(axis=1) != 127) or q.min() < -127:
        bad.append("code range")
    if np.any(np.sign(q) * np.sign(x) < 0):
        bad.append("sign flipped")
    # integer brute force of the projection on a small case
    xq = rng.integers(-127, 128, size=(2, 3, 8)).astype(np.int8)
    sx = rng.random((2, 3)).astype(np.float32) + 0.1
    Wq = rng.integers(-127, 128, size=(8, 6)).astype(np.int8)
    swv = (rng.random(6).astype(np.float32) - 0.5)
    out = M.w8a8_project(xq, sx, Wq, swv)
    for b in range(2):
        for n in range(3):
            for c in range(6):
                acc = sum(int(xq[b, n, k]) * int(Wq[k, c]) for k in range(8))
                if out[b, n, c] != float(acc) * float(sx[b, n]) * float(swv[c]):
                    bad.append(f"projection ({b},{n},{c})")
    return bad


def test_w8a8_pins_hold():
    assert w8a8_battery(O) == []


def test_w8a8_forward_is_fused_forward_on_dequantised_inputs():
    rng = np.random.default_rng(3)
    B, N, C, H = 1, 40, 64, 2
    x = rng.standard_normal((B, N, C)).astype(np.float32)
    W = (0.05 * rng.standard_normal((C, 3 * C))).astype(np.float32)
    xq, sx = O.quantize_i8(x)
    Wq, sw = O.quantize_i8(W, axis=0)
    gq = (1 + 0.1 * rng.standard_normal(C)).astype(np.float32)
    gk = (1 + 0.1 * rng.standard_normal(C)).astype(np.float32)
    got = O.w8a8_fused_forward(xq, sx, Wq, sw, gq, gk, H, 1e-6)
    xd = xq.astype(np.float64) * sx[..., None]
    Wd = Wq.astype(np.float64) * sw[None, :]
    ref = O.fused_forward(xd, Wd, gq, gk, H, 1e-6)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)
    toks = [0, 7, 39]
    part = O.w8a8_fused_forward(xq, sx, Wq, sw, gq, gk, H, 1e-6, tokens=toks)
    np.testing.assert_allclose(part, got.reshape(N, C)[toks], rtol=1e-12, atol=1e-13)


MUTATIONS = {
    "scale_over_128": ("amax / np.float32(127.0)", "amax / np.float32(128.0)"),
    "truncate_not_round": ("q = np.rint((x32 / safe).astype(np.float32))",
                           "q = np.trunc((x32 / safe).astype(np.float32))"),
    "round_half_up": ("q = np.rint((x32 / safe).astype(np.float32))",
                      "q = np.floor((x32 / safe).astype(np.float32) + 0.5)"),
    "peak_without_abs": ("amax = np.max(np.abs(x32), axis=axis, keepdims=True)",
                         "amax = np.max(x32, axis=axis, keepdims=True)"),
    "token_scale_dropped": ("return acc * np.asarray(sx, dtype=np.float64)[..., None] * sw",
                            "return acc * sw"),
    "channel_scale_on_rows": ("return acc * np.asarray(sx, dtype=np.float64)[..., None] * sw",
                              "return acc * np.asarray(sx, dtype=np.float64)[..., None] * sw[0]"),
    "weights_transposed": ("acc = np.matmul(xq, Wq)", "acc = np.matmul(xq, Wq[::-1])"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_w8a8_battery_catches_planted_mistake(name):
    old, new = MUTATIONS[name]
    src = open(O.__file__).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    mod = types.ModuleType(f"oracle_{name}")
    mod.__file__ = O.__file__
    exec(compile(src.replace(old, new), O.__file__, "exec"), mod.__dict__)
    assert w8a8_battery(mod), f"planted mistake {name} went unnoticed"
