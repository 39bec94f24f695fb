"""Pins of the oracle's Mix-FFN ("Sana: Efficient High-Resolution Image Synthesis
with Linear Diffusion Transformers", sections 2.2 and 2.3: 1x1 expand, 3x3
depthwise convolution with zero padding, GLU, 1x1 project) against what the
mathematics fixes: a hand-derived worked example, a pure-Python brute force,
torch's grouped conv2d / glu / silu (a different implementation of the textbook
operations), closed forms, and plausible mistakes planted in a copy of the oracle,
each of which the battery must notice."""
import math
import types

import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

from oracle import oracle as O

LN3 = math.log(3.0)


def _worked_example(mod):
    """One value channel and one gate channel (F = 1) on a 3x3 grid.
    u(y, x) = 3y + x + 1 on the value channel, 0 on the gate channel; value kernel
    w(i, j) = 3i + j + 1, value bias 1/2; gate kernel 0, gate bias ln 3, so the gate
    is sigmoid(ln 3) = 3/4 and silu(ln 3) = (3/4) ln 3 everywhere.  By hand, the
    cross-correlation (tap (i, j) reads u(y + i - 1, x + j - 1), zero outside):
      (0,0) 5*1 + 6*2 + 8*4 + 9*5 = 94          (0,1) 4*1+5*2+6*3+7*4+8*5+9*6 = 154
      (0,2) 4*2 + 5*3 + 7*5 + 8*6 = 106         (1,0) 2*1+3*2+5*4+6*5+8*7+9*8 = 186
      (1,1) 1+4+9+16+25+36+49+64+81 = 285        (1,2) 1*2+2*3+4*5+5*6+7*8+8*9 = 186
      (2,0) 2*4 + 3*5 + 5*7 + 6*8 = 106         (2,1) 1*4+2*5+3*6+4*7+5*8+6*9 = 154
      (2,2) 1*5 + 2*6 + 4*8 + 5*9 = 94
    (a flipped kernel, true convolution, would give 26 at (0, 0))."""
    conv = np.array([94, 154, 106, 186, 285, 186, 106, 154, 94], dtype=np.float64) + 0.5
    u = np.zeros((1, 9, 2))
    u[0, :, 0] = np.arange(1, 10)
    wdw = np.zeros((2, 3, 3))
    wdw[0] = np.arange(1, 10).reshape(3, 3)
    bdw = np.array([0.5, LN3])
    bad = []
    if not np.allclose(mod.depthwise_conv3x3(u, wdw, bdw, 3, 3)[0, :, 0], conv, rtol=0, atol=1e-12):
        bad.append("worked example: convolution")
    if not np.allclose(mod.dwconv_glu(u, wdw, bdw, 3, 3, "sigmoid")[0, :, 0], 0.75 * conv,
                       rtol=1e-14, atol=0):
        bad.append("worked example: GLU (sigmoid gate)")
    if not np.allclose(mod.dwconv_glu(u, wdw, bdw, 3, 3, "silu")[0, :, 0], 0.75 * LN3 * conv,
                       rtol=1e-14, atol=0):
        bad.append("worked example: GLU (SiLU gate)")
    return bad


def _brute_force(mod):
    """Pure-Python loops on a non-square grid (the token index n = y * Ws + x)."""
    rng = np.random.default_rng(1)
    B, Hs, Ws, Cc = 2, 3, 4, 4
    u = rng.standard_normal((B, Hs * Ws, Cc))
    w = rng.standard_normal((Cc, 3, 3))
    bias = rng.standard_normal(Cc)
    ref = np.zeros_like(u)
    for b in range(B):
        for y in range(Hs):
            for x in range(Ws):
                for c in range(Cc):
                    s = bias[c]
                    for i in range(3):
                        for j in range(3):
                            yy, xx = y + i - 1, x + j - 1
                            if 0 <= yy < Hs and 0 <= xx < Ws:
                                s += w[c, i, j] * u[b, yy * Ws + xx, c]
                    ref[b, y * Ws + x, c] = s
    got = mod.depthwise_conv3x3(u, w, bias, Hs, Ws)
    return [] if np.allclose(got, ref, rtol=1e-13, atol=1e-13) else ["brute force"]


def _torch_composite(mod):
    """The whole Mix-FFN against torch's linear / grouped conv2d / glu / silu in
    fp64, with and without biases, both gates, a non-square grid."""
    rng = np.random.default_rng(2)
    B, Hs, Ws, C, F = 2, 5, 7, 16, 12
    x = rng.standard_normal((B, Hs * Ws, C))
    W1 = rng.standard_normal((C, 2 * F)) / 4
    b1 = rng.standard_normal(2 * F)
    wdw = rng.standard_normal((2 * F, 3, 3)) / 3
    bdw = rng.standard_normal(2 * F)
    W2 = rng.standard_normal((F, C)) / 4
    b2 = rng.standard_normal(C)
    bad = []
    for gate in ("sigmoid", "silu"):
        for biased in (True, False):
            bb1, bbd, bb2 = (b1, bdw, b2) if biased else (None, None, None)
            t = lambda a: None if a is None else torch.tensor(a)
            u = Fn.linear(torch.tensor(x), torch.tensor(W1).T, t(bb1))
            c = Fn.conv2d(u.reshape(B, Hs, Ws, 2 * F).permute(0, 3, 1, 2), torch.tensor(wdw)[:, None],
                          t(bbd), padding=1, groups=2 * F)
            c = c.permute(0, 2, 3, 1).reshape(B, Hs * Ws, 2 * F)
            h = Fn.glu(c, -1) if gate == "sigmoid" else c[..., :F] * Fn.silu(c[..., F:])
            ref = Fn.linear(h, torch.tensor(W2).T, t(bb2)).numpy()
            got = mod.mixffn_forward(x, W1, bb1, wdw, bbd, W2, bb2, Hs, Ws, gate)
            if not np.allclose(got, ref, rtol=1e-12, atol=1e-12):
                bad.append(f"torch composite ({gate}, bias={biased})")
            tok = [0, 6, 7, 20, 34, 35, 41, 69]
            got_s = mod.mixffn_forward(x, W1, bb1, wdw, bbd, W2, bb2, Hs, Ws, gate, tokens=tok)
            if not np.allclose(got_s, ref.reshape(-1, C)[tok], rtol=1e-12, atol=1e-12):
                bad.append(f"sampled tokens ({gate}, bias={biased})")
    return bad


def _closed_forms(mod):
    """A constant input sees only the taps inside the grid (corner: a 2x2 block of
    the kernel, edge: 2x3 or 3x2, interior: all 9); a centre-only kernel is the
    identity; the gate of a large positive pre-activation passes the value."""
    bad = []
    rng = np.random.default_rng(3)
    Hs, Ws, Cc = 4, 5, 3
    w = rng.standard_normal((Cc, 3, 3))
    got = mod.depthwise_conv3x3(np.ones((1, Hs * Ws, Cc)), w, None, Hs, Ws).reshape(Hs, Ws, Cc)
    exp = {(0, 0): w[:, 1:, 1:].sum((1, 2)), (0, 2): w[:, 1:, :].sum((1, 2)),
           (2, 0): w[:, :, 1:].sum((1, 2)), (2, 2): w.sum((1, 2)),
           (Hs - 1, Ws - 1): w[:, :2, :2].sum((1, 2)), (Hs - 1, 2): w[:, :2, :].sum((1, 2)),
           (2, Ws - 1): w[:, :, :2].sum((1, 2)), (0, Ws - 1): w[:, 1:, :2].sum((1, 2))}
    for (y, x), e in exp.items():
        if not np.allclose(got[y, x], e, rtol=1e-13, atol=1e-13):
            bad.append(f"constant input at ({y}, {x})")
    centre = np.zeros((Cc, 3, 3))
    centre[:, 1, 1] = 1.0
    u = rng.standard_normal((2, Hs * Ws, Cc))
    if not np.array_equal(mod.depthwise_conv3x3(u, centre, None, Hs, Ws), u):
        bad.append("centre-only kernel is not the identity")
    c = np.concatenate([rng.standard_normal((1, 5, 2)), np.full((1, 5, 2), 60.0)], axis=-1)
    if not np.allclose(mod.glu(c, "sigmoid"), c[..., :2], rtol=1e-15, atol=0):
        bad.append("sigmoid gate of +60 does not pass the value")
    if not np.allclose(mod.glu(c, "silu"), 60.0 * c[..., :2], rtol=1e-15, atol=0):
        bad.append("silu gate of +60 is not 60 x the value")
    return bad


def _linear_pin(mod):
    """The 1x1 convolutions as plain sums over the input channels."""
    rng = np.random.default_rng(4)
    x = rng.standard_normal((2, 3, 5))
    W = rng.standard_normal((5, 4))
    b = rng.standard_normal(4)
    ref = np.zeros((2, 3, 4))
    for i in range(2):
        for n in range(3):
            for c in range(4):
                ref[i, n, c] = b[c] + sum(x[i, n, k] * W[k, c] for k in range(5))
    return [] if np.allclose(mod.linear(x, W, b), ref, rtol=1e-13, atol=1e-13) else ["linear"]


def mixffn_battery(mod):
    return (_worked_example(mod) + _brute_force(mod) + _torch_composite(mod) +
            _closed_forms(mod) + _linear_pin(mod))


def test_mixffn_pins_hold():
    assert mixffn_battery(O) == []


MUTATIONS = {
    "kernel_flipped": ("out += w[:, i, j] * padded[:, i:i + Hs, j:j + Ws, :]",
                       "out += w[:, 2 - i, 2 - j] * padded[:, i:i + Hs, j:j + Ws, :]"),
    "kernel_transposed": ("out += w[:, i, j] * padded[:, i:i + Hs, j:j + Ws, :]",
                          "out += w[:, j, i] * padded[:, i:i + Hs, j:j + Ws, :]"),
    "grid_transposed": ("padded[:, 1:Hs + 1, 1:Ws + 1, :] = u.reshape(B, Hs, Ws, Cc)",
                        "padded[:, 1:Hs + 1, 1:Ws + 1, :] = "
                        "u.reshape(B, Ws, Hs, Cc).transpose(0, 2, 1, 3)"),
    "conv_bias_dropped": ("        out += _f64(bdw)\n", "        out += 0.0\n"),
    "value_and_gate_swapped": ("a, z = c[..., :F], c[..., F:]", "z, a = c[..., :F], c[..., F:]"),
    "gate_sign": ("sig = 1.0 / (1.0 + np.exp(-z))", "sig = 1.0 / (1.0 + np.exp(z))"),
    "silu_without_z": ("return a * (z * sig)", "return a * sig"),
    "expand_bias_dropped": ("        y = y + _f64(b)\n", "        y = y + 0.0\n"),
    "sampled_padding_keeps_bias": ("u = u * inside", "u = u * 1.0"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mixffn_battery_catches_planted_mistake(name):
    old, new = MUTATIONS[name]
    src = open(O.__file__).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    mod = types.ModuleType(f"oracle_{name}")
    mod.__file__ = O.__file__
    exec(compile(src.replace(old, new), O.__file__, "exec"), mod.__dict__)
    assert mixffn_battery(mod), f"planted mistake {name} went unnoticed"
