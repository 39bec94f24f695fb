"""fp64 CPU oracle for SANA's multi-head ReLU linear attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA library (``relu_linear_attention_attn_b200``) and imports nothing from
it; both sides are fed the same seeded inputs by the tests.

The arithmetic lives in ``sana_oracle.c`` (plain fp64 loops written from
Eq. (1) of "Sana: Efficient High-Resolution Image Synthesis with Linear
Diffusion Transformers", section 2.1, and the QK-Norm bullet of "SANA 1.5:
Efficient Scaling of Training-Time and Inference-Time Compute in Linear
Diffusion Transformer", section "Model architecture").  This file marshals
arrays to fp64 and adds one library step: the QKV projection ``x @ Wqkv`` of
the fused variant (section 7, on-device deployment, of the Sana notes: the
ReLU(K)^T V reduction fused with the QKV projection), done as an fp64 numpy
matmul.

``quadratic_forward`` is Eq. (1) in its O(N^2) form, the CPU brute force the
benchmark times on the tiny workload; it is pinned against ``forward`` and the
tests' independent quadratic form.

Pins (checked by ``tests/test_oracle_pins.py``): the quadratic form of Eq. (1)
brute-forced on tiny inputs, hand-derived worked examples in
``tests/golden/``, closed forms (N = 1, one-hot keys, constant values),
invariants (linearity in V, token permutation, scale invariance), and
torch's own ``rms_norm`` for the feature map.

The W8A8 prologue (``quantize_i8``, ``w8a8_project``, ``w8a8_fused_forward``)
is pinned by ``tests/test_oracle_w8a8.py``: hand-derived codes and a
hand-derived projection (``tests/golden/w8a8_quantize.json``), a pure-Python
integer brute force, the half-step rounding bound, and equality with the fused
forward on the dequantised tensors.

The prefix (causal) form ``causal_forward`` (C: ``oracle_causal_forward_f64``,
the running state over tokens) is pinned by ``tests/test_oracle_causal.py``:
hand-derived examples, a masked quadratic form with a textbook RMSNorm, the last
token against the non-causal forward, the first token's closed form, causality.

The Mix-FFN (``linear``, ``depthwise_conv3x3``, ``glu``, ``dwconv_glu``,
``mixffn_forward``) is pinned by ``tests/test_oracle_mixffn.py``: a hand-derived
3x3 worked example (cross-correlation orientation, zero padding, exact gate
values), a pure-Python brute force, torch's grouped ``conv2d``, ``glu`` and
``silu``, and closed forms of a constant input and of a centre-only kernel.

The backward (``backward``: hand-derived gradients of the forward with respect to
q, k, v and the gains) is pinned by ``tests/test_oracle_backward.py``: automatic
differentiation of an independently written fp64 torch forward, central
finite differences of ``forward``, and the closed form of dV.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sana_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_sana_oracle.so")

NORM_OFF = 0
NORM_PER_HEAD = 1
NORM_FULL_C = 2

_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile sana_oracle.c into oracle/_sana_oracle.so with gcc (no fast-math,
    no FMA contraction, so fp64 operations happen in the written order)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-o", tmp, _SRC, "-lpthread", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(lib):
    """Declare the C signatures on a loaded oracle library."""
    dp = ctypes.POINTER(ctypes.c_double)
    i64p = ctypes.POINTER(ctypes.c_int64)
    i64, ci, cd = ctypes.c_int64, ctypes.c_int, ctypes.c_double
    lib.oracle_phi_f64.argtypes = [dp, dp, dp, i64, ci, ci, cd, ci, ci]
    lib.oracle_kv_state_f64.argtypes = [dp, dp, dp, dp, i64, i64, ci, ci, cd, ci, ci]
    lib.oracle_apply_f64.argtypes = [dp, dp, dp, dp, i64p, i64, i64, i64, ci, ci, cd, ci, ci]
    lib.oracle_forward_f64.argtypes = [dp, dp, dp, dp, dp, dp, i64, i64, ci, ci, cd, ci, ci]
    lib.oracle_causal_forward_f64.argtypes = [dp, dp, dp, dp, dp, dp, i64, i64, ci, ci, cd, ci,
                                              ci]
    for f in (lib.oracle_phi_f64, lib.oracle_kv_state_f64, lib.oracle_apply_f64,
              lib.oracle_forward_f64, lib.oracle_causal_forward_f64):
        f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


def host_threads() -> int:
    """Threads the oracle uses by default: the cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _f64(a) -> np.ndarray:
    """Any array-like (numpy, torch CPU tensor of any float dtype) -> C-contiguous fp64.
    bf16 and fp32 values are exactly representable in fp64, so nothing is rounded."""
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor, converted without importing torch here
        a = a.detach().cpu()
        if str(a.dtype) in ("torch.bfloat16", "torch.float16"):
            a = a.float()
        a = a.double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _norm_mode(gq, gk, scope: str) -> int:
    if gq is None and gk is None:
        return NORM_OFF
    if gq is None or gk is None:
        raise ValueError("gq and gk must both be given (norm on) or both be None (norm off)")
    if scope == "head":
        return NORM_PER_HEAD
    if scope == "full":
        return NORM_FULL_C
    raise ValueError("scope must be 'head' or 'full'")


def phi(x, g, H: int, eps: float, scope: str = "head", nthreads: int = 0) -> np.ndarray:
    """phi(x) = ReLU(RMSNorm(x) * g) per token; g None = norm off (plain ReLU).
    x: (..., C).  Returns fp64 of the same shape."""
    x = _f64(x)
    g = _f64(g)
    C = x.shape[-1]
    mode = NORM_OFF if g is None else (NORM_PER_HEAD if scope == "head" else NORM_FULL_C)
    out = np.empty_like(x)
    T = x.size // C if C else 0
    rc = _load().oracle_phi_f64(_ptr(x), _ptr(g), _ptr(out), T, C, H, float(eps), mode,
                                nthreads or host_threads())
    if rc != 0:
        raise ValueError("oracle_phi_f64 rejected its arguments")
    return out


def kv_state(k, v, gk, H: int, eps: float, scope: str = "head", nthreads: int = 0,
             norm: bool | None = None) -> np.ndarray:
    """S[b,h] = sum_n phi(K_n)^T [V_n | 1], shape (B, H, D, D+1), fp64.
    Norm is on iff gk is given (pass norm=False to force it off)."""
    k = _f64(k)
    v = _f64(v)
    gk = _f64(gk)
    B, N, C = k.shape
    if v.shape != k.shape:
        raise ValueError("k and v must have the same shape")
    D = C // H
    mode = NORM_OFF if (gk is None or norm is False) else (
        NORM_PER_HEAD if scope == "head" else NORM_FULL_C)
    S = np.empty((B, H, D, D + 1), dtype=np.float64)
    rc = _load().oracle_kv_state_f64(_ptr(k), _ptr(v), _ptr(gk), _ptr(S), B, N, C, H,
                                     float(eps), mode, nthreads or host_threads())
    if rc != 0:
        raise ValueError("oracle_kv_state_f64 rejected its arguments")
    return S


def apply(q, gq, S, H: int, eps: float, tokens=None, scope: str = "head",
          nthreads: int = 0) -> np.ndarray:
    """O = phi(Q) S[:, :D] / (phi(Q) S[:, D] + eps).
    q: (B, N, C); S: (B, H, D, D+1).  tokens: optional flat indices b*N+n; then the
    result is (len(tokens), C), otherwise (B, N, C)."""
    q = _f64(q)
    gq = _f64(gq)
    S = _f64(S)
    B, N, C = q.shape
    mode = NORM_OFF if gq is None else (NORM_PER_HEAD if scope == "head" else NORM_FULL_C)
    if tokens is None:
        out = np.empty((B, N, C), dtype=np.float64)
        tp, T = None, 0
    else:
        tok = np.ascontiguousarray(np.asarray(tokens, dtype=np.int64))
        T = tok.size
        out = np.empty((T, C), dtype=np.float64)
        tp = tok.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))
    rc = _load().oracle_apply_f64(_ptr(q), _ptr(gq), _ptr(S), _ptr(out), tp, T, B, N, C, H,
                                  float(eps), mode, nthreads or host_threads())
    if rc != 0:
        raise ValueError("oracle_apply_f64 rejected its arguments")
    return out


def forward(q, k, v, gq, gk, H: int, eps: float, scope: str = "head",
            nthreads: int = 0) -> np.ndarray:
    """Eq. (1) with QK-RMSNorm: (B, N, C) fp64 output.  gq = gk = None: norm off."""
    mode = _norm_mode(gq, gk, scope)
    q, k, v, gq, gk = (_f64(a) for a in (q, k, v, gq, gk))
    B, N, C = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same (B, N, C) shape")
    out = np.empty((B, N, C), dtype=np.float64)
    rc = _load().oracle_forward_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(gq), _ptr(gk), _ptr(out),
                                    B, N, C, H, float(eps), mode, nthreads or host_threads())
    if rc != 0:
        raise ValueError("oracle_forward_f64 rejected its arguments")
    return out


def quadratic_forward(q, k, v, gq, gk, H: int, eps: float) -> np.ndarray:
    """Eq. (1) as the O(N^2) sum it reorders: per (b, h), A_ij = phi(Q_i).phi(K_j),
    O_i = sum_j A_ij V_j / (sum_j A_ij + eps).  Equal to ``forward`` up to rounding
    (associativity); used as the brute-force CPU timing on small inputs."""
    pq, pk, vv = phi(q, gq, H, eps), phi(k, gk, H, eps), _f64(v)
    B, N, C = pq.shape
    D = C // H
    out = np.empty_like(vv)
    for b in range(B):
        for h in range(H):
            cols = slice(h * D, (h + 1) * D)
            A = np.matmul(pq[b, :, cols], pk[b, :, cols].T)
            out[b, :, cols] = np.matmul(A, vv[b, :, cols]) / (A.sum(axis=1)[:, None] + eps)
    return out


def causal_forward(q, k, v, gq, gk, H: int, eps: float, nthreads: int = 0) -> np.ndarray:
    """The prefix form: token n attends to keys j <= n only (the running sums
    of the state), per-head QK-RMSNorm as in forward().  (B, N, C) fp64."""
    mode = _norm_mode(gq, gk, "head")
    q, k, v, gq, gk = (_f64(a) for a in (q, k, v, gq, gk))
    B, N, C = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same (B, N, C) shape")
    out = np.empty((B, N, C), dtype=np.float64)
    rc = _load().oracle_causal_forward_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(gq), _ptr(gk),
                                           _ptr(out), B, N, C, H, float(eps), mode,
                                           nthreads or host_threads())
    if rc != 0:
        raise ValueError("oracle_causal_forward_f64 rejected its arguments")
    return out


def qkv_project(x, W, rows=None) -> np.ndarray:
    """[Q | K | V] = x @ Wqkv in fp64 (a library matmul step).
    x: (B, N, C); W: (C, 3C) with columns [0,C) = Q, [C,2C) = K, [2C,3C) = V.
    rows: optional column range (lo, hi) of W to project onto."""
    x = _f64(x)
    W = _f64(W)
    if rows is not None:
        W = W[:, rows[0]:rows[1]]
    return np.matmul(x, W)


def fused_forward(x, W, gq, gk, H: int, eps: float, tokens=None, nthreads: int = 0):
    """The fused variant end to end: projection, then Eq. (1) with QK-RMSNorm.
    The projected Q, K, V stay in fp64 (no intermediate rounding).
    tokens: optional flat token indices; then only those rows of O are formed
    (K and V are still projected for every token, since the state needs them)."""
    x = _f64(x)
    B, N, C = x.shape
    kvp = qkv_project(x, W, rows=(C, 3 * C))
    k, v = kvp[..., :C], kvp[..., C:]
    S = kv_state(np.ascontiguousarray(k), np.ascontiguousarray(v), gk, H, eps,
                 nthreads=nthreads, norm=gk is not None)
    if tokens is None:
        q = qkv_project(x, W, rows=(0, C))
        return apply(q, gq, S, H, eps, nthreads=nthreads)
    tok = np.asarray(tokens, dtype=np.int64)
    xs = x.reshape(B * N, C)[tok]
    q = qkv_project(xs, W, rows=(0, C))
    # apply() indexes q by flat token; give it a (B, N, C) view with only the
    # sampled rows filled, which it never reads past.
    qfull = np.zeros((B * N, C), dtype=np.float64)
    qfull[tok] = q
    return apply(qfull.reshape(B, N, C), gq, S, H, eps, tokens=tok, nthreads=nthreads)


# ----------------------------------------------------------------------------- W8A8
# The W8A8 prologue of the fused variant ("Sana: Efficient High-Resolution Image
# Synthesis with Linear Diffusion Transformers", section 7, on-device deployment:
# linear layers in 8-bit weights and activations, attention kept in full
# precision).  The pages do not state the scale granularity; the reading here is
# symmetric int8 with one scale per token of x and one per output channel of Wqkv.
# Codes are integers decided by floating point, so they are formed in fp32 exactly
# as stated below (IEEE division, round half to even), the precision the kernels
# use, and compared bit for bit.

def quantize_i8(x, axis: int = -1):
    """Symmetric int8 codes along `axis`: scale = max|x| / 127 (fp32), code =
    round_half_even(x / scale) in fp32, clipped to [-127, 127].  A slice that is
    all zero gets scale 0 and zero codes.  Returns (codes int8, scales fp32 with
    `axis` removed)."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x32), axis=axis, keepdims=True)
    s = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    q = np.rint((x32 / safe).astype(np.float32))
    q = np.where(s > 0, q, np.float32(0.0))
    q = np.clip(q, -127, 127).astype(np.int8)
    return q, np.squeeze(s, axis=axis)


def w8a8_project(xq, sx, Wq, sw, rows=None) -> np.ndarray:
    """Dequantised projection of int8 codes: (xq @ Wq)[n, c] * sx[n] * sw[c].
    xq: (..., C) int8, sx: (...) scales; Wq: (C, 3C) int8, sw: (3C,) scales.
    The integer products sum exactly in fp64 (|sum| <= 127^2 * C < 2^53)."""
    xq = np.asarray(xq).astype(np.float64)
    Wq = np.asarray(Wq).astype(np.float64)
    sw = np.asarray(sw, dtype=np.float64)
    if rows is not None:
        Wq = Wq[:, rows[0]:rows[1]]
        sw = sw[rows[0]:rows[1]]
    acc = np.matmul(xq, Wq)
    return acc * np.asarray(sx, dtype=np.float64)[..., None] * sw


def w8a8_fused_forward(xq, sx, Wq, sw, gq, gk, H: int, eps: float, tokens=None,
                       nthreads: int = 0):
    """The fused variant on int8 codes: dequantised projection, then Eq. (1) with
    QK-RMSNorm in fp64.  tokens: optional flat token indices of O to form."""
    xq = np.asarray(xq)
    B, N, C = xq.shape
    kvp = w8a8_project(xq, sx, Wq, sw, rows=(C, 3 * C))
    k, v = kvp[..., :C], kvp[..., C:]
    S = kv_state(np.ascontiguousarray(k), np.ascontiguousarray(v), gk, H, eps,
                 nthreads=nthreads, norm=gk is not None)
    if tokens is None:
        q = w8a8_project(xq, sx, Wq, sw, rows=(0, C))
        return apply(q, gq, S, H, eps, nthreads=nthreads)
    tok = np.asarray(tokens, dtype=np.int64)
    q = w8a8_project(xq.reshape(B * N, C)[tok], np.asarray(sx).reshape(B * N)[tok], Wq, sw,
                     rows=(0, C))
    qfull = np.zeros((B * N, C), dtype=np.float64)
    qfull[tok] = q
    return apply(qfull.reshape(B, N, C), gq, S, H, eps, tokens=tok, nthreads=nthreads)


# ----------------------------------------------------------------------------- backward
# Gradients of Eq. (1) with the per-head QK-RMSNorm feature map, for training with
# the op ("Sana ..." section 2.1 defines only the forward; the gradients below are
# derived from it).  Per (b, h), with u = g * x * r, r = (mean_d x^2 + eps)^(-1/2),
# phi = ReLU(u), S = sum_j phi(K_j)^T V_j, z = sum_j phi(K_j):
#   num_i = phi(Q_i) S,  den_i = phi(Q_i) . z + eps,  O_i = num_i / den_i
#   dnum_i = dO_i / den_i,               dden_i = -(dO_i . O_i) / den_i
#   dphi(Q_i) = dnum_i S^T + dden_i z
#   dS = sum_i phi(Q_i)^T dnum_i,        dz = sum_i phi(Q_i) dden_i
#   dphi(K_j) = dS V_j + dz,             dV_j = phi(K_j) dS
# and through the feature map (du = dphi where u > 0, else 0):
#   dg[d] += du[d] x[d] r,   dx[c] = g[c] r du[c] - (r^3 x[c] / D) sum_d du[d] g[d] x[d]
# (norm off: dx = dphi where x > 0).

def _phi_fwd(x, g, H: int, eps: float):
    """(phi, u, r) of x (B, N, C) per head; r has shape (B, N, H, 1)."""
    B, N, C = x.shape
    D = C // H
    xh = x.reshape(B, N, H, D)
    if g is None:
        return np.maximum(xh, 0.0), xh, None
    r = 1.0 / np.sqrt((xh * xh).mean(-1, keepdims=True) + eps)
    u = g.reshape(1, 1, H, D) * xh * r
    return np.maximum(u, 0.0), u, r


def _phi_bwd(dphi, x, g, u, r, H: int):
    """(dx (B, N, C), dg (C,) or None) through the feature map."""
    B, N, C = x.shape
    D = C // H
    xh = x.reshape(B, N, H, D)
    du = np.where(u > 0.0, dphi, 0.0)
    if g is None:
        return du.reshape(B, N, C), None
    gh = g.reshape(1, 1, H, D)
    dg = (du * xh * r).sum(axis=(0, 1)).reshape(C)
    t = (du * gh * xh).sum(-1, keepdims=True)
    dx = gh * r * du - (r ** 3) * xh * t / D
    return dx.reshape(B, N, C), dg


def backward(q, k, v, gq, gk, dout, H: int, eps: float):
    """Gradients of the forward() output with respect to q, k, v and the gains:
    returns (dq, dk, dv, dgq, dgk), fp64; dgq, dgk are None with the norm off."""
    q, k, v, dout = (_f64(a) for a in (q, k, v, dout))
    gq, gk = _f64(gq), _f64(gk)
    B, N, C = q.shape
    D = C // H
    pq, uq, rq = _phi_fwd(q, gq, H, eps)
    pk, uk, rk = _phi_fwd(k, gk, H, eps)
    vh = v.reshape(B, N, H, D)
    do = dout.reshape(B, N, H, D)
    S = np.einsum("bnhd,bnhe->bhde", pk, vh)
    z = pk.sum(axis=1)                                        # (B, H, D)
    num = np.einsum("bnhd,bhde->bnhe", pq, S)
    den = np.einsum("bnhd,bhd->bnh", pq, z)[..., None] + eps
    o = num / den
    dnum = do / den
    dden = -(do * o).sum(-1, keepdims=True) / den
    dpq = np.einsum("bnhe,bhde->bnhd", dnum, S) + dden * z[:, None]
    dS = np.einsum("bnhd,bnhe->bhde", pq, dnum)
    dz = np.einsum("bnhd,bnh->bhd", pq, dden[..., 0])
    dpk = np.einsum("bhde,bnhe->bnhd", dS, vh) + dz[:, None]
    dv = np.einsum("bnhd,bhde->bnhe", pk, dS)
    dq, dgq = _phi_bwd(dpq, q, gq, uq, rq, H)
    dk, dgk = _phi_bwd(dpk, k, gk, uk, rk, H)
    return dq, dk, dv.reshape(B, N, C), dgq, dgk


# ----------------------------------------------------------------------------- Mix-FFN
# The Mix-FFN of the Linear DiT block ("Sana: Efficient High-Resolution Image
# Synthesis with Linear Diffusion Transformers", section 2.2: an inverted residual
# block, a 3x3 depthwise convolution and a GLU take the place of the MLP FFN;
# section 2.3: the convolution's zero padding is what carries position; "SANA 1.5",
# section "Model architecture": C = 2240, FFN width 5600).  The pages leave the
# rest open; the reading here, with tokens n = y * Ws + x on an (Hs, Ws) grid:
#   U  = X W1 + b1                                  1x1 expand, C -> 2F
#   Cv[y, x, c] = bdw[c] + sum_{i, j in 0..2} wdw[c, i, j] U[y + i - 1, x + j - 1, c]
#                                                   depthwise 3x3 cross-correlation,
#                                                   zero outside the grid
#   Hg = Cv[..., :F] * gate(Cv[..., F:])            GLU: the first half gated by the
#                                                   second; gate = sigmoid (the GLU's
#                                                   definition) or SiLU
#   Y  = Hg W2 + b2                                 1x1 project, F -> C
# Biases are optional (None: no bias).

def linear(x, W, b=None) -> np.ndarray:
    """x @ W (+ b) in fp64: x (..., K), W (K, Nc) row-major, b (Nc,) or None."""
    y = np.matmul(_f64(x), _f64(W))
    if b is not None:
        y = y + _f64(b)
    return y


def depthwise_conv3x3(u, wdw, bdw, Hs: int, Ws: int) -> np.ndarray:
    """Depthwise 3x3 cross-correlation with zero padding of u (B, Hs*Ws, Cc) on the
    row-major (Hs, Ws) token grid; wdw (Cc, 3, 3), tap (i, j) reads the token at
    (y + i - 1, x + j - 1); bdw (Cc,) or None."""
    u = _f64(u)
    B, N, Cc = u.shape
    if N != Hs * Ws:
        raise ValueError("N must equal Hs * Ws")
    w = _f64(wdw).reshape(Cc, 3, 3)
    padded = np.zeros((B, Hs + 2, Ws + 2, Cc))
    padded[:, 1:Hs + 1, 1:Ws + 1, :] = u.reshape(B, Hs, Ws, Cc)
    out = np.zeros((B, Hs, Ws, Cc))
    for i in range(3):
        for j in range(3):
            out += w[:, i, j] * padded[:, i:i + Hs, j:j + Ws, :]
    if bdw is not None:
        out += _f64(bdw)
    return out.reshape(B, N, Cc)


def glu(c, gate: str = "sigmoid") -> np.ndarray:
    """GLU over the last axis (2F -> F): value c[..., :F] times gate(c[..., F:]),
    gate = sigmoid(z) = 1 / (1 + exp(-z)) or silu(z) = z * sigmoid(z)."""
    c = _f64(c)
    F = c.shape[-1] // 2
    a, z = c[..., :F], c[..., F:]
    with np.errstate(over="ignore"):
        sig = 1.0 / (1.0 + np.exp(-z))
    if gate == "sigmoid":
        return a * sig
    if gate == "silu":
        return a * (z * sig)
    raise ValueError(f"unknown gate {gate!r}")


def dwconv_glu(u, wdw, bdw, Hs: int, Ws: int, gate: str = "sigmoid") -> np.ndarray:
    """The Mix-FFN middle: GLU of the depthwise 3x3 convolution of u (B, N, 2F)."""
    return glu(depthwise_conv3x3(u, wdw, bdw, Hs, Ws), gate)


def mixffn_forward(x, W1, b1, wdw, bdw, W2, b2, Hs: int, Ws: int, gate: str = "sigmoid",
                   tokens=None) -> np.ndarray:
    """The whole Mix-FFN: x (B, N, C) -> (B, N, C).  tokens: optional flat token
    indices (b * N + n) of Y to form; only the expand of their 3x3 neighbourhoods is
    computed, and the result has shape (len(tokens), C)."""
    x = _f64(x)
    B, N, C = x.shape
    if tokens is None:
        return linear(dwconv_glu(linear(x, W1, b1), wdw, bdw, Hs, Ws, gate), W2, b2)
    tok = np.asarray(tokens, dtype=np.int64)
    rows = []
    for t in tok:
        b, n = divmod(int(t), N)
        y0, x0 = divmod(n, Ws)
        # the 3x3 neighbourhood as its own 3x3 grid, zero where it leaves the grid
        xs = np.zeros((1, 9, C))
        for i in range(3):
            for j in range(3):
                yy, xx = y0 + i - 1, x0 + j - 1
                if 0 <= yy < Hs and 0 <= xx < Ws:
                    xs[0, 3 * i + j] = x[b, yy * Ws + xx]
        u = linear(xs, W1, b1)
        inside = np.array([[0 <= y0 + i - 1 < Hs and 0 <= x0 + j - 1 < Ws for j in range(3)]
                           for i in range(3)], dtype=np.float64).reshape(1, 9, 1)
        u = u * inside                      # outside the grid U is zero, bias included
        c = depthwise_conv3x3(u, wdw, bdw, 3, 3)[:, 4]
        rows.append(linear(glu(c, gate), W2, b2)[0])
    return np.stack(rows) if rows else np.zeros((0, _f64(W2).shape[-1]))
