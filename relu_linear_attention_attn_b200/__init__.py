"""Python binding of the B200 SANA ReLU-linear-attention library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libsana_linattn.so`` (declared in ``include/sana_linattn.h``).
PyTorch provides device memory and the current stream.  There is no CPU or
PyTorch fallback: if the shared library is missing, ``load()`` raises.

    import relu_linear_attention_attn_b200 as sla
    out = sla.forward(q, k, v, gq, gk, H=70, eps=1e-6)     # (B, N, C) bf16/fp32
    out = sla.qkv_fused(x, Wqkv, gq, gk, H=70, eps=1e-6)   # bf16
    out = sla.forward_causal(q, k, v, gq, gk, H=70, eps=1e-6)
    dq, dk, dv, dgq, dgk = sla.backward(q, k, v, gq, gk, dout, H=70, eps=1e-6)
    y = sla.mixffn_forward(x, W1, b1, wdw, bdw, W2, b2, Hs=64, Ws=64)   # Mix-FFN tail

The Mix-FFN calls are declared in ``include/sana_mixffn.h``.
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = ["load", "lib_path", "workspace_bytes", "forward", "forward_noalloc", "forward_pass1", "forward_pass2", "forward_kernels", "kv_state", "apply", "qkv_fused",
           "qkv_fused_w8a8", "quantize_rows_i8", "quantize_cols_i8", "forward_causal",
           "backward", "gemm_bias", "mixffn_dwconv_glu", "mixffn_workspace_bytes",
           "mixffn_forward", "GATES",
           "device_error", "selftest_wait_timeout", "selftest_launch_failure", "SanaError", "STATUS", "BF16", "F32"]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libsana_linattn.so"

BF16, F32 = 0, 1
GATES = {"sigmoid": 0, "silu": 1}
STATUS = {0: "SANA_OK", -1: "SANA_EINVAL", -2: "SANA_EALIGN", -3: "SANA_EUNSUPPORTED",
          -4: "SANA_EWORKSPACE", -5: "SANA_ECUDA", -6: "SANA_ESCRATCH"}

_lib = None
_lock = threading.Lock()


class SanaError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} -> {STATUS.get(status, status)} ({status}): {msg}")
        self.status = status


def lib_path() -> str:
    return os.path.join(_PKG, _LIB_NAME)


def _declare(lib):
    vp, fp = ctypes.c_void_p, ctypes.c_void_p
    i64, ci, cf, sz = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.sana_linattn_workspace_bytes.argtypes = [i64, i64, ci, ci, ci]
    lib.sana_linattn_workspace_bytes.restype = sz
    lib.sana_linattn_forward.argtypes = [vp, vp, vp, fp, fp, vp, i64, i64, ci, ci, cf, ci, vp, sz,
                                         vp]
    lib.sana_linattn_kv_state.argtypes = [vp, vp, fp, fp, i64, i64, ci, ci, cf, ci, vp, sz, vp]
    lib.sana_linattn_apply.argtypes = [vp, fp, fp, vp, i64, i64, ci, ci, cf, ci, vp]
    lib.sana_linattn_forward_pass1.argtypes = [vp, vp, fp, i64, i64, ci, ci, cf, vp, sz, vp]
    lib.sana_linattn_forward_pass2.argtypes = [vp, fp, vp, i64, i64, ci, ci, cf, vp, sz, vp]
    lib.sana_linattn_forward_pass1.restype = ctypes.c_int
    lib.sana_linattn_forward_pass2.restype = ctypes.c_int
    lib.sana_linattn_qkv_fused.argtypes = [vp, vp, fp, fp, vp, i64, i64, ci, ci, cf, vp, sz, vp]
    for f in (lib.sana_linattn_forward, lib.sana_linattn_kv_state, lib.sana_linattn_apply,
              lib.sana_linattn_qkv_fused):
        f.restype = ctypes.c_int
    lib.sana_linattn_backward_workspace_bytes.argtypes = [i64, i64, ci, ci]
    lib.sana_linattn_backward_workspace_bytes.restype = sz
    lib.sana_linattn_backward.argtypes = [vp, vp, vp, fp, fp, vp, vp, vp, vp, fp, fp, i64, i64,
                                          ci, ci, cf, ci, vp, sz, vp]
    lib.sana_linattn_backward.restype = ctypes.c_int
    lib.sana_linattn_backward_with_state.argtypes = [vp, vp, vp, fp, fp, fp, vp, vp, vp, vp, fp,
                                                     fp, i64, i64, ci, ci, cf, ci, vp, sz, vp]
    lib.sana_linattn_backward_with_state.restype = ctypes.c_int
    lib.sana_linattn_forward_causal.argtypes = [vp, vp, vp, fp, fp, vp, i64, i64, ci, ci, cf, ci,
                                                vp, sz, vp]
    lib.sana_linattn_forward_causal.restype = ctypes.c_int
    lib.sana_linattn_qkv_fused_w8a8.argtypes = [vp, fp, vp, fp, fp, fp, vp, i64, i64, ci, ci, cf,
                                                vp, sz, vp]
    lib.sana_linattn_qkv_fused_w8a8.restype = ctypes.c_int
    lib.sana_quantize_rows_i8.argtypes = [vp, ci, vp, fp, i64, ci, vp]
    lib.sana_quantize_rows_i8.restype = ctypes.c_int
    lib.sana_quantize_cols_i8.argtypes = [vp, ci, vp, fp, i64, ci, vp]
    lib.sana_quantize_cols_i8.restype = ctypes.c_int
    lib.sana_linattn_forward_noalloc.argtypes = [vp, vp, vp, fp, fp, vp, i64, i64, ci, ci, cf, ci,
                                                 vp]
    lib.sana_linattn_forward_noalloc.restype = ctypes.c_int
    lib.sana_linattn_device_error.argtypes = [ctypes.POINTER(ci), ctypes.POINTER(ci), ci]
    lib.sana_linattn_device_error.restype = ctypes.c_int
    lib.sana_linattn_selftest_launch_failure.argtypes = [vp]
    lib.sana_linattn_selftest_launch_failure.restype = ctypes.c_int
    lib.sana_linattn_selftest_wait_timeout.argtypes = [i64, vp]
    lib.sana_linattn_selftest_wait_timeout.restype = ctypes.c_int
    lib.sana_gemm_bias_bf16.argtypes = [vp, vp, fp, vp, i64, ci, ci, vp]
    lib.sana_gemm_bias_bf16.restype = ctypes.c_int
    lib.sana_mixffn_dwconv_glu.argtypes = [vp, fp, fp, vp, i64, ci, ci, ci, ci, vp]
    lib.sana_mixffn_dwconv_glu.restype = ctypes.c_int
    lib.sana_mixffn_workspace_bytes.argtypes = [i64, ci, ci, ci, ci]
    lib.sana_mixffn_workspace_bytes.restype = sz
    lib.sana_mixffn_forward.argtypes = [vp, vp, fp, fp, fp, vp, fp, vp, i64, ci, ci, ci, ci, ci,
                                        vp, sz, vp]
    lib.sana_mixffn_forward.restype = ctypes.c_int
    lib.sana_linattn_forward_kernels.argtypes = [i64, i64, ci, ci, ci]
    lib.sana_linattn_forward_kernels.restype = ctypes.c_int
    lib.sana_linattn_strerror.argtypes = [ci]
    lib.sana_linattn_strerror.restype = ctypes.c_char_p
    return lib


def load():
    """Load the in-tree CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            path = lib_path()
            if not os.path.exists(path):
                raise RuntimeError(
                    f"{path} is missing: build it with `python -m relu_linear_attention_attn_b200"
                    ".build` (there is no fallback implementation)")
            _lib = _declare(ctypes.CDLL(path))
    return _lib


def _check(fn: str, rc: int):
    if rc != 0:
        raise SanaError(fn, rc, load().sana_linattn_strerror(rc).decode())


def workspace_bytes(B: int, N: int, C: int, H: int, fused: bool = False) -> int:
    return int(load().sana_linattn_workspace_bytes(B, N, C, H, 1 if fused else 0))


# --------------------------------------------------------------------------- torch marshalling
def forward_kernels(B: int, N: int, C: int, H: int, dtype: str = "bf16") -> int:
    """How many kernels forward() launches for this shape: 1 (one cluster launch),
    2 (the two persistent passes), 3 (the CUDA-core path), 0 when empty."""
    rc = load().sana_linattn_forward_kernels(B, N, C, H, {"bf16": 0, "f32": 1}[dtype])
    _check("sana_linattn_forward_kernels", min(rc, 0))
    return rc


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _dev(t, name: str):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _gain(g, name: str):
    if g is None:
        return None
    torch = _torch()
    if g.dtype != torch.float32:
        raise TypeError(f"{name} must be float32")
    return _dev(g, name)


def _stream(stream) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _workspace(nbytes: int, device, workspace, stream=None):
    torch = _torch()
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        # the library runs on `stream`: keep the caching allocator from handing this
        # block to other work on the current stream before that stream's use of it ends
        if stream is not None and stream != torch.cuda.current_stream(device):
            workspace.record_stream(stream)
    if workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError(f"workspace needs {nbytes} bytes")
    return workspace, workspace.numel() * workspace.element_size()


def forward(q, k, v, gq, gk, H: int, eps: float, out=None, workspace=None, stream=None):
    """Eq. (1) with QK-RMSNorm on projected q, k, v of shape (B, N, C).
    gq, gk: float32 [C] tensors, or both None to switch the norm off."""
    B, N, C = q.shape
    if k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share shape and dtype")
    dt = _dtype_code(q)
    if out is None:
        out = _torch().empty_like(q)
    ws, wsb = _workspace(workspace_bytes(B, N, C, H), q.device, workspace, stream)
    rc = load().sana_linattn_forward(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _gain(gq, "gq"),
                                     _gain(gk, "gk"), _dev(out, "out"), B, N, C, H, float(eps), dt,
                                     None if ws is None else ws.data_ptr(), wsb, _stream(stream))
    _check("sana_linattn_forward", rc)
    return out


def backward(q, k, v, gq, gk, dout, H: int, eps: float, grads=None, workspace=None,
             stream=None, kv=None):
    """Gradients of forward()'s output: returns (dq, dk, dv, dgq, dgk); dgq, dgk
    (float32 [C]) are None with the norm off.  `grads`, when given, is that tuple
    preallocated (the results are written into it).  `kv`, when given, is the
    forward's state (kv_state() of the same k, v, gk, eps): it is used instead of
    being formed again (sana_linattn_backward_with_state)."""
    torch = _torch()
    B, N, C = q.shape
    for t, n in ((k, "k"), (v, "v"), (dout, "dout")):
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError(f"{n} must match q in shape and dtype")
    dt = _dtype_code(q)
    if grads is not None:
        dq, dk, dv, dgq, dgk = grads
        for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
            if t.shape != q.shape or t.dtype != q.dtype:
                raise ValueError(f"{n} must match q in shape and dtype")
        for t, n in ((dgq, "dgq"), (dgk, "dgk")):
            if (t is None) != (gq is None) or (t is not None and (t.shape != (C,) or
                                                                   t.dtype != torch.float32)):
                raise ValueError(f"{n} must be float32 [C] exactly when the gains are given")
    else:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        dgq = dgk = None
        if gq is not None:
            dgq = torch.empty(C, dtype=torch.float32, device=q.device)
            dgk = torch.empty(C, dtype=torch.float32, device=q.device)
    ws, wsb = _workspace(int(load().sana_linattn_backward_workspace_bytes(B, N, C, H)), q.device,
                         workspace, stream)
    wsp = None if ws is None else ws.data_ptr()
    if kv is None:
        rc = load().sana_linattn_backward(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"),
                                          _gain(gq, "gq"), _gain(gk, "gk"), _dev(dout, "dout"),
                                          _dev(dq, "dq"), _dev(dk, "dk"), _dev(dv, "dv"),
                                          _dev(dgq, "dgq"), _dev(dgk, "dgk"), B, N, C, H,
                                          float(eps), dt, wsp, wsb, _stream(stream))
        _check("sana_linattn_backward", rc)
    else:
        if kv.dtype != torch.float32 or kv.shape != (B, H, C // H, C // H + 1):
            raise ValueError("kv must be float32 (B, H, D, D+1), as kv_state() returns")
        rc = load().sana_linattn_backward_with_state(
            _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _gain(gq, "gq"), _gain(gk, "gk"),
            _dev(kv, "kv"), _dev(dout, "dout"), _dev(dq, "dq"), _dev(dk, "dk"), _dev(dv, "dv"),
            _dev(dgq, "dgq"), _dev(dgk, "dgk"), B, N, C, H, float(eps), dt, wsp, wsb,
            _stream(stream))
        _check("sana_linattn_backward_with_state", rc)
    return dq, dk, dv, dgq, dgk


def forward_causal(q, k, v, gq, gk, H: int, eps: float, out=None, workspace=None, stream=None):
    """The prefix (causal) form: token n attends to keys j <= n.  Same arguments as
    forward()."""
    B, N, C = q.shape
    if k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share shape and dtype")
    dt = _dtype_code(q)
    if out is None:
        out = _torch().empty_like(q)
    ws, wsb = _workspace(int(load().sana_linattn_workspace_bytes(B, N, C, H, 2)), q.device,
                         workspace, stream)
    rc = load().sana_linattn_forward_causal(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"),
                                            _gain(gq, "gq"), _gain(gk, "gk"), _dev(out, "out"),
                                            B, N, C, H, float(eps), dt,
                                            None if ws is None else ws.data_ptr(), wsb,
                                            _stream(stream))
    _check("sana_linattn_forward_causal", rc)
    return out


def forward_noalloc(q, k, v, gq, gk, H: int, eps: float, out=None, stream=None):
    """forward() without a workspace: the library's static 16 MiB device scratch is
    used instead, for callers that cannot allocate device memory (see
    sana_linattn_forward_noalloc in include/sana_linattn.h).  Only `out` is
    allocated here when not given."""
    B, N, C = q.shape
    if k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share shape and dtype")
    dt = _dtype_code(q)
    if out is None:
        out = _torch().empty_like(q)
    rc = load().sana_linattn_forward_noalloc(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"),
                                             _gain(gq, "gq"), _gain(gk, "gk"), _dev(out, "out"),
                                             B, N, C, H, float(eps), dt, _stream(stream))
    _check("sana_linattn_forward_noalloc", rc)
    return out


def forward_pass1(k, v, gk, H: int, eps: float, workspace, stream=None):
    """The forward's first pass alone: the split-N partial states into `workspace`
    (uint8, at least workspace_bytes(B, N, C, H)).  bf16 only."""
    B, N, C = k.shape
    if v.shape != k.shape or v.dtype != k.dtype:
        raise ValueError("k, v must share shape and dtype")
    if _dtype_code(k) != BF16:
        raise TypeError("the forward's passes run on bf16 inputs")
    ws, wsb = _workspace(workspace_bytes(B, N, C, H), k.device, workspace, stream)
    rc = load().sana_linattn_forward_pass1(_dev(k, "k"), _dev(v, "v"), _gain(gk, "gk"), B, N, C,
                                           H, float(eps), None if ws is None else ws.data_ptr(),
                                           wsb, _stream(stream))
    _check("sana_linattn_forward_pass1", rc)
    return ws


def forward_pass2(q, gq, H: int, eps: float, workspace, out=None, stream=None):
    """The forward's second pass alone, from the partial states forward_pass1 left
    in `workspace` for the same shapes."""
    B, N, C = q.shape
    if _dtype_code(q) != BF16:
        raise TypeError("the forward's passes run on bf16 inputs")
    if out is None:
        out = _torch().empty_like(q)
    wsb = workspace.numel() * workspace.element_size()
    rc = load().sana_linattn_forward_pass2(_dev(q, "q"), _gain(gq, "gq"), _dev(out, "out"), B, N,
                                           C, H, float(eps), workspace.data_ptr(), wsb,
                                           _stream(stream))
    _check("sana_linattn_forward_pass2", rc)
    return out


def kv_state(k, v, gk, H: int, eps: float, kv=None, workspace=None, stream=None):
    """State S (B, H, D, D+1) fp32 of Eq. (1): sum_n phi(K_n)^T [V_n | 1]."""
    torch = _torch()
    B, N, C = k.shape
    D = C // H
    dt = _dtype_code(k)
    if kv is None:
        kv = torch.empty((B, H, D, D + 1), dtype=torch.float32, device=k.device)
    ws, wsb = _workspace(workspace_bytes(B, N, C, H), k.device, workspace, stream)
    rc = load().sana_linattn_kv_state(_dev(k, "k"), _dev(v, "v"), _gain(gk, "gk"), _dev(kv, "kv"),
                                      B, N, C, H, float(eps), dt,
                                      None if ws is None else ws.data_ptr(), wsb, _stream(stream))
    _check("sana_linattn_kv_state", rc)
    return kv


def apply(q, gq, kv, H: int, eps: float, out=None, stream=None):
    """O = phi(Q) S[:, :D] / (phi(Q) S[:, D] + eps) with a given state kv."""
    B, N, C = q.shape
    dt = _dtype_code(q)
    if out is None:
        out = _torch().empty_like(q)
    rc = load().sana_linattn_apply(_dev(q, "q"), _gain(gq, "gq"), _dev(kv, "kv"), _dev(out, "out"),
                                   B, N, C, H, float(eps), dt, _stream(stream))
    _check("sana_linattn_apply", rc)
    return out


def device_error(clear: bool = True):
    """(code, site) of the device-side error word (0, 0 when no bounded wait gave up).
    Synchronous; call after synchronising the work of interest."""
    code, site = ctypes.c_int(0), ctypes.c_int(0)
    _check("sana_linattn_device_error",
           load().sana_linattn_device_error(ctypes.byref(code), ctypes.byref(site),
                                            1 if clear else 0))
    return code.value, site.value


def selftest_launch_failure(stream=None) -> int:
    """Enqueue a launch the runtime rejects (see include/sana_linattn.h) and return
    the library's status for it (SANA_ECUDA = -5); raises nothing."""
    return int(load().sana_linattn_selftest_launch_failure(_stream(stream)))


def selftest_wait_timeout(limit_us: int = 20000, stream=None):
    """Enqueue the bounded-wait self-test (see include/sana_linattn.h)."""
    _check("sana_linattn_selftest_wait_timeout",
           load().sana_linattn_selftest_wait_timeout(int(limit_us), _stream(stream)))


def quantize_rows_i8(x, out=None, scales=None, stream=None):
    """Symmetric int8 codes of each row of x (..., cols) (bf16 or fp32): returns
    (codes int8 of x's shape, scales fp32 of x.shape[:-1]); scale = max|row| / 127,
    code = round_half_even(x / scale) clamped to [-127, 127]."""
    torch = _torch()
    cols = x.shape[-1]
    rows = x.numel() // cols if cols else 0
    if out is None:
        out = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    rc = load().sana_quantize_rows_i8(_dev(x, "x"), _dtype_code(x), _dev(out, "codes"),
                                      _dev(scales, "scales"), rows, cols, _stream(stream))
    _check("sana_quantize_rows_i8", rc)
    return out, scales


def quantize_cols_i8(w, out=None, scales=None, stream=None):
    """Symmetric int8 codes of each column of w (K, cols) (bf16 or fp32): returns
    (codes int8 (K, cols), scales fp32 (cols,))."""
    torch = _torch()
    K, cols = w.shape
    if out is None:
        out = torch.empty(w.shape, dtype=torch.int8, device=w.device)
    if scales is None:
        scales = torch.empty((cols,), dtype=torch.float32, device=w.device)
    rc = load().sana_quantize_cols_i8(_dev(w, "w"), _dtype_code(w), _dev(out, "codes"),
                                      _dev(scales, "scales"), K, cols, _stream(stream))
    _check("sana_quantize_cols_i8", rc)
    return out, scales


def qkv_fused_w8a8(xq, sx, Wq, sw, gq, gk, H: int, eps: float, out=None, workspace=None,
                   stream=None):
    """The fused variant with a W8A8 prologue: int8 codes xq (B, N, C) with
    per-token scales sx (B, N), int8 Wq (C, 3C) with per-channel scales sw (3C,);
    returns O (B, N, C) bf16."""
    torch = _torch()
    B, N, C = xq.shape
    if xq.dtype != torch.int8 or Wq.dtype != torch.int8:
        raise TypeError("the W8A8 path takes int8 xq and Wq")
    if tuple(Wq.shape) != (C, 3 * C) or tuple(sx.shape) != (B, N) or tuple(sw.shape) != (3 * C,):
        raise ValueError("shapes: xq (B, N, C), sx (B, N), Wq (C, 3C), sw (3C,)")
    if out is None:
        out = torch.empty((B, N, C), dtype=torch.bfloat16, device=xq.device)
    ws, wsb = _workspace(workspace_bytes(B, N, C, H, fused=True), xq.device, workspace, stream)
    rc = load().sana_linattn_qkv_fused_w8a8(_dev(xq, "xq"), _dev(sx, "sx"), _dev(Wq, "Wq"),
                                            _dev(sw, "sw"), _gain(gq, "gq"), _gain(gk, "gk"),
                                            _dev(out, "out"), B, N, C, H, float(eps),
                                            None if ws is None else ws.data_ptr(), wsb,
                                            _stream(stream))
    _check("sana_linattn_qkv_fused_w8a8", rc)
    return out


def qkv_fused(x, W, gq, gk, H: int, eps: float, out=None, workspace=None, stream=None):
    """The fused variant: [Q|K|V] = x @ Wqkv, QK-RMSNorm, ReLU, Eq. (1).  bf16 in and out."""
    torch = _torch()
    B, N, C = x.shape
    if x.dtype != torch.bfloat16 or W.dtype != torch.bfloat16:
        raise TypeError("the fused path takes bf16 x and Wqkv")
    if tuple(W.shape) != (C, 3 * C):
        raise ValueError("Wqkv must be (C, 3C)")
    if out is None:
        out = torch.empty_like(x)
    ws, wsb = _workspace(workspace_bytes(B, N, C, H, fused=True), x.device, workspace, stream)
    rc = load().sana_linattn_qkv_fused(_dev(x, "x"), _dev(W, "Wqkv"), _gain(gq, "gq"),
                                       _gain(gk, "gk"), _dev(out, "out"), B, N, C, H, float(eps),
                                       None if ws is None else ws.data_ptr(), wsb,
                                       _stream(stream))
    _check("sana_linattn_qkv_fused", rc)
    return out


# --------------------------------------------------------------------------- Mix-FFN
# (declared in include/sana_mixffn.h)
def _bf16(t, name: str):
    if t.dtype != _torch().bfloat16:
        raise TypeError(f"{name} must be bfloat16")
    return _dev(t, name)


def _gate(gate: str) -> int:
    if gate not in GATES:
        raise ValueError(f"gate must be one of {sorted(GATES)}")
    return GATES[gate]


def gemm_bias(A, W, bias=None, out=None, stream=None):
    """out[M, Nc] = A[M, K] @ W[K, Nc] (+ bias) in bf16 with fp32 accumulation.
    A may have leading batch dimensions (flattened into M)."""
    K, Nc = W.shape
    if A.shape[-1] != K:
        raise ValueError("A's last dimension must equal W's first")
    M = A.numel() // K
    if out is None:
        out = _torch().empty(*A.shape[:-1], Nc, dtype=A.dtype, device=A.device)
    if out.numel() != M * Nc:
        raise ValueError("out must hold M x Nc elements")
    rc = load().sana_gemm_bias_bf16(_bf16(A, "A"), _bf16(W, "W"), _gain(bias, "bias"),
                                    _bf16(out, "out"), M, K, Nc, _stream(stream))
    _check("sana_gemm_bias_bf16", rc)
    return out


def mixffn_dwconv_glu(u, wdw, bdw, Hs: int, Ws: int, gate: str = "sigmoid", out=None,
                      stream=None):
    """GLU of the depthwise 3x3 convolution of u (B, Hs*Ws, 2F) bf16 on the row-major
    (Hs, Ws) grid; wdw float32 (2F, 3, 3), bdw float32 [2F] or None -> (B, N, F)."""
    B, N, C2 = u.shape
    if N != Hs * Ws or C2 % 2:
        raise ValueError("u must be (B, Hs*Ws, 2F)")
    F = C2 // 2
    if tuple(wdw.shape) != (C2, 3, 3):
        raise ValueError("wdw must be (2F, 3, 3)")
    if out is None:
        out = _torch().empty(B, N, F, dtype=u.dtype, device=u.device)
    rc = load().sana_mixffn_dwconv_glu(_bf16(u, "u"), _gain(wdw, "wdw"), _gain(bdw, "bdw"),
                                       _bf16(out, "out"), B, Hs, Ws, F, _gate(gate),
                                       _stream(stream))
    _check("sana_mixffn_dwconv_glu", rc)
    return out


def mixffn_workspace_bytes(B: int, Hs: int, Ws: int, C: int, F: int) -> int:
    return int(load().sana_mixffn_workspace_bytes(B, Hs, Ws, C, F))


def mixffn_forward(x, W1, b1, wdw, bdw, W2, b2, Hs: int, Ws: int, gate: str = "sigmoid",
                   out=None, workspace=None, stream=None):
    """The Mix-FFN of x (B, Hs*Ws, C) bf16: 1x1 expand (W1: (C, 2F)), depthwise 3x3 +
    GLU, 1x1 project (W2: (F, C)); biases float32 or None."""
    B, N, C = x.shape
    F = W2.shape[0]
    if N != Hs * Ws or tuple(W1.shape) != (C, 2 * F) or tuple(W2.shape) != (F, C):
        raise ValueError("shapes must be x (B, Hs*Ws, C), W1 (C, 2F), W2 (F, C)")
    if tuple(wdw.shape) != (2 * F, 3, 3):
        raise ValueError("wdw must be (2F, 3, 3)")
    if out is None:
        out = _torch().empty_like(x)
    ws, wsb = _workspace(mixffn_workspace_bytes(B, Hs, Ws, C, F), x.device, workspace, stream)
    rc = load().sana_mixffn_forward(_bf16(x, "x"), _bf16(W1, "W1"), _gain(b1, "b1"),
                                    _gain(wdw, "wdw"), _gain(bdw, "bdw"), _bf16(W2, "W2"),
                                    _gain(b2, "b2"), _bf16(out, "out"), B, Hs, Ws, C, F,
                                    _gate(gate), None if ws is None else ws.data_ptr(), wsb,
                                    _stream(stream))
    _check("sana_mixffn_forward", rc)
    return out
