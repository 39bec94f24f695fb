"""Parity of the W8A8 prologue (through the C ABI) with the fp64 oracle.

Codes and scales are integer/fp32 results of a stated rule, so the GPU's must
equal the oracle's bit for bit.  The fused W8A8 op is fed the oracle's codes and
compared with the oracle's forward on them under the bf16 output tolerance."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from parity import assert_close, sample_tokens
from relu_linear_attention_attn_b200.synthetic import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _codes_equal(q_gpu, s_gpu, q_ref, s_ref, what):
    qg = q_gpu.cpu().numpy()
    sg = s_gpu.cpu().numpy()
    assert np.array_equal(sg.view(np.uint32), np.asarray(s_ref, np.float32).view(np.uint32)), \
        f"{what}: scales differ at {np.argwhere(sg != s_ref)[:5].tolist()}"
    bad = np.argwhere(qg != q_ref)
    assert bad.size == 0, f"{what}: {len(bad)} codes differ, first {bad[:5].tolist()}"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_quantize_rows_bit_exact(cuda_lib, dtype):
    w = WORKLOADS["w8a8-2048px-b4"].scaled(B=2, N=300, dtype=dtype, seed=51)
    x = make_inputs(w)["x"].clone()
    x[0, 7] = 0                        # an all-zero row: scale 0, codes 0
    x[1, 3] *= 1e-30 if dtype == "f32" else 1.0   # a tiny-magnitude row
    q, s = cuda_lib.quantize_rows_i8(x.cuda())
    torch.cuda.synchronize()
    q_ref, s_ref = O.quantize_i8(x.float().numpy())
    _codes_equal(q, s, q_ref, s_ref, f"rows {dtype}")
    assert float(s[0, 7]) == 0.0 and int(q[0, 7].abs().max()) == 0


def test_quantize_cols_bit_exact_full_wqkv(cuda_lib):
    W = make_inputs(WORKLOADS["w8a8-2048px-b4"])["W"]
    q, s = cuda_lib.quantize_cols_i8(W.cuda())
    torch.cuda.synchronize()
    q_ref, s_ref = O.quantize_i8(W.float().numpy(), axis=0)
    _codes_equal(q, s, q_ref, s_ref, "columns of Wqkv")


def _oracle_codes(x):
    xq, sx = O.quantize_i8(x["x"].float().numpy())
    Wq, sw = O.quantize_i8(x["W"].float().numpy(), axis=0)
    return xq, sx, Wq, sw


def _run(cuda_lib, xq, sx, Wq, sw, x, w):
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    out = cuda_lib.qkv_fused_w8a8(dev(xq), dev(sx), dev(Wq), dev(sw),
                                  None if x["gq"] is None else x["gq"].cuda(),
                                  None if x["gk"] is None else x["gk"].cuda(), w.H, w.eps)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("B,N,gains", [(1, 1, "random"), (1, 300, "random"), (2, 129, "off"),
                                       (1, 1000, "ones")])
def test_w8a8_small_full_parity(cuda_lib, B, N, gains):
    w = WORKLOADS["w8a8-2048px-b4"].scaled(B=B, N=N, gains=gains, seed=60 + N)
    x = make_inputs(w)
    xq, sx, Wq, sw = _oracle_codes(x)
    out = _run(cuda_lib, xq, sx, Wq, sw, x, w)
    ref = O.w8a8_fused_forward(xq, sx, Wq, sw, x["gq"], x["gk"], w.H, w.eps)
    assert_close(out, ref, "bf16", f"w8a8 {B}x{N} {gains}")


def test_w8a8_full_size_sampled_parity(cuda_lib):
    w = WORKLOADS["w8a8-2048px-b4"]
    x = make_inputs(w)
    xq, sx, Wq, sw = _oracle_codes(x)
    out = _run(cuda_lib, xq, sx, Wq, sw, x, w)
    tok = sample_tokens(w.B, w.N, n=256)
    ref = O.w8a8_fused_forward(xq, sx, Wq, sw, x["gq"], x["gk"], w.H, w.eps, tokens=tok)
    got = out.reshape(w.B * w.N, w.C)[torch.from_numpy(tok).cuda()]
    assert_close(got, ref, "bf16", w.name)


def test_w8a8_with_gpu_codes_is_deterministic(cuda_lib):
    """The GPU's own quantisation feeding the W8A8 op twice gives identical bits."""
    w = WORKLOADS["w8a8-2048px-b4"].scaled(B=1, N=1024, seed=77)
    x = make_inputs(w)
    xq, sx = cuda_lib.quantize_rows_i8(x["x"].cuda())
    Wq, sw = cuda_lib.quantize_cols_i8(x["W"].cuda())
    a = cuda_lib.qkv_fused_w8a8(xq, sx, Wq, sw, x["gq"].cuda(), x["gk"].cuda(), w.H, w.eps)
    b = cuda_lib.qkv_fused_w8a8(xq, sx, Wq, sw, x["gq"].cuda(), x["gk"].cuda(), w.H, w.eps)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
