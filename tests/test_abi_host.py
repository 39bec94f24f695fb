"""Host-side checks of the C ABI (no GPU needed).

The library must load, export every symbol that include/*.h declares, size its
workspace, and reject bad arguments with the documented status before touching
the device.  The rejection tests pass fake device addresses; every call below
carries at least one violation, so nothing is launched.  They are skipped on a
machine with a GPU (the GPU suite repeats them with real buffers)."""
import ctypes
import glob
import os
import re

import pytest
import torch

import relu_linear_attention_attn_b200 as sla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, EINVAL, EALIGN, EUNSUP, EWS, ECUDA = 0, -1, -2, -3, -4, -5


def declared_symbols():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names += re.findall(r"SANA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return sorted(set(names))


def test_library_builds_for_sm100a_and_loads():
    lib = sla.load()
    assert os.path.exists(sla.lib_path())
    assert lib is not None


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert "sana_linattn_forward" in names and "sana_linattn_qkv_fused" in names
    lib = ctypes.CDLL(sla.lib_path())
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_strerror_covers_every_status():
    lib = sla.load()
    for code in (OK, EINVAL, EALIGN, EUNSUP, EWS, ECUDA, 12345):
        s = lib.sana_linattn_strerror(code)
        assert s and len(s) > 3


def test_workspace_bytes():
    ws = sla.workspace_bytes
    assert ws(0, 1024, 2240, 70) == 0 and ws(1, 0, 2240, 70) == 0
    assert ws(1, 1024, 2240, 71) == 0            # C % H != 0
    assert ws(1, 1024, 2240, 35) == 0            # D = 64 unsupported
    a = ws(1, 1024, 2240, 70)
    b = ws(8, 4096, 2240, 70)
    assert 0 < a < b and a % 256 == 0 and b % 256 == 0
    # the fused path keeps Q, K, V on chip: its workspace is states and partials only
    f = ws(4, 4096, 2240, 70, fused=True)
    assert 2 * 4 * 70 * 32 * 33 * 4 <= f < 64 << 20
    # the state alone: B*H*D*(D+1) fp32, the partials at least as much again
    assert a >= 2 * 1 * 70 * 32 * 33 * 4


def test_forward_kernel_count_follows_the_dispatch():
    """Short problems on the tensor cores are one cluster launch (clusters of
    ceil(N / 128) <= 8 CTAs per batch item and group of 4 heads, at most 400 CTAs);
    longer or larger ones the two persistent passes; fp32 or C > 4096 the CUDA-core
    path (3 launches)."""
    fk = sla.forward_kernels
    assert fk(1, 1024, 2240, 70) == 1              # the 1024px latent, batch 1: 8 x 18 CTAs
    assert fk(2, 1024, 2240, 70) == 1              # 288 CTAs
    assert fk(3, 777, 2240, 70) == 1               # 3 x 18 x 7 = 378
    assert fk(3, 1024, 2240, 70) == 2              # 432 > 400
    assert fk(1, 1025, 2240, 70) == 2              # longer than 8 x 128 tokens
    assert fk(8, 4096, 2240, 70) == 2
    assert fk(1, 1, 32, 1) == 1
    assert fk(1, 1024, 2240, 70, "f32") == 3
    assert fk(1, 256, 4128, 129) == 3              # gains of more than 4096 channels
    assert fk(0, 1024, 2240, 70) == 0 and fk(1, 0, 2240, 70) == 0
    with pytest.raises(sla.SanaError):
        fk(1, 1024, 2240, 71)                      # C % H != 0


FAKE = 1 << 36   # a 256-byte-aligned address that is never dereferenced


@pytest.fixture()
def lib():
    if torch.cuda.is_available():
        pytest.skip("fake-pointer rejection tests run on CPU-only machines")
    return sla.load()


def _fwd(lib, q=FAKE, k=FAKE + (1 << 30), v=FAKE + (2 << 30), gq=FAKE + (3 << 30),
         gk=FAKE + (3 << 30) + 65536, out=FAKE + (4 << 30), B=1, N=1024, C=2240, H=70,
         eps=1e-6, dtype=0, ws=FAKE + (6 << 30), wsb=1 << 30):
    return lib.sana_linattn_forward(q, k, v, gq, gk, out, B, N, C, H, eps, dtype, ws, wsb, None)


@pytest.mark.parametrize("kw,status", [
    (dict(H=35), EUNSUP),                      # D = 64
    (dict(H=71), EINVAL),                      # C % H != 0
    (dict(C=0), EINVAL),
    (dict(B=-1), EINVAL),
    (dict(N=-5), EINVAL),
    (dict(eps=-1e-6), EINVAL),
    (dict(eps=float("nan")), EINVAL),
    (dict(eps=float("inf")), EINVAL),
    (dict(gq=None), EINVAL),                   # only one gain given
    (dict(gk=None), EINVAL),
    (dict(q=None), EINVAL),
    (dict(out=None), EINVAL),
    (dict(dtype=7), EINVAL),
    (dict(q=FAKE + 2), EALIGN),
    (dict(out=FAKE + (4 << 30) + 8), EALIGN),
    (dict(gq=FAKE + (3 << 30) + 2), EALIGN),
    (dict(ws=None), EWS),
    (dict(wsb=1024), EWS),
    (dict(ws=FAKE + (6 << 30) + 16), EALIGN),
    (dict(out=FAKE + 4096), EINVAL),           # out overlaps q
    (dict(ws=FAKE + (1 << 30) + 256), EINVAL),  # workspace overlaps k
    (dict(B=1 << 20), EUNSUP),                  # beyond the grid's batch limit
])
def test_forward_rejects_bad_arguments(lib, kw, status):
    assert _fwd(lib, **kw) == status


def test_empty_problem_is_a_no_op(lib):
    assert _fwd(lib, B=0) == OK
    assert _fwd(lib, N=0) == OK
    assert lib.sana_linattn_apply(FAKE, None, FAKE + (1 << 30), FAKE + (2 << 30), 3, 0, 2240, 70,
                                  1e-6, 0, None) == OK


def test_other_entry_points_reject_bad_arguments(lib):
    # kv_state: misaligned k, workspace too small, bad dtype
    assert lib.sana_linattn_kv_state(FAKE + 4, FAKE + (1 << 30), None, FAKE + (2 << 30), 1, 64,
                                     2240, 70, 1e-6, 0, FAKE + (3 << 30), 1 << 30, None) == EALIGN
    assert lib.sana_linattn_kv_state(FAKE, FAKE + (1 << 30), None, FAKE + (2 << 30), 1, 64,
                                     2240, 70, 1e-6, 0, FAKE + (3 << 30), 16, None) == EWS
    assert lib.sana_linattn_kv_state(FAKE, FAKE + (1 << 30), None, FAKE + (2 << 30), 1, 64,
                                     2240, 70, 1e-6, 9, FAKE + (3 << 30), 1 << 30, None) == EINVAL
    # apply: D = 16, out overlapping the state
    assert lib.sana_linattn_apply(FAKE, None, FAKE + (1 << 30), FAKE + (2 << 30), 1, 64, 2240, 140,
                                  1e-6, 0, None) == EUNSUP
    assert lib.sana_linattn_apply(FAKE, None, FAKE + (1 << 30), FAKE + (1 << 30) + 256, 1, 64,
                                  2240, 70, 1e-6, 0, None) == EINVAL
    # fused: misaligned W, too-small workspace, one gain
    args = [FAKE, FAKE + (1 << 30), None, None, FAKE + (2 << 30), 4, 4096, 2240, 70, 1e-6,
            FAKE + (4 << 30), 1 << 34, None]
    a = list(args)
    a[1] += 2
    assert lib.sana_linattn_qkv_fused(*a) == EALIGN
    a = list(args)
    a[11] = 4096
    assert lib.sana_linattn_qkv_fused(*a) == EWS
    a = list(args)
    a[2] = FAKE + (3 << 30)
    assert lib.sana_linattn_qkv_fused(*a) == EINVAL


def test_w8a8_and_quantize_entry_points_reject_bad_arguments(lib):
    # W8A8 fused: misaligned xq, one gain, too-small workspace, overlap of out and xq
    args = [FAKE, FAKE + (1 << 30), FAKE + (2 << 30), FAKE + (3 << 30), None, None,
            FAKE + (4 << 30), 4, 4096, 2240, 70, 1e-6, FAKE + (5 << 30), 1 << 34, None]
    a = list(args)
    a[0] += 8
    assert lib.sana_linattn_qkv_fused_w8a8(*a) == EALIGN
    a = list(args)
    a[4] = FAKE + (6 << 30)
    assert lib.sana_linattn_qkv_fused_w8a8(*a) == EINVAL
    a = list(args)
    a[13] = 4096
    assert lib.sana_linattn_qkv_fused_w8a8(*a) == EWS
    a = list(args)
    a[6] = FAKE + 64
    assert lib.sana_linattn_qkv_fused_w8a8(*a) == EINVAL
    a = list(args)
    a[10] = 35                                   # D = 64
    assert lib.sana_linattn_qkv_fused_w8a8(*a) == EUNSUP
    # quantisation: cols not a multiple of 8, bad dtype, misaligned, overlapping
    assert lib.sana_quantize_rows_i8(FAKE, 0, FAKE + (1 << 30), FAKE + (2 << 30), 16, 12,
                                     None) == EINVAL
    assert lib.sana_quantize_rows_i8(FAKE, 5, FAKE + (1 << 30), FAKE + (2 << 30), 16, 16,
                                     None) == EINVAL
    assert lib.sana_quantize_rows_i8(FAKE + 2, 0, FAKE + (1 << 30), FAKE + (2 << 30), 16, 16,
                                     None) == EALIGN
    assert lib.sana_quantize_rows_i8(FAKE, 0, FAKE + 8, FAKE + (2 << 30), 16, 16, None) == EINVAL
    assert lib.sana_quantize_rows_i8(FAKE, 0, FAKE + (1 << 30), FAKE + (2 << 30), 0, 16,
                                     None) == OK
    assert lib.sana_quantize_cols_i8(FAKE, 0, FAKE + 4, FAKE + (2 << 30), 64, 64, None) == EINVAL
    assert lib.sana_quantize_cols_i8(FAKE, 0, FAKE + (1 << 30), FAKE + (2 << 30) + 2, 64, 64,
                                     None) == EALIGN


def test_causal_entry_point_rejects_bad_arguments(lib):
    ws_need = lib.sana_linattn_workspace_bytes(2, 1000, 2240, 70, 2)
    simt = 2 * 70 * 16 * 1056 * 4               # one state per 64-token chunk
    tc = 2 * (2 * 70 * 8 * 2 * 1056 * 4)        # two partial slots + the prefix per 128 tokens
    assert ws_need == max(simt, tc)
    args = [FAKE, FAKE + (1 << 30), FAKE + (2 << 30), None, None, FAKE + (4 << 30), 2, 1000,
            2240, 70, 1e-6, 0, FAKE + (6 << 30), ws_need, None]
    a = list(args)
    a[0] += 2
    assert lib.sana_linattn_forward_causal(*a) == EALIGN
    a = list(args)
    a[13] = ws_need - 4
    assert lib.sana_linattn_forward_causal(*a) == EWS
    a = list(args)
    a[3] = FAKE + (3 << 30)
    assert lib.sana_linattn_forward_causal(*a) == EINVAL
    a = list(args)
    a[9] = 35
    assert lib.sana_linattn_forward_causal(*a) == EUNSUP
    a = list(args)
    a[5] = FAKE + 64
    assert lib.sana_linattn_forward_causal(*a) == EINVAL


def test_backward_entry_point_rejects_bad_arguments(lib):
    need = lib.sana_linattn_backward_workspace_bytes(1, 256, 2240, 70)
    assert need > 1 * 256 * 70 * 33 * 4
    base = [FAKE, FAKE + (1 << 30), FAKE + (2 << 30), FAKE + (3 << 30), FAKE + (3 << 30) + 65536,
            FAKE + (4 << 30), FAKE + (5 << 30), FAKE + (6 << 30), FAKE + (7 << 30),
            FAKE + (8 << 30), FAKE + (8 << 30) + 65536, 1, 256, 2240, 70, 1e-6, 0,
            FAKE + (9 << 30), need, None]
    a = list(base)
    a[9] = None                                  # gains given, one gain gradient missing
    assert lib.sana_linattn_backward(*a) == EINVAL
    a = list(base)
    a[6] += 2                                    # misaligned dq
    assert lib.sana_linattn_backward(*a) == EALIGN
    a = list(base)
    a[7] = FAKE + 64                             # dk overlaps q
    assert lib.sana_linattn_backward(*a) == EINVAL
    a = list(base)
    a[18] = need - 256
    assert lib.sana_linattn_backward(*a) == EWS
    a = list(base)
    a[14] = 35
    assert lib.sana_linattn_backward(*a) == EUNSUP
    # with the forward's state: (q, k, v, gq, gk, kv, dout, ...)
    kv = FAKE + (10 << 30)
    w = base[:5] + [kv] + base[5:]
    a = list(w)
    a[5] = None                                  # the state is required
    assert lib.sana_linattn_backward_with_state(*a) == EINVAL
    a = list(w)
    a[5] = kv + 4                                # misaligned state
    assert lib.sana_linattn_backward_with_state(*a) == EALIGN
    a = list(w)
    a[5] = base[18 - 1] + 256                    # the state inside the workspace
    assert lib.sana_linattn_backward_with_state(*a) == EINVAL
    a = list(w)
    a[5] = base[6]                               # the state overlaps dq
    assert lib.sana_linattn_backward_with_state(*a) == EINVAL



def test_mixffn_entry_points_reject_bad_arguments(lib):
    G = 1 << 30
    # GEMM: K and Nc multiples of 8, aligned pointers, D apart from the operands
    base = [FAKE, FAKE + G, FAKE + 2 * G, FAKE + 3 * G, 1000, 2240, 11200, None]
    a = list(base)
    a[5] = 2244
    assert lib.sana_gemm_bias_bf16(*a) == EINVAL
    a = list(base)
    a[6] = 0
    assert lib.sana_gemm_bias_bf16(*a) == EINVAL
    a = list(base)
    a[0] += 8
    assert lib.sana_gemm_bias_bf16(*a) == EALIGN
    a = list(base)
    a[2] += 2
    assert lib.sana_gemm_bias_bf16(*a) == EALIGN
    a = list(base)
    a[3] = FAKE + 64                              # D overlaps A
    assert lib.sana_gemm_bias_bf16(*a) == EINVAL
    a = list(base)
    a[4] = 1 << 31
    assert lib.sana_gemm_bias_bf16(*a) == EUNSUP
    a = list(base)
    a[4] = 0                                      # empty: nothing to do
    assert lib.sana_gemm_bias_bf16(*a) == OK
    # depthwise conv + GLU
    base = [FAKE, FAKE + G, FAKE + 2 * G, FAKE + 3 * G, 2, 64, 64, 5600, 0, None]
    a = list(base)
    a[7] = 5604
    assert lib.sana_mixffn_dwconv_glu(*a) == EINVAL
    a = list(base)
    a[8] = 2
    assert lib.sana_mixffn_dwconv_glu(*a) == EINVAL
    a = list(base)
    a[3] += 4
    assert lib.sana_mixffn_dwconv_glu(*a) == EALIGN
    a = list(base)
    a[3] = FAKE + 128                             # h overlaps u
    assert lib.sana_mixffn_dwconv_glu(*a) == EINVAL
    a = list(base)
    a[4] = 70000
    assert lib.sana_mixffn_dwconv_glu(*a) == EUNSUP
    # the whole Mix-FFN
    need = lib.sana_mixffn_workspace_bytes(2, 64, 64, 2240, 5600)
    tok = 2 * 64 * 64
    assert need == tok * 2 * 5600 * 2 + tok * 5600 * 2
    assert lib.sana_mixffn_workspace_bytes(2, 64, 64, 2240, 5601) == 0
    base = [FAKE, FAKE + G, None, FAKE + 2 * G, None, FAKE + 3 * G, None, FAKE + 4 * G, 2, 64, 64,
            2240, 5600, 0, FAKE + 5 * G, need, None]
    a = list(base)
    a[15] = need - 256
    assert lib.sana_mixffn_forward(*a) == EWS
    a = list(base)
    a[14] = FAKE + 5 * G + 16
    assert lib.sana_mixffn_forward(*a) == EALIGN
    a = list(base)
    a[14] = FAKE + 4 * G                          # workspace overlaps y
    assert lib.sana_mixffn_forward(*a) == EINVAL
    a = list(base)
    a[7] = FAKE + 64                              # y overlaps x
    assert lib.sana_mixffn_forward(*a) == EINVAL
    a = list(base)
    a[11] = 2242
    assert lib.sana_mixffn_forward(*a) == EINVAL
    a = list(base)
    a[13] = 5
    assert lib.sana_mixffn_forward(*a) == EINVAL
    a = list(base)
    a[0] += 2
    assert lib.sana_mixffn_forward(*a) == EALIGN


def test_guard_band_helper_detects_writes_outside_the_region():
    """The canary helper the GPU tests wrap outputs and workspaces in (checked here on
    CPU tensors)."""
    from parity import Guarded
    g = Guarded(1000, "cpu", guard=64, align=256)
    assert g.region.data_ptr() % 256 == 0 and g.region.numel() == 1000 and g.intact()
    g.region.fill_(1)
    assert g.intact()
    x = g.view(torch.bfloat16, (10, 50))
    x.fill_(3.0)
    assert g.intact()
    g.buf[g.off + 1000] = 0
    assert not g.intact()
    h = Guarded(64, "cpu", guard=64, align=256)
    h.buf[h.off - 1] = 7
    assert not h.intact()
