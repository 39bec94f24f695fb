"""Tolerances and helpers for comparing the CUDA path with the fp64 oracle.

Tolerances (applied to the library's output against the fp64 oracle on the
same dtype-rounded inputs):
  bf16 output : max|O - O_ref| <= 2e-2 and mean|O - O_ref| <= 2e-3, and, as a
                stricter guard derived from the arithmetic (bf16 operands carry
                a relative rounding of up to 2^-8 ~ 3.9e-3, the unit roundoff of
                bf16's 8 significant bits, and the output one more), the
                normwise relative error ||O - O_ref||_2 / ||O_ref||_2 <= 2e-2.
  fp32 output : max|O - O_ref| <= 5e-5 * max|O_ref| (normwise relative).
"""
from __future__ import annotations

import numpy as np
import torch

BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
BF16_REL_L2 = 2e-2
F32_NORMWISE = 5e-5


def to_np(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().double().numpy()
    return np.asarray(t, dtype=np.float64)


def errors(got, ref) -> dict:
    g, r = to_np(got), to_np(ref)
    d = np.abs(g - r)
    return dict(max_abs=float(d.max()) if d.size else 0.0,
                mean_abs=float(d.mean()) if d.size else 0.0,
                rel_l2=float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300)),
                normwise=float(d.max() / max(np.abs(r).max(), 1e-300)) if d.size else 0.0,
                finite=bool(np.isfinite(g).all()))


def assert_close(got, ref, dtype: str, what: str = ""):
    e = errors(got, ref)
    assert e["finite"], f"{what}: non-finite output {e}"
    if dtype == "bf16":
        ok = (e["max_abs"] <= BF16_MAX_ABS and e["mean_abs"] <= BF16_MEAN_ABS
              and e["rel_l2"] <= BF16_REL_L2)
    else:
        ok = e["normwise"] <= F32_NORMWISE
    assert ok, f"{what}: parity failed ({dtype}) {e}"
    return e


def sample_tokens(B: int, N: int, n: int = 512, seed: int = 0) -> np.ndarray:
    """Random flat token indices plus every batch's first and last token and the
    tokens either side of the 128-token tile edges."""
    rng = np.random.default_rng(seed)
    t = set(rng.integers(0, B * N, size=n).tolist())
    for b in range(B):
        for off in (0, 1, 63, 64, 127, 128, 129, N - 2, N - 1):
            if 0 <= off < N:
                t.add(b * N + off)
    return np.array(sorted(t), dtype=np.int64)


def to_dev(inp: dict, device="cuda") -> dict:
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


# ----------------------------------------------------------------------------- guard bands
CANARY = 0x5A


class Guarded:
    """A buffer of `nbytes` (offset `align`-aligned) inside a larger uint8 buffer whose
    `guard` bytes on each side hold a canary; `intact()` says whether anything wrote
    outside the region.  `view(dtype, shape)` is the region as a typed tensor."""

    def __init__(self, nbytes: int, device, guard: int = 4096, align: int = 256):
        self.nbytes = int(nbytes)
        self.buf = torch.full((self.nbytes + 2 * guard + align,), CANARY, dtype=torch.uint8,
                              device=device)
        base = self.buf.data_ptr()
        self.off = guard + (-(base + guard)) % align
        self.region = self.buf[self.off:self.off + self.nbytes]

    def view(self, dtype, shape):
        return self.region.view(dtype).view(shape)

    def intact(self) -> bool:
        return bool((self.buf[:self.off] == CANARY).all()) and \
            bool((self.buf[self.off + self.nbytes:] == CANARY).all())
