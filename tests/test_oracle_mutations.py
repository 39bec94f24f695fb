"""Plant plausible mistakes in a copy of the C oracle (on the CPU) and check that
the pin battery notices every one: a transposed operand, a dropped term, a wrong
index, a wrong sign, a missing square root, a missing eps, a skipped token."""
import ctypes
import os
import subprocess

import pytest

from oracle import oracle as O
from oracle_checks import battery

SRC = os.path.join(os.path.dirname(O.__file__), "sana_oracle.c")

MUTATIONS = {
    "transposed_state": ("S[d * (D + 1) + e] += kk[d] * vv[e];",
                         "S[d * (D + 1) + e] += kk[e] * vv[d];"),
    "normaliser_dropped": ("S[d * (D + 1) + D] += kk[d];", "S[d * (D + 1) + D] += 1.0;"),
    "eps_dropped_from_denominator": ("num / (den + c->eps)", "num / den"),
    "mean_square_not_divided": ("r = 1.0 / sqrt(ss / (double)D + eps)", "r = 1.0 / sqrt(ss + eps)"),
    "sqrt_missing": ("r = 1.0 / sqrt(ss / (double)D + eps)", "r = 1.0 / (ss / (double)D + eps)"),
    "relu_missing_after_norm": ("out[d] = y > 0.0 ? y : 0.0;", "out[d] = y;"),
    "relu_flipped": ("out[d] = y > 0.0 ? y : 0.0;",
                     "out[d] = y < 0.0 ? -y : 0.0;"),
    "relu_missing_norm_off": ("out[d] = xh[d] > 0.0 ? xh[d] : 0.0;", "out[d] = xh[d];"),
    "gain_index_ignores_head": ("g[h * D + d] * (xh[d] * r)", "g[d] * (xh[d] * r)"),
    "apply_reads_state_transposed": ("num += qq[d] * S[d * (D + 1) + e];",
                                     "num += qq[d] * S[e * (D + 1) + d];"),
    "apply_ignores_batch": ("c->S + ((size_t)b * c->H + h) * D * (D + 1)",
                            "c->S + ((size_t)h) * D * (D + 1)"),
    "last_token_skipped": ("for (int64_t n = 0; n < c->N; ++n)",
                           "for (int64_t n = 0; n + 1 < c->N; ++n)"),
    "den_uses_value_column": ("den += qq[d] * S[d * (D + 1) + D];",
                              "den += qq[d] * S[d * (D + 1) + 0];"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_battery_catches_planted_mistake(name, tmp_path, monkeypatch):
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
    assert battery(O), f"planted mistake {name} went unnoticed"
