"""The pins catch plausible mistakes: each mutant below plants one mistake in a temporary copy
of the oracle's C source (never in the committed one), and the pin suite must fail on it."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "delta_sign": ("S[e] = a * (S[e] - beta * k[i] * u[j]) + beta * k[i] * v[j];",
                   "S[e] = a * (S[e] + beta * k[i] * u[j]) + beta * k[i] * v[j];"),
    "drop_gate": ("S[e] = a * (S[e] - beta * k[i] * u[j]) + beta * k[i] * v[j];",
                  "S[e] = (S[e] - beta * k[i] * u[j]) + beta * k[i] * v[j];"),
    "u_from_query": ("acc += k[i] * a * S[(size_t)i * dv + j];",
                     "acc += q[i] * a * S[(size_t)i * dv + j];"),
    "readout_with_key": ("for (int i = 0; i < dk; ++i) acc += q[i] * S[(size_t)i * dv + j];",
                         "for (int i = 0; i < dk; ++i) acc += k[i] * S[(size_t)i * dv + j];"),
    "decay_first_without_gate": ("double a = (gate == ORC_GATE_CHANNEL_DECAY_FIRST) ? alpha[i] : 1.0;",
                                 "double a = 1.0;"),
    "column_weight_index": ("acc += w[i] * S[(size_t)i * dv + j] * S[(size_t)i * dv + j];",
                            "acc += w[j % dk] * S[(size_t)i * dv + j] * S[(size_t)i * dv + j];"),
    "bf16_truncates": ("double r = orc_round_half_even(ldexp(a, 7 - e));", "double r = floor(ldexp(a, 7 - e));"),
    "bf16_scale_stored_as_fp32": ("if (sfmt == ORC_SCALE_BF16) return orc_bf16_to_double(orc_double_to_bf16(v));",
                                  "if (sfmt == ORC_SCALE_BF16) return (double)(float)v;"),
    "fit_column_unweighted": ("num += w[i] * a * S[(size_t)i * dv + j];", "num += a * S[(size_t)i * dv + j];"),
    "fit_row_without_column_scale": ("double a = cs[j] * (double)Q[(size_t)i * dv + j];",
                                     "double a = (double)Q[(size_t)i * dv + j];"),
    "row_scale_from_unrounded_column": ("cs[j] = stored_scale(sfmt, c);\n", "cs[j] = c;\n"),
    "column_scale_no_sqrt": ("double c = sqrt(acc / W);", "double c = acc / W;"),
    "row_scale_ignores_column": ("double t = fabs(S[(size_t)i * dv + j] / cs[j]);",
                                 "double t = fabs(S[(size_t)i * dv + j]);"),
    "round_half_up": ("n = (fmod(f, 2.0) == 0.0) ? f : f + 1.0;", "n = f + 1.0;"),
    "offset_binary_off_by_one": ("            u[e] = (int32_t)qv + (1 << (bits - 1));",
                                 "            u[e] = (int32_t)qv + (1 << (bits - 1)) - 1;"),
    "uniform_offset_off_by_one": ("\n        u[e] = (int32_t)qv + (1 << (bits - 1));",
                                  "\n        u[e] = (int32_t)qv + (1 << (bits - 1)) - 1;"),
    "uniform_scale_without_qmax": ("double s = m / (double)qmax;", "double s = m;"),
    "uniform_scale_never_one": ("    if (s == 0.0) s = 1.0;\n    float sf", "    float sf"),
    "uniform_dequant_offset": ("S[e] = s * (double)(u[e] - (1 << (bits - 1)));",
                               "S[e] = s * (double)(u[e] - (1 << (bits - 1)) + 1);"),
    "pack_msb_first": ("out[bit / 8] |= (uint8_t)(1u << (bit % 8));",
                       "out[bit / 8] |= (uint8_t)(1u << (7 - bit % 8));"),
    "half_truncates": ("double r = orc_round_half_even(ldexp(a, 10 - e));",
                       "double r = floor(ldexp(a, 10 - e));"),
    "wy_substitution_sign": ("rhs -= beta[t] * A[(size_t)t * C + s] * Tm[(size_t)s * C + c];",
                             "rhs += beta[t] * A[(size_t)t * C + s] * Tm[(size_t)s * C + c];"),
    "wy_decay_exponent": ("acc += k[(size_t)s * dk + i] * exp(gC - g[s]) * U[(size_t)s * dv + j];",
                          "acc += k[(size_t)s * dk + i] * exp(g[s]) * U[(size_t)s * dv + j];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    shutil.copytree(os.path.join(ROOT, "oracle"), tmp_path / "oracle",
                    ignore=shutil.ignore_patterns("_build", "__pycache__"))
    os.makedirs(tmp_path / "tests")
    for f in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), tmp_path / "tests" / f)
    shutil.copy(os.path.join(ROOT, "pytest.ini"), tmp_path / "pytest.ini")
    src_path = tmp_path / "oracle" / "stq_oracle.c"
    src = src_path.read_text()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    src_path.write_text(src.replace(old, new))
    proc = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           "-W", "ignore::RuntimeWarning", "tests/test_oracle_pins.py"],
                          cwd=tmp_path, capture_output=True, text=True, timeout=600)
    assert proc.returncode != 0, f"mutant {name} survived the pins:\n{proc.stdout[-2000:]}"
    assert "failed" in proc.stdout or "error" in proc.stdout.lower()
