"""The oracle's pins must catch plausible mistakes.

Each case below plants one mistake in a copy of the oracle's C source (on the
CPU, in a temporary directory), builds it, and runs the pin suite
``tests/test_oracle.py`` against that build in a child process.  The suite must
fail for every mutant; a mutant that survives means a pin is missing.
"""
from __future__ import annotations

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SOURCE = os.path.join(ROOT, "oracle", "qknorm_oracle.c")

# (name, text in the source, replacement, how many occurrences to change: None = all)
MUTANTS = [
    ("drop_eps", "sqrt(S / (double)H + eps)", "sqrt(S / (double)H)", None),
    ("sum_not_mean", "sqrt(S / (double)H + eps)", "sqrt(S + eps)", None),
    ("shard_width_divisor", "S / (double)H_full + eps", "S / (double)h_shard + eps", None),
    ("sqrt_not_rsqrt", "double r = 1.0 / sqrt(S / (double)H + eps);", "double r = sqrt(S / (double)H + eps);", None),
    ("decode_sign_flipped", "return sign ? -v : v;", "return sign ? v : -v;", None),
    ("exponent_bias_off_by_one", "expo - 134", "expo - 133", None),
    ("truncate_not_rne", "double n = nearbyint(ldexp(a, -q));", "double n = trunc(ldexp(a, -q));", None),
    ("round_half_away", "double n = nearbyint(ldexp(a, -q));", "double n = round(ldexp(a, -q));", None),
    ("gamma_indexed_by_token", "double g = load_elem(gamma, gamma_dtype(dtype), j);",
     "double g = load_elem(gamma, gamma_dtype(dtype), t);", None),
    ("e4m3_exponent_bias", "ldexp((double)(8 + mant), expo - 10)", "ldexp((double)(8 + mant), expo - 9)", None),
    ("e4m3_no_saturation", "    if (r > 448.0)\n        r = 448.0;\n", "", None),
    ("f16_subnormal_scale", "ldexp((double)mant, -24);", "ldexp((double)mant, -25);", None),
    ("f16_encode_bias", "((er - 1 + 15) << 10)", "((er - 1 + 14) << 10)", None),
    ("f16_subnormal_threshold", "round_to_grid(a, 11, -14)", "round_to_grid(a, 11, -15)", None),
    ("gamma_type_e4m3", "return dtype == ORACLE_E4M3 ? ORACLE_BF16 : dtype;", "return dtype;", None),
    ("heads_divide_by_row_width", "sqrt(S / (double)head_dim + eps)", "sqrt(S / (double)W + eps)", None),
    ("heads_gamma_by_column", "double g = load_elem(gamma, gamma_dtype(dtype), j);\n                double yv",
     "double g = load_elem(gamma, gamma_dtype(dtype), c0 + j);\n                double yv", None),
    ("stride_ignored", "double v = load_elem(x, dtype, t * x_stride + j);\n            double g",
     "double v = load_elem(x, dtype, t * (int64_t)H + j);\n            double g", 1),
    ("drop_last_shard", "for (int32_t p = 0; p < P; ++p)", "for (int32_t p = 0; p + 1 < P; ++p)", None),
    ("square_missing", "S += v * v;", "S += v * fabs(v) * 0.5 + v * v * 0.5;", None),
    ("proj_w_transposed", "load_elem(w, dtype, (int64_t)n * w_stride + d)",
     "load_elem(w, dtype, (int64_t)(d % N) * w_stride + (n % D))", None),
    ("proj_drop_last_term", "for (int32_t d = 0; d < D; ++d)", "for (int32_t d = 0; d + 1 < D; ++d)", None),
    ("proj_row_index", "const int64_t t = rows[i];", "const int64_t t = i < T ? i : T - 1;", None),
    ("proj_float_accumulation", "double acc = 0.0;\n            for (int32_t d",
     "float acc = 0.0f;\n            for (int32_t d", None),
]


def _mutate(src: str, old: str, new: str, occurrence) -> str:
    assert old in src, f"mutation anchor not found: {old!r}"
    return src.replace(old, new) if occurrence is None else src.replace(old, new, occurrence)


@pytest.mark.parametrize("name,old,new,occurrence", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new, occurrence):
    with open(SOURCE) as f:
        src = f.read()
    mutant_c = tmp_path / f"{name}.c"
    mutant_c.write_text(_mutate(src, old, new, occurrence))
    lib = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-shared",
                    "-fPIC", str(mutant_c), "-o", str(lib), "-lm"], check=True)
    env = dict(os.environ, QKNORM_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} survived the pin suite:\n{r.stdout[-2000:]}"
