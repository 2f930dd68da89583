"""Plant plausible mistakes in the oracle and check that its pins catch each one.

Each mutant is a copy of the oracle's C source with one textual change,
compiled into a temporary directory; the pin suite is then run against it in a
subprocess and must fail.  The committed oracle is never modified.
"""
from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
SRC = ROOT / "oracle" / "segpaged_oracle.c"

MUTANTS = {
    "window_one_too_wide": ("(j >= p - window + 1)", "(j >= p - window)"),
    "window_excludes_query": ("(j >= p - window + 1)", "(j >= p - window + 2)"),
    "sink_one_too_wide": ("(j < sink)", "(j <= sink)"),
    "sink_dropped": ("(j < sink) ||", "0 ||"),
    "not_causal": ("if (j > p) return 0;", ""),
    "scale_dropped": ("s[j] = scale * acc;", "s[j] = acc;"),
    "values_from_keys": ("o[t] += e * v[j * d + t];", "o[t] += e * k[j * d + t];"),
    "transposed_key_index": ("acc += qr[t] * k[j * d + t];", "acc += qr[t] * k[t * d + j % d];"),
    "lse_without_max": ("*lse = m + log(denom);", "*lse = log(denom);"),
    "dense_treated_as_local": ("if (kind == ORACLE_GLOBAL || kind == ORACLE_DENSE) return 1;",
                               "if (kind == ORACLE_GLOBAL) return 1;"),
    "stored_only_last_query": ("for (int64_t p = q0; p < L && !keep; ++p)", "for (int64_t p = L - 1; p < L && !keep; ++p)"),
    # RETRIEVAL heads: visibility of kept blocks and the top-p block selection
    "retrieval_kept_blocks_ignored": ("return kind == ORACLE_RETRIEVAL && sel[j / block] != 0;", "return 0;"),
    "retrieval_kept_block_shifted": ("&& sel[j / block] != 0;", "&& sel[(j + 1) / block] != 0;"),
    "retrieval_ties_to_higher_block": ("if (best < 0 || mass[i] > mass[best]) best = i;",
                                       "if (best < 0 || mass[i] >= mass[best]) best = i;"),
    "retrieval_least_important_first": ("mass[i] > mass[best]", "mass[i] < mass[best]"),
    "retrieval_threshold_strict": ("if (run >= target) {", "if (run > target) {"),
    "retrieval_sink_blocks_are_candidates": ("if (taken[i] || (i + 1) * block <= sink) continue;",
                                             "if (taken[i]) continue;"),
    "retrieval_top_p_one_drops_empty_blocks": ("} else if (top_p < 1.0f) {", "} else if (top_p <= 1.0f) {"),
    # attention mass per block (retrieval importance scoring pass)
    "block_mass_not_averaged": ("mass[j / block] += a[j] / z / (double)g;", "mass[j / block] += a[j] / z;"),
    "block_mass_shifted_block": ("mass[j / block] += a[j] / z / (double)g;",
                                 "mass[(j > 0 ? j - 1 : 0) / block] += a[j] / z / (double)g;"),
    "block_mass_scale_dropped": ("a[j] = scale * acc;", "a[j] = acc;"),
    "block_mass_rotated_dims": ("acc += qh[t] * k[j * d + t];", "acc += qh[t] * k[j * d + (t + 1) % d];"),
    "block_mass_base_two": ("a[j] = exp(a[j] - m);", "a[j] = exp2(a[j] - m);"),
    "block_mass_first_query_only": ("const double* qh = q + h * d;", "const double* qh = q;"),
    # FP8 E4M3 encoder / decoder
    "e4m3_bias_8": ("ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)"),
    "e4m3_subnormal_step": ("ldexp((double)m, -9)", "ldexp((double)m, -10)"),
    "e4m3_ties_up": ("(down < up || (down == up && ((lo - 1) & 1) == 0))", "(down < up)"),
    "e4m3_saturates_to_nan": ("if (a >= 448.0) return sgn | 0x7E;", "if (a >= 448.0) return sgn | 0x7F;"),
    "e4m3_inv_scale_dropped": ("oracle_e4m3_encode_f32(x[i] * inv_scale)", "oracle_e4m3_encode_f32(x[i])"),
    "e4m3_decode_scale_dropped": ("values[i] = oracle_e4m3_value(codes[i]) * scale;",
                                  "values[i] = oracle_e4m3_value(codes[i]);"),
}


@pytest.mark.slow
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = SRC.read_text()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", str(mut), "-o", str(lib), "-lm"],
                   check=True)
    env = dict(os.environ, SEGPAGED_ORACLE_LIB=str(lib), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        str(ROOT / "tests" / "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
