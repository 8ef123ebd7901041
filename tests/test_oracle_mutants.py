"""The pins must catch plausible mistakes in the oracle.

Each case plants one mistake in a private copy of the oracle's C source
(on the CPU, in a temporary directory), builds it, and runs the pin suite
against it in a subprocess: the suite must fail.  The real oracle is not
touched.
"""
import os
import subprocess
import sys

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

MUTANTS = {
    "rotation_sign": ("y[j] = c * xa - sn * xb;\n        y[j + h] = sn * xa + c * xb;",
                      "y[j] = c * xa + sn * xb;\n        y[j + h] = -sn * xa + c * xb;"),
    "pair_index": ("int p = (j >> (s + 1)) * h + (j & (h - 1));", "int p = j / 2;"),
    "stage_order": ("for (int s = 0; s < L; s++) stage_apply(y, d, s, angles + (size_t)s * (d / 2), 1.0);",
                    "for (int s = L - 1; s >= 0; s--) stage_apply(y, d, s, angles + (size_t)s * (d / 2), 1.0);"),
    "transpose_keeps_sign": ("stage_apply(y, d, s, angles + (size_t)s * (d / 2), -1.0);",
                             "stage_apply(y, d, s, angles + (size_t)s * (d / 2), 1.0);"),
    "input_not_transposed": ("oracle_butterfly_vec(d, theta_e, 1, x, xr);",
                             "oracle_butterfly_vec(d, theta_e, 0, x, xr);"),
    "theta_phi_swapped": ("oracle_butterfly_vec(d, phi_e, 0, z, u);",
                          "oracle_butterfly_vec(d, theta_e, 0, z, u);"),
    "alpha_dropped": ("u[i] *= (double)alpha;", "u[i] *= 1.0;"),
    "ternary_sign": ("else if (row[c] == -1) acc -= x[c];", "else if (row[c] == -1) acc += x[c];"),
    "ties_to_higher_index": ("return a < b;", "return a > b;"),
    "gate_normaliser": ("g[j] = exp(v[j] - m) / z;", "g[j] = exp(v[j] - m) / (z + 1e-3);"),
    "pack_codes_swapped": ("return v == 1 ? 1u : (v == -1 ? 3u : 0u);",
                           "return v == 1 ? 3u : (v == -1 ? 1u : 0u);"),
    "bucket_unstable": ("for (int i = 0; i < R; i++) perm[start[topk_idx[i]]++] = i;",
                        "for (int i = R - 1; i >= 0; i--) perm[start[topk_idx[i]]++] = i;"),
    "gate_dropped_in_sum": ("yt[i] += g[(size_t)t * k + j] * u[i];", "yt[i] += u[i];"),
    "offsets_inclusive": ("for (int e = 0; e <= N; e++) offsets[e] = start[e];",
                          "for (int e = 0; e <= N; e++) offsets[e] = start[e < N ? e + 1 : N];"),
    "zero_weight_as_plus_one": ("if (row[c] == 1) acc += x[c];", "if (row[c] >= 0) acc += x[c];"),
    "nan_not_rejected": ("if (isnan(logits[i])) return ORACLE_ERR_NONFINITE;",
                         "if (0 && isnan(logits[i])) return ORACLE_ERR_NONFINITE;"),
    "pack_bit_order_reversed": ("word |= code_of(w[(size_t)r * d + 16 * wd + i]) << (2 * i);",
                                "word |= code_of(w[(size_t)r * d + 16 * wd + i]) << (2 * (15 - i));"),
    "all_minus_inf_gate": ("for (int j = 0; j < k; j++) g[j] = 1.0 / k;",
                           "for (int j = 0; j < k; j++) g[j] = j == 0 ? 1.0 : 0.0;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    src = open(os.path.join(ROOT, "oracle", "bfmoe_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mut_src = tmp_path / "mutant.c"
    mut_src.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", str(mut_src), "-o", str(lib),
                    "-lm"], check=True)
    env = dict(os.environ, ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_oracle_pins.py")], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
