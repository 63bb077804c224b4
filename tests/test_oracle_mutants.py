"""Planted mistakes in the oracle must fail its pins (CPU only).

Each mutant is a copy of ``oracle/gn_oracle.c`` with one plausible mistake (a dropped term,
a wrong sign, a wrong index, a wrong constant). It is compiled into a temporary directory
and the pin suite runs against it in a child process; the suite must fail for every mutant.
The mistakes are planted only in these throw-away copies of the CPU oracle.
"""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gn_oracle.c")

MUTANTS = {
    "rms_bwd_drops_centering": ("dx[j] = r * (g * wp[j] - xh * c);", "dx[j] = r * (g * wp[j]);"),
    "rms_eps_outside_sqrt": ("return 1.0 / sqrt(ss / (double)n + eps);",
                             "return 1.0 / (sqrt(ss / (double)n) + eps);"),
    "rms_mean_over_n_minus_1": ("return 1.0 / sqrt(ss / (double)n + eps);",
                                "return 1.0 / sqrt(ss / (double)(n - 1) + eps);"),
    "gemma_offset_dropped": ("wp[j] = (gemma ? 1.0 : 0.0) + rd(w, w_dt, j);", "wp[j] = rd(w, w_dt, j);"),
    "gelu_without_cubic": ("double t = tanh(gelu_k() * (z + GELU_C * z * z * z));\n    return",
                           "double t = tanh(gelu_k() * z);\n    return"),
    "gelu_grad_missing_3": ("(1.0 + 3.0 * GELU_C * z * z)", "(1.0 + GELU_C * z * z)"),
    "silu_wrong_sign": ("return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    "ln_unbiased_variance": ("v /= (double)n;", "v /= (double)(n - 1);"),
    "ln_bwd_drops_mean_term": ("dx[j] = s * (g * w[j] - c1 - xh * c2);", "dx[j] = s * (g * w[j] - xh * c2);"),
    "ln_bias_ignored": ("bv[j] = b ? rd(b, dt, j) : 0.0;", "bv[j] = 0.0;"),
    "rope_sign_swapped": ("out[2 * i] = a * co - c * si;", "out[2 * i] = a * co + c * si;"),
    "rope_half_split_pairs": ("double a = x[2 * i], c = x[2 * i + 1];", "double a = x[i], c = x[i + d / 2];"),
    "rope_table_row_from_batch": ("rd_row(cos_t, tab_dt, s * (D / 2), D / 2, cs);",
                                  "rd_row(cos_t, tab_dt, ((s + b) % S) * (D / 2), D / 2, cs);"),
    "qk_bwd_forward_rotation": ("rope_row(grow, cs, sn, D, -1, u);", "rope_row(grow, cs, sn, D, +1, u);"),
    "dw_without_xhat": ("if (dw_acc) dw_acc[j] += g * xh;", "if (dw_acc) dw_acc[j] += g;"),
    "bf16_widen_wrong_shift": ("[i]) << 16;", "[i]) << 15;"),
    "norm_linear_transposed_weight": ("acc += xn[k] * wt[n * K + k];", "acc += xn[k] * wt[k * N + n];"),
    "norm_linear_drops_bias": ("double acc = bias ? rd(bias, bias_dt, n) : 0.0;", "double acc = 0.0;"),
    "norm_linear_uncentred": ("xn[k] = (row[k] - mu) * s * gv[k] + bv[k];", "xn[k] = row[k] * s * gv[k] + bv[k];"),
    "linear_bwd_drops_act_grad": ("gr[n] = rd(dy, dy_dt, m * N + n) * oracle_act_grad(act, z);",
                                  "gr[n] = rd(dy, dy_dt, m * N + n);"),
    "linear_bwd_dx_from_wrong_column": ("acc += gr[n] * wt[n * K + k];", "acc += gr[n] * wt[n * K + (K - 1 - k)];"),
}


def _run_mutant(name, tmp):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert old in src, f"mutant {name}: pattern not found in the oracle"
    path = os.path.join(tmp, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(tmp, f"lib_{name}.so")
    subprocess.run(["gcc", "-std=c11", "-D_DEFAULT_SOURCE", "-O2", "-fPIC", "-shared", "-I",
                    os.path.join(ROOT, "oracle"), "-o", lib, path, "-lm"], check=True)
    env = dict(os.environ, GN_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    return name, r.returncode


def test_every_planted_mistake_fails_the_pins():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max(1, min(8, os.cpu_count() or 1))) as ex:
            results = dict(ex.map(lambda n: _run_mutant(n, tmp), MUTANTS))
    survivors = [n for n, rc in results.items() if rc == 0]
    assert not survivors, f"pins did not catch: {survivors}"
    # rc 1 = tests failed (as wanted); anything else would be a crash of the harness
    assert all(rc == 1 for rc in results.values()), results
