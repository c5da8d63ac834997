"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a temporary copy of the oracle's C source
(on the CPU only), rebuilds it there, runs the pin suite against the copy,
and requires at least one pin to fail."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "silu_sign": ("return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    "nibble_order": ("int nib = (j % 2 == 0) ? (byte & 0xF) : (byte >> 4);",
                     "int nib = (j % 2 == 1) ? (byte & 0xF) : (byte >> 4);"),
    "twos_complement": ("int v = (nib >= 8) ? nib - 16 : nib;",
                        "int v = (nib >= 8) ? nib - 8 : nib;"),
    "dropped_scale": ("return (double)scale[i] * (double)v;", "return (double)v;"),
    "x_mask_strict": ("mx[i] = fabs(bf16_value(x[i])) >= (double)tau_x;",
                      "mx[i] = fabs(bf16_value(x[i])) > (double)tau_x;"),
    "s_mask_strict": ("if (mask_s) mask_s[j] = fabs(s) >= (double)tau_s;",
                      "if (mask_s) mask_s[j] = fabs(s) > (double)tau_s;"),
    "stage2_sparse_x": ("double xi = bf16_value(x[i]);\n                u += xi",
                        "double xi = bf16_value(x[i]) * (fabs(bf16_value(x[i])) >= 1.0);\n"
                        "                u += xi"),
    "down_transposed": ("y[k] += s * bf16_value(w_down[(size_t)j * d_model + k]);",
                        "y[k] += s * bf16_value(w_down[(size_t)(k % d_ff) * d_model + (j % d_model)]);"),
    "round_truncates": ("v = (int)nearbyintf(r);", "v = (int)r;"),
    "scale_over_8": ("float s = amax / 7.0f;", "float s = amax / 8.0f;"),
    "up_gate_swapped": ("s = u * activation(g, act);\n            for",
                        "s = g * activation(u, act);\n            for"),
    "gelu_half_dropped": ("return 0.5 * z * (1.0 + erf(z / sqrt(2.0)));",
                          "return z * (1.0 + erf(z / sqrt(2.0)));"),
    "gelu_scale": ("return 0.5 * z * (1.0 + erf(z / sqrt(2.0)));",
                   "return 0.5 * z * (1.0 + erf(z));"),
    "rank_ceil": ("double r = floor((1.0 - keep) * (double)n);",
                  "double r = ceil((1.0 - keep) * (double)n);"),
    "budget_term": ("s2 = e + 2.0 * alpha * (1.0 - s1) / 3.0;",
                    "s2 = e + alpha * (1.0 - s1) / 3.0;"),
    "rms_sum_not_mean": ("sqrt(ss / (double)d + eps)", "sqrt(ss + eps)"),
    "rms_eps_dropped": ("sqrt(ss / (double)d + eps)", "sqrt(ss / (double)d)"),
    "bf16_truncates": ("nearbyint(fabs(v) / q) * q", "floor(fabs(v) / q) * q"),
    "bf16_proxy_transposed": ("u[j] += xi * (pw_up ? bf16_value(pw_up[(size_t)j * d_model + i])",
                              "u[j] += xi * (pw_up ? bf16_value(pw_up[((size_t)i * d_ff + j) % ((size_t)d_ff * d_model)])"),
    "hist_upper_edge": ("    return (float)sel * w;", "    return (float)(sel + 1) * w;"),
    "hist_no_subsample": ("    long k = (n + max_samples - 1) / max_samples;",
                          "    long k = 1;"),
}


@pytest.fixture(scope="module")
def source():
    return open(os.path.join(ROOT, "oracle", "prox_oracle.c")).read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, source, tmp_path):
    before, after = MUTANTS[name]
    assert before in source, f"mutant anchor for {name} no longer in the oracle"
    ign = shutil.ignore_patterns("*.so", "__pycache__", "*.tmp*")
    shutil.copytree(os.path.join(ROOT, "oracle"), tmp_path / "oracle", ignore=ign)
    shutil.copytree(os.path.join(ROOT, "tests"), tmp_path / "tests", ignore=ign)
    pkg = tmp_path / "free_ffn_activation_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "free_ffn_activation_b200", "synth.py"), pkg / "synth.py")
    (pkg / "__init__.py").write_text("")
    (tmp_path / "oracle" / "prox_oracle.c").write_text(source.replace(before, after))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_oracle_pins.py"], cwd=tmp_path, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 1, f"mutant {name} survived:\n{r.stdout[-2000:]}"
