"""The pins must be sharp: plant one plausible mistake at a time in a copy
of the oracle's C source (on the CPU), build it, and check that the pin
suite fails against that copy."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

MUTANTS = {
    "q4_offset": ("W[(long)r * K + k] = s * (double)(c - 8);",
                  "W[(long)r * K + k] = s * (double)(c - 7);"),
    "q4_nibble_order": ("int c = (k % 2 == 0) ? (byte & 0xf) : (byte >> 4);",
                        "int c = (k % 2 == 0) ? (byte >> 4) : (byte & 0xf);"),
    "q2_min_dropped": ("W[(long)r * K + k] = s * (double)q + m;",
                       "W[(long)r * K + k] = s * (double)q + 0.0 * m;"),
    "silu_sign": ("return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    "gate_up_swapped": ("a[r] = orc_silu(g) * u;", "a[r] = orc_silu(u) * g;"),
    "down_transposed": ("acc += Wd[(long)o * f + r] * a[r];",
                        "acc += Wd[(long)r * d + o] * a[r];"),
    "tie_to_higher_id": ("if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;",
                         "if (!taken[e] && (best < 0 || l[e] >= l[best])) best = e;"),
    "softmax_not_renormalised": ("w[(long)t * k + j] = exp(l[idx[(long)t * k + j]] - lmax) / den;",
                                 "w[(long)t * k + j] = exp(l[idx[(long)t * k + j]] - lmax);"),
    "shared_dropped": ("acc += yshared[(long)t * d + o];", "acc += 0.0;"),
    "bias_dropped": ("if (bias) acc += (double)bias[e];", "if (bias) acc += 0.0;"),
    "eps_outside_sqrt": ("double inv = 1.0 / sqrt(ss / (double)d + eps);",
                         "double inv = 1.0 / (sqrt(ss / (double)d) + eps);"),
    "q4_round_half_away": ("double t = rint(w[i] / s);", "double t = round(w[i] / s);"),
    "q2_round_half_away": ("double t = rint((w[i] - m) / s);", "double t = round((w[i] - m) / s);"),
    "q4_clamp_low_7": ("q = t < -8.0 ? -8 : t > 7.0 ? 7 : (int)t;",
                       "q = t < -7.0 ? -7 : t > 7.0 ? 7 : (int)t;"),
    "bucket_descending": ("for (int t = 0; t < T; ++t)\n    for (int j = 0; j < k; ++j) {\n      int e = idx[(long)t * k + j];\n      perm",
                          "for (int t = T - 1; t >= 0; --t)\n    for (int j = 0; j < k; ++j) {\n      int e = idx[(long)t * k + j];\n      perm"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not found: {name}"
    mut = tmp_path / "moe_oracle.c"
    mut.write_text(src.replace(old, new))
    hdr = os.path.join(ROOT, "oracle", "moe_oracle.h")
    (tmp_path / "moe_oracle.h").write_text(open(hdr).read())
    so = tmp_path / "liboracle_mut.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared",
                           "-ffp-contract=off", "-o", str(so), str(mut), "-lm"])
    env = dict(os.environ, MOE_ORACLE_SO=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"planted mistake {name} passed every pin:\n{r.stdout[-2000:]}"
