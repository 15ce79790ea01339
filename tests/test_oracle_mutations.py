"""The oracle's pins catch plausible mistakes planted in the oracle.

Each case copies the oracle's C source, plants one mistake (a dropped term,
a wrong sign, index or constant, a transposed operand, the wrong rounding
rule), builds it with the oracle's own flags into a temporary library and
runs the pin tests against it in a fresh process.  The pins must fail for
every mutant.  Everything here runs on the CPU.
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "gamma_signed_mean": ("row += fabs((double)W[n * K + k]);", "row += (double)W[n * K + k];"),
    "gamma_fp32_accumulate": ("double row = 0.0;", "float row = 0.0f;"),
    "gamma_divides_by_rows": ("return (float)(total / (double)(N * K));", "return (float)(total / (double)(K));"),
    "ternary_no_eps": ("float d = gamma + ORACLE_EPS;", "float d = gamma;"),
    "ternary_round_half_away": ("float t = rintf(r);", "float t = roundf(r);"),
    "ternary_no_clamp": ("if (t > 1.0f) t = 1.0f;", ";"),
    "pack_swapped_fields": ("word |= code << (8 * b + 2 * j);", "word |= code << (8 * j + 2 * b);"),
    "pack_signed_code": ("uint32_t code = (uint32_t)(t + 1);", "uint32_t code = (uint32_t)(t & 3);"),
    "act_scale_128": ("float scale = 127.0f / fmaxf(amax, ORACLE_EPS);", "float scale = 128.0f / fmaxf(amax, ORACLE_EPS);"),
    "act_round_half_away": ("float v = rintf(x[m * K + k] * scale);", "float v = roundf(x[m * K + k] * scale);"),
    "act_signed_max": ("float a = fabsf(x[m * K + k]);", "float a = x[m * K + k];"),
    "act_rowsum_of_abs": ("sum += (int8_t)v;", "sum += abs((int8_t)v);"),
    "act_scale_without_eps": ("float scale = 127.0f / fmaxf(amax, ORACLE_EPS);", "float scale = 127.0f / amax;"),
    "unpack_wrong_field": ("uint32_t code = (word >> (8 * b + 2 * j)) & 3u;", "uint32_t code = (word >> (8 * j + 2 * b)) & 3u;"),
    "bf16_truncates": ("double r = rint(ldexp(a, -qexp));", "double r = floor(ldexp(a, -qexp));"),
    "bf16_no_subnormal_spacing": ("if (qexp < -133) qexp = -133;", ";"),
    "acc_transposed_weight": ("(int64_t)T[n * K + k];", "(int64_t)T[k * N + n];"),
    "dequant_multiplies_scale": ("(double)gamma / (double)s[m];", "(double)gamma * (double)s[m];"),
    "dequant_gamma_plus_eps": ("(double)gamma / (double)s[m];", "((double)gamma + 1e-5) / (double)s[m];"),
    "bf16_via_fp32": ("double r = rint(ldexp(a, -qexp));", "double r = rint(ldexp((double)(float)a, -qexp));"),
    "rms_divides_by_k_minus_1": ("double ms = ss / (double)K;", "double ms = ss / (double)(K - 1);"),
    "rms_eps_outside_sqrt": ("float r = (float)(1.0 / sqrt(ms + (double)eps));",
                             "float r = (float)(1.0 / (sqrt(ms) + (double)eps));"),
    "rms_gain_ignored": ("if (g) v = v * g[k];", ";"),
    "rms_sum_of_abs": ("ss += v * v;", "ss += fabs(v);"),
    "rms_no_bf16_rounding": ("if (g) v = v * g[k];\n      if (out_bf16) {", "if (g) v = v * g[k];\n      if (0) {"),
    "glu_relu_not_squared": ("h = (g * g) * up[i];", "h = g * up[i];"),
    "glu_relu_not_clamped": ("float g = gate[i] > 0.0f ? gate[i] : 0.0f;", "float g = gate[i];"),
    "glu_silu_wrong_sign": ("h = (float)(z / (1.0 + exp(-z)) * (double)up[i]);",
                            "h = (float)(z / (1.0 + exp(z)) * (double)up[i]);"),
    "glu_silu_ignores_up": ("h = (float)(z / (1.0 + exp(-z)) * (double)up[i]);", "h = (float)(z / (1.0 + exp(-z)));"),
    "ste_input_without_gamma": ("dx[m * K + k] = (double)gamma * sum;", "dx[m * K + k] = sum;"),
    "ste_xhat_multiplies_scale": ("float v = (float)q[m * K + k] / s[m];", "float v = (float)q[m * K + k] * s[m];"),
    "ste_xhat_not_rounded": ("xhat[m * K + k] = v;", "xhat[m * K + k] = (float)q[m * K + k] / s[m];"),
    "ste_weight_reversed_k": ("sum += (double)dy[m * N + n] * (double)xhat[m * K + k];",
                              "sum += (double)dy[m * N + n] * (double)xhat[m * K + (K - 1 - k)];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, tmp_path):
    before, after = MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(before) == 1, "mutation site not found: " + name
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(before, after))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, str(mutated), "-o", str(so), "-lm"])
    env = dict(os.environ, BITLINEAR_ORACLE_LIB=str(so))
    res = subprocess.run(
        [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
         os.path.join(ROOT, "tests", "test_oracle_pins.py")],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=600,
    )
    assert res.returncode != 0, "pins did not catch mutant %s:\n%s" % (name, res.stdout[-2000:])
