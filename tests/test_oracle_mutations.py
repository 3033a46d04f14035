"""Plant mistakes in the oracle (on the CPU) and check that the pins catch each.

Each mutation edits one line of the oracle's C source, builds it into a
temporary library, and runs the pin suite against that build in a child
process.  A plausible slip anywhere in the oracle (a dropped term, a wrong
sign or index, a swapped operand, another rounding rule) must fail a pin.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "kvq_oracle.c")

MUTATIONS = {
    "butterfly_sign": ("t[i + h] = a - b;\n            }\n    for (int i = 0; i < D; ++i)\n        y[i] = t[i] * 0.0625f;",
                       "t[i + h] = b - a;\n            }\n    for (int i = 0; i < D; ++i)\n        y[i] = t[i] * 0.0625f;"),
    "fwht_dropped_stage": ("for (int h = 1; h < D; h <<= 1)\n        for (int i = 0; i < D; ++i)\n            if ((i & h) == 0) {\n                float a",
                           "for (int h = 2; h < D; h <<= 1)\n        for (int i = 0; i < D; ++i)\n            if ((i & h) == 0) {\n                float a"),
    "fwht_no_normalisation": ("y[i] = t[i] * 0.0625f;", "y[i] = t[i] * 0.125f;"),
    "q4_scale_sign": ("float d32 = xb[imax] / -8.0f;", "float d32 = xb[imax] / 8.0f;"),
    "q4_tie_last_index": ("if (fabsf(xb[j]) > amax) {", "if (fabsf(xb[j]) >= amax) {"),
    "q4_reciprocal_multiply": ("float r = rintf(xb[j] / df);", "float r = rintf(xb[j] * (1.0f / df));"),
    "q4_truncate": ("float r = rintf(xb[j] / df);", "float r = truncf(xb[j] / df);"),
    "q4_no_clamp_high": ("if (c > 15) c = 15;", "if (c > 16) c = 16;"),
    "int8_range_128": ("if (c < -127) c = -127;", "if (c < -128) c = -128;"),
    "int8_divisor": ("float d32 = amax / 127.0f;", "float d32 = amax / 128.0f;"),
    "f16_ties_away": ("if (rem > half || (rem == half && (q & 1u)))\n        q += 1;\n    if (e >= -14)",
                      "if (rem >= half)\n        q += 1;\n    if (e >= -14)"),
    "dequant_offset": ("out[j] = (double)((int)c[j] - 8) * (double)oracle_f16_to_f32(s[j / 32]);",
                       "out[j] = (double)((int)c[j] - 7) * (double)oracle_f16_to_f32(s[j / 32]);"),
    "dequant_scale_index": ("out[j] = (double)ci[j] * (double)oracle_f16_to_f32(s[j / 64]);",
                            "out[j] = (double)ci[j] * (double)oracle_f16_to_f32(s[j / 32 % 4]);"),
    "softmax_scale": ("s[(size_t)h * T + t] = acc / 16.0;", "s[(size_t)h * T + t] = acc / 8.0;"),
    "no_max_subtraction_merge": ("la[h] = la[h] * fa + lb[h] * fb;", "la[h] = la[h] + lb[h] * fb;"),
    "k8v4_rotates_k": ("case ORACLE_K8V4: *k_part = PART_INT8; *v_part = PART_Q4_0; *k_rot = 0; *v_rot = 1; return 0;",
                       "case ORACLE_K8V4: *k_part = PART_INT8; *v_part = PART_Q4_0; *k_rot = 1; *v_rot = 1; return 0;"),
    "no_unrotation": ("if (vrot) oracle_fwht256_f64(tmp, out + D * h);", "if (0) oracle_fwht256_f64(tmp, out + D * h);"),
    "q8_bytes": ("case ORACLE_Q4_0: return 2 * (128 + 8 * 2);", "case ORACLE_Q4_0: return 2 * (128 + 4 * 2);"),
    # fp8 / nvfp4 codecs
    "e4m3_bias": ("v = ldexp(8.0 + m, e - 10);", "v = ldexp(8.0 + m, e - 9);"),
    "e4m3_subnormal_step": ("v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    "small_format_no_saturation": ("return r > vmax ? vmax : r;", "return r;"),
    "small_format_ties_away": ("double r = rint(a / quantum) * quantum;", "double r = round(a / quantum) * quantum;"),
    "e2m1_exponent": ("double v = (e == 0) ? 0.5 * m : ldexp(2.0 + m, e - 2);",
                      "double v = (e == 0) ? 0.5 * m : ldexp(2.0 + m, e - 1);"),
    "fp8_divisor": ("float dq = amax / 448.0f;", "float dq = amax / 240.0f;"),
    "nvfp4_divisor": ("uint8_t sb = oracle_f32_to_e4m3(amax / 6.0f);", "uint8_t sb = oracle_f32_to_e4m3(amax / 4.0f);"),
    "nvfp4_block_32": ("(double)oracle_e4m3_to_f32((uint8_t)s[j / 16]);", "(double)oracle_e4m3_to_f32((uint8_t)s[j / 32]);"),
    "fp8_bytes": ("case ORACLE_FP8: return 2 * (256 + 1 * 2);", "case ORACLE_FP8: return 2 * (256 + 2 * 2);"),
}
PIN_FILES = ("test_oracle_pins.py", "test_oracle_fp_formats.py")


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    with tempfile.TemporaryDirectory() as d:
        csrc = os.path.join(d, "m.c")
        so = os.path.join(d, "libm.so")
        open(csrc, "w").write(src.replace(old, new))
        subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-o", so, csrc, "-lm"],
                       check=True)
        env = dict(os.environ, KVQ_ORACLE_LIB=so)
        r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider"] +
                           [os.path.join(ROOT, "tests", f) for f in PIN_FILES],
                           env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
        assert r.returncode != 0, f"mutation {name} survived the pins:\n{r.stdout[-2000:]}"
