"""Plants plausible mistakes in the oracle (on the CPU) and checks that the
pins in test_oracle_pins.py catch every one of them."""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "oracle.c")

# (name, exact text in oracle.c, replacement)
MUTATIONS = [
    ("pack_msb_first", "out[n * words + bitpos / 32] |= code << (bitpos % 32);",
     "out[n * words + bitpos / 32] |= code << (32 - bits - bitpos % 32);"),
    ("round_half_away", "float r = rintf(t);", "float r = roundf(t);"),
    ("int8_round_half_away", "float t = rintf(w[r * C + c] / s);", "float t = roundf(w[r * C + c] / s);"),
    ("scale_wrong_levels", "float scale = (mx - mn) / qmax;", "float scale = (mx - mn) / (qmax + 1.0f);"),
    ("dequant_sign", "fmaf((float)q[n * K + k], scales[n * G + k / g], biases[n * G + k / g])",
     "fmaf((float)q[n * K + k], scales[n * G + k / g], -biases[n * G + k / g])"),
    ("dequant_group_index", "scales[n * G + k / g], biases[n * G + k / g]",
     "scales[n * G + k / (2 * g)], biases[n * G + k / (2 * g)]"),
    ("matmul_drops_bias", "                if (bias)\n                    acc += (double)bias[n];",
     "                if (bias)\n                    acc += 0.0;"),
    ("bitlinear_row_map", "const int64_t r = n % R;\n            const int j = (int)(n / R);",
     "const int64_t r = n / 4;\n            const int j = (int)(n % 4);"),
    ("bitlinear_offset", "int v = (int)((P[r * K + k] >> (2 * j)) & 3u) - 1;",
     "int v = (int)((P[r * K + k] >> (2 * j)) & 3u) - 2;"),
    ("bitlinear_no_invert", "const float scale = invert ? 1.0f / ws : ws;", "const float scale = ws;"),
    ("int4_nibble_swap", "P[i * N + n] = (uint8_t)((c[0] << 4) | c[1]);",
     "P[i * N + n] = (uint8_t)((c[1] << 4) | c[0]);"),
    ("w4a8_zero_point", "int64_t p = (int64_t)qx[m * K + k] * (int64_t)(c - 8);",
     "int64_t p = (int64_t)qx[m * K + k] * (int64_t)(c - 7);"),
    ("w4a8_nibble_read", "int c = (k % 2 == 0) ? (byte >> 4) : (byte & 15);",
     "int c = (k % 2 == 0) ? (byte & 15) : (byte >> 4);"),
    ("int8_absmax_scale", "float s = amax / 127.0f;\n        if (s == 0.0f)\n            s = 1.0f;\n        scale[r] = s;",
     "float s = amax / 128.0f;\n        if (s == 0.0f)\n            s = 1.0f;\n        scale[r] = s;"),
    ("pack_drops_straddle", "                out[n * words + bitpos / 32 + 1] |= code >> (32 - bitpos % 32);",
     "                out[n * words + bitpos / 32 + 1] |= 0u;"),
    ("unpack_drops_straddle", "                v |= packed[n * words + bitpos / 32 + 1] << (32 - bitpos % 32);",
     "                v |= 0u;"),
    ("f16_ties_away", "    if (frac > 0.5 || (frac == 0.5 && fmod(fl, 2.0) != 0.0))", "    if (frac >= 0.5)"),
    ("f16_subnormal_spacing", "    if (q < -24)\n        q = -24;", "    if (q < -25)\n        q = -25;"),
    ("percentile_index_n", "const float h = (float)(n - 1) * q;", "const float h = (float)n * q;"),
    ("percentile_lerp_side", "r = t < 0.5f ? a + d * t : b - d * (1.0f - t);", "r = t < 0.5f ? a + d * t : b - d * t;"),
    ("percentile_no_zero_fallback", "        if (row_clip == 0.0f)\n            row_clip = amax;", "        if (row_clip < 0.0f)\n            row_clip = amax;"),
    ("percentile_no_clip", "            if (v < -row_clip) v = -row_clip;\n            if (v > row_clip) v = row_clip;", "            (void)row_clip;"),
    ("groups_scale_row_major", "scale_w[grp * N + n] = s;", "scale_w[n * G + grp] = s;"),
    ("pergroup_scale_index", "const double sw = (double)scale_w[grp * N + n];", "const double sw = (double)scale_w[n * G + grp];"),
    ("pergroup_m1_quantizes_x", "const int fp_act = M == 1;", "const int fp_act = 0;"),
    ("pergroup_drops_s_x", "                out *= (double)s_x[m];", "                out *= 1.0;"),
    ("groups_absmax_scale", "            float s = amax / 127.0f;\n            if (s == 0.0f)\n                s = 1.0f;\n            scale_w[grp * N + n] = s;",
     "            float s = amax / 128.0f;\n            if (s == 0.0f)\n                s = 1.0f;\n            scale_w[grp * N + n] = s;"),
    ("w8a8_scale_drop", "double sc = (double)s_x[m] * (double)scale_w[n];\n            double out = (double)acc * sc;\n            if (bias)\n                out += (double)bias[n];\n            y[m * N + n] = out;\n            absdot[m * N + n] = (double)mag * sc;\n        }\n    return overflow ? ORC_EOVERFLOW : 0;\n}\n\n/*\n * [W4]",
     "double sc = (double)scale_w[n];\n            double out = (double)acc * sc;\n            if (bias)\n                out += (double)bias[n];\n            y[m * N + n] = out;\n            absdot[m * N + n] = (double)mag * sc;\n        }\n    return overflow ? ORC_EOVERFLOW : 0;\n}\n\n/*\n * [W4]"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = tmp_path / "oracle_mut.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "liboracle_mut.so"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-std=c11",
                           "-shared", "-fPIC", "-o", str(so), str(mutated), "-lm"])
    env = dict(os.environ, ORACLE_SO_OVERRIDE=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"planted mistake {name} passed every pin:\n{r.stdout[-2000:]}"
