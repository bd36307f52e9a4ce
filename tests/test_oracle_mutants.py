"""Plant plausible mistakes in a copy of the oracle and require that the pins
catch every one: a dropped term, a wrong sign, a wrong index, a transposed
operand, the wrong rounding, the wrong qmax, the epsilon in the wrong place.

The mistakes are planted on the CPU only, in a temporary copy of
``oracle/qk_oracle.c``; the real oracle is untouched.
"""
import os
import shutil
import subprocess

import pytest

import oracle_pins
from oracle.oracle import Oracle, load

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "qk_oracle.c")

# (name, original text, planted text) -- the original must occur exactly once.
MUTANTS = [
    ("qmax_128", "float s = fmaxf(amax, 1e-12f) / 127.0f;", "float s = fmaxf(amax, 1e-12f) / 128.0f;"),
    ("eps_after_divide", "float s = fmaxf(amax, 1e-12f) / 127.0f;",
     "float s = fmaxf(amax / 127.0f, 1e-12f);"),
    ("round_half_away", "float r = nearbyintf(y);", "float r = roundf(y);"),
    ("round_truncate", "float r = nearbyintf(y);", "float r = truncf(y);"),
    ("absmax_signed", "float a = fabsf(x[i]);", "float a = x[i];"),
    ("gemm_dropped_first_term", "for (int i = 0; i < k; ++i) s += (int64_t)ar[i] * (int64_t)wr[i];",
     "for (int i = 1; i < k; ++i) s += (int64_t)ar[i] * (int64_t)wr[i];"),
    ("gemm_transposed_w", "const int8_t* wr = j->w + (int64_t)c * k;",
     "const int8_t* wr = j->w + (int64_t)(c % (j->m1 > 0 ? j->m1 : 1)) * k;"),
    ("gemm_int8_wrap", "if (s > INT32_MAX || s < INT32_MIN) j->overflow = 1;", ""),
    ("epi_wrong_scale_index", "o = o * sw[c];", "o = o * sw[r % n];"),
    ("epi_wrong_sign", "o = o * sa[r];", "o = o * -sa[r];"),
    ("epi_dropped_alpha", "      o = o * alpha;\n      out[", "      out["),
    ("epi_scales_multiplied_first", "      o = o * sa[r];\n      o = o * sw[c];",
     "      o = o * (sa[r] * sw[c]);"),
    ("epi_sw_before_sa", "      o = o * sa[r];\n      o = o * sw[c];", "      o = o * sw[c];\n      o = o * sa[r];"),
    ("epi_alpha_first", "      o = o * sa[r];\n      o = o * sw[c];\n      o = o * alpha;",
     "      o = o * alpha;\n      o = o * sa[r];\n      o = o * sw[c];"),
    ("group_unfused", "f = fmaf((float)(int32_t)p, j->sw[(int64_t)c * ng + g], f);",
     "f = f + (float)(int32_t)p * j->sw[(int64_t)c * ng + g];"),
    ("group_descending", "for (int g = 0; g < ng; ++g) {", "for (int g = ng - 1; g >= 0; --g) {"),
    ("group_sa_alpha_first", "float o = f * j->sa[r];\n        o = o * j->alpha;",
     "float o = f * (j->sa[r] * j->alpha);"),
    ("group_scale_transposed", "f = fmaf((float)(int32_t)p, j->sw[(int64_t)c * ng + g], f);",
     "f = fmaf((float)(int32_t)p, j->sw[(int64_t)g * ng + c % ng], f);"),
    ("group_dropped_last", "for (int g = 0; g < ng; ++g) {", "for (int g = 0; g < ng - 1; ++g) {"),
    ("exp_wrong_coeff", "p = fmaf(p, r, (float)(1.0 / 24.0));", "p = fmaf(p, r, (float)(1.0 / 25.0));"),
    ("exp_wrong_sign", "float e = qko_exp(-g);", "float e = qko_exp(g);"),
    ("silu_times", "return g / d;", "return g * d;"),
    ("bf16_round_half_up", "u += 0x7fffu + lsb;", "u += 0x8000u;"),
    ("bf16_truncate", "u += 0x7fffu + lsb;", "u += 0u * lsb;"),
    ("bf16_widen_wrong", "uint32_t u = ((uint32_t)b) << 16;", "uint32_t u = ((uint32_t)b) << 15;"),
    ("silu_ld_ignored", "float u = qko_load(up, dtype, (int64_t)r * ld + i);",
     "float u = qko_load(up, dtype, (int64_t)r * k + i);"),
    ("fp8_ties_away", "const float steps = nearbyintf(a / spacing); /* ties to even */",
     "const float steps = roundf(a / spacing);"),
    ("fp8_no_subnormal_floor", "if (E < -6) E = -6;", ""),
    ("fp8_bias_8", "return sign | (uint8_t)(((E2 + 7) << 3) | m);",
     "return sign | (uint8_t)(((E2 + 8) << 3) | m);"),
    ("fp8_decode_bias", ": ldexpf((float)(8 + m), e - 10);", ": ldexpf((float)(8 + m), e - 11);"),
    ("fp8_qmax_240", "float s = fmaxf(amax, 1e-12f) / 448.0f;", "float s = fmaxf(amax, 1e-12f) / 240.0f;"),
    ("fp8_ub_ignored", "if (ub && s > *ub) s = *ub;", ""),
    ("fp8_absmax_signed", "float ax = fabsf(x[i]);", "float ax = x[i];"),
    ("fp8_clamp_240", "if (y > 448.0f) y = 448.0f;", "if (y > 240.0f) y = 240.0f;"),
    ("fp8_silu_up_from_gate", "float uv = qko_load(up, dtype, (int64_t)r * ld + i);",
     "float uv = qko_load(gate, dtype, (int64_t)r * ld + i);"),
    ("asym_ties_away", "float r = nearbyintf(x[i] * inv) + z;", "float r = roundf(x[i] * inv) + z;"),
    ("asym_range_without_zero", "float lo = 0.0f, hi = 0.0f;", "float lo = x[0], hi = x[0];"),
    ("asym_qrange_256", "const float s = fmaxf(hi - lo, 1e-12f) / 255.0f;",
     "const float s = fmaxf(hi - lo, 1e-12f) / 256.0f;"),
    ("asym_zp_sign", "float z = nearbyintf(-128.0f - lo * inv);", "float z = nearbyintf(-128.0f + lo * inv);"),
    ("asym_clamp_127", "if (r < -128.0f) r = -128.0f;", "if (r < -127.0f) r = -127.0f;"),
    ("asym_gemm_zp_ignored", "s += ((int64_t)a[(int64_t)r * k + i] - zp[r]) * (int64_t)w[(int64_t)c * k + i];",
     "s += ((int64_t)a[(int64_t)r * k + i]) * (int64_t)w[(int64_t)c * k + i];"),
    ("asym_wsum_dropped", "for (int i = 0; i < k; ++i) t += w[(int64_t)c * k + i];",
     "for (int i = 1; i < k; ++i) t += w[(int64_t)c * k + i];"),
    ("static_ties_away", "float r = nearbyintf(qko_load(x, dtype, i) * inv);",
     "float r = roundf(qko_load(x, dtype, i) * inv);"),
    ("static_no_saturation", "    if (r > 127.0f) r = 127.0f;\n    if (r < -127.0f) r = -127.0f;\n    q[i] = (int8_t)(int)r;\n  }\n  return QKO_OK;",
     "    q[i] = (int8_t)(int)r;\n  }\n  return QKO_OK;"),
    ("fp8_gemm_units", ": (int64_t)(8 + m) << (e - 1);", ": (int64_t)(8 + m) << e;"),
    ("fp8_gemm_dropped_term", "for (int i = 0; i < j->k; ++i) s += qko_e4m3_units(ar[i]) * qko_e4m3_units(wr[i]);",
     "for (int i = 1; i < j->k; ++i) s += qko_e4m3_units(ar[i]) * qko_e4m3_units(wr[i]);"),
]


@pytest.fixture(scope="module")
def workdir(tmp_path_factory):
    return tmp_path_factory.mktemp("mutants")


@pytest.mark.parametrize("name,orig,planted", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(workdir, name, orig, planted):
    if shutil.which("gcc") is None:
        pytest.skip("gcc missing")
    text = open(SRC).read()
    assert text.count(orig) == 1, f"mutation anchor for {name} not unique"
    src = os.path.join(workdir, f"{name}.c")
    lib = os.path.join(workdir, f"lib{name}.so")
    with open(src, "w") as f:
        f.write(text.replace(orig, planted))
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
                    "-o", lib, src, "-lm"], check=True)
    O = Oracle(load(lib), nthreads=2)
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(O)
        except (AssertionError, OverflowError, ValueError) as e:  # a pin caught it
            failed.append(pin.__name__)
            del e
    assert failed, f"planted mistake {name} passed every pin"
