"""Plants plausible mistakes in a copy of the oracle, on the CPU, and checks
that the pins in test_oracle.py catch every one of them.  The real oracle
is never modified; each mutant is compiled to a temporary library and the
pin suite is run against it in a subprocess."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gemm_oracle.c")

MUTANTS = {
    "dropped_bias": ("s += bias[j];", "(void)bias;"),
    "wrong_sign": ("s += a * b;", "s -= a * b;"),
    "relu_clamps_positive": ("if (relu && s < 0.0)\n                s = 0.0;",
                             "if (relu && s > 0.0)\n                s = 0.0;"),
    "relu_before_bias": (
        "            if (bias)\n                s += bias[j];\n"
        "            if (relu && s < 0.0)\n                s = 0.0;\n"
        "            out[",
        "            if (relu && s < 0.0)\n                s = 0.0;\n"
        "            if (bias)\n                s += bias[j];\n"
        "            out["),
    "transposed_b": ("double b = b_colmajor ? B[(int64_t)j * ldb + k]\n"
                     "                                      : B[(int64_t)k * ldb + j];",
                     "double b = b_colmajor ? B[(int64_t)k * ldb + j]\n"
                     "                                      : B[(int64_t)j * ldb + k];"),
    "leading_dim_ignored": ("decode(src[(int64_t)r * ld + c], dtype)",
                            "decode(src[(int64_t)r * cols + c], dtype)"),
    "sampled_lda_ignored": ("decode(A[(int64_t)i * lda + k], dtype)",
                            "decode(A[(int64_t)i * K + k], dtype)"),
    "sampled_b_transposed": ("decode(b_colmajor ? B[(int64_t)j * ldb + k]\n"
                             "                                     : B[(int64_t)k * ldb + j], dtype)",
                             "decode(b_colmajor ? B[(int64_t)k * ldb + j]\n"
                             "                                     : B[(int64_t)j * ldb + k], dtype)"),
    "last_k_dropped": ("for (int k = 0; k < K; ++k) {\n                double a = A[",
                       "for (int k = 0; k < K - 1; ++k) {\n                double a = A["),
    "f16_exponent_off_by_one": ("ldexp((double)(1024 + f), e - 25)",
                                "ldexp((double)(1024 + f), e - 24)"),
    "f16_subnormal_scale": ("ldexp((double)f, -24)", "ldexp((double)f, -25)"),
    "bf16_exponent_off_by_one": ("ldexp((double)(128 + f), e - 134)",
                                 "ldexp((double)(128 + f), e - 133)"),
    "bf16_fraction_width": ("int f = h & 0x7f;", "int f = h & 0x3f;"),
    "f32_lda_ignored": ("a[(size_t)i * K + k] = (double)A[(int64_t)i * lda + k];",
                        "a[(size_t)i * K + k] = (double)A[(int64_t)i * K + k];"),
    "conv_pad_sign": ("const int ih = oh * sh - ph + kh * dh;",
                      "const int ih = oh * sh + ph + kh * dh;"),
    "conv_dilation_ignored": ("const int iw = ow * sw - pw + kw * dw;",
                              "const int iw = ow * sw - pw + kw;"),
    "grouped_b_not_advanced": ("B ? B + (int64_t)g * strideB : NULL", "B"),
    "grouped_bias_not_advanced": ("bias ? bias + (int64_t)g * N : NULL,\n                                 relu",
                                  "bias,\n                                 relu"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new)
    c = tmp_path / "mutant.c"
    so = tmp_path / "mutant.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                           "-o", str(so), str(c), "-lm"])
    env = dict(os.environ, GEMM_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
