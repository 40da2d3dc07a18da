"""The pins bite: copies of the C++ oracle with one planted mistake each (a wrong constant,
a dropped term, a wrong index or operand, a wrong rounding) are compiled and run against
the pins of tests/test_oracle_quant.py and tests/test_oracle_decoder.py; every copy must
fail at least one pin.  The mistakes are planted in copies on the CPU; the oracle itself is
not touched."""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "fg_oracle.cpp")
PINS = [os.path.join(ROOT, "tests", "test_oracle_quant.py"), os.path.join(ROOT, "tests", "test_oracle_decoder.py")]

# (name, text in fg_oracle.cpp, replacement); each text must occur in the source
MUTANTS = [
    ("scale divides by 16", "const float s32 = d / 15.0f;", "const float s32 = d / 16.0f;"),
    ("codes truncate instead of rounding", "float c = std::nearbyintf(r);", "float c = std::floor(r);"),
    ("scale not rounded to fp16", "const float s = h2f(s16);", "const float s = s32;"),
    ("nibbles swapped", "packed[r * (cols / 2) + j] = uint8_t((q[r * cols + 2 * j] & 15) | ((q[r * cols + 2 * j + 1] & 15) << 4));",
     "packed[r * (cols / 2) + j] = uint8_t((q[r * cols + 2 * j + 1] & 15) | ((q[r * cols + 2 * j] & 15) << 4));"),
    ("dequant drops the min", "return h2d(mn) + double(code) * h2d(s);", "return double(code) * h2d(s);"),
    ("fp16 rounding truncates", "double n = std::nearbyint(std::ldexp(a, 10 - e));", "double n = std::floor(std::ldexp(a, 10 - e));"),
    ("LayerNorm eps outside the root", "const double inv = std::sqrt(var + eps);", "const double inv = std::sqrt(var) + eps;"),
    ("LayerNorm drops beta", "* h2d(gamma[i]) + h2d(beta[i]));", "* h2d(gamma[i]));"),
    ("LN2 reads the block input (decode)", "orc_layernorm(x1.data(), B, h, ly->ln2_g", "orc_layernorm(xin.data(), B, h, ly->ln2_g"),
    ("LN2 reads the block input (prefill)", "orc_layernorm(x1.data(), BL, h, ly->ln2_g", "orc_layernorm(x, BL, h, ly->ln2_g"),
    ("linear drops the residual", "if (r) v += h2d(r[i * N + j]);", "(void)r;"),
    ("ReLU after the residual", "if (relu && v < 0.0) v = 0.0;\n        if (r) v += h2d(r[i * N + j]);",
     "if (r) v += h2d(r[i * N + j]);\n        if (relu && v < 0.0) v = 0.0;"),
    ("attention without 1/sqrt(hd)", "const double scale = 1.0 / std::sqrt(double(hd));", "const double scale = 1.0;"),
    ("prefill attention not causal", "for (int t = 0; t <= i; ++t)", "for (int t = 0; t < L; ++t)"),
    ("decode attends without the new token", "orc_decode_attention(qkv.data(), 3 * h, c, pos + 1, att.data());",
     "orc_decode_attention(qkv.data(), 3 * h, c, pos > 0 ? pos : 1, att.data());"),
    ("decode attention keys from the value cache", "orc_code_values(c->k_codes + row0 * (hd / 2), c->k_params",
     "orc_code_values(c->v_codes + row0 * (hd / 2), c->v_params"),
    ("generation skips the last prompt position", "x.data() + (size_t(b) * L + L - 1) * h",
     "x.data() + (size_t(b) * L + L - 2) * h"),
    ("position offset by one", "orc_embed(m, prev.data(), B, 1, L + step - 1, xd.data());",
     "orc_embed(m, prev.data(), B, 1, L + step, xd.data());"),
    ("argmax ties to the highest id", "if (logits[i * V + v] > logits[i * V + best]) best = v;",
     "if (logits[i * V + v] >= logits[i * V + best]) best = v;"),
    ("KV appended one position late", "const int64_t slot = (int64_t(b) * nh + j) * c->capacity + pos + t;",
     "const int64_t slot = (int64_t(b) * nh + j) * c->capacity + pos + t + 1;"),
    ("LM head reads E transposed", "acc += h2d(a[i * K + k]) * h2d(E[int64_t(v) * K + k]);",
     "acc += h2d(a[i * K + k]) * h2d(E[(int64_t(k) * V + v) % (int64_t(V) * K)]);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site not found: {name}"
    with tempfile.TemporaryDirectory() as d:
        mut = os.path.join(d, "mutant.cpp")
        so = os.path.join(d, "libmutant.so")
        with open(mut, "w") as f:
            f.write(src.replace(old, new))
        r = subprocess.run(["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared",
                            "-fPIC", "-o", so, mut], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
        env = dict(os.environ, FG_ORACLE_LIB=so, OMP_NUM_THREADS="2")
        r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider"] + PINS,
                           capture_output=True, text=True, env=env, cwd=ROOT, timeout=600)
        assert r.returncode != 0, f"no pin caught the planted mistake '{name}'\n{r.stdout[-2000:]}"
