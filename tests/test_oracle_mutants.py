"""Plants plausible mistakes in a copy of the oracle and checks that the pins catch each one.

Every mutant is built from a modified copy of oracle/hqq_oracle.c in a temporary folder and
run against tests/test_oracle_pins.py in a child process; the pins must fail for each.
"""
import os
import subprocess
import sys
import tempfile

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "hqq_oracle.c")

MUTANTS = {
    "t sign": ("float t = w * s + z;", "float t = w * s - z;"),
    "z0 from max": ("*z_out = 0.0f - mn * s;", "*z_out = 0.0f - mx * s;"),
    "s0 transposed": ("1.0f : qmax / d;", "1.0f : d / qmax;"),
    "no scale clamp": ("if (s > scale_max) s = scale_max;", ""),
    "no upper clip": ("if (q > qmax) q = qmax;", ""),
    "w_hat times s": ("float w_hat = (q - z) / s;", "float w_hat = (q - z) * s;"),
    "e sign": ("term[j] = q - (w[j] - e) * s;", "term[j] = q - (w[j] + e) * s;"),
    "e dropped": ("term[j] = q - (w[j] - e) * s;", "term[j] = q - w[j] * s;"),
    "mean over g-1": ("hqo_pairwise_sum(term, g) / (float)g;",
                      "hqo_pairwise_sum(term, g) / (float)(g - 1);"),
    "signed error": ("absr[j] = fabsf(r);", "absr[j] = r;"),
    "sequential sum": ("return pairwise(x, n, lo, len / 2) + pairwise(x, n, lo + len / 2, len / 2);",
                       "{ float a = 0.0f; for (int64_t i = lo; i < lo + len; i++) a = a + (i < n ? x[i] : 0.0f); return a; }"),
    "accept ties": ("if (!have_best || total < best) {", "if (!have_best || total <= best) {"),
    "keep unmeasured z": ("memcpy(z_out, z, sizeof(float) * (size_t)G);   /* z_i",
                          "memcpy(z_out, znext, sizeof(float) * (size_t)G);   /* z_i"),
    "beta not updated": ("beta = beta * kappa;", ""),
    "axis0 index": ("return axis == 1 ? k * g + j : j * G + k;", "return axis == 1 ? k * g + j : k * g + j;"),
    "1-bit one per byte": ("case 1: return (n + 7) / 8;", "case 1: return n;"),
    "nibble order": ("packed[i / per] |= (uint8_t)(codes[i] << (nbits * (i % per)));",
                     "packed[i / per] |= (uint8_t)(codes[i] << (nbits * (per - 1 - i % per)));"),
    "dequant group index": ("int64_t k = axis == 1 ? n / g : n % G;", "int64_t k = axis == 1 ? n / g : n / g;"),
    "dequant adds z": ("float v = ((float)codes[n] - zf) * df;", "float v = ((float)codes[n] + zf) * df;"),
    "half truncates": ("float m = rintf(ldexpf(a, 10 - expo));", "float m = truncf(ldexpf(a, 10 - expo));"),
    "delta not inverted": ("scale_h[k] = hqo_float_to_half(1.0f / s[k]);", "scale_h[k] = hqo_float_to_half(s[k]);"),
    "gemv transposed": ("(double)hqo_half_to_float(w[r * cols + c])", "(double)hqo_half_to_float(w[(c * rows + r) % N])"),
    "gemv x reversed": ("(double)hqo_half_to_float(x_h[c]);", "(double)hqo_half_to_float(x_h[cols - 1 - c]);"),
    "gemv signed magnitude": ("mag += fabs(p);", "mag += p;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not found once: {old!r}"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, str(mut), "-o", str(lib), "-lm"])
    env = dict(os.environ, HQO_LIB_OVERRIDE=str(lib))
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode != 0, f"mutant '{name}' passed every pin:\n{res.stdout[-2000:]}"
