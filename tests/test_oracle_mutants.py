"""Each plausible mistake planted in a copy of the oracle must fail a pin.

The copy is patched as text, compiled with gcc into a temporary directory and
exercised in a subprocess (so a crash also counts as caught). The oracle source
itself is never modified.
"""

import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

from oracle import build as oracle_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "stem_oracle.c")

# (name, original text, planted mistake)
MUTANTS = [
    ("budget-sign", "exp(-(double)i / tau)", "exp((double)i / tau)"),
    ("budget-index", "ceil(rho * (double)(i + 1))", "ceil(rho * (double)(i))"),
    ("budget-no-clamp",
     "ceil(rho * (double)(i + 1));\n    double kk = want > (double)k_min ? want : (double)k_min;\n"
     "    if (kk > (double)(i + 1)) kk = (double)(i + 1);",
     "ceil(rho * (double)(i + 1));\n    double kk = want > (double)k_min ? want : (double)k_min;\n"),
    ("linear-no-cap",
     "ceil(k_lin);\n    double kk = want > (double)k_min ? want : (double)k_min;\n"
     "    if (kk > (double)(i + 1)) kk = (double)(i + 1);",
     "ceil(k_lin);\n    double kk = want > (double)k_min ? want : (double)k_min;\n"),
    ("linear-no-floor", "double want = ceil(k_lin);\n    double kk = want > (double)k_min ? want : (double)k_min;",
     "double want = ceil(k_lin);\n    double kk = want;"),
    ("pool-divisor", "qbar[u * D + d] = acc / n;", "qbar[u * D + d] = acc / (n - 1);"),
    ("pool-no-sqrt", "const double norm = sqrt(sq);", "const double norm = sq;"),
    ("pool-norm-of-mean", "sq += x * x;", "sq += x;"),
    ("metric-no-scale", "mrow[j] = dot * scale; /* s_ij", "mrow[j] = dot; /* s_ij"),
    ("metric-no-vnorm", "mrow[j] = p * vnorm[bg * nb + j];", "mrow[j] = p;"),
    ("metric-softmax-sign", "z += exp(mrow[j] - mx);", "z += exp(mx - mrow[j]);"),
    ("metric-gqa",
     "const int64_t bg = b * Hkv + h / G;\n    const double* qi = qbar + u * D;\n"
     "    double* mrow = m + bh * T + (int64_t)i * (i + 1) / 2;\n    double mx",
     "const int64_t bg = b * Hkv + h % Hkv;\n    const double* qi = qbar + u * D;\n"
     "    double* mrow = m + bh * T + (int64_t)i * (i + 1) / 2;\n    double mx"),
    ("additive-gqa",
     "const int64_t bg = b * Hkv + h / G;\n    const double* qi = qbar + u * D;\n"
     "    double* mrow = m + bh * T + (int64_t)i * (i + 1) / 2;\n    for",
     "const int64_t bg = b * Hkv + h % Hkv;\n    const double* qi = qbar + u * D;\n"
     "    double* mrow = m + bh * T + (int64_t)i * (i + 1) / 2;\n    for"),
    ("select-tie-order", "return (a->j > b->j) - (a->j < b->j);", "return (a->j < b->j) - (a->j > b->j);"),
    ("select-shift", "c[j - 1].m = mrow[j];", "c[j - 1].m = mrow[j - 1];"),
    ("select-no-sink", "chosen[n++] = 0;\n", "chosen[n++] = 1;\n"),
    ("attn-no-causal", "int last = (j == i) ? r : block - 1;", "int last = block - 1;"),
    ("attn-no-scale", "logit[nkeys] = dot * scale;", "logit[nkeys] = dot;"),
    ("attn-no-normalise", "const double w = logit[c] / z;", "const double w = logit[c];"),
    ("linear-denominator", "(double)i / (double)(nb - 1)", "(double)i / (double)nb"),
    ("linear-direction", "k_start * (1.0 - (1.0 - mu) * t)", "k_start * (mu + (1.0 - mu) * t)"),
    ("linear-floor", "double want = ceil(k_lin);", "double want = floor(k_lin);"),
    ("pool-max-is-mean", "vnorm[u] = vmax ? nmax : nacc / n;", "vnorm[u] = nacc / n;"),
    ("additive-no-clamp", "if (clamp && energy < 0.0) energy = 0.0;", ""),
    ("additive-no-square", "double energy = log(n * n);", "double energy = log(n);"),
    ("additive-no-scale", "mrow[j] = dot * scale + (beta", "mrow[j] = dot + (beta"),
    ("ragged-nb-floor", "  const int nb = (S + block - 1) / block;\n  const int64_t nq",
     "  const int nb = S / block;\n  const int64_t nq"),
    ("ragged-divisor", "qbar[u * D + d] = acc / n;", "qbar[u * D + d] = acc / block;"),
    ("ragged-vnorm-divisor", "vnorm[u] = vmax ? nmax : nacc / n;",
     "vnorm[u] = vmax ? nmax : nacc / block;"),
    ("ragged-last-rows", "for (int r = 0; r < block && (int64_t)i * block + r < S; ++r) {",
     "for (int r = 0; r < block && (int64_t)i * block + r < S - 1; ++r) {"),
    ("antidiag-main-diagonal", "(int64_t)w * stride + (stride - 1 - s);", "(int64_t)w * stride + s;"),
    ("antidiag-no-stride-scale", "const double scale = 1.0 / ((double)stride * sqrt((double)D));",
     "const double scale = 1.0 / sqrt((double)D);"),
    ("antidiag-strict-mask", "for (int w = 0; w <= u; ++w) {\n          double acc = 0.0;",
     "for (int w = 0; w < u; ++w) {\n          double acc = 0.0;"),
    ("antidiag-divisor", "prow[w / R] += exp(a[w] - mx) / z / n_i;",
     "prow[w / R] += exp(a[w] - mx) / z / R;"),
    ("antidiag-block-map", "prow[w / R] += exp(a[w] - mx) / z / n_i;",
     "prow[w / stride] += exp(a[w] - mx) / z / n_i;"),
    ("antidiag-gqa", "const int64_t kbase = (b * Hkv + h / G) * (int64_t)S;",
     "const int64_t kbase = (b * Hkv + h % Hkv) * (int64_t)S;"),
    ("antidiag-unnormalised", "prow[w / R] += exp(a[w] - mx) / z / n_i;",
     "prow[w / R] += exp(a[w] - mx) / n_i;"),
]


def _check(mutant, tmp):
    name, old, new = mutant
    src = open(SRC).read()
    assert src.count(old) == 1, f"{name}: pattern must occur exactly once"
    d = os.path.join(tmp, name)
    os.makedirs(d)
    csrc = os.path.join(d, "m.c")
    lib = os.path.join(d, "libm.so")
    with open(csrc, "w") as f:
        f.write(src.replace(old, new))
    flags = [f for f in oracle_build.CFLAGS if not f.startswith("-W")]  # as the oracle itself
    subprocess.run(["gcc"] + flags + ["-w", "-o", lib, csrc, "-lm"], check=True)
    env = dict(os.environ, STEM_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-c", "from tests import pins; pins.run_all()"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max_workers=4) as ex:
            results = list(ex.map(lambda m: _check(m, tmp), MUTANTS))
    survivors = [name for name, rc in results if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
