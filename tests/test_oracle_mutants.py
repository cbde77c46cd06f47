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

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "stem_oracle.c")

# (name, original text, planted mistake)
MUTANTS = [
    ("budget-sign", "exp(-(double)i / tau)", "exp((double)i / tau)"),
    ("budget-index", "ceil(rho * (double)(i + 1))", "ceil(rho * (double)(i))"),
    ("budget-no-clamp", "if (kk > (double)(i + 1)) kk = (double)(i + 1);", ""),
    ("pool-divisor", "qbar[u * D + d] = acc / block;", "qbar[u * D + d] = acc / (block - 1);"),
    ("pool-no-sqrt", "nacc += sqrt(sq);", "nacc += sq;"),
    ("pool-norm-of-mean", "sq += x * x;", "sq += x;"),
    ("metric-no-scale", "mrow[j] = dot * scale; /* s_ij", "mrow[j] = dot; /* s_ij"),
    ("metric-no-vnorm", "mrow[j] = p * vnorm[bg * nb + j];", "mrow[j] = p;"),
    ("metric-softmax-sign", "z += exp(mrow[j] - mx);", "z += exp(mx - mrow[j]);"),
    ("metric-gqa", "const int64_t bg = b * Hkv + h / G;", "const int64_t bg = b * Hkv + h % Hkv;"),
    ("select-tie-order", "return (a->j > b->j) - (a->j < b->j);", "return (a->j < b->j) - (a->j > b->j);"),
    ("select-shift", "c[j - 1].m = mrow[j];", "c[j - 1].m = mrow[j - 1];"),
    ("select-no-sink", "chosen[n++] = 0;\n", "chosen[n++] = 1;\n"),
    ("attn-no-causal", "const int last = (j == i) ? r : block - 1;", "const int last = block - 1;"),
    ("attn-no-scale", "logit[nkeys] = dot * scale;", "logit[nkeys] = dot;"),
    ("attn-no-normalise", "const double w = logit[c] / z;", "const double w = logit[c];"),
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
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-w", "-o", lib, csrc, "-lm"],
                   check=True)
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
