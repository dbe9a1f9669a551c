"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
catch each one.

Every mutation is a one-line change to a copy of oracle/dash_oracle.c, built
into a temporary library that the pin tests then load (through the oracle
package's DASH_ORACLE_LIB override).  A mutation that no pin detects would
mean the pins leave that part of the oracle unchecked.
"""
import os
import subprocess
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
SRC = ROOT / "oracle" / "dash_oracle.c"

# (name, original text, mutated text) -- each must occur in the source
MUTATIONS = [
    ("entmax exponent alpha-1 instead of 1/(alpha-1)",
     "const double k = 1.0 / (alpha - 1.0);\n    memcpy", "const double k = (alpha - 1.0);\n    memcpy"),
    ("alpha=1.5 closed form takes the larger root", "return m - sqrt(disc);", "return m + sqrt(disc);"),
    ("alpha=2 closed form off by one", "return (S1 - 1.0) / ks;", "return (S1 - 1.0) / (ks + 1);"),
    ("diagonal branch drops the query's own key", "for (int64_t t = d0; t <= d1; ++t) {\n        const float *kt",
     "for (int64_t t = d0; t < d1; ++t) {\n        const float *kt"),
    ("routing bias sign flipped", "(log(w[c]) - mu) / cf->sigma", "(mu - log(w[c])) / cf->sigma"),
    ("routing bias multiplied by sigma", "(log(w[c]) - mu) / cf->sigma", "(log(w[c]) - mu) * cf->sigma"),
    ("own chunk routed as well", "nvis = first_local < n_chunks ? first_local : n_chunks;",
     "nvis = first_local + 1 < n_chunks ? first_local + 1 : n_chunks;"),
    ("group prior not averaged", "wg[c] += ph[c] / g;", "wg[c] += ph[c];"),
    ("Stage-1 scale 1/d instead of 1/sqrt(d)", "const double zscale = gamma / sqrt((double)d);",
     "const double zscale = gamma / (double)d;"),
    ("Stage-2 scale dropped", "const double scale = 1.0 / sqrt((double)d);\n    /* gather",
     "const double scale = 1.0;\n    /* gather"),
    ("pooling divides by B on a partial chunk", "out[e] /= cnt;", "out[e] /= (double)B;"),
    ("support decided by >= instead of >", "if (s[c] > tau_h) rt[c] = 1;", "if (s[c] >= tau_h - 1e-3) rt[c] = 1;"),
    ("learned pooling drops 1/sqrt(d)", "score[j] = acc * inv_sqrt_d;", "score[j] = acc;"),
    ("learned pooling weights not normalised", "const double a = exp(score[j] - smax) / z;",
     "const double a = exp(score[j] - smax);"),
    ("learned pooling uses chunk 0's query everywhere", "const float *qb = Qbar + ((size_t)c * hkv + r) * d;",
     "const float *qb = Qbar + (size_t)r * d;"),
    ("two-block window drops the previous chunk",
     "const int first_local = ci - (local - 1) > 0 ? ci - (local - 1) : 0;", "const int first_local = ci;"),
    ("forward ignores the learned query", "if (Qbar)\n        dash_oracle_pool_q(", "if (0)\n        dash_oracle_pool_q("),
]


@pytest.mark.parametrize("name,orig,mut", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_mutation(tmp_path, name, orig, mut):
    src = SRC.read_text()
    assert src.count(orig) == 1, "mutation anchor not unique: " + name
    msrc = tmp_path / "dash_oracle_mut.c"
    msrc.write_text(src.replace(orig, mut))
    lib = tmp_path / "libdash_oracle_mut.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fvisibility=hidden", str(msrc),
                    "-o", str(lib), "-lm"], check=True)
    env = dict(os.environ, DASH_ORACLE_LIB=str(lib), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        str(ROOT / "tests" / "test_oracle_pins.py")], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    # a failed pin or a crash of the broken oracle both count as detection
    assert r.returncode != 0, "no pin detected the planted mistake: " + name
