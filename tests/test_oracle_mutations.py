"""Plant plausible mistakes in a copy of the oracle and check the pins fail.

Each mutation edits one expression of ``oracle/oracle.c`` (a sign, a bit
order, an index, a dropped term), compiles the edited copy into a temporary
library, and runs ``tests/test_oracle.py`` against it in a subprocess.  The
pins must reject every mutant.  The real oracle is never modified.

Edits that cannot change any result are not listed: the salient padding is
zeroed twice (x and alpha_c past nS are both 0), so giving it alpha_c = 1 or a
set pattern bit changes nothing, and e takes fabs of a whole product, so
dropping the fabs of its row scale changes nothing either.
"""

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTATIONS = [
    ("sign convention", "? +1 : -1;", "? -1 : +1;"),
    ("bit order within a byte", "(row_bits[j >> 3] >> (j & 7))", "(row_bits[j >> 3] >> (7 - (j & 7)))"),
    ("salient term dropped", "Wrow[w->s_idx[t]] += ar * ac * sign_at(bits, t);",
     "Wrow[w->s_idx[t]] += 0.0 * ar * ac * sign_at(bits, t);"),
    ("salient column index", "Wrow[w->s_idx[t]] += ar", "Wrow[t] += ar"),
    ("alpha_c indexed backwards", "w->alpha_c[(size_t)k * N + j] : 1.0;\n            Wrow",
     "w->alpha_c[(size_t)k * N + (N - 1 - j)] : 1.0;\n            Wrow"),
    ("alpha_r of base 0 for every base", "const double ar = w->alpha_r[(size_t)k * M + i];\n        for (int64_t j",
     "const double ar = w->alpha_r[i];\n        for (int64_t j"),
    ("LUT entry sign", "s += ((p >> t) & 1) ? z : -z;", "s += ((p >> t) & 1) ? -z : z;"),
    ("LUT pattern bit order", "p |= (int64_t)bit << t;", "p |= (int64_t)bit << (g - 1 - t);"),
    ("LUT salient term dropped", "acc += w->s_alpha_r[(size_t)k * M + i] * s;", "acc += 0.0 * s;"),
    ("fp16 exponent bias", "e - 25);", "e - 24);"),
    ("last column dropped", "acc += Wrow[j] * xb[j];", "if (j + 1 < N) acc += Wrow[j] * xb[j];"),
    ("tolerance magnitude signed", "mag += fabs(Wrow[j] * xb[j]);", "mag += Wrow[j] * xb[j];"),
    ("salient x gather", "x_S[t] = x[s_idx[t]];", "x_S[t] = x[t];"),
    ("e: salient bases dropped", "m2 += fabs(ar * w->s_alpha_c[(size_t)k * w->nS + t] * xb[w->s_idx[t]]);",
     "m2 += 0.0 * fabs(ar * w->s_alpha_c[(size_t)k * w->nS + t] * xb[w->s_idx[t]]);"),
    ("e: salient x not gathered", "* xb[w->s_idx[t]]);", "* xb[t]);"),
    ("e: global alpha_c dropped", "m2 += fabs(ar * ac * xb[j]);", "m2 += fabs(ar * xb[j]);"),
    ("fp16 subnormal scale", "ldexp((double)m, -24)", "ldexp((double)m, -25)"),
    ("bf16 decode shift", "(uint32_t)b << 16", "(uint32_t)b << 15"),
    ("dense batch stride", "const double *xb = x + (size_t)b * N;\n                double acc",
     "const double *xb = x;\n                double acc"),
    ("LUT batch stride", "const double *xb = x + (size_t)b * N;\n        lut_tables",
     "const double *xb = x;\n        lut_tables"),
    ("salient alpha_c of base 0", "s_alpha_c[(size_t)k * w->nS + t];\n            Wrow", "s_alpha_c[t];\n            Wrow"),
    ("salient alpha_r of base 0", "const double ar = w->s_alpha_r[(size_t)k * M + i];\n        for (int64_t t",
     "const double ar = w->s_alpha_r[i];\n        for (int64_t t"),
    ("LUT alpha_r of base 0", "acc += w->alpha_r[(size_t)k * M + i] * s;", "acc += w->alpha_r[i] * s;"),
    ("gather padding not zero", "            x_S[t] = 0.0;", "            x_S[t] = 1.0;"),
    ("salient index bound off by one", "if ((int64_t)w->s_idx[t] >= w->N) return ORACLE_EINVAL;",
     "if ((int64_t)w->s_idx[t] > w->N) return ORACLE_EINVAL;"),
    ("more salient columns than columns accepted", "if (w->nS < 0 || w->nS > w->N) return ORACLE_EINVAL;",
     "if (w->nS < 0) return ORACLE_EINVAL;"),
    ("fp16 infinity read as NaN", "v = m ? NAN : INFINITY;", "v = NAN;"),
    ("fp16 sign dropped", "return sign ? -v : v;", "return v;"),
    ("dequantised row index", "dequant_row(w, i, Wout + (size_t)r * w->N);", "dequant_row(w, r, Wout + (size_t)r * w->N);"),
    ("sampled row index", "            dequant_row(w, i, Wrow);", "            dequant_row(w, r, Wrow);"),
    ("magnitude without x", "mag += fabs(Wrow[j] * xb[j]);", "mag += fabs(Wrow[j]);"),
    ("salient groups rounded down", "const int64_t nSg = nS > 0 ? (nS + g - 1) / g * g : 0;",
     "const int64_t nSg = nS > 0 ? nS / g * g : 0;"),
]


def _run_mutant(name, old, new, workdir):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for '{name}' not unique"
    tag = "".join(c if c.isalnum() else "_" for c in name)
    mutated = os.path.join(workdir, f"oracle_{tag}.c")
    with open(mutated, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(workdir, f"liboracle_{tag}.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", lib,
                    mutated, "-lm"], check=True)
    env = dict(os.environ, FB_ORACLE_LIB=lib, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle.py"),
                        "-x", "-q", "-p", "no:cacheprovider"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    return name, r.returncode, r.stdout[-1500:]


def test_pins_reject_every_mutant(tmp_path):
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda m: _run_mutant(*m, str(tmp_path)), MUTATIONS))
    accepted = [(n, out) for n, rc, out in results if rc == 0]
    assert not accepted, "pins accepted mutants: " + "; ".join(n for n, _ in accepted)
    assert len(results) == len(MUTATIONS)
