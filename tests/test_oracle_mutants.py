"""The pins catch plausible mistakes in the oracle.

Each case plants one mistake in a copy of ``oracle/csa_oracle.c`` (a text
substitution that must match the source exactly once), builds it, and runs
the oracle's pin suites (``test_oracle_pins.py``, ``test_oracle_mx.py``,
``test_oracle_stream.py``, ``test_oracle_mixed.py``) against that build in a
child process.  The planted
build must fail at least two pins.  The real oracle is never modified; the
mutants live in a temporary directory.
"""
import os
import re
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "csa_oracle.c")

# (name, text in the oracle, planted replacement)
MUTANTS = [
    ("RoPE rotates the wrong way",
     "x[d0 + 2 * i] = x0 * cs - x1 * sn;\n    x[d0 + 2 * i + 1] = x0 * sn + x1 * cs;",
     "x[d0 + 2 * i] = x0 * cs + x1 * sn;\n    x[d0 + 2 * i + 1] = -x0 * sn + x1 * cs;"),
    ("RoPE frequency exponent without the factor 2",
     "pow(base, -2.0 * (double)i / (double)r)", "pow(base, -1.0 * (double)i / (double)r)"),
    ("RMSNorm without eps",
     "1.0 / sqrt(ss / (double)c + eps)", "1.0 / sqrt(ss / (double)c)"),
    ("RMSNorm mean over c - 1",
     "1.0 / sqrt(ss / (double)c + eps)", "1.0 / sqrt(ss / (double)(c - 1) + eps)"),
    ("visibility one token early",
     "int64_t v = (pos + 1) / m;", "int64_t v = (pos + 2) / m;"),
    ("group b pooled over the entry's own block",
     "int64_t tok = m * (s - 1) + j;", "int64_t tok = m * s + j;"),
    ("compression logits of channel 0 for every channel",
     "int zc = (z_cols == 1) ? 0 : ch;", "int zc = 0;"),
    ("entry rotated at its last token",
     "orc_norm_rope(e, f, (double)(pos0 + m * s));",
     "orc_norm_rope(e, f, (double)(pos0 + m * s + m - 1));"),
    ("indexer without the ReLU",
     "(dot > 0.0 ? dot : 0.0)", "dot"),
    ("indexer head weights read transposed",
     "acc += w[t * HI + h] *", "acc += w[h * Tq + t] *"),
    ("top-k ties to the higher index",
     "return (a->s < b->s) ? -1 : (a->s > b->s) ? 1 : 0;",
     "return (a->s > b->s) ? -1 : (a->s < b->s) ? 1 : 0;"),
    ("sink dropped from the denominator",
     "double zs = sink ? sink[h] : -INFINITY;", "double zs = -INFINITY;"),
    ("window without the query's own token",
     "int64_t jhi = pos;", "int64_t jhi = pos - 1;"),
    ("output rotated by +pos",
     "orc_rope_inplace(o, c, f->rope_dims, f->rope_base, -(double)pos);",
     "orc_rope_inplace(o, c, f->rope_dims, f->rope_base, (double)pos);"),
    ("logit scale 1/c",
     "scale = 1.0 / sqrt((double)c);", "scale = 1.0 / (double)c;"),
    ("E4M3 exponent bias 8",
     "ldexp(1.0 + (double)m / 8.0, e - 7)", "ldexp(1.0 + (double)m / 8.0, e - 8)"),
    ("E4M3 ties to the odd code",
     "double err = fabs(orc_e4m3_value((uint8_t)c) - a);\n"
     "    if (err < best_err || (err == best_err && (c & 1) == 0)) {",
     "double err = fabs(orc_e4m3_value((uint8_t)c) - a);\n"
     "    if (err < best_err || (err == best_err && (c & 1) == 1)) {"),
    ("E2M1 ties to the odd code",
     "double err = fabs(orc_e2m1_value((uint8_t)c) - a);\n"
     "    if (err < best_err || (err == best_err && (c & 1) == 0)) {",
     "double err = fabs(orc_e2m1_value((uint8_t)c) - a);\n"
     "    if (err < best_err || (err == best_err && (c & 1) == 1)) {"),
    ("MX scale without E4M3's largest exponent",
     "e = (int)floor(log2(amax)) - 8;", "e = (int)floor(log2(amax));"),
    ("stream hands a block's b rows on before pooling it",
     "  orc_pool(c, ns, rows, lg, z_cols, entry, NULL);\n  free(rows);",
     "  if (overlap) memcpy(prev_b, cur_b, sizeof(double) * (size_t)m * c);\n"
     "  orc_pool(c, ns, rows, lg, z_cols, entry, NULL);\n  free(rows);"),
    ("stream entry rotated at the completing token",
     "  orc_norm_rope(entry, f, (double)(pos0 + m * s));\n  if (overlap) {",
     "  orc_norm_rope(entry, f, (double)(pos0 + t));\n  if (overlap) {"),
    ("BF16 rounding by truncation",
     "double y = rint(x / q) * q;", "double y = trunc(x / q) * q;"),
    ("mixed storage keeps the first r dims in BF16",
     "for (int d = 0; d < r; ++d) rope[i * r + d] = orc_bf16_round(x[i * c + cq + d]);",
     "for (int d = 0; d < r; ++d) rope[i * r + d] = orc_bf16_round(x[i * c + d]);"),
    ("FP4 tensor scale without the element format's maximum",
     "double g = amax > 0.0 ? amax / (448.0 * 6.0) : 1.0;",
     "double g = amax > 0.0 ? amax / 448.0 : 1.0;"),
    ("E2M1 exponent bias 0",
     "ldexp(1.0 + 0.5 * (double)m, e - 1)", "ldexp(1.0 + 0.5 * (double)m, e)"),
    ("MX-FP4 scale with E4M3's largest exponent",
     "e = (int)floor(log2(amax)) - 2;", "e = (int)floor(log2(amax)) - 8;"),
]


def _build(tmp, i, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutant {i}: the planted text no longer matches the oracle"
    path = os.path.join(tmp, f"mutant{i}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(tmp, f"libmutant{i}.so")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", path, "-o",
                           lib, "-lm"])
    return lib


def _failed_pins(lib):
    env = dict(os.environ, CSA_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    p = subprocess.run([sys.executable, "-m", "pytest",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                        os.path.join(ROOT, "tests", "test_oracle_mx.py"),
                        os.path.join(ROOT, "tests", "test_oracle_stream.py"),
                        os.path.join(ROOT, "tests", "test_oracle_mixed.py"), "-q", "-p",
                        "no:cacheprovider", "--maxfail=2", "-m", "not gpu"], env=env,
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    m = re.search(r"(\d+) failed", p.stdout)
    return int(m.group(1)) if m else 0, p.stdout[-2000:]


def test_every_planted_mistake_fails_pins(tmp_path):
    libs = [_build(str(tmp_path), i, old, new) for i, (_, old, new) in enumerate(MUTANTS)]
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 2)) as ex:
        results = list(ex.map(_failed_pins, libs))
    caught = {name: n for (name, _, _), (n, _) in zip(MUTANTS, results)}
    missed = [name for name, n in caught.items() if n < 2]
    assert not missed, f"pins failed by each planted mistake: {caught}"


def test_the_unmodified_oracle_passes_the_pins(tmp_path):
    """The harness itself: a copy built the same way, unmodified, fails none."""
    lib = _build(str(tmp_path), 99, "#include <math.h>", "#include <math.h>")
    n, out = _failed_pins(lib)
    assert n == 0, out
