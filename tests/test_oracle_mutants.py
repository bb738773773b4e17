"""The oracle's pins must catch plausible mistakes.

Each case below alters one line of a private copy of the oracle's C source (a
dropped term, a flipped sign, a transposed operand, a wrong tie rule, an
off-by-one), compiles it, and runs the pin suite against that copy in a
separate process.  The pins pass on the real oracle (test_oracle_pins.py);
here every altered copy must make at least one of them fail.
"""
import concurrent.futures
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "muse_oracle.c")

MUTANTS = {
    "splitmix-shift": ("z = (z ^ (z >> 30))", "z = (z ^ (z >> 31))"),
    "fisher-yates-range": ("int j = c + (int)(r % (uint64_t)(n - c));",
                           "int j = (int)(r % (uint64_t)n);"),
    "assign-ties-high": ("if (d < bd) {", "if (d <= bd) {"),
    "empty-cluster-not-kept": ("    if (counts[c] > 0)\n      for (int d = 0; d < D; ++d)\n"
                               "        cent[(size_t)c * D + d] = sum",
                               "    if (counts[c] >= 0)\n      for (int d = 0; d < D; ++d)\n"
                               "        cent[(size_t)c * D + d] = sum"),
    "monopole-sum-of-keys": ("S[(size_t)j * D + e] += v[e];", "S[(size_t)j * D + e] += k[e];"),
    "dipole-transposed": ("v[e] * (k[d] - mu[(size_t)j * D + d])",
                          "v[d] * (k[e] - mu[(size_t)j * D + e])"),
    "dipole-sign": ("x += scale * dot(Me, nu, D);", "x -= scale * dot(Me, nu, D);"),
    "far-field-drops-logW": ("lam = scale * dot(x, kb->mu + (size_t)j * D, D) + logW[ij];",
                             "lam = scale * dot(x, kb->mu + (size_t)j * D, D);"),
    "score-drops-log-n": ("score[ij] = scale * dot(nu, mu, D) + log((double)nj);",
                          "score[ij] = scale * dot(nu, mu, D);"),
    "select-ties-high": ("if (best < 0 || score[ij] > bs) {", "if (best < 0 || score[ij] >= bs) {"),
    "tilted-uses-q-not-residual": ("g += (x[d] - nu[d]) * kh[d];", "g += x[d] * kh[d];"),
    "tilted-logW-drops-max": ("logW[ij] = mx + log(z);", "logW[ij] = log(z);"),
    "exact-uses-centroid": ("scale * dot(x, kb->K + (size_t)t * D, D)",
                            "scale * dot(nu, kb->K + (size_t)t * D, D)"),
    "online-softmax-no-rescale": ("*l = *l * sc + 1.0;", "*l = *l + 1.0;"),
    "local-block-reads-future": ("for (int t = t0; t <= q; ++t) {", "for (int t = t0; t < t0 + L; ++t) {"),
    "causal-level-skips-top": ("for (int lv = 0; lv < levels; ++lv) {",
                               "for (int lv = 0; lv + 1 < levels; ++lv) {"),
    "fine-query-dipole-uses-centroid": (
        "scale * dot(kb->M + ((size_t)j * D + e) * D, x, D) / (double)kb->count[j];",
        "scale * dot(kb->M + ((size_t)j * D + e) * D, nu, D) / (double)kb->count[j];"),
    "fine-query-dipole-sign": (
        "uq[e] = val[e] + scale * dot(", "uq[e] = val[e] - scale * dot("),
    "tilted-dipole-about-centroid": ("g += (x[d] - nu[d]) * (k[d] - kh[d]);",
                                     "g += (x[d] - nu[d]) * (k[d] - mu[d]);"),
    "tilted-dipole-uses-q": ("g += (x[d] - nu[d]) * (k[d] - kh[d]);", "g += x[d] * (k[d] - kh[d]);"),
    "tilted-dipole-sign": ("uq[e] += scale * w * g * kb->V", "uq[e] -= scale * w * g * kb->V"),
}


def _run_mutant(name, tmpdir):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/absent"
    path = os.path.join(tmpdir, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    so = os.path.join(tmpdir, f"{name}.so")
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", so, path, "-lm"])
    env = dict(os.environ, MUSE_ORACLE_SO=so, OMP_NUM_THREADS="1")
    p = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, p.returncode, p.stdout[-400:]


def test_every_mutant_is_caught():
    with tempfile.TemporaryDirectory() as tmp:
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            results = list(ex.map(lambda n: _run_mutant(n, tmp), list(MUTANTS)))
    survivors = [(n, out) for n, rc, out in results if rc == 0]
    assert not survivors, survivors
