"""The block-accumulation oracle's pins must catch plausible mistakes.

Each case alters one line of a private copy of oracle/muse_v4.py, loads the
copy as its own module and runs the pins of test_v4_oracle.py against it: at
least one must fail.
"""
import importlib.util
import os

import pytest

import test_v4_oracle as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "muse_v4.py")

MUTANTS = {
    "prefix-includes-own-block": ("out[b] = out[b - 1] + x[b - 1]", "out[b] = out[b - 1] + x[b]"),
    "ties-to-the-higher-index": ("idx.sort(key=lambda j: (-scores[j], j))",
                                 "idx.sort(key=lambda j: (-scores[j], -j))"),
    "cluster-score-drops-log-n": ("sc[j] = scale * _dot(nu[i], mu) + math.log(pn[b, j])",
                                  "sc[j] = scale * _dot(nu[i], mu)"),
    "block-score-uses-prefix-count": ("+ math.log(bn[bb, j])", "+ math.log(pn[b, j])"),
    "far-keeps-retrieved-blocks": ("rem = np.nonzero(before & (ka == j) & ~retrieved)[0]",
                                   "rem = np.nonzero(before & (ka == j))[0]"),
    "local-block-reads-ahead": ("loc = np.arange(t0, t + 1)", "loc = np.arange(t0, t0 + L)"),
    "dipole-sign": ("u = (S + scale * M @ nu[i]) / n", "u = (S - scale * M @ nu[i]) / n"),
    "far-logit-drops-log-n": ("lg = np.concatenate([scale * (far_mu @ q[t]) + far_ln,",
                              "lg = np.concatenate([scale * (far_mu @ q[t]),"),
}


def _load(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/absent"
    path = tmp_path / f"v4mut_{name.replace('-', '_')}.py"
    path.write_text(src.replace(old, new).replace("from . import default", "from oracle import default"))
    spec = importlib.util.spec_from_file_location(path.stem, path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    mod = _load(name, tmp_path)
    caught = []
    for pin in pins.PINS:
        for mode in ("monopole", "dipole"):
            try:
                pin(mod, mode)
            except (AssertionError, ValueError, IndexError) as e:
                caught.append(f"{pin.__name__}[{mode}]: {str(e)[:60]}")
    assert caught, f"mutant {name} passed every pin"
