"""The gradient oracle's pins must catch plausible mistakes.

Each case alters one line of a private copy of oracle/muse_backward.py (a term
cut off from the chain rule, a dropped or sign-flipped term, a swapped
operand), loads the copy as its own module, and runs the pins of
test_backward_oracle.py against it: at least one must fail.
"""
import importlib.util
import os

import pytest

import test_backward_oracle as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "muse_backward.py")

MUTANTS = {
    "key-centroid-held-constant": ("mu = (A.T @ k) / n", "mu = (A.T @ k.detach()) / n"),
    "query-centroid-held-constant": ("nu = (Aq.T @ q) / m", "nu = (Aq.T @ q.detach()) / m"),
    "cross-moment-about-origin": (' - torch.einsum("je,jd->jed", S, mu)', ""),
    "dipole-sign": ("(S[None] + scale * torch.einsum", "(S[None] - scale * torch.einsum"),
    "far-logit-drops-log-n": (" + torch.log(n.clamp(min=1.0))[None]", ""),
    "exact-values-are-keys": ("P[:, Ck:] @ v", "P[:, Ck:] @ k"),
    "selected-clusters-also-far": ("far_ok = (~R) & (n > 0)[None, :]", "far_ok = (n > 0)[None, :].expand(Cq, -1)"),
    "causal-local-block-reads-ahead": ("torch.where(kl <= pos[:, None],", "torch.where(kl >= 0,"),
    "causal-level-reads-the-query-block": ("k[k0:k0 + s], v[k0:k0 + s],", "k[q0:q0 + s], v[q0:q0 + s],"),
}


def _load_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/absent"
    path = tmp_path / f"mut_{name.replace('-', '_')}.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(path.stem, path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    mod = _load_mutant(name, tmp_path)
    caught = []
    for pin in pins.PINS:
        for mode in ("monopole", "dipole"):
            try:
                pin(mod, mode)
            except (AssertionError, RuntimeError, ValueError) as e:
                caught.append(f"{pin.__name__}[{mode}]: {str(e)[:80]}")
    assert caught, f"mutant {name} passed every pin"
