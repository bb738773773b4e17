"""Pins of the gradient oracle (oracle/muse_backward.py), CPU only.

The gradient oracle differentiates, with the clusterings and selections held
fixed, the same operator the C oracle evaluates.  It is pinned by:
  * central finite differences of the C oracle's own forward (an independent
    implementation), with the clusterings teacher-forced and the selections
    checked unchanged at both probe points;
  * the special cases that reduce to exact softmax attention (singleton key
    clusters; every cluster retrieved), against the textbook closed form of
    the attention gradient;
  * two invariants of the operator: translating every key by one vector
    leaves O unchanged (so the key gradient sums to zero over the tokens of a
    key set), and translating every value by c moves O by c (so the value
    gradient sums to the sum of dO over the queries reading that key set);
  * the same three for the causal operator (finite differences of the C
    oracle's causal forward; singleton key clusters at every level against the
    causal closed form; the translation invariants);
  * the mutants of test_backward_mutants.py, each caught by one of these.
"""
import numpy as np
import pytest

import oracle
from oracle import muse_backward as mb
from clustered_multipole_approximation_b200.inputs import clustered_qkv


def exact_grads_closed_form(q, k, v, dO, scale):
    """Softmax attention O = P V with P = softmax(s q k^T): dV = P^T dO,
    dS = P * (dO V^T - rowsum(dO * O)), dQ = s dS K, dK = s dS^T Q."""
    Sx = scale * q @ k.T
    P = np.exp(Sx - Sx.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    O = P @ v
    dV = P.T @ dO
    dS = P * (dO @ v.T - (dO * O).sum(1, keepdims=True))
    return O, scale * dS @ k, scale * dS.T @ q, dV


def small_case(seed, N=80, D=8, Hq=2, Hkv=1, centres=4):
    Q, K, V = clustered_qkv(1, Hq, Hkv, N, D, centres, 0.4, 0.0, "f32", seed)
    rng = np.random.default_rng(seed)
    dO = rng.standard_normal(Q.shape)
    return Q.astype(np.float64), K.astype(np.float64), V.astype(np.float64), dO


def forced_forward(Q, K, V, Cq, Ck, topk, scale, mode, qa, ka):
    return oracle.muse_acausal(Q, K, V, Cq, Ck, 4, 11, topk, scale, mode, q_assign_in=qa,
                               k_assign_in=ka)


# --- pins as functions of the gradient module, so the mutant tests reuse them --
def pin_finite_differences(mod, mode, seed=3, Cq=5, Ck=6, topk=2, scale=0.7, eps=1e-5):
    Q, K, V, dO = small_case(seed)
    r0 = oracle.muse_acausal(Q, K, V, Cq, Ck, 4, 11, topk, scale, mode)
    qa, ka, sel = r0["q_assign"], r0["k_assign"], r0["selected"]
    O, dQ, dK, dV = mod.muse_acausal_grads(Q, K, V, dO, qa, ka, sel, Cq, Ck, scale, mode)
    np.testing.assert_allclose(O, r0["O"], rtol=0, atol=1e-12)
    rng = np.random.default_rng(seed + 100)
    for which, g in (("Q", dQ), ("K", dK), ("V", dV)):
        h = rng.standard_normal(g.shape)
        X = {"Q": Q, "K": K, "V": V}

        def f(sign):
            Y = dict(X)
            Y[which] = X[which] + sign * eps * h
            r = forced_forward(Y["Q"], Y["K"], Y["V"], Cq, Ck, topk, scale, mode, qa, ka)
            assert (r["selected"] == sel).all(), "selection moved under the probe"
            return float((r["O"] * dO).sum())

        fd = (f(+1) - f(-1)) / (2 * eps)
        an = float((g * h).sum())
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (which, fd, an)


def pin_exact_special_cases(mod, mode, seed=5):
    Q, K, V, dO = small_case(seed, N=48, Hq=1)
    N = Q.shape[2]
    q, k, v, g = Q[0, 0], K[0, 0], V[0, 0], dO[0, 0]
    Oe, dQe, dKe, dVe = exact_grads_closed_form(q, k, v, g, 0.9)
    rng = np.random.default_rng(seed)
    qa = rng.integers(0, 3, (1, 1, N)).astype(np.int32)
    # singleton key clusters, nothing retrieved: every far term is one key
    ka = np.arange(N, dtype=np.int32)[None, None]
    none = np.zeros((1, 1, 3, 0), np.int32)
    O, dQ, dK, dV = mod.muse_acausal_grads(Q[:, :1], K, V, dO[:, :1], qa, ka, none, 3, N, 0.9, mode)
    for a, b in ((O, Oe), (dQ, dQe), (dK, dKe), (dV, dVe)):
        np.testing.assert_allclose(a[0, 0], b, rtol=0, atol=1e-10)
    # four key clusters, all four retrieved by every query cluster
    ka = rng.integers(0, 4, (1, 1, N)).astype(np.int32)
    allsel = np.tile(np.arange(4, dtype=np.int32), (1, 1, 3, 1))
    O, dQ, dK, dV = mod.muse_acausal_grads(Q[:, :1], K, V, dO[:, :1], qa, ka, allsel, 3, 4, 0.9,
                                           mode)
    for a, b in ((O, Oe), (dQ, dQe), (dK, dKe), (dV, dVe)):
        np.testing.assert_allclose(a[0, 0], b, rtol=0, atol=1e-10)


def pin_translation_invariants(mod, mode, seed=7, Cq=5, Ck=6, topk=2, scale=0.8):
    Q, K, V, dO = small_case(seed, Hq=4, Hkv=2)
    r = oracle.muse_acausal(Q, K, V, Cq, Ck, 4, 11, topk, scale, mode)
    _, _, dK, dV = mod.muse_acausal_grads(Q, K, V, dO, r["q_assign"], r["k_assign"],
                                          r["selected"], Cq, Ck, scale, mode)
    G = 2
    for hk in range(2):
        np.testing.assert_allclose(dK[0, hk].sum(0), 0.0, rtol=0, atol=1e-10)
        want = dO[0, hk * G:(hk + 1) * G].sum((0, 1))
        np.testing.assert_allclose(dV[0, hk].sum(0), want, rtol=0, atol=1e-10)


def causal_exact_grads(q, k, v, dO, scale):
    """The closed form of exact_grads_closed_form with the causal mask."""
    N = q.shape[0]
    Sx = scale * q @ k.T
    Sx[np.triu_indices(N, 1)] = -np.inf
    P = np.exp(Sx - Sx.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    O = P @ v
    dS = P * (dO @ v.T - (dO * O).sum(1, keepdims=True))
    return O, scale * dS @ k, scale * dS.T @ q, P.T @ dO


def pin_causal_finite_differences(mod, mode, seed=9, L=32, C=5, topk=2, scale=0.7, eps=1e-5):
    Q, K, V, dO = small_case(seed, N=256)
    r0 = oracle.muse_causal(Q, K, V, L, C, 4, 11, topk, scale, mode)
    qa, ka, sel = r0["q_assign"], r0["k_assign"], r0.get("selected")
    O, dQ, dK, dV = mod.muse_causal_grads(Q, K, V, dO, qa, ka, sel, L, C, scale, mode)
    np.testing.assert_allclose(O, r0["O"], rtol=0, atol=1e-12)
    rng = np.random.default_rng(seed + 100)
    for which, g in (("Q", dQ), ("K", dK), ("V", dV)):
        h = rng.standard_normal(g.shape)
        X = {"Q": Q, "K": K, "V": V}

        def f(sign):
            Y = dict(X)
            Y[which] = X[which] + sign * eps * h
            r = oracle.muse_causal(Y["Q"], Y["K"], Y["V"], L, C, 4, 11, topk, scale, mode,
                                   q_assign_in=qa, k_assign_in=ka)
            if sel is not None:
                assert (r["selected"] == sel).all(), "selection moved under the probe"
            return float((r["O"] * dO).sum())

        fd = (f(+1) - f(-1)) / (2 * eps)
        an = float((g * h).sum())
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (which, fd, an)


def pin_causal_singletons_are_exact(mod, mode, L=16):
    Q, K, V, dO = small_case(10, N=128, Hq=1)
    N = 128
    lv = oracle.causal_levels(N, L)
    ka = np.zeros((1, 1, lv, N // 2), np.int32)
    qa = np.zeros((1, 1, lv, N // 2), np.int32)
    for l in range(lv):
        s = L << l
        ka[0, 0, l] = np.tile(np.arange(s), N // (2 * s))  # every key its own cluster
    O, dQ, dK, dV = mod.muse_causal_grads(Q[:, :1], K, V, dO[:, :1], qa, ka, None, L, N, 0.9, mode)
    Oe, dQe, dKe, dVe = causal_exact_grads(Q[0, 0], K[0, 0], V[0, 0], dO[0, 0], 0.9)
    for a, b in ((O, Oe), (dQ, dQe), (dK, dKe), (dV, dVe)):
        np.testing.assert_allclose(a[0, 0], b, rtol=0, atol=1e-10)


def pin_causal_translation_invariants(mod, mode, L=32, C=6, topk=2, scale=0.8):
    Q, K, V, dO = small_case(11, N=256, Hq=2, Hkv=2)
    r = oracle.muse_causal(Q, K, V, L, C, 4, 11, topk, scale, mode)
    _, _, dK, dV = mod.muse_causal_grads(Q, K, V, dO, r["q_assign"], r["k_assign"],
                                         r.get("selected"), L, C, scale, mode)
    for hk in range(2):
        np.testing.assert_allclose(dK[0, hk].sum(0), 0.0, rtol=0, atol=1e-10)
        np.testing.assert_allclose(dV[0, hk].sum(0), dO[0, hk].sum(0), rtol=0, atol=1e-10)


PINS = (pin_finite_differences, pin_exact_special_cases, pin_translation_invariants,
        pin_causal_finite_differences, pin_causal_singletons_are_exact,
        pin_causal_translation_invariants)


@pytest.mark.parametrize("mode", ["monopole", "dipole"])
@pytest.mark.parametrize("pin", [pin_causal_finite_differences, pin_causal_singletons_are_exact,
                                 pin_causal_translation_invariants], ids=lambda p: p.__name__)
def test_causal_gradient_pin(pin, mode):
    pin(mb, mode)


@pytest.mark.parametrize("mode", ["monopole", "dipole"])
def test_gradient_matches_finite_differences_of_the_c_oracle(mode):
    pin_finite_differences(mb, mode)


@pytest.mark.parametrize("mode", ["monopole", "dipole"])
def test_gradient_reduces_to_exact_attention_gradient(mode):
    pin_exact_special_cases(mb, mode)


@pytest.mark.parametrize("mode", ["monopole", "dipole"])
def test_gradient_respects_key_and_value_translation(mode):
    pin_translation_invariants(mb, mode)


def test_gradient_oracle_refuses_tilted():
    Q, K, V, dO = small_case(1, N=16, Hq=1)
    z = np.zeros((1, 1, 16), np.int32)
    with pytest.raises(ValueError):
        mb.muse_acausal_grads(Q[:, :1], K, V, dO[:, :1], z, z, None, 1, 1, 1.0, "tilted")
