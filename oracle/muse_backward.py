"""fp64 CPU oracle for the gradients of the MuSe operator, acausal and causal
-- TEST INFRASTRUCTURE ONLY.

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It shares nothing with the CUDA library.

What is differentiated.  The pages use MuSe as a drop-in attention layer for
pretraining (gist.science page "Multipole Semantic Attention: A Fast
Approximation of Softmax Attention for Pretraining", Experimental Results:
1B-parameter models trained with MuSe), so gradients flow through the layer.
The clustering is a piecewise-constant function of the inputs (an assignment
changes only where a token crosses a cell boundary), and so is the selection
of the retrieved clusters (newx.sg page, Abstract: hierarchical two-stage
attention; gist.science page, Core Mechanisms, "Retrieval-Augmented
Approximation").  Both are held fixed, as given by the forward pass.  Every
other quantity is differentiated as the function of Q, K and V it is:

  n_j  = |{t : a(t) = j}|                    (constant)
  mu_j = (1 / n_j) sum_{a(t) = j} k_t         key centroid
  S_j  = sum_{a(t) = j} v_t                   summed values (monopole)
  M_j  = sum_{a(t) = j} v_t (k_t - mu_j)^T    value-key cross moment (dipole)
  nu_i = (1 / m_i) sum_{b(q) = i} q           query centroid
  u_ij = S_j / n_j                            MONOPOLE
  u_ij = (S_j + s M_j nu_i) / n_j             DIPOLE (first-order term of
                                              exp(s nu_i . (k_t - mu_j)))

and the output of a query q of cluster i is one softmax over the far terms
(key clusters j outside R_i with n_j > 0: logit s q.mu_j + log n_j, value
u_ij) and the exact terms (keys t of the clusters in R_i: logit s q.k_t,
value v_t).  The gradient is taken by reverse-mode automatic differentiation
of that expression (torch.autograd, float64), the library routine serving as
the chain-rule step; the expression itself is written out below term by
term, with no blocking or reordering.
"""
from __future__ import annotations

import numpy as np
import torch


def _problem_terms(q, k, v, q_assign, k_assign, sel, Cq, Ck, scale, mode):
    """The terms one MuSe problem (a query set against a key set with their
    clusterings and selections) gives each of its queries: far logits
    [nq, Ck] and values [nq, Ck, D], exact logits [nq, nk] (values: the rows
    of v); -inf marks an absent term."""
    N = q.shape[0]
    A = torch.zeros(k.shape[0], Ck, dtype=torch.float64)
    A[torch.arange(k.shape[0]), torch.as_tensor(k_assign, dtype=torch.long)] = 1.0
    n = A.sum(0)
    mu = (A.T @ k) / n.clamp(min=1.0)[:, None]
    S = A.T @ v
    Aq = torch.zeros(N, Cq, dtype=torch.float64)
    qa = torch.as_tensor(q_assign, dtype=torch.long)
    Aq[torch.arange(N), qa] = 1.0
    m = Aq.sum(0)
    nu = (Aq.T @ q) / m.clamp(min=1.0)[:, None]
    if mode == "monopole":
        U = (S / n.clamp(min=1.0)[:, None])[None].expand(Cq, Ck, -1)
    elif mode == "dipole":
        M = torch.einsum("tj,te,td->jed", A, v, k) - torch.einsum("je,jd->jed", S, mu)
        U = (S[None] + scale * torch.einsum("jed,id->ije", M, nu)) / n.clamp(min=1.0)[None, :, None]
    else:
        raise ValueError(f"no gradient oracle for mode {mode!r}")
    R = torch.zeros(Cq, Ck, dtype=torch.bool)
    for i in range(Cq):
        for j in sel[i]:
            if j >= 0:
                R[i, int(j)] = True
    far_ok = (~R) & (n > 0)[None, :]
    ka = torch.as_tensor(k_assign, dtype=torch.long)
    ex_ok = R[qa][:, ka]
    ninf = torch.tensor(-np.inf, dtype=torch.float64)
    lf = torch.where(far_ok[qa], scale * (q @ mu.T) + torch.log(n.clamp(min=1.0))[None], ninf)
    le = torch.where(ex_ok, scale * (q @ k.T), ninf)
    return lf, U[qa], le


def _head_forward(q, k, v, q_assign, k_assign, sel, Cq, Ck, scale, mode):
    """O of one q-head (torch float64 tensors; q, k, v may require grad)."""
    lf, uq, le = _problem_terms(q, k, v, q_assign, k_assign, sel, Cq, Ck, scale, mode)
    P = torch.softmax(torch.cat([lf, le], 1), 1)
    return torch.einsum("qj,qje->qe", P[:, :Ck], uq) + P[:, Ck:] @ v


def _causal_head_forward(q, k, v, qa_lv, ka_lv, sel_p, L, C, scale, mode):
    """O of one q-head of the causal operator (newx.sg page, Abstract: the
    hierarchical block decomposition with exact local blocks).  Level l has
    blocks of s = L 2^l; pair p's queries [(2p+1)s, (2p+2)s) see the MuSe
    terms of the key block [2p s, (2p+1)s), clustered inside the two blocks
    (C_eff = min(C, s)); every query also sees the keys of its own L-block up
    to itself; all terms meet in one softmax.  qa_lv / ka_lv [levels, N/2]
    (entry (l, p s + r): row r of pair p's block), sel_p [pairs, C, k1]
    numbered level by level."""
    N, D = q.shape
    NB = N // L
    ninf = torch.tensor(-np.inf, dtype=torch.float64)
    pos = torch.arange(N)
    kl = (pos // L)[:, None] * L + torch.arange(L)[None, :]  # the own block's keys
    logits = [torch.where(kl <= pos[:, None], scale * torch.einsum("qd,qrd->qr", q, k[kl]), ninf)]
    values = [v[kl]]
    pb, lv, s = 0, 0, L
    while s < N:
        Ce, npairs = min(C, s), NB // (2 * (s // L))
        lf_l = torch.full((N, Ce), -np.inf, dtype=torch.float64)
        uq_l = torch.zeros((N, Ce, D), dtype=torch.float64)
        le_l = torch.full((N, s), -np.inf, dtype=torch.float64)
        kidx = torch.zeros((N, s), dtype=torch.long)
        for p in range(npairs):
            k0, q0 = 2 * p * s, (2 * p + 1) * s
            sel = sel_p[pb + p, :Ce] if sel_p is not None else [[]] * Ce
            lf, uq, le = _problem_terms(q[q0:q0 + s], k[k0:k0 + s], v[k0:k0 + s],
                                        qa_lv[lv, p * s:(p + 1) * s], ka_lv[lv, p * s:(p + 1) * s],
                                        sel, Ce, Ce, scale, mode)
            lf_l[q0:q0 + s] = lf
            uq_l[q0:q0 + s] = uq
            le_l[q0:q0 + s] = le
            kidx[q0:q0 + s] = torch.arange(k0, k0 + s)
        logits += [lf_l, le_l]
        values += [uq_l, v[kidx]]
        pb += npairs
        lv += 1
        s *= 2
    P = torch.softmax(torch.cat(logits, 1), 1)
    return torch.einsum("qt,qtd->qd", P, torch.cat(values, 1))


def muse_acausal_grads(Q, K, V, dO, q_assign, k_assign, selected, Cq, Ck, scale=1.0,
                       mode="dipole", hq_mask=None):
    """Gradients of <dO, O> with respect to Q, K and V for the acausal
    operator with the given clusterings and selections.

    Q [B,Hq,N,D], K and V [B,Hkv,Nk,D], dO [B,Hq,N,D]; q_assign [B,Hq,N],
    k_assign [B,Hkv,Nk], selected [B,Hq,Cq,k1] (-1 padded; k1 may be 0).
    Returns (O, dQ, dK, dV) as float64 arrays; with hq_mask only the marked
    q-heads are computed (their dK, dV contributions included)."""
    B, Hq = Q.shape[:2]
    Hkv = K.shape[1]
    G = Hq // Hkv
    O = np.zeros(Q.shape)
    dQ = np.zeros(Q.shape)
    dK = np.zeros(K.shape)
    dV = np.zeros(V.shape)
    for b in range(B):
        for h in range(Hq):
            if hq_mask is not None and not hq_mask[b, h]:
                continue
            hk = h // G
            q = torch.tensor(np.asarray(Q[b, h], np.float64), requires_grad=True)
            k = torch.tensor(np.asarray(K[b, hk], np.float64), requires_grad=True)
            v = torch.tensor(np.asarray(V[b, hk], np.float64), requires_grad=True)
            sel = selected[b, h] if selected is not None and selected.shape[-1] else [[]] * Cq
            o = _head_forward(q, k, v, q_assign[b, h], k_assign[b, hk], sel, Cq, Ck, scale, mode)
            g = torch.tensor(np.asarray(dO[b, h], np.float64))
            gq, gk, gv = torch.autograd.grad((o * g).sum(), (q, k, v))
            O[b, h] = o.detach().numpy()
            dQ[b, h] = gq.numpy()
            dK[b, hk] += gk.numpy()
            dV[b, hk] += gv.numpy()
    return O, dQ, dK, dV


def muse_causal_grads(Q, K, V, dO, q_assign, k_assign, selected, L, C, scale=1.0, mode="dipole",
                      hq_mask=None):
    """Gradients of <dO, O> for the causal operator with the given per-level
    clusterings (q_assign [B,Hq,levels,N/2], k_assign [B,Hkv,levels,N/2]) and
    selections (selected [B,Hq,N/L - 1,C,k1], or None for k1 = 0), held
    fixed.  Returns (O, dQ, dK, dV) as float64 arrays."""
    B, Hq = Q.shape[:2]
    G = Hq // K.shape[1]
    O = np.zeros(Q.shape)
    dQ = np.zeros(Q.shape)
    dK = np.zeros(K.shape)
    dV = np.zeros(V.shape)
    for b in range(B):
        for h in range(Hq):
            if hq_mask is not None and not hq_mask[b, h]:
                continue
            hk = h // G
            q = torch.tensor(np.asarray(Q[b, h], np.float64), requires_grad=True)
            k = torch.tensor(np.asarray(K[b, hk], np.float64), requires_grad=True)
            v = torch.tensor(np.asarray(V[b, hk], np.float64), requires_grad=True)
            sel = selected[b, h] if selected is not None and selected.shape[-1] else None
            o = _causal_head_forward(q, k, v, q_assign[b, h], k_assign[b, hk], sel, L, C, scale,
                                     mode)
            g = torch.tensor(np.asarray(dO[b, h], np.float64))
            gq, gk, gv = torch.autograd.grad((o * g).sum(), (q, k, v))
            O[b, h] = o.detach().numpy()
            dQ[b, h] = gq.numpy()
            dK[b, hk] += gk.numpy()
            dV[b, hk] += gv.numpy()
    return O, dQ, dK, dV
