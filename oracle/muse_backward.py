"""fp64 CPU oracle for the gradients of the acausal MuSe operator -- TEST
INFRASTRUCTURE ONLY.

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


def _head_forward(q, k, v, q_assign, k_assign, sel, Cq, Ck, scale, mode):
    """O of one q-head (torch float64 tensors; q, k, v may require grad)."""
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
    P = torch.softmax(torch.cat([lf, le], 1), 1)
    return torch.einsum("qj,qje->qe", P[:, :Ck], U[qa]) + P[:, Ck:] @ v


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
