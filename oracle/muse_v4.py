"""fp64 CPU oracle of the causal operator with causal accumulation of block
summaries and two-level retrieval -- TEST INFRASTRUCTURE ONLY.

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It shares nothing with the CUDA library.

Source: gist.science page "Multipole Semantic Attention: A Fast Approximation
of Softmax Attention for Pretraining", Technical Summary, Core Mechanisms:
  * "Causal Accumulation": the context is cut into spatial blocks and the
    summaries are accumulated causally along them, so a block reads the
    summaries of every preceding block;
  * "Retrieval-Augmented Approximation": the top-k1 key clusters are selected
    by their summary scores, then within each selected cluster the top-k2
    spatial blocks; exact attention covers the retrieved (cluster, block)
    pairs and the local block diagonal, the summaries cover the rest.
The readings taken where the page is silent:
  * both roles are clustered over the whole sequence of a (b, head) (the
    acausal operator's seeded Lloyd k-means, so the clusterings are those of
    muse_attn_fwd); only the summaries are causal;
  * block summaries of key cluster j in block b: n_jb, the key sum and the
    value sum over the members of j in b (token order); the prefix summary of
    block b is the sum of the block summaries of blocks 0 .. b-1, accumulated
    in block order;
  * cluster score of (i, j) at query block b: s nu_i . mu_j^{<b} + log n_j^{<b}
    over the clusters with n_j^{<b} > 0; block score of (i, j, b'):
    s nu_i . mu_jb' + log n_jb' over the blocks b' < b with n_jb' > 0; both in
    fp64 with the dot product in dimension order, top-k with ties to the
    lowest index;
  * the far term of key cluster j for query cluster i at block b is the
    summary of the members of j before block b that are not in a retrieved
    block (omitted when empty): logit s q.mu + log n, value S / n (MONOPOLE)
    or (S + s M nu_i) / n with M = sum v (k - mu)^T about that set's own
    centroid (DIPOLE);
  * the local block diagonal: the keys of the query's own block up to the
    query; queries of block 0 read nothing else.
"""
from __future__ import annotations

import math

import numpy as np


def _dot(a, b):
    """Sum of a * b over the last axis, accumulated in dimension order (fp64,
    no fused multiply-add), so the scores are reproducible bit for bit."""
    return np.cumsum(a * b, axis=-1)[..., -1]


def _topk(scores, k):
    """Indices of the k largest finite scores, best first, ties to the lowest
    index."""
    idx = [j for j in range(len(scores)) if np.isfinite(scores[j])]
    idx.sort(key=lambda j: (-scores[j], j))
    return idx[:k]


def block_summaries(k, ka, L, Ck):
    """n [NB, Ck], key sums [NB, Ck, D] of every (block, key cluster), each
    summed in token order."""
    N, D = k.shape
    NB = N // L
    n = np.zeros((NB, Ck), np.int64)
    ks = np.zeros((NB, Ck, D))
    for t in range(N):
        b, j = t // L, ka[t]
        n[b, j] += 1
        ks[b, j] += k[t]
    return n, ks


def prefix(x):
    """Exclusive prefix over blocks, accumulated in block order."""
    out = np.zeros_like(x)
    for b in range(1, x.shape[0]):
        out[b] = out[b - 1] + x[b - 1]
    return out


def head_v4(q, k, v, qa, ka, nu, L, Ck, k1, k2, scale, mode):
    """O, cluster selections [NB, Cq, k1], block selections [NB, Cq, k1, k2]
    and exact-key counts of one q-head (fp64)."""
    N, D = q.shape
    Cq = nu.shape[0]
    NB = N // L
    bn, bk = block_summaries(k, ka, L, Ck)
    pn, pk = prefix(bn), prefix(bk)
    O = np.zeros((N, D))
    nex = np.zeros(N, np.int64)
    sel1 = np.full((NB, Cq, max(k1, 1)), -1, np.int64)
    sel2 = np.full((NB, Cq, max(k1, 1), max(k2, 1)), -1, np.int64)
    blk = np.arange(N) // L
    for b in range(NB):
        t0 = b * L
        for i in range(Cq):
            rows = [t for t in range(t0, t0 + L) if qa[t] == i]
            if not rows:
                continue
            # 1. clusters, by the prefix summaries
            R = []
            if b > 0 and k1 > 0:
                sc = np.full(Ck, -np.inf)
                for j in range(Ck):
                    if pn[b, j] > 0:
                        mu = pk[b, j] / pn[b, j]
                        sc[j] = scale * _dot(nu[i], mu) + math.log(pn[b, j])
                R = _topk(sc, k1)
            # 2. blocks within each selected cluster, by the block summaries
            picked = {}
            for r, j in enumerate(R):
                sc = np.full(b, -np.inf)
                for bb in range(b):
                    if bn[bb, j] > 0:
                        sc[bb] = scale * _dot(nu[i], bk[bb, j] / bn[bb, j]) + math.log(bn[bb, j])
                picked[j] = _topk(sc, k2)
                sel1[b, i, r] = j
                for r2, bb in enumerate(picked[j]):
                    sel2[b, i, r, r2] = bb
            # 3. the terms: retrieved keys, far summaries, local block
            before = np.arange(N) < t0
            retrieved = np.zeros(N, bool)
            for j, bbs in picked.items():
                for bb in bbs:
                    retrieved |= (ka == j) & (blk == bb)
            ex = np.nonzero(retrieved)[0]
            far_mu, far_ln, far_u = np.zeros((0, D)), [], np.zeros((0, D))
            for j in range(Ck):
                rem = np.nonzero(before & (ka == j) & ~retrieved)[0]
                if len(rem) == 0:
                    continue
                kr, vr = k[rem], v[rem]
                n = len(rem)
                mu = kr.sum(0) / n
                S = vr.sum(0)
                if mode == "monopole":
                    u = S / n
                elif mode == "dipole":
                    M = vr.T @ (kr - mu)
                    u = (S + scale * M @ nu[i]) / n
                else:
                    raise ValueError(f"no v4 oracle for mode {mode!r}")
                far_mu = np.vstack([far_mu, mu])
                far_ln.append(math.log(n))
                far_u = np.vstack([far_u, u])
            far_ln = np.array(far_ln)
            for t in rows:
                loc = np.arange(t0, t + 1)
                keys = np.concatenate([k[ex], k[loc]])
                vals = np.concatenate([v[ex], v[loc]])
                lg = np.concatenate([scale * (far_mu @ q[t]) + far_ln, scale * (keys @ q[t])])
                xs = np.concatenate([far_u, vals])
                w = np.exp(lg - lg.max())
                O[t] = (w[:, None] * xs).sum(0) / w.sum()
                nex[t] = len(ex) + len(loc)
    return O, sel1[..., :k1], sel2[..., :k1, :k2], nex


def muse_v4(Q, K, V, L, Cq, Ck, iters, seed, k1, k2, scale=1.0, mode="dipole", hq_mask=None,
            q_assign_in=None, k_assign_in=None):
    """The causal operator with block-summary accumulation (see the module
    docstring).  Q [B,Hq,N,D], K and V [B,Hkv,N,D]; N % L == 0.  Returns a
    dict with O, the clusterings, sel1 [B,Hq,NB,Cq,k1], sel2
    [B,Hq,NB,Cq,k1,k2] (-1 padded) and n_exact [B,Hq,N]."""
    from . import default

    orc = default()
    B, Hq, N, D = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    NB = N // L
    r = orc.muse_acausal(Q, K, V, Cq, Ck, iters, seed, 0, scale, "monopole", hq_mask=hq_mask,
                         q_assign_in=q_assign_in, k_assign_in=k_assign_in)
    O = np.zeros(Q.shape)
    sel1 = np.full((B, Hq, NB, Cq, k1), -1, np.int64)
    sel2 = np.full((B, Hq, NB, Cq, k1, k2), -1, np.int64)
    nex = np.zeros((B, Hq, N), np.int64)
    for b in range(B):
        for h in range(Hq):
            if hq_mask is not None and not hq_mask[b, h]:
                continue
            hk = h // G
            qa, ka = r["q_assign"][b, h], r["k_assign"][b, hk]
            o, s1, s2, ne = head_v4(np.asarray(Q[b, h], np.float64), np.asarray(K[b, hk], np.float64),
                                    np.asarray(V[b, hk], np.float64), qa, ka, r["q_cent"][b, h], L,
                                    Ck, k1, k2, scale, mode)
            O[b, h], sel1[b, h], sel2[b, h], nex[b, h] = o, s1, s2, ne
    return dict(O=O, q_assign=r["q_assign"], k_assign=r["k_assign"], q_cent=r["q_cent"],
                sel1=sel1, sel2=sel2, n_exact=nex)
