"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Assignments, cluster counts, retrieval sets and exact-key counts must match
bit for bit (a k-means mismatch is tolerated only as a documented near tie);
outputs must match within 1e-5 (fp32 inputs) or 2e-3 (bf16 inputs) max-abs,
and the relative squared error against exact attention within 1e-3 of the
oracle's.
"""
import concurrent.futures
import os

import numpy as np
import pytest
import torch

import clustered_multipole_approximation_b200 as muse
import oracle
from clustered_multipole_approximation_b200 import build
from clustered_multipole_approximation_b200.inputs import WORKLOADS, clustered_qkv, make_inputs
from helpers import TOL, assert_assign_match, assert_close, rse, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    muse.load_library()


def gpu_acausal(Q, K, V, dtype, C, iters, seed, topk, scale=1.0, mode="dipole", Cq=None):
    q, k, v = to_dev(Q, dtype), to_dev(K, dtype), to_dev(V, dtype)
    O, dbg = muse.muse_attn_fwd(q, k, v, Cq=Cq or C, Ck=C, iters=iters, seed=seed, topk=topk,
                                scale=scale, mode=mode, debug=True, out_dtype=torch.float32)
    Ob = muse.muse_attn_fwd(q, k, v, Cq=Cq or C, Ck=C, iters=iters, seed=seed, topk=topk,
                            scale=scale, mode=mode)
    torch.cuda.synchronize()
    # the input-dtype output is the fp32 result rounded once
    assert torch.equal(Ob, O.to(Ob.dtype))
    assert int(dbg["device_error"].item()) == 0
    return O.cpu().numpy(), {n: t.cpu().numpy() for n, t in dbg.items()}


def check_acausal(Q, K, V, dtype, C, iters, seed, topk, scale=1.0, mode="dipole", heads=None,
                  Cq=None, check_rse=True):
    B, Hq = Q.shape[:2]
    Hkv = K.shape[1]
    G = Hq // Hkv
    O, g = gpu_acausal(Q, K, V, dtype, C, iters, seed, topk, scale, mode, Cq)
    mask = None
    if heads is not None:
        mask = np.zeros((B, Hq), np.uint8)
        for b, h in heads:
            mask[b, h] = 1
    r = oracle.muse_acausal(Q, K, V, Cq or C, C, iters, seed, topk, scale, mode, hq_mask=mask)
    sel_heads = [(b, h) for b in range(B) for h in range(Hq)] if heads is None else heads
    for b, h in sel_heads:
        hk = h // G
        assert_assign_match(g["k_assign"][b, hk], r["k_assign"][b, hk], what=f"k_assign b{b}h{hk}")
        assert_assign_match(g["q_assign"][b, h], r["q_assign"][b, h], what=f"q_assign b{b}h{h}")
        assert (g["k_counts"][b, hk] == r["k_count"][b, hk]).all()
        np.testing.assert_allclose(g["k_centroids"][b, hk], r["k_cent"][b, hk], rtol=2e-7, atol=1e-7)
        np.testing.assert_allclose(g["q_centroids"][b, h], r["q_cent"][b, h], rtol=2e-7, atol=1e-7)
        if topk > 0:
            qc = np.bincount(r["q_assign"][b, h], minlength=Cq or C)
            live = qc > 0  # rows of empty query clusters are never used
            assert (g["selected"][b, h][live] == r["selected"][b, h][live]).all(), f"R b{b}h{h}"
        assert (g["n_exact"][b, h] == r["n_exact"][b, h]).all()
        assert_close(O[b, h], r["O"][b, h], TOL[dtype], f"O b{b}h{h}")
    if check_rse:
        E = oracle.exact_attention(Q, K, V, scale, hq_mask=mask)
        idx = tuple(np.array(sel_heads).T)
        r_gpu = rse(O[idx], E[idx])
        r_orc = rse(r["O"][idx], E[idx])
        assert abs(r_gpu - r_orc) < 1e-3, (r_gpu, r_orc)
    return O, g, r


# ---------------------------------------------------------------------------
# acausal
# ---------------------------------------------------------------------------
def test_workload_acausal_f32_n1k():
    w = WORKLOADS["acausal-f32-n1k"]
    Q, K, V = make_inputs(w)
    check_acausal(Q, K, V, w.dtype, w.C, w.iters, w.cluster_seed, w.topk, w.scale, w.mode)


@pytest.mark.parametrize("mode", ["dipole", "monopole"])
def test_workload_acausal_bf16_h8_n8k(mode):
    """The 8-head 8k layer, every head against the oracle."""
    w = WORKLOADS["acausal-bf16-h8-n8k"]
    Q, K, V = make_inputs(w)
    check_acausal(Q, K, V, w.dtype, w.C, w.iters, w.cluster_seed, w.topk, w.scale, mode)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("mode", ["monopole", "dipole", "tilted", "tilted_dipole"])
def test_small_acausal_gqa_ragged(dtype, D, mode):
    Q, K, V = clustered_qkv(2, 4, 2, 1000, D, 12, 0.3, 0.0, dtype, 31 + D)
    check_acausal(Q, K, V, dtype, 13, 5, 77, 3, 1.0, mode, Cq=11)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_singleton_key_clusters_match_exact_attention(dtype):
    Q, K, V = clustered_qkv(1, 2, 1, 256, 64, 8, 0.3, 0.0, dtype, 5)
    O, _, _ = check_acausal(Q, K, V, dtype, 256, 2, 3, 0, 1.0, "dipole", Cq=16)
    E = oracle.exact_attention(Q, K, V)
    assert_close(O, E, TOL[dtype], "O vs exact")


def test_retrieving_all_clusters_is_exact():
    Q, K, V = clustered_qkv(1, 1, 1, 512, 64, 8, 0.3, 0.0, "f32", 6)
    O, _, _ = check_acausal(Q, K, V, "f32", 8, 4, 9, 8)
    assert_close(O, oracle.exact_attention(Q, K, V), 1e-5, "O vs exact")


def test_duplicate_tokens_and_empty_clusters():
    rng = np.random.default_rng(0)
    base = rng.standard_normal((5, 64)).astype(np.float32) * 0.4
    Q = base[rng.integers(0, 5, (1, 1, 300))].astype(np.float32)
    K = base[rng.integers(0, 5, (1, 1, 300))].astype(np.float32)
    V = rng.standard_normal((1, 1, 300, 64)).astype(np.float32)
    # 9 clusters over 5 distinct points: several clusters end up empty
    _, g, r = check_acausal(Q, K, V, "f32", 9, 3, 4, 2, check_rse=False)
    assert (r["k_count"] == 0).any()


def test_single_cluster_and_topk_zero():
    Q, K, V = clustered_qkv(1, 1, 1, 300, 64, 4, 0.3, 0.0, "bf16", 8)
    check_acausal(Q, K, V, "bf16", 1, 2, 1, 0, 1.0, "dipole", Cq=1)


def test_repeatable_bit_for_bit():
    Q, K, V = clustered_qkv(1, 2, 2, 2048, 64, 16, 0.3, 0.0, "bf16", 12)
    a, _ = gpu_acausal(Q, K, V, "bf16", 32, 5, 3, 4)
    b, _ = gpu_acausal(Q, K, V, "bf16", 32, 5, 3, 4)
    assert (a == b).all()


# ---------------------------------------------------------------------------
# clustering and summaries on their own
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_muse_cluster_seeded(dtype):
    X, _, _ = clustered_qkv(2, 3, 3, 777, 64, 10, 0.3, 0.0, dtype, 40)
    x = to_dev(X, dtype)
    for role in (0, 1):
        a, c, n = muse.muse_cluster(x, 12, 6, 1234, role=role)
        a, c, n = a.cpu().numpy(), c.cpu().numpy(), n.cpu().numpy()
        for b in range(2):
            for h in range(3):
                ra, rc, rn, _ = oracle.kmeans(X[b, h], 12, 6, 1234, b * 3 + h, role)
                assert_assign_match(a[b, h], ra, what=f"assign b{b}h{h}")
                assert (n[b, h] == rn).all()
                np.testing.assert_allclose(c[b, h], rc, rtol=2e-7, atol=1e-7)


@pytest.mark.parametrize("C,D,N", [(1, 64, 300), (16, 64, 500), (100, 128, 1000), (256, 64, 2000),
                                   (300, 128, 1500), (1024, 64, 3000)])
def test_muse_cluster_bf16_cluster_counts(C, D, N):
    # C > 256 exercises several tensor-core passes per tile
    X, _, _ = clustered_qkv(1, 2, 2, N, D, 24, 0.3, 0.0, "bf16", 43 + C)
    a, c, n = muse.muse_cluster(to_dev(X, "bf16"), C, 3, 99, role=1)
    for h in range(2):
        ra, rc, rn, _ = oracle.kmeans(X[0, h], C, 3, 99, h, 1)
        assert_assign_match(a[0, h].cpu().numpy(), ra, what=f"assign h{h}")
        assert (n[0, h].cpu().numpy() == rn).all()
        np.testing.assert_allclose(c[0, h].cpu().numpy(), rc, rtol=2e-7, atol=1e-7)


@pytest.mark.parametrize("spread", ["wide", "narrow"])
def test_muse_cluster_sums_outside_the_exactness_certificate(spread):
    """Centroid sums are taken in any order only when the problem's exponent
    range certifies them exact; a problem whose values span too many binades
    (here tokens scaled by 2^40 next to tokens scaled by 2^-40) goes through
    the sequential-order kernel.  Both must equal the oracle bit for bit."""
    X, _, _ = clustered_qkv(1, 2, 2, 1500, 64, 12, 0.3, 0.0, "f32", 44)
    if spread == "wide":
        X[0, 0, ::7] *= 2.0 ** 40
        X[0, 0, 3::7] *= 2.0 ** -40
    Xb = to_dev(X, "bf16")
    Xr = Xb.float().cpu().numpy()
    a, c, n = muse.muse_cluster(Xb, 20, 4, 5, role=0)
    torch.cuda.synchronize()
    for h in range(2):
        ra, rc, rn, _ = oracle.kmeans(Xr[0, h], 20, 4, 5, h, 0)
        assert_assign_match(a[0, h].cpu().numpy(), ra, what=f"assign h{h}")
        assert (n[0, h].cpu().numpy() == rn).all()
        np.testing.assert_allclose(c[0, h].cpu().numpy(), rc, rtol=2e-7, atol=1e-30)


def test_muse_cluster_one_round_from_given_centroids():
    X, _, _ = clustered_qkv(1, 2, 2, 1500, 128, 20, 0.3, 0.0, "bf16", 41)
    rng = np.random.default_rng(1)
    init = rng.standard_normal((1, 2, 24, 128)).astype(np.float32) * 0.3
    a, c, n = muse.muse_cluster(to_dev(X, "bf16"), 24, 1, 0, init=torch.from_numpy(init).cuda())
    for h in range(2):
        ra, _ = oracle.kmeans_assign(X[0, h], init[0, h])
        rc, rn = oracle.kmeans_update(X[0, h], ra, init[0, h])
        assert_assign_match(a[0, h].cpu().numpy(), ra, X[0, h].astype(np.float64),
                            init[0, h].astype(np.float64))
        np.testing.assert_allclose(c[0, h].cpu().numpy(), rc, rtol=2e-7, atol=1e-7)


@pytest.mark.parametrize("dtype,D", [("f32", 64), ("bf16", 64), ("bf16", 128)])
def test_muse_summarize(dtype, D):
    """Counts, centroids, monopole sums S and dipole moments M of a given
    assignment against the oracle (bf16 inputs are exact in the oracle's
    fp64; the GPU accumulates S and M in fp32)."""
    K, _, V = clustered_qkv(1, 2, 2, 600, D, 6, 0.3, 0.0, dtype, 42 + D)
    rng = np.random.default_rng(3)
    assign = rng.integers(0, 7, (1, 2, 600)).astype(np.int32)
    assign[0, 1][assign[0, 1] == 3] = 4  # cluster 3 empty in head 1
    cnt, mu, S, M = muse.muse_summarize(to_dev(K, dtype), to_dev(V, dtype),
                                        torch.from_numpy(assign).cuda(), 7)
    torch.cuda.synchronize()
    for h in range(2):
        rmu, rn = oracle.kmeans_update(K[0, h], assign[0, h], np.zeros((7, D)))
        rS, rM = oracle.summaries(K[0, h], V[0, h], 7, assign[0, h], rmu)
        assert (cnt[0, h].cpu().numpy() == rn).all()
        np.testing.assert_allclose(mu[0, h].cpu().numpy(), rmu, rtol=1e-6, atol=1e-6)
        np.testing.assert_allclose(S[0, h].cpu().numpy(), rS, rtol=1e-5, atol=1e-4)
        np.testing.assert_allclose(M[0, h].cpu().numpy(), rM, rtol=1e-4, atol=1e-4)
    assert (cnt[0, 1, 3] == 0).item() and (mu[0, 1, 3] == 0).all().item()


def _golden_init_cases():
    path = os.path.join(os.path.dirname(__file__), "golden", "init_indices.txt")
    cases = []
    for ln in open(path):
        if ln.startswith("#") or not ln.strip():
            continue
        head, idx = ln.split(":")
        n, C, seed, sid, role = map(int, head.split())
        cases.append((n, C, seed, sid, role, np.array(idx.split(), dtype=np.int64)))
    return cases


@pytest.mark.parametrize("case", range(7))
def test_gpu_seeded_start_rows_match_golden(case):
    """The GPU's seeded start rows are the stored ones: one Lloyd round from
    them (assignment to those rows, then the means) is what muse_cluster
    computes with iters = 1 for the stream (b = 0, h = sid) and role."""
    n, C, seed, sid, role, idx = _golden_init_cases()[case]
    X, _, _ = clustered_qkv(1, sid + 1, sid + 1, n, 64, 8, 0.3, 0.0, "bf16", 90 + case)
    a, c, cnt = muse.muse_cluster(to_dev(X, "bf16"), C, 1, seed, role=role)
    torch.cuda.synchronize()
    Xh = X[0, sid].astype(np.float64)
    start = Xh[idx]
    ra, _ = oracle.kmeans_assign(Xh, start)
    rc, rn = oracle.kmeans_update(Xh, ra, start)
    assert_assign_match(a[0, sid].cpu().numpy(), ra, what="round-1 assignment")
    assert (cnt[0, sid].cpu().numpy() == rn).all()
    np.testing.assert_allclose(c[0, sid].cpu().numpy(), rc, rtol=2e-7, atol=1e-7)


def test_v_outside_unit_range_large_and_tiny():
    """V far from N(0, 1): large values (up to 3e4, still inside fp16) and tiny
    ones (down to 1e-7, below fp16's normal range).  The output is linear in
    V, so the bf16 tolerance scales with max |v|."""
    Q, K, V = clustered_qkv(1, 2, 1, 1024, 64, 8, 0.3, 0.0, "bf16", 70)
    rng = np.random.default_rng(5)
    scale = np.where(rng.random(V.shape) < 0.5, 3e4 / 4, 1e-7).astype(np.float32)
    V = (V * scale).astype(np.float32)
    big = float(np.abs(V).max())
    q, k, v = to_dev(Q, "bf16"), to_dev(K, "bf16"), to_dev(V, "bf16")
    Vb = v.float().cpu().numpy()
    O, dbg = muse.muse_attn_fwd(q, k, v, Cq=16, Ck=16, iters=4, seed=3, topk=2, debug=True,
                                out_dtype=torch.float32)
    muse.device_status(dbg["device_error"])
    r = oracle.muse_acausal(Q, K, Vb, 16, 16, 4, 3, 2)
    assert_close(O.cpu().numpy(), r["O"], TOL["bf16"] * big / 4.0, "O with large / tiny V")


def test_v_beyond_fp16_is_reported():
    """A finite bf16 value of V beyond fp16's range cannot enter the fp16
    PV operand: the call still returns MUSE_OK (nothing is synchronised), and
    the device error word reports MUSE_DEVERR_V_RANGE."""
    Q, K, V = clustered_qkv(1, 1, 1, 512, 64, 8, 0.3, 0.0, "bf16", 71)
    V[0, 0, 7, 3] = 1.0e5
    q, k, v = to_dev(Q, "bf16"), to_dev(K, "bf16"), to_dev(V, "bf16")
    _, dbg = muse.muse_attn_fwd(q, k, v, Cq=8, Ck=8, iters=2, seed=1, topk=1, debug=True)
    with pytest.raises(muse.MuseError) as e:
        muse.device_status(dbg["device_error"])
    assert e.value.status == 5 and "fp16" in str(e.value)
    assert int(dbg["device_error"].item()) == 4


def test_team_barrier_that_runs_out_is_reported_and_context_survives():
    """Failure path of the persistent k-means' cooperative barrier: one CTA
    per problem skips its first arrival (test hook), every wait gives up after
    a few thousand polls, the kernel records MUSE_DEVERR_TEAM_BARRIER and
    returns; the next call, without the hook, is correct."""
    X, _, _ = clustered_qkv(1, 4, 4, 4096, 64, 16, 0.3, 0.0, "bf16", 72)
    x = to_dev(X, "bf16")
    err = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    muse.inject_barrier_fault(1, 4096)
    try:
        muse.muse_cluster(x, 64, 3, 5, role=0, device_error=err)
        with pytest.raises(muse.MuseError) as e:
            muse.device_status(err)
    finally:
        muse.inject_barrier_fault(-1)
    assert e.value.status == 5 and int(err.item()) & 2
    a, c, n = muse.muse_cluster(x, 64, 3, 5, role=0, device_error=err)
    muse.device_status(err)
    ra, rc, rn, _ = oracle.kmeans(X[0, 2], 64, 3, 5, 2, 0)
    assert_assign_match(a[0, 2].cpu().numpy(), ra)
    np.testing.assert_allclose(c[0, 2].cpu().numpy(), rc, rtol=2e-7, atol=1e-7)


# ---------------------------------------------------------------------------
# causal
# ---------------------------------------------------------------------------
def gpu_causal(Q, K, V, dtype, L, C, iters, seed, topk, scale=1.0, mode="dipole"):
    q, k, v = to_dev(Q, dtype), to_dev(K, dtype), to_dev(V, dtype)
    O, dbg = muse.muse_attn_fwd_causal(q, k, v, C=C, block=L, iters=iters, seed=seed, topk=topk,
                                       scale=scale, mode=mode, debug=True,
                                       out_dtype=torch.float32)
    Ob = muse.muse_attn_fwd_causal(q, k, v, C=C, block=L, iters=iters, seed=seed, topk=topk,
                                   scale=scale, mode=mode)
    torch.cuda.synchronize()
    assert torch.equal(Ob, O.to(Ob.dtype))
    assert int(dbg["device_error"].item()) == 0
    return O.cpu().numpy(), {n: t.cpu().numpy() for n, t in dbg.items()}


def causal_problems(N, L):
    """(problem index, level, pair, block size) of the hierarchical
    decomposition, numbered level by level as the causal debug layouts are."""
    out, k = [], 0
    for lv in range(oracle.causal_levels(N, L)):
        s = L << lv
        for p in range(N // (2 * s)):
            out.append((k, lv, p, s))
            k += 1
    return out


def assert_causal_selected(g_sel, r_sel, q_assign, N, L, C, what):
    """Retrieval sets of every block problem of one head, bit for bit, on the
    rows of non-empty query clusters (the rows stage 2 uses)."""
    for k, lv, p, s in causal_problems(N, L):
        Ce = min(C, s)
        live = np.bincount(q_assign[lv, p * s:(p + 1) * s], minlength=Ce) > 0
        assert (g_sel[k, :Ce][live] == r_sel[k, :Ce][live]).all(), f"{what} R lv{lv} p{p}"


def check_causal(Q, K, V, dtype, L, C, iters, seed, topk, scale=1.0, mode="dipole", heads=None,
                 rse_heads=None):
    B, Hq, N = Q.shape[:3]
    G = Hq // K.shape[1]
    O, g = gpu_causal(Q, K, V, dtype, L, C, iters, seed, topk, scale, mode)
    mask = None
    if heads is not None:
        mask = np.zeros((B, Hq), np.uint8)
        for b, h in heads:
            mask[b, h] = 1
    r = oracle.muse_causal(Q, K, V, L, C, iters, seed, topk, scale, mode, hq_mask=mask)
    sel = [(b, h) for b in range(B) for h in range(Hq)] if heads is None else heads
    for b, h in sel:
        assert_assign_match(g["k_assign"][b, h // G], r["k_assign"][b, h // G], what="k_assign")
        assert_assign_match(g["q_assign"][b, h], r["q_assign"][b, h], what="q_assign")
        if "selected" in r:
            assert_causal_selected(g["selected"][b, h], r["selected"][b, h], r["q_assign"][b, h],
                                   N, L, C, f"b{b}h{h}")
        assert (g["n_exact"][b, h] == r["n_exact"][b, h]).all()
        assert_close(O[b, h], r["O"][b, h], TOL[dtype], f"O b{b}h{h}")
    rh = sel if rse_heads is None else rse_heads
    rmask = np.zeros((B, Hq), np.uint8)
    for b, h in rh:
        rmask[b, h] = 1
    E = oracle.exact_attention(Q, K, V, scale, causal=True, hq_mask=rmask)
    idx = tuple(np.array(rh).T)
    assert abs(rse(O[idx], E[idx]) - rse(r["O"][idx], E[idx])) < 1e-3
    return O, g, r


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["monopole", "dipole", "tilted", "tilted_dipole"])
def test_small_causal_gqa(dtype, mode):
    Q, K, V = clustered_qkv(1, 4, 2, 1024, 64, 8, 0.3, 0.0, dtype, 50)
    check_causal(Q, K, V, dtype, 64, 12, 4, 21, 2, 1.0, mode)


def test_causal_d128_clusters_above_block_size():
    # C = 96 > L = 64: level 0 uses singleton clusters (C_eff = 64)
    Q, K, V = clustered_qkv(2, 2, 2, 512, 128, 8, 0.3, 0.0, "bf16", 51)
    check_causal(Q, K, V, "bf16", 64, 96, 3, 2, 4)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("topk", [0, 3])
def test_causal_low_levels_per_key_token(D, topk):
    """Levels with at most 8 keys per cluster (s = 128 and 256 with C = 32)
    take the far field one key token at a time; the levels above (s = 512,
    1024) keep the per-cluster tables.  Every head against the oracle, with a
    heavy-tailed norm factor on q and k."""
    Q, K, V = clustered_qkv(1, 4, 2, 2048, D, 24, 0.3, 0.5, "bf16", 60 + D + topk)
    muse.profile_read()
    muse.profile_enable(True)
    try:
        check_causal(Q, K, V, "bf16", 128, 32, 4, 61, topk)
    finally:
        muse.profile_enable(False)
        launched = muse.profile_read()
    assert "stage2_dense" in launched and "stage2_attn" in launched, launched


def test_causal_single_block_is_exact():
    Q, K, V = clustered_qkv(1, 2, 1, 256, 64, 8, 0.3, 0.0, "f32", 52)
    O, _ = gpu_causal(Q, K, V, "f32", 256, 8, 3, 1, 2)
    assert_close(O, oracle.exact_attention(Q, K, V, causal=True), 1e-5, "O vs exact causal")


def test_causal_never_reads_the_future_on_gpu():
    Q, K, V = clustered_qkv(1, 2, 1, 1024, 64, 8, 0.3, 0.0, "bf16", 53)
    base, _ = gpu_causal(Q, K, V, "bf16", 128, 16, 4, 7, 2)
    for t0 in (0, 127, 128, 500, 1000):
        K2, V2 = K.copy(), V.copy()
        K2[:, :, t0 + 1:] *= -1.5
        V2[:, :, t0 + 1:] += 1.0
        o, _ = gpu_causal(Q, K2, V2, "bf16", 128, 16, 4, 7, 2)
        assert (o[:, :, : t0 + 1] == base[:, :, : t0 + 1]).all(), t0


# ---------------------------------------------------------------------------
# fine-query dipole: the first-order term taken at each query (M_j q)
def _stages_launched(fn):
    muse.profile_read()
    muse.profile_enable(True)
    try:
        out = fn()
    finally:
        muse.profile_enable(False)
        launched = muse.profile_read()
    return out, launched


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("topk", [0, 3])
def test_small_acausal_fine_query_dipole(D, topk):
    """GQA, Cq != Ck, every head against the oracle; the far field runs per
    key token (the per-cluster-pair summaries are not formed)."""
    Q, K, V = clustered_qkv(2, 4, 2, 1024, D, 12, 0.3, 0.5, "bf16", 90 + D + topk)
    _, launched = _stages_launched(
        lambda: check_acausal(Q, K, V, "bf16", 13, 5, 77, topk, 1.0, "dipole_q", Cq=11))
    assert "stage2_dense" in launched, launched
    assert "stage1_summaries" not in launched and "stage2_attn" not in launched, launched


def test_fine_query_dipole_is_closer_to_exact_than_dipole():
    """Taking the dipole at each query instead of at its cluster centroid
    removes the (q - nu_i) part of the expansion error: on a spread-out
    layer the GPU's fine-query output is nearer exact attention."""
    Q, K, V = clustered_qkv(1, 2, 2, 2048, 64, 8, 0.6, 0.0, "bf16", 95)
    Oq, _ = gpu_acausal(Q, K, V, "bf16", 32, 6, 5, 2, 1.0, "dipole_q")
    Od, _ = gpu_acausal(Q, K, V, "bf16", 32, 6, 5, 2, 1.0, "dipole")
    E = oracle.exact_attention(Q, K, V)
    assert rse(Oq, E) < rse(Od, E), (rse(Oq, E), rse(Od, E))


@pytest.mark.parametrize("D", [64, 128])
def test_small_causal_fine_query_dipole(D):
    """Every level (s = 128, 256, 512) per key token, every head."""
    Q, K, V = clustered_qkv(1, 4, 2, 1024, D, 8, 0.3, 0.0, "bf16", 96 + D)
    _, launched = _stages_launched(
        lambda: check_causal(Q, K, V, "bf16", 128, 12, 4, 21, 2, 1.0, "dipole_q"))
    assert "stage2_dense" in launched and "stage2_attn" not in launched, launched


def test_workload_acausal_bf16_h8_n8k_fine_query_dipole():
    """The 8-head 8k layer in the fine-query mode, heads 0 and 5 against the
    oracle."""
    w = WORKLOADS["acausal-bf16-h8-n8k"]
    Q, K, V = make_inputs(w)
    check_acausal(Q, K, V, w.dtype, w.C, w.iters, w.cluster_seed, w.topk, w.scale, "dipole_q",
                  heads=[(0, 0), (0, 5)])


def test_workload_causal_b2h8_n16k_fine_query_dipole():
    """The 16k causal layer in the fine-query mode (levels s = 512 .. 8192
    per key token), head (1, 3) against the oracle."""
    w = WORKLOADS["causal-bf16-b2h8-n16k"]
    Q, K, V = make_inputs(w)
    check_causal(Q, K, V, w.dtype, w.block, w.C, w.iters, w.cluster_seed, w.topk, w.scale,
                 "dipole_q", heads=[(1, 3)])


def test_tilted_dipole_runs_per_key_token_and_beats_tilted():
    """The tilted per-pair dipole takes its own stage 2 (no per-cluster-pair
    stage-2 kernel runs) and lands nearer exact attention than TILTED."""
    Q, K, V = clustered_qkv(1, 2, 2, 2048, 64, 8, 0.6, 0.0, "bf16", 95)
    _, launched = _stages_launched(
        lambda: gpu_acausal(Q, K, V, "bf16", 32, 6, 5, 2, 1.0, "tilted_dipole"))
    assert "stage2_tdip" in launched and "stage2_attn" not in launched, launched
    Ot, _ = gpu_acausal(Q, K, V, "bf16", 32, 6, 5, 2, 1.0, "tilted_dipole")
    Oi, _ = gpu_acausal(Q, K, V, "bf16", 32, 6, 5, 2, 1.0, "tilted")
    E = oracle.exact_attention(Q, K, V)
    assert rse(Ot, E) < 0.5 * rse(Oi, E), (rse(Ot, E), rse(Oi, E))


def test_workload_acausal_bf16_h8_n8k_tilted_dipole():
    """The 8-head 8k layer in the tilted per-pair dipole mode, head 4 against
    the oracle."""
    w = WORKLOADS["acausal-bf16-h8-n8k"]
    Q, K, V = make_inputs(w)
    check_acausal(Q, K, V, w.dtype, w.C, w.iters, w.cluster_seed, w.topk, w.scale,
                  "tilted_dipole", heads=[(0, 4)])


@pytest.mark.parametrize("case", ["f32", "n_not_128", "block_not_128", "clusters_above_256"])
def test_fine_query_dipole_unsupported_shapes_are_refused(case):
    dtype = "f32" if case == "f32" else "bf16"
    N = 1000 if case == "n_not_128" else 1024
    Q, K, V = clustered_qkv(1, 1, 1, N, 64, 8, 0.3, 0.0, dtype, 97)
    q, k, v = to_dev(Q, dtype), to_dev(K, dtype), to_dev(V, dtype)
    with pytest.raises(muse.MuseError, match="DIPOLE_Q"):
        if case == "block_not_128":
            muse.muse_attn_fwd_causal(q, k, v, C=8, block=64, iters=2, seed=1, topk=1,
                                      mode="dipole_q")
        else:
            C = 300 if case == "clusters_above_256" else 8
            muse.muse_attn_fwd(q, k, v, Cq=C, Ck=C, iters=2, seed=1, topk=1, mode="dipole_q")
    torch.cuda.synchronize()


def test_workload_causal_b2h8_n16k():
    """The B=2, H=8 16k causal layer, every head against the oracle."""
    w = WORKLOADS["causal-bf16-b2h8-n16k"]
    Q, K, V = make_inputs(w)
    check_causal(Q, K, V, w.dtype, w.block, w.C, w.iters, w.cluster_seed, w.topk, w.scale,
                 w.mode, rse_heads=[(0, 0), (1, 7)])


# q-heads of the GQA layers checked against the oracle: the first kv-group
# whole and the last q-head (kv-heads 0 and 7)
GQA_HEADS = [0, 1, 2, 3, 31]


@pytest.mark.parametrize("name", ["causal-gqa32x8-n64k-d64", "causal-gqa32x8-n32k-d128"])
def test_workload_causal_gqa_full_size(name):
    """Full-size GQA causal workloads, on q-heads 0-3 and 31 and their
    kv-heads 0 and 7:
    - every (level, pair) k-means problem of both roles against the oracle's
      own k-means (untethered), bit for bit;
    - the oracle fed the GPU's clusterings (teacher-forced, which the line
      above shows equal to the oracle's own) for the retrieval sets of every
      block problem, the exact-key counts and the outputs;
    - the relative squared error against exact causal attention on those
      heads, GPU against oracle within 1e-3."""
    w = WORKLOADS[name]
    Q, K, V = make_inputs(w)
    O, g = gpu_causal(Q, K, V, w.dtype, w.block, w.C, w.iters, w.cluster_seed, w.topk, w.scale,
                      w.mode)
    assert np.isfinite(O).all()
    N, L, C = w.N, w.block, w.C
    G = w.Hq // w.Hkv
    levels = oracle.causal_levels(N, L)
    pmax = (N // L) // 2
    kv_heads = sorted({h // G for h in GQA_HEADS})
    jobs = []
    for role, heads, X in ((0, kv_heads, K), (1, GQA_HEADS, Q)):
        for h in heads:
            for _, lv, p, s in causal_problems(N, L):
                jobs.append((role, h, lv, p, s, X))

    def run(job):
        role, h, lv, p, s, X = job
        blk = X[0, h, (2 * p + role) * s:(2 * p + role + 1) * s]
        sid = (h * levels + lv) * pmax + p
        return oracle.kmeans(blk, min(C, s), w.iters, w.cluster_seed, sid, role)[0]

    # ctypes releases the GIL: the oracle's k-means problems run in parallel
    with concurrent.futures.ThreadPoolExecutor(os.cpu_count() or 4) as ex:
        results = list(ex.map(run, jobs))
    for (role, h, lv, p, s, _), ra in zip(jobs, results):
        ga = (g["k_assign"] if role == 0 else g["q_assign"])[0, h, lv, p * s:(p + 1) * s]
        assert_assign_match(ga, ra, what=f"{'kq'[role]} h{h} lv{lv} p{p}")

    def forced(h):
        mask = np.zeros((1, w.Hq), np.uint8)
        mask[0, h] = 1
        return oracle.muse_causal(Q, K, V, L, C, w.iters, w.cluster_seed, w.topk, w.scale,
                                  w.mode, hq_mask=mask, q_assign_in=g["q_assign"],
                                  k_assign_in=g["k_assign"])

    with concurrent.futures.ThreadPoolExecutor(len(GQA_HEADS)) as ex:
        rs = list(ex.map(forced, GQA_HEADS))
    for h, r in zip(GQA_HEADS, rs):
        assert_causal_selected(g["selected"][0, h], r["selected"][0, h], g["q_assign"][0, h],
                               N, L, C, f"h{h}")
        assert (g["n_exact"][0, h] == r["n_exact"][0, h]).all(), f"n_exact h{h}"
        assert_close(O[0, h], r["O"][0, h], TOL[w.dtype], f"O head {h}")
    # exact causal attention is O(N^2) per head in fp64: the relative squared
    # error is taken over 512 sampled query rows per head (the first and last
    # rows, block edges and random rows), for the GPU and the oracle alike
    rng = np.random.default_rng(11)
    rows = np.unique(np.concatenate([[0, 1, L - 1, L, N - 1], rng.integers(0, N, 507)]))
    E = np.stack([oracle.exact_attention_rows(Q, K, V, 0, h, rows, w.scale, causal=True)
                  for h in GQA_HEADS])
    r_gpu = rse(O[0, GQA_HEADS][:, rows], E)
    r_orc = rse(np.stack([r["O"][0, h][rows] for h, r in zip(GQA_HEADS, rs)]), E)
    assert abs(r_gpu - r_orc) < 1e-3, (r_gpu, r_orc)


@pytest.mark.parametrize("causal", [False, True])
def test_sharded_layer_equals_whole_layer_on_gpu(causal):
    """The layer split into (batch, kv-head) units over 3 ranks, each shard run
    by the CUDA operator with the whole layer's stream ids, reassembles to the
    whole-layer output bit for bit.  The ranks run one after another on this
    GPU (the path needs no exchange)."""
    from clustered_multipole_approximation_b200 import sharding
    Q, K, V = clustered_qkv(2, 8, 4, 1024, 64, 8, 0.3, 0.0, "bf16", 81)
    q, k, v = to_dev(Q, "bf16"), to_dev(K, "bf16"), to_dev(V, "bf16")
    kw = dict(iters=4, seed=9, topk=2, out_dtype=torch.float32)
    kw.update(dict(C=12, block=128) if causal else dict(Cq=12, Ck=10))
    fn = muse.muse_attn_fwd_causal if causal else muse.muse_attn_fwd
    whole = fn(q, k, v, **kw)
    world = 3
    plan = sharding.partition(2, 4, world)
    shards = [sharding.muse_attn_fwd_sharded(q, k, v, rank=r, world=world, causal=causal, **kw)[0]
              for r in range(world)]
    torch.cuda.synchronize()
    O = sharding.assemble(shards, plan, 2, 8, 4)
    assert torch.equal(O, whole)
