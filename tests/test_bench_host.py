"""Host-side logic of the benchmark's roofline accounting (no GPU): the
far-field rows and retrieved keys it counts from the clusterings and
retrieval sets must agree with the exact-key counts the oracle reports, and
the level table with the causal decomposition."""
import numpy as np
import pytest

import bench
import oracle
from clustered_multipole_approximation_b200.inputs import WORKLOADS, clustered_qkv


def _as_debug(r, C, topk):
    d = dict(q_assign=r["q_assign"], k_assign=r["k_assign"], n_exact=r["n_exact"])
    if topk > 0:
        d["selected"] = r["selected"]
    return d


@pytest.mark.parametrize("topk", [0, 2])
def test_counted_retrieval_matches_exact_key_counts_causal(topk):
    w = WORKLOADS["causal-bf16-b2h8-n16k"].replace(B=1, Hq=4, Hkv=2, N=1024, block=128, C=16,
                                                   iters=3, topk=topk)
    Q, K, V = clustered_qkv(1, 4, 2, 1024, 64, 8, 0.3, 0.0, "bf16", 3)
    r = oracle.muse_causal(Q, K, V, w.block, w.C, w.iters, w.cluster_seed, topk)
    work, f_alg, nbytes, retrieved = bench.algorithmic_work(w, "dipole", _as_debug(r, w.C, topk))
    local = (1024 // 128) * 128 * 129 / 2 * 4
    assert retrieved == pytest.approx(r["n_exact"].sum() - local)
    assert f_alg == pytest.approx(sum(work.values()))
    assert nbytes == (4 * 1024 * 64 * 2 + 2 * 2 * 1024 * 64) * 2


def test_counted_retrieval_matches_exact_key_counts_acausal():
    w = WORKLOADS["acausal-bf16-h8-n8k"].replace(Hq=2, Hkv=2, N=1000, C=12, iters=3, topk=3)
    Q, K, V = clustered_qkv(1, 2, 2, 1000, 64, 8, 0.3, 0.0, "bf16", 4)
    r = oracle.muse_acausal(Q, K, V, 12, 12, 3, w.cluster_seed, 3)
    _, _, _, retrieved = bench.algorithmic_work(w, "dipole", _as_debug(r, 12, 3))
    assert retrieved == r["n_exact"].sum()
    far, exact = bench.retrieval_rows(w, "dipole", _as_debug(r, 12, 3))
    # every query sees each non-empty key cluster once: far or retrieved
    nonempty = [(r["k_count"][0, h] > 0).sum() for h in range(2)]
    sel = r["selected"]
    assert far[0] + sum(int(((sel[0, h] >= 0).sum(-1))[r["q_assign"][0, h]].sum())
                        for h in range(2)) == 1000 * sum(nonempty)


def test_level_table_tiles_the_causal_decomposition():
    w = WORKLOADS["causal-gqa32x8-n64k-d64"]
    lt = bench.level_table(w, "dipole")
    assert [s for s, *_ in lt] == [1024 << l for l in range(6)]
    assert sum(npairs for _, npairs, _, _ in lt) == w.N // w.block - 1
    assert [d for *_, d in lt] == [True, True, False, False, False, False]
    assert [d for *_, d in bench.level_table(w, "monopole")] == [False] * 6
    # the fine-query dipole runs per key token at every level, acausal included
    assert [d for *_, d in bench.level_table(w, "dipole_q")] == [True] * 6
    a = WORKLOADS["acausal-bf16-h8-n8k"]
    assert bench.level_table(a, "dipole") == [(8192, 1, 128, False)]
    assert bench.level_table(a, "dipole_q") == [(8192, 1, 128, True)]


def test_backward_and_variant_work_accounting():
    """The backward's counted work has every kernel's share where it runs
    (the causal form adds the local blocks), and the per-key-token variants
    count their stage 2 against the kernel that runs it."""
    a = WORKLOADS["acausal-bf16-h8-n8k"]
    c = WORKLOADS["causal-bf16-b2h8-n16k"]

    def fake_dbg(w):
        rng = np.random.default_rng(0)
        lv = len(bench.level_table(w, "dipole"))
        if w.causal:
            return {"q_assign": rng.integers(0, min(w.C, w.block), (w.B, w.Hq, lv, w.N // 2)),
                    "k_assign": rng.integers(0, min(w.C, w.block), (w.B, w.Hkv, lv, w.N // 2))}
        return {"q_assign": rng.integers(0, w.C, (w.B, w.Hq, w.N)),
                "k_assign": rng.integers(0, w.C, (w.B, w.Hkv, w.N))}

    wa = bench.backward_work(a, "dipole", fake_dbg(a))
    assert wa["bwd_query"] > 0 and wa["bwd_u_table"] > 0 and wa["bwd_local"] == 0
    wc = bench.backward_work(c, "dipole", fake_dbg(c))
    assert wc["bwd_local"] > 0 and wc["bwd_query"] > 0
    assert bench.backward_work(a, "monopole", fake_dbg(a))["bwd_u_table"] == 0
    work, *_ = bench.algorithmic_work(a, "tilted_dipole", fake_dbg(a))
    assert work["stage2_tdip"] > 0 and work["stage2_attn"] == 0
    work, *_ = bench.algorithmic_work(a, "dipole_q", fake_dbg(a))
    assert work["stage2_dense"] > 0 and work["stage2_attn"] == 0
