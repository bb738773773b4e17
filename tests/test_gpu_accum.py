"""Parity of the block-accumulation causal operator (muse_attn_fwd_causal_accum,
through the C ABI) with its fp64 oracle (oracle/muse_v4.py).

Assignments, both selections (clusters, then blocks within them) and the
exact-key counts must match bit for bit; outputs within 1e-5 (fp32 inputs) or
2e-3 (bf16 inputs) max-abs on the fp32 output; the relative squared error
against exact causal attention within 1e-3 of the oracle's.
"""
import numpy as np
import pytest
import torch

import clustered_multipole_approximation_b200 as muse
import oracle
from clustered_multipole_approximation_b200 import build
from clustered_multipole_approximation_b200.inputs import WORKLOADS, clustered_qkv, make_inputs
from helpers import TOL, assert_assign_match, assert_close, rse, to_dev
from oracle.muse_v4 import muse_v4

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    muse.load_library()


def gpu_accum(Q, K, V, dtype, L, Cq, Ck, iters, seed, k1, k2, scale, mode):
    q, k, v = to_dev(Q, dtype), to_dev(K, dtype), to_dev(V, dtype)
    kw = dict(Cq=Cq, Ck=Ck, block=L, iters=iters, seed=seed, topk=k1, topk2=k2, scale=scale,
              mode=mode)
    O, dbg = muse.muse_attn_fwd_causal_accum(q, k, v, debug=True, out_dtype=torch.float32, **kw)
    Ob = muse.muse_attn_fwd_causal_accum(q, k, v, **kw)
    torch.cuda.synchronize()
    assert torch.equal(Ob, O.to(Ob.dtype))
    assert int(dbg["device_error"].item()) == 0
    return O.cpu().numpy(), {n: t.cpu().numpy() for n, t in dbg.items()}


def check_accum(Q, K, V, dtype, L, Cq, Ck, iters, seed, k1, k2, scale, mode, heads=None):
    B, Hq, N = Q.shape[:3]
    G = Hq // K.shape[1]
    O, g = gpu_accum(Q, K, V, dtype, L, Cq, Ck, iters, seed, k1, k2, scale, mode)
    mask = None
    if heads is not None:
        mask = np.zeros((B, Hq), np.uint8)
        for b, h in heads:
            mask[b, h] = 1
    r = muse_v4(Q, K, V, L, Cq, Ck, iters, seed, k1, k2, scale, mode, hq_mask=mask)
    hs = [(b, h) for b in range(B) for h in range(Hq)] if heads is None else heads
    for b, h in hs:
        assert_assign_match(g["k_assign"][b, h // G], r["k_assign"][b, h // G], what="k_assign")
        assert_assign_match(g["q_assign"][b, h], r["q_assign"][b, h], what="q_assign")
        if k1 > 0 and k2 > 0:
            assert (g["sel1"][b, h] == r["sel1"][b, h]).all(), f"sel1 b{b}h{h}"
            assert (g["sel2"][b, h] == r["sel2"][b, h]).all(), f"sel2 b{b}h{h}"
        assert (g["n_exact"][b, h] == r["n_exact"][b, h]).all(), f"n_exact b{b}h{h}"
        assert_close(O[b, h], r["O"][b, h], TOL[dtype], f"O b{b}h{h}")
    rmask = np.zeros((B, Hq), np.uint8)
    for b, h in hs:
        rmask[b, h] = 1
    E = oracle.exact_attention(Q, K, V, scale, causal=True, hq_mask=rmask)
    idx = tuple(np.array(hs).T)
    assert abs(rse(O[idx], E[idx]) - rse(r["O"][idx], E[idx])) < 1e-3
    return O, g, r


@pytest.mark.parametrize("dtype,D", [("f32", 64), ("f32", 128), ("bf16", 64), ("bf16", 128)])
@pytest.mark.parametrize("mode", ["monopole", "dipole"])
def test_small_accum_gqa(dtype, D, mode):
    Q, K, V = clustered_qkv(1, 4, 2, 1024, D, 10, 0.35, 0.0, dtype, 141 + D)
    check_accum(Q, K, V, dtype, 128, 12, 16, 4, 21, 3, 2, 0.75, mode)


def test_accum_ragged_blocks_bf16_simt_local():
    # L = 96 is not a multiple of 128: the local blocks take the SIMT kernel
    Q, K, V = clustered_qkv(2, 2, 1, 960, 64, 8, 0.3, 0.0, "bf16", 142)
    check_accum(Q, K, V, "bf16", 96, 9, 11, 4, 5, 2, 3, 1.0, "dipole")


def test_accum_one_block_is_exact_causal_attention():
    Q, K, V = clustered_qkv(1, 2, 1, 512, 64, 8, 0.3, 0.0, "f32", 143)
    O, _, _ = check_accum(Q, K, V, "f32", 512, 8, 8, 3, 5, 2, 1, 1.0, "dipole")
    assert_close(O, oracle.exact_attention(Q, K, V, causal=True), 1e-5, "O vs exact")


def test_accum_retrieving_everything_is_exact_causal_attention():
    Q, K, V = clustered_qkv(1, 2, 2, 512, 64, 8, 0.3, 0.0, "f32", 144)
    O, _, _ = check_accum(Q, K, V, "f32", 64, 8, 8, 3, 5, 8, 8, 1.0, "dipole")
    assert_close(O, oracle.exact_attention(Q, K, V, causal=True), 1e-5, "O vs exact")


@pytest.mark.parametrize("k1,k2", [(0, 0), (3, 0), (16, 1)])
def test_accum_retrieval_budgets(k1, k2):
    Q, K, V = clustered_qkv(1, 2, 1, 1024, 64, 12, 0.3, 0.5, "bf16", 145)
    check_accum(Q, K, V, "bf16", 128, 16, 16, 4, 9, k1, k2, 1.0, "dipole")


@pytest.mark.parametrize("mode", ["monopole", "dipole"])
def test_accum_clusters_with_empty_prefixes(mode):
    # 64 key clusters and blocks of 64: the first blocks' prefixes leave most
    # key clusters without a member
    Q, K, V = clustered_qkv(1, 2, 1, 1024, 64, 16, 0.4, 0.0, "bf16", 149)
    O, _, _ = check_accum(Q, K, V, "bf16", 64, 32, 64, 4, 11, 2, 1, 1.0, mode)
    assert np.isfinite(O).all()


def test_accum_many_retrieved_keys():
    # 4 clusters over blocks of 1024: each retrieved (cluster, block) pair
    # holds ~256 keys, so a query cluster retrieves more keys than the
    # stage-2 kernel lists in shared memory at once
    Q, K, V = clustered_qkv(1, 1, 1, 4096, 64, 4, 0.3, 0.0, "bf16", 148)
    _, g, _ = check_accum(Q, K, V, "bf16", 1024, 4, 4, 3, 7, 4, 2, 1.0, "dipole")
    assert g["n_exact"].max() > 1024 + 1024


def test_accum_never_reads_the_future_on_gpu():
    """Changing the values after position t0 changes no output up to t0 (the
    clusterings read only keys and queries, so they stay as they were)."""
    Q, K, V = clustered_qkv(1, 1, 1, 1024, 64, 8, 0.3, 0.0, "bf16", 146)
    kw = dict(Cq=8, Ck=8, block=128, iters=4, seed=3, topk=2, topk2=2, scale=1.0)
    q, k, v = to_dev(Q, "bf16"), to_dev(K, "bf16"), to_dev(V, "bf16")
    base = muse.muse_attn_fwd_causal_accum(q, k, v, **kw)
    t0 = 700
    v2 = v.clone()
    v2[:, :, t0 + 1:] = torch.flip(v2[:, :, t0 + 1:], dims=[2])  # values only: clusterings fixed
    out = muse.muse_attn_fwd_causal_accum(q, k, v2, **kw)
    torch.cuda.synchronize()
    assert torch.equal(out[:, :, :t0 + 1], base[:, :, :t0 + 1])
    assert not torch.equal(out[:, :, t0 + 1:], base[:, :, t0 + 1:])


def test_workload_causal_b2h8_n16k_accum():
    """The 16k causal layer (B=2, 8 heads, C=64, blocks of 512) with k1 = 4
    key clusters and k2 = 2 blocks each, heads (0, 1) and (1, 6) against the
    oracle."""
    w = WORKLOADS["causal-bf16-b2h8-n16k"]
    Q, K, V = make_inputs(w)
    check_accum(Q, K, V, w.dtype, w.block, w.C, w.C, w.iters, w.cluster_seed, 4, 2, w.scale,
                "dipole", heads=[(0, 1), (1, 6)])


@pytest.mark.parametrize("case", ["tilted", "clusters_above_256", "k2_above_blocks"])
def test_accum_unsupported_arguments_are_refused(case):
    Q, K, V = clustered_qkv(1, 1, 1, 1024, 64, 8, 0.3, 0.0, "bf16", 147)
    q, k, v = (to_dev(x, "bf16") for x in (Q, K, V))
    kw = dict(Cq=8, Ck=8, block=128, iters=2, seed=1, topk=2, topk2=2, mode="dipole")
    if case == "tilted":
        kw["mode"] = "tilted"
    elif case == "clusters_above_256":
        kw["Ck"] = 300
    else:
        kw["topk2"] = 9
    with pytest.raises(muse.MuseError):
        muse.muse_attn_fwd_causal_accum(q, k, v, **kw)
