"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): each
rank runs its own layer, the job time is the slowest rank's, and throughput is
every rank's tokens over that time.  The operator itself has no collective."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from clustered_multipole_approximation_b200.inputs import WORKLOADS


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [120.0, 150.0][rank]
        m = bench.max_over_ranks(local_ms, world)
        w = WORKLOADS["acausal-bf16-h8-n8k"]
        out[rank] = (m, bench.rank_data_seed(w, rank),
                     bench.whole_job_throughput(w.B * w.N, world, 10, m))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert out[0][0] == out[1][0] == 150.0
    assert out[0][1] != out[1][1]          # independent layers per rank
    assert out[0][2] == pytest.approx(8192 * 2 * 10 / 0.150)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_throughput(100, 1, 4, 2000.0) == pytest.approx(200.0)


# ---------------------------------------------------------------------------
# one layer sharded by (batch, kv-head) units across ranks
# ---------------------------------------------------------------------------
from clustered_multipole_approximation_b200 import sharding  # noqa: E402


def test_partition_covers_every_unit_once():
    for B, Hkv, world in [(1, 8, 2), (1, 3, 2), (2, 8, 8), (1, 2, 4), (3, 5, 4), (1, 1, 3)]:
        plan = sharding.partition(B, Hkv, world)
        assert len(plan) == world
        seen = [u for a, b in plan for u in range(a, b)]
        assert seen == list(range(B * Hkv))  # contiguous, in order, each once
        sizes = [b - a for a, b in plan]
        assert max(sizes) - min(sizes) <= 1


def _oracle_forward(causal):
    import oracle

    def fwd(q, k, v, *, key_stream0, query_stream0, **kw):
        f = oracle.muse_causal if causal else oracle.muse_acausal
        r = f(q.numpy(), k.numpy(), v.numpy(), key_stream0=key_stream0,
              query_stream0=query_stream0, **kw)
        return torch.from_numpy(r["O"])
    return fwd


def _layer():
    from clustered_multipole_approximation_b200.inputs import clustered_qkv
    Q, K, V = clustered_qkv(1, 6, 3, 256, 64, 8, 0.3, 0.0, "f32", 17)
    return (torch.from_numpy(x).double() for x in (Q, K, V))


def _shard_worker(rank, world, port, out, causal):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = _layer()
        kw = dict(L=64, C=6) if causal else dict(Cq=7, Ck=6)
        O = sharding.muse_attn_fwd_sharded(q, k, v, rank=rank, world=world, causal=causal,
                                           gather=True, forward=_oracle_forward(causal),
                                           iters=3, seed=5, topk=2, **kw)
        out[rank] = O.numpy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("causal", [False, True])
def test_two_ranks_rebuild_the_single_process_layer(causal):
    """Each rank runs its units (3 kv-heads over 2 ranks: 2 + 1) with the
    stream ids of the whole layer; the all-gathered output equals the
    single-process output bit for bit (the fp64 oracle stands in for the
    operator on CPU)."""
    import oracle
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_shard_worker, args=(world, _free_port(), out, causal), nprocs=world,
                       start_method="spawn")
    q, k, v = _layer()
    if causal:
        ref = oracle.muse_causal(q.numpy(), k.numpy(), v.numpy(), 64, 6, 3, 5, 2)["O"]
    else:
        ref = oracle.muse_acausal(q.numpy(), k.numpy(), v.numpy(), 7, 6, 3, 5, 2)["O"]
    for r in range(world):
        assert (out[r] == ref).all()
