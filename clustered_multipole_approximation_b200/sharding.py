"""Sharding one MuSe layer across ranks (one process per GPU).

Every (batch, kv-head) unit of a layer is independent: its keys are clustered
and summarised once, and its q-heads' queries are clustered and attend only to
those keys (the hierarchical causal blocks stay inside one sequence).  A layer
therefore splits across ranks by contiguous runs of units with no exchange on
the data path; the only collective is the optional all-gather that rebuilds
the whole output on every rank.

Each rank's units run as one call of the operator, each unit a batch entry
with Hkv = 1 and Hq = G = Hq / Hkv.  The call passes the stream ids of its
first unit (key_stream0 = u0, query_stream0 = G u0), so every unit draws the
same seeded k-means starts as in the whole-layer call, and the shards are bit
for bit the whole layer's rows.
"""
from __future__ import annotations

import torch


def partition(B: int, Hkv: int, world: int) -> list[tuple[int, int]]:
    """Contiguous, balanced runs [u0, u1) of the B * Hkv units, one per rank
    (unit u is (b, kv-head) = divmod(u, Hkv)); ranks past the units get an
    empty run."""
    U = B * Hkv
    base, extra = divmod(U, world)
    out, u = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((u, u + n))
        u += n
    return out


def shard_inputs(q, k, v, u0: int, u1: int):
    """The units [u0, u1) as batch entries: q [U, G, N, D], k and v [U, 1, N, D]
    (contiguous copies)."""
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    units = [divmod(u, Hkv) for u in range(u0, u1)]
    qs = torch.stack([q[b, h * G:(h + 1) * G] for b, h in units]) if units else q.new_empty(0, G, N, D)
    ks = torch.stack([k[b, h:h + 1] for b, h in units]) if units else k.new_empty(0, 1, N, D)
    vs = torch.stack([v[b, h:h + 1] for b, h in units]) if units else v.new_empty(0, 1, N, D)
    return qs.contiguous(), ks.contiguous(), vs.contiguous()


def assemble(shards, plan, B: int, Hq: int, Hkv: int):
    """The whole-layer output [B, Hq, N, D] from the ranks' shard outputs
    (shard r: [u1 - u0, G, N, D])."""
    G = Hq // Hkv
    ref = next(s for s in shards if s.shape[0] > 0)
    O = ref.new_empty(B, Hq, ref.shape[2], ref.shape[3])
    for (u0, u1), s in zip(plan, shards):
        for i, u in enumerate(range(u0, u1)):
            b, h = divmod(u, Hkv)
            O[b, h * G:(h + 1) * G] = s[i]
    return O


def muse_attn_fwd_sharded(q, k, v, *, rank: int, world: int, causal: bool = False,
                          gather: bool = False, group=None, forward=None, **params):
    """This rank's share of one MuSe layer.

    q [B,Hq,N,D], k and v [B,Hkv,N,D] hold the whole layer on every rank (or
    at least this rank's units).  Runs the operator on units
    partition(B, Hkv, world)[rank] and returns (O_shard [U_r, G, N, D],
    (u0, u1)); with gather=True it all-gathers the shards over
    torch.distributed (`group`, NCCL for CUDA tensors) and returns the whole
    O [B,Hq,N,D] instead.  `params` are those of muse_attn_fwd /
    muse_attn_fwd_causal; `forward` replaces the operator (a callable with
    their signature), for tests."""
    if forward is None:
        import clustered_multipole_approximation_b200 as muse
        forward = muse.muse_attn_fwd_causal if causal else muse.muse_attn_fwd
    B, Hq = q.shape[:2]
    Hkv = k.shape[1]
    G = Hq // Hkv
    plan = partition(B, Hkv, world)
    u0, u1 = plan[rank]
    qs, ks, vs = shard_inputs(q, k, v, u0, u1)
    if u1 > u0:
        o = forward(qs, ks, vs, key_stream0=u0, query_stream0=G * u0, **params)
    else:
        o = torch.empty(0, G, q.shape[2], q.shape[3], dtype=params.get("out_dtype") or q.dtype,
                        device=q.device)
    if not gather:
        return o, (u0, u1)
    import torch.distributed as dist
    most = max(b - a for a, b in plan)
    padded = o.new_zeros(most, *o.shape[1:])
    padded[:o.shape[0]] = o
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded, group=group)
    return assemble([p[:b - a] for p, (a, b) in zip(parts, plan)], plan, B, Hq, Hkv)
