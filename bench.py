#!/usr/bin/env python
"""Benchmark of the MuSe forward operator; rank 0 prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl muse|reference]
                    [--workload NAME] [--mode dipole|monopole|tilted|dipole_q]

A step is one full forward call of the operator (k-means of queries and keys,
summaries, selection, far field + exact retrieval) over one layer of synthetic
clustered inputs already resident in HBM.  Between timed steps the L2 cache is
flushed by writing a 512 MiB buffer; only the operator's own interval is
timed (CUDA events on the launching stream).  With N > 1 (torchrun) every rank
runs its own layer (weak scaling, no collective on the data path) and the time
is the max over ranks.

The headline line is the 8-head 8k acausal layer (DIPOLE).  The default run
also times every other configuration with N >= 8k (the MONOPOLE variant of
the 8k layer and the three causal layers) and reports each under
"workloads", with its own roofline figures.

--impl reference times the fp64 CPU oracle (the plain statement of the
method) on the host cores, each step a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from clustered_multipole_approximation_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "MuSe attn fwd tokens/s/layer at 8k–64k; % of roofline; rel. sq. error vs exact"
UNIT = "tokens/s/layer"
DEFAULT_WORKLOAD = "acausal-bf16-h8-n8k"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="muse", choices=["muse", "reference"])
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(WORKLOADS))
    p.add_argument("--mode", default=None, choices=[None, "dipole", "monopole", "tilted", "dipole_q",
                                                       "tilted_dipole"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--accum", action="store_true",
                   help="time only the block-accumulation causal form of a causal workload")
    p.add_argument("--backward", action="store_true",
                   help="time only the backward pass of an acausal workload (one JSON line)")
    p.add_argument("--no-side", action="store_true",
                   help="skip the other N >= 8k configurations of the default run")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.dev = device_index
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        time.sleep(0.3)

    def stop(self):
        if self.p is None:
            return None
        time.sleep(0.3)
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.f.read().splitlines():
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.f.name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# algorithmic work of one call (what the method must compute)
# ---------------------------------------------------------------------------
# DRAM bytes (read + write) of one launch of a kernel on a workload, from one ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum, caches flushed as in the
# timed region).  An entry is removed whenever its kernel changes.
NCU_TRAFFIC: dict = {
    # k-means of the 8k x 8-head layer: its resident launch read 18.05 MB and wrote
    # 1 KB; the call's second launch (sequential order) finds every problem certified
    # exact and exits at once -- the average over the call's two launches
    ("acausal-bf16-h8-n8k", "kmeans"): (18_046_976 + 1_024) / 2,
}

# The library's per-kernel profiling names -> what they compute.
TENSOR_KERNELS = ("kmeans", "stage1_summaries", "stage2_attn", "stage2_dense", "stage2_tdip",
                  "causal_local_merge")
# Launches that together do one algorithmic step: the persistent k-means runs
# the problems whose centroid sums are certified exact with every token tile
# resident in shared memory, and the rest in sequential order.
KERNEL_GROUPS = {"kmeans_resident": "kmeans", "kmeans_ordered": "kmeans"}


def level_table(w, mode):
    """(block size s, pairs per head, effective clusters, per-key-token far field)
    of every level; the acausal operator is one level with one block problem.
    The per-key-token form runs where the library's dense-level rule admits it:
    bf16 DIPOLE, C <= 256, s a multiple of 128, s <= 2048 and s <= 8 C_eff; and
    at every level in the fine-query mode (DIPOLE_Q)."""
    fq = mode == "dipole_q"
    if not w.causal:
        return [(w.N, 1, w.C, fq)]
    out, s = [], w.block
    while s < w.N:
        ce = min(w.C, s)
        dense = fq or (w.dtype == "bf16" and mode == "dipole" and w.C <= 256 and s % 128 == 0
                       and s <= 2048 and s <= 8 * ce)
        out.append((s, w.N // (2 * s), ce, dense))
        s *= 2
    return out


def retrieval_rows(w, mode, dbg):
    """Far-field rows and exact retrieved keys summed over every query, per
    level, counted from the actual clusterings and retrieval sets: a query of
    cluster i in block problem p has one far row per non-empty key cluster
    outside R_i and one exact key per member of R_i's clusters."""
    G = w.Hq // w.Hkv
    qa, ka = dbg["q_assign"], dbg["k_assign"]
    sel = dbg.get("selected")
    far = []
    exact = []
    pbase = 0
    for lv, (s, npairs, ce, _dense) in enumerate(level_table(w, mode)):
        f_lv = e_lv = 0.0
        for b in range(w.B):
            for h in range(w.Hq):
                if w.causal:
                    qb = qa[b, h, lv].reshape(npairs, s)
                    kb = ka[b, h // G, lv].reshape(npairs, s)
                    sl = sel[b, h, pbase:pbase + npairs, :ce] if sel is not None else None
                else:
                    qb, kb = qa[b, h][None], ka[b, h // G][None]
                    sl = sel[b, h][None] if sel is not None else None
                off = (np.arange(npairs) * ce)[:, None]
                nq = np.bincount((qb + off).ravel(), minlength=npairs * ce).reshape(npairs, ce)
                nk = np.bincount((kb + off).ravel(), minlength=npairs * ce).reshape(npairs, ce)
                nonempty = (nk > 0).sum(1, keepdims=True)
                if sl is None or sl.shape[-1] == 0:
                    nsel = np.zeros((npairs, ce))
                    ex = np.zeros((npairs, ce))
                else:
                    ok = sl >= 0
                    nsel = ok.sum(-1)
                    got = np.take_along_axis(nk[:, None, :].repeat(ce, 1),
                                             np.where(ok, sl, 0), axis=2)
                    ex = (got * ok).sum(-1)
                f_lv += float((nq * (nonempty - nsel)).sum())
                e_lv += float((nq * ex).sum())
        far.append(f_lv)
        exact.append(e_lv)
        pbase += npairs
    return far, exact


def algorithmic_work(w, mode, dbg):
    """Per-call algorithmic FLOPs of each kernel and of the whole operator
    (a multiply-add counts 2 FLOPs), and the operator's algorithmic bytes:
      k-means       T * 2 * tokens * C_eff * D per role (every level);
      stage 1       min(2 C_eff^2 D^2 + 2 s D^2, 4 s C_eff D) per query problem
                    (the dipole contraction; 0 for MONOPOLE and DIPOLE_Q);
      stage 2       4 D per far row and per exact retrieved key; DIPOLE_Q and
                    TILTED_DIPOLE
                    (per key token: q.k_t, the factor's q.(k_t - mu) and
                    the weighted v_t) 4 D per (query, key) pair of the block
                    plus 2 D per (query, key cluster) for q.mu_j;
      local block   4 D per (query, key) pair of the causal local block;
      bytes         Q, K and V read once, O written once."""
    B, Hq, Hkv, D = w.B, w.Hq, w.Hkv, w.D
    far, exact = retrieval_rows(w, mode, dbg)
    work = dict.fromkeys(TENSOR_KERNELS, 0.0)
    for lv, (s, npairs, ce, dense) in enumerate(level_table(w, mode)):
        toks = npairs * s
        work["kmeans"] += w.iters * 2.0 * toks * ce * D * B * (Hq + Hkv)
        if not dense and mode != "monopole":
            work["stage1_summaries"] += npairs * B * Hq * min(2.0 * ce * ce * D * D + 2.0 * s * D * D,
                                                              4.0 * s * ce * D)
        if mode == "dipole_q":
            work["stage2_dense"] += B * Hq * toks * (4.0 * D * s + 2.0 * D * ce)
        elif mode == "tilted_dipole":  # per key token: q.k_t, nu.k_t, the weighted v_t
            work["stage2_tdip"] += B * Hq * toks * (4.0 * D * s + 2.0 * D * ce)
        else:
            work["stage2_dense" if dense else "stage2_attn"] += 4.0 * D * (far[lv] + exact[lv])
    if w.causal:
        L = w.block
        work["causal_local_merge"] = 4.0 * D * B * Hq * (w.N // L) * L * (L + 1) / 2
    elt = 2 if w.dtype == "bf16" else 4
    nbytes = (B * Hq * w.N * D * 2 + 2 * B * Hkv * w.N * D) * elt
    retrieved = sum(exact)
    return work, sum(work.values()), nbytes, retrieved

# ---------------------------------------------------------------------------
# multi-rank plumbing (one independent layer per rank, no data-path collective)
# ---------------------------------------------------------------------------
def rank_data_seed(w, rank: int) -> int:
    """Each rank draws its own layer of the workload."""
    return w.data_seed + rank


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The slowest rank's value (every rank gets it)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_throughput(tokens_per_rank: int, world: int, steps: int, max_ms: float) -> float:
    """Tokens processed by all ranks per second of the slowest rank."""
    return tokens_per_rank * world * steps / (max_ms / 1e3)


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
def run_muse(w, mode, steps, warmup, rank, world, device, e2e_leg=True):
    """Times `steps` calls of the operator on workload `w` (inputs resident in
    HBM, L2 flushed between calls) and, with e2e_leg, the same through host
    buffers; returns the measurements and the roofline figures."""
    import clustered_multipole_approximation_b200 as muse

    Q, K, V = make_inputs(w, seed=rank_data_seed(w, rank))
    cast = (lambda x: torch.from_numpy(x).to(torch.bfloat16)) if w.dtype == "bf16" else torch.from_numpy
    hq, hk, hv = cast(Q).pin_memory(), cast(K).pin_memory(), cast(V).pin_memory()
    del Q, K, V
    q, k, v = hq.to(device), hk.to(device), hv.to(device)
    out = torch.empty_like(q)
    kw = dict(iters=w.iters, seed=w.cluster_seed, topk=w.topk, scale=w.scale, mode=mode)
    if w.causal:
        kw.update(C=w.C, block=w.block)
        fn = muse.muse_attn_fwd_causal
        params = muse.make_params(w.C, w.C, w.iters, w.cluster_seed, w.topk, w.block, w.scale, mode)
    else:
        kw.update(Cq=w.C, Ck=w.C)
        fn = muse.muse_attn_fwd
        params = muse.make_params(w.C, w.C, w.iters, w.cluster_seed, w.topk, 0, w.scale, mode)
    ws = torch.empty(muse.workspace_size(q, k, params, w.causal), dtype=torch.uint8, device=device)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def step():
        fn(q, k, v, out=out, workspace=ws, **kw)

    # one untimed call with inspection outputs: retrieval counts and accuracy
    o_chk, dbg = fn(q, k, v, debug=True, workspace=ws, **kw)
    muse.device_status(dbg["device_error"])
    dbg = {n: t.cpu().numpy() for n, t in dbg.items()}
    G = w.Hq // w.Hkv
    num = den = 0.0
    for h0 in range(0, w.Hq, G):  # exact attention one kv-group at a time (memory)
        qq = q[:, h0:h0 + G].float()
        kk = k[:, h0 // G:h0 // G + 1].float().expand(-1, G, -1, -1)
        vv = v[:, h0 // G:h0 // G + 1].float().expand(-1, G, -1, -1)
        from torch.nn.attention import SDPBackend, sdpa_kernel
        with sdpa_kernel([SDPBackend.EFFICIENT_ATTENTION]):  # never the N^2-memory path
            E = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, is_causal=w.causal,
                                                                 scale=w.scale)
        num += float(((o_chk[:, h0:h0 + G].float() - E) ** 2).sum())
        den += float((E ** 2).sum())
        del E, qq, kk, vv
    rse_val = num / den
    del o_chk
    torch.cuda.synchronize()

    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clk = Clocks(device.index if device.index is not None else 0)
    clk.start()
    muse.profile_read()
    muse.profile_enable(True)
    evs = []
    for _ in range(steps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize()
    muse.profile_enable(False)
    prof = muse.profile_read()
    clocks = clk.stop()
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world, device)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    tokens = w.B * w.N
    value = whole_job_throughput(tokens, world, steps, total_ms)
    ms_per_step = total_ms / steps

    e2e = None
    if e2e_leg:
        # end to end through the public API: host inputs in, host output back
        ho = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        e2e_ms = 0.0
        for i in range(warmup + steps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            step()
            ho.copy_(out, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
            if i >= warmup:
                e2e_ms += e0.elapsed_time(e1)
        e2e_ms = max_over_ranks(e2e_ms, world, device)
        e2e = {"value": whole_job_throughput(tokens, world, steps, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(hq.numel() * hq.element_size()
                                         + hk.numel() * hk.element_size()
                                         + hv.numel() * hv.element_size()),
               "d2h_bytes_per_step": int(ho.numel() * ho.element_size())}

    # roofline: the dominant kernel, and the whole operator
    pk, how = peaks()
    work, f_alg, b_alg, retrieved = algorithmic_work(w, mode, dbg)
    exact_total = float(np.asarray(dbg["n_exact"], dtype=np.float64).sum())
    local = work["causal_local_merge"] / (4.0 * w.D) if w.causal else 0.0
    # the counted retrieval equals the library's own exact-key count
    assert abs(exact_total - local - retrieved) < 0.5, (exact_total, local, retrieved)
    launches = sum(n for n, _ in prof.values())
    grouped = {}
    for n, (c, t) in prof.items():
        g = KERNEL_GROUPS.get(n, n)
        c0, t0 = grouped.get(g, (0, 0.0))
        grouped[g] = (c0 + c, t0 + t)
    dom = max(grouped, key=lambda n: grouped[n][1])
    dom_launches, dom_ms = grouped[dom]
    peak = pk["bf16_tflops"]
    roofline = {"kernel": dom, "bound": "tensor", "achieved": None, "peak": peak,
                "unit": "TFLOP/s", "frac": None, "traffic": NCU_TRAFFIC.get((w.name, dom)),
                "peak_source": f"{how} bf16 dense (burst)",
                "launches_per_call": dom_launches / steps,
                "avg_launch_ms": dom_ms / dom_launches}
    if work.get(dom):
        per_call_ms = dom_ms / steps
        ach = work[dom] / (per_call_ms / 1e3) / 1e12
        roofline.update(achieved=ach, frac=ach / peak,
                        frac_of_sustained_peak=ach / pk["bf16_tflops_sustained"],
                        flops_per_launch=work[dom] / (dom_launches / steps))
    t_roof = max(f_alg / (peak * 1e12), b_alg / (pk["hbm_gbs"] * 1e9))
    whole = {"algorithmic_tflop": f_alg / 1e12, "algorithmic_gb": b_alg / 1e9,
             "roofline_ms": t_roof * 1e3,
             "achieved_tflops": f_alg / (ms_per_step / 1e3) / 1e12,
             "frac": t_roof / (ms_per_step / 1e3),
             "frac_of_bf16_sustained_peak":
                 f_alg / (ms_per_step / 1e3) / 1e12 / pk["bf16_tflops_sustained"],
             "flops_by_kernel": {n: f for n, f in work.items() if f}}
    tot = sum(x[1] for x in prof.values())
    kernels = {}
    for n, (c, t) in sorted(prof.items(), key=lambda kv: -kv[1][1]):
        e = {"launches": c, "ms_per_call": round(t / steps, 4), "share": round(t / tot, 4)}
        if work.get(n):
            e["tflops"] = round(work[n] / (t / steps / 1e3) / 1e12, 2)
        kernels[n] = e
    for g in set(KERNEL_GROUPS.values()):
        if g in grouped and work.get(g):
            c, t = grouped[g]
            kernels[g + " (all launches)"] = {"ms_per_call": round(t / steps, 4),
                                              "tflops": round(work[g] / (t / steps / 1e3) / 1e12, 2)}
    del q, k, v, out, ws, flush
    torch.cuda.empty_cache()
    return dict(value=value, ms_per_step=ms_per_step, e2e=e2e, roofline=roofline, clocks=clocks,
                gpu_launches=launches, kernels=kernels, rse=rse_val, mode=mode, whole_op=whole)


# ---------------------------------------------------------------------------
# the backward pass (acausal): gradients of <dO, O> through the C ABI
# ---------------------------------------------------------------------------
BWD_KERNELS = ("bwd_key_stats", "bwd_u_table", "bwd_lse", "bwd_query", "bwd_local", "bwd_cluster",
               "bwd_query_nu")


def backward_work(w, mode, dbg):
    """Algorithmic FLOPs of one backward call per kernel (multiply-add = 2):
      bwd_key_stats  S_j: D per key; M_j (DIPOLE): 2 D^2 per key, per kv-head;
      bwd_u_table    (DIPOLE) 2 C_k D^2 per query cluster, per q-head;
      bwd_query      10 D per far row (logit, dO.u, dq, dmu, du) and per exact
                     key (logit, dO.v, dq, dk, dv);
      bwd_cluster    (DIPOLE) dM and dnu: 4 C_q D^2 per key cluster, per
                     q-head; the members' chain: 4 D^2 per key, per kv-head;
                     (MONOPOLE: 2 D per key)."""
    far, exact = retrieval_rows(w, mode, dbg)
    B, Hq, Hkv, D, N = w.B, w.Hq, w.Hkv, w.D, w.N
    dip = mode == "dipole"
    work = dict.fromkeys(BWD_KERNELS, 0.0)
    for s, npairs, ce, _dense in level_table(w, mode):
        toks = npairs * s  # key tokens (and query tokens) of the level's problems, per head
        work["bwd_key_stats"] += B * Hkv * toks * (D + (2.0 * D * D if dip else 0.0))
        if dip:
            work["bwd_u_table"] += B * Hq * npairs * ce * 2.0 * ce * D * D
            work["bwd_cluster"] += B * Hq * npairs * ce * 4.0 * ce * D * D + B * Hkv * toks * 4.0 * D * D
            work["bwd_query_nu"] += B * Hq * toks * D
        else:
            work["bwd_cluster"] += B * Hkv * toks * 2.0 * D
    work["bwd_query"] = 10.0 * D * (sum(far) + sum(exact))
    if w.causal:  # the local blocks: 10 D per (query, key) pair, keys up to the query
        work["bwd_local"] = 10.0 * D * B * Hq * (N // w.block) * w.block * (w.block + 1) / 2
    return work


def run_backward(w, mode, steps, warmup, device):
    """Times `steps` backward calls on workload `w` after one forward call that
    fills the shared workspace (inputs and dO resident, L2 flushed between
    calls); returns ms per call, per-kernel times and the algorithmic rate."""
    import clustered_multipole_approximation_b200 as muse

    Q, K, V = make_inputs(w)
    cast = (lambda x: torch.from_numpy(x).to(torch.bfloat16)) if w.dtype == "bf16" else torch.from_numpy
    q, k, v = cast(Q).to(device), cast(K).to(device), cast(V).to(device)
    del Q, K, V
    if w.causal:
        kw = dict(C=w.C, block=w.block, iters=w.iters, seed=w.cluster_seed, topk=w.topk,
                  scale=w.scale, mode=mode)
        p = muse.make_params(w.C, w.C, w.iters, w.cluster_seed, w.topk, w.block, w.scale, mode)
        fwd, bwd = muse.muse_attn_fwd_causal, muse.muse_attn_bwd_causal
    else:
        kw = dict(Cq=w.C, Ck=w.C, iters=w.iters, seed=w.cluster_seed, topk=w.topk, scale=w.scale,
                  mode=mode)
        p = muse.make_params(w.C, w.C, w.iters, w.cluster_seed, w.topk, 0, w.scale, mode)
        fwd, bwd = muse.muse_attn_fwd, muse.muse_attn_bwd
    ws = torch.empty(muse.backward_workspace_size(q, k, p, causal=w.causal), dtype=torch.uint8,
                     device=device)
    o, dbg = fwd(q, k, v, workspace=ws, debug=True, **kw)
    dbg = {n: t.cpu().numpy() for n, t in dbg.items()}
    do = torch.randn(o.shape, generator=torch.Generator(device=device).manual_seed(7),
                     device=device).to(o.dtype)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        flush.zero_()
        bwd(q, k, v, do, workspace=ws, **kw)
    torch.cuda.synchronize()
    muse.profile_read()
    muse.profile_enable(True)
    total = 0.0
    for _ in range(steps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        bwd(q, k, v, do, workspace=ws, **kw)
        e1.record(stream)
        torch.cuda.synchronize()
        total += e0.elapsed_time(e1)
    muse.profile_enable(False)
    prof = muse.profile_read()
    work = backward_work(w, mode, dbg)
    ms = total / steps
    kernels = {}
    for n, (c, t) in sorted(prof.items(), key=lambda kv: -kv[1][1]):
        e = {"launches": c, "ms_per_call": round(t / steps, 4)}
        if work.get(n):
            e["tflops"] = round(work[n] / (t / steps / 1e3) / 1e12, 3)
        kernels[n] = e
    del q, k, v, o, do, ws, flush
    torch.cuda.empty_cache()
    return {"config": config_of(w, mode), "ms_per_call": ms, "steps": steps, "warmup": warmup,
            "algorithmic_gflop": sum(work.values()) / 1e9,
            "achieved_tflops": sum(work.values()) / (ms / 1e3) / 1e12,
            "arithmetic": "fp32 CUDA cores", "kernels": kernels}


# ---------------------------------------------------------------------------
# the causal operator with block-summary accumulation and cluster/block retrieval
# ---------------------------------------------------------------------------
ACCUM_K1, ACCUM_K2 = 4, 2  # no workload states k1 / k2 for this form: 4 clusters, 2 blocks each


def run_accum_bench(w, mode, steps, warmup, device, k1=ACCUM_K1, k2=ACCUM_K2):
    """Times `steps` calls of muse_attn_fwd_causal_accum on the causal
    workload `w` (inputs resident, L2 flushed between calls); returns
    tokens/s, ms per call, per-kernel times and the RSE against exact causal
    attention."""
    import clustered_multipole_approximation_b200 as muse

    Q, K, V = make_inputs(w)
    cast = (lambda x: torch.from_numpy(x).to(torch.bfloat16)) if w.dtype == "bf16" else torch.from_numpy
    q, k, v = cast(Q).to(device), cast(K).to(device), cast(V).to(device)
    del Q, K, V
    kw = dict(Cq=w.C, Ck=w.C, block=w.block, iters=w.iters, seed=w.cluster_seed, topk=k1,
              topk2=k2, scale=w.scale, mode=mode)
    p = muse.make_params(w.C, w.C, w.iters, w.cluster_seed, k1, w.block, w.scale, mode)
    ws = torch.empty(muse.accum_workspace_size(q, k, p, k2), dtype=torch.uint8, device=device)
    out = torch.empty_like(q)
    o = muse.muse_attn_fwd_causal_accum(q, k, v, workspace=ws, out_dtype=torch.float32, **kw)
    G = w.Hq // w.Hkv
    num = den = 0.0
    from torch.nn.attention import SDPBackend, sdpa_kernel
    for h0 in range(0, w.Hq, G):
        qq = q[:, h0:h0 + G].float()
        kk = k[:, h0 // G:h0 // G + 1].float().expand(-1, G, -1, -1)
        vv = v[:, h0 // G:h0 // G + 1].float().expand(-1, G, -1, -1)
        with sdpa_kernel([SDPBackend.EFFICIENT_ATTENTION]):
            E = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, is_causal=True,
                                                                 scale=w.scale)
        num += float(((o[:, h0:h0 + G] - E) ** 2).sum())
        den += float((E ** 2).sum())
        del E, qq, kk, vv
    del o
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        flush.zero_()
        muse.muse_attn_fwd_causal_accum(q, k, v, out=out, workspace=ws, **kw)
    torch.cuda.synchronize()
    muse.profile_read()
    muse.profile_enable(True)
    total = 0.0
    for _ in range(steps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        muse.muse_attn_fwd_causal_accum(q, k, v, out=out, workspace=ws, **kw)
        e1.record(stream)
        torch.cuda.synchronize()
        total += e0.elapsed_time(e1)
    muse.profile_enable(False)
    prof = muse.profile_read()
    ms = total / steps
    tot = sum(t for _, t in prof.values())
    kernels = {n: {"launches": c, "ms_per_call": round(t / steps, 4), "share": round(t / tot, 4)}
               for n, (c, t) in sorted(prof.items(), key=lambda kv: -kv[1][1])}
    del q, k, v, out, ws, flush
    torch.cuda.empty_cache()
    if not np.isfinite(num / den):
        raise RuntimeError("non-finite output from the block-accumulation form")
    cfg = dict(config_of(w, mode), topk=k1, topk2=k2, form="block-summary accumulation")
    return {"config": cfg, "value": w.B * w.N / (ms / 1e3), "unit": UNIT, "ms_per_call": ms,
            "steps": steps, "warmup": warmup, "rse_vs_exact": num / den, "kernels": kernels}


# ---------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(w, mode, heads):
    """Time the fp64 oracle on the first `heads` q-heads of one layer; returns
    (seconds, per-layer tokens/s extrapolated by head count, threads used)."""
    import oracle
    Q, K, V = make_inputs(w)
    mask = np.zeros((w.B, w.Hq), np.uint8)
    mask.reshape(-1)[:heads] = 1
    t0 = time.perf_counter()
    if w.causal:
        oracle.muse_causal(Q, K, V, w.block, w.C, w.iters, w.cluster_seed, w.topk, w.scale, mode,
                           hq_mask=mask)
    else:
        oracle.muse_acausal(Q, K, V, w.C, w.C, w.iters, w.cluster_seed, w.topk, w.scale, mode,
                            hq_mask=mask)
    dt = time.perf_counter() - t0
    frac = heads / (w.B * w.Hq)
    G = w.Hq // w.Hkv
    kv_groups = -(-heads // G)
    threads = min(oracle.num_threads(), kv_groups)
    return dt, w.B * w.N * frac / dt, threads


def run_reference(args, w):
    mode = args.mode or w.mode
    heads = 1
    vals = []
    for i in range(args.warmup + args.steps):
        dt, tps, thr = oracle_sample(w, mode, heads)
        if i >= args.warmup:
            vals.append(dt)
    t = sum(vals)
    value = w.B * w.N * (heads / (w.B * w.Hq)) * args.steps / t
    sample = f"q-head 0 of one layer per step ({heads}/{w.B * w.Hq} heads), extrapolated by head count"
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(w, mode),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def config_of(w, mode):
    c = {"workload": w.name, "causal": w.causal, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N,
         "D": w.D, "C": w.C, "iters": w.iters, "topk": w.topk, "mode": mode,
         "input_dtype": w.dtype, "l2": "flushed: 512 MiB write between timed steps"}
    if w.causal:
        c["block"] = w.block
    return c


# Configurations timed next to the headline one in the default run (one line
# each under "workloads"): every configuration with N >= 8k.
SIDE_WORKLOADS = [("acausal-bf16-h8-n8k", "monopole"), ("causal-bf16-b2h8-n16k", None),
                  ("causal-gqa32x8-n64k-d64", None), ("causal-gqa32x8-n32k-d128", None)]


def side_entry(r, w, steps, warmup):
    return {"config": config_of(w, r["mode"]), "value": r["value"], "unit": UNIT,
            "ms_per_step": r["ms_per_step"], "steps": steps, "warmup": warmup,
            "roofline": r["roofline"], "whole_operator": r["whole_op"],
            "rse_vs_exact": r["rse"], "kernels": r["kernels"], "clocks": r["clocks"],
            "gpu_launches": r["gpu_launches"]}


def main():
    args = parse()
    w = WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    mode = args.mode or w.mode
    if args.accum:
        if rank == 0:
            print(json.dumps(run_accum_bench(w, mode, args.steps, args.warmup, device)), flush=True)
        return
    if args.backward:
        if rank == 0:
            print(json.dumps(run_backward(w, mode, args.steps, args.warmup, device)), flush=True)
        return
    r = run_muse(w, mode, args.steps, args.warmup, rank, world, device)
    line = {"metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32",
            "data": "synthetic", "config": config_of(w, r["mode"]),
            "parallelism": f"replicas x{world} (independent layers, no collective)",
            "e2e": r["e2e"], "roofline": r["roofline"], "clocks": r["clocks"],
            "gpu_launches": r["gpu_launches"], "rse_vs_exact": r["rse"], "kernels": r["kernels"],
            "whole_operator": r["whole_op"]}
    if world == 1 and not args.no_side and args.workload == DEFAULT_WORKLOAD and args.mode is None:
        side = {}
        for name, m in SIDE_WORKLOADS:
            sw = WORKLOADS[name]
            sm = m or sw.mode
            big = sw.B * sw.Hq * sw.N >= 1 << 20
            st, wu = (6, 3) if big else (args.steps, args.warmup)
            rr = run_muse(sw, sm, st, wu, rank, world, device, e2e_leg=False)
            side[f"{name}/{sm}"] = side_entry(rr, sw, st, wu)
        line["workloads"] = side
    if world == 1 and not args.no_side and args.workload == DEFAULT_WORKLOAD and args.mode is None:
        cw = WORKLOADS["causal-bf16-b2h8-n16k"]
        line["backward"] = {m: run_backward(w, m, args.steps, args.warmup, device)
                            for m in ("dipole", "monopole")}
        line["backward"]["causal-16k/dipole"] = run_backward(cw, "dipole", args.steps, args.warmup,
                                                             device)
        line["accum"] = {m: run_accum_bench(cw, m, args.steps, args.warmup, device)
                         for m in ("dipole", "monopole")}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        heads = min(w.B * w.Hq, 8)
        dt, tps, thr = oracle_sample(w, r["mode"], heads)
        line["cpu_baseline"] = {"value": tps, "unit": UNIT, "cores": thr, "kind": "oracle",
                                "sample": f"{heads} of {w.B * w.Hq} q-heads of one layer, "
                                          f"{dt:.1f} s, extrapolated by head count"}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
