#!/usr/bin/env python
"""Benchmark of the MuSe forward operator; rank 0 prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl muse|reference]
                    [--workload NAME] [--mode dipole|monopole|tilted]

A step is one full forward call of the operator (k-means of queries and keys,
summaries, selection, far field + exact retrieval) over one layer of synthetic
clustered inputs already resident in HBM.  Between timed steps the L2 cache is
flushed by writing a 512 MiB buffer; only the operator's own interval is
timed (CUDA events on the launching stream).  With N > 1 (torchrun) every rank
runs its own layer (weak scaling, no collective on the data path) and the time
is the max over ranks.

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
    p.add_argument("--mode", default=None, choices=[None, "dipole", "monopole", "tilted"])
    p.add_argument("--no-cpu-baseline", action="store_true")
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
# algorithmic work per kernel launch (what the method must compute)
# ---------------------------------------------------------------------------
# DRAM bytes (read + write) of one launch of a kernel on a workload, from one ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum, caches flushed as in the
# timed region).  An entry is removed whenever its kernel changes.
NCU_TRAFFIC = {
    ("acausal-bf16-h8-n8k", "kmeans_fused"): 18_488_064 + 3_584,
}


def algorithmic_work(w, mode, dbg):
    """Per-launch algorithmic FLOPs and bytes of the acausal kernels, from the
    shapes and the actual retrieval counts.  A multiply-add counts 2 FLOPs."""
    B, Hq, Hkv, N, D, C = w.B, w.Hq, w.Hkv, w.N, w.D, w.C
    G = Hq // Hkv
    elt = 2 if w.dtype == "bf16" else 4
    roles = [B * Hkv, B * Hq]
    work = {}
    # one assign launch per role and round: distances of every token to C centroids
    work["kmeans_assign"] = dict(
        flops=sum(2.0 * N * C * D * r for r in roles) / 2,
        bytes=sum(N * D * elt * r + N * 4 * r for r in roles) / 2)
    work["kmeans_reduce"] = dict(flops=sum(N * D * r for r in roles) / 2,
                                 bytes=sum(N * D * elt * r for r in roles) / 2)
    # the persistent k-means: every round of both clusterings in one launch
    work["kmeans_fused"] = dict(flops=w.iters * sum(2.0 * N * C * D * r for r in roles),
                                bytes=w.iters * sum(N * D * elt * r for r in roles))
    # stage 1: the dipole contraction sum_t v_t (1 + s nu_i.k~_t) for every (i, t)
    s1 = 0.0 if mode == "monopole" else 4.0 * N * D * C * B * Hq
    work["stage1_summaries"] = dict(flops=s1, bytes=B * Hq * C * C * D * 4.0)
    # stage 2: QK^T and PV for every far-field cluster and every retrieved key
    k_counts = dbg["k_counts"]
    q_assign = dbg["q_assign"]
    sel = dbg.get("selected")
    far_rows = 0.0
    for b in range(B):
        for h in range(Hq):
            nonempty = int((k_counts[b, h // G] > 0).sum())
            nq = np.bincount(q_assign[b, h], minlength=C)
            nsel = (sel[b, h] >= 0).sum(-1) if sel is not None else np.zeros(C)
            far_rows += float((nq * (nonempty - nsel)).sum())
    exact = float(np.asarray(dbg["n_exact"], dtype=np.float64).sum())
    work["stage2_attn"] = dict(flops=4.0 * D * (far_rows + exact),
                               bytes=2.0 * B * Hq * N * D * elt + B * Hq * C * C * D * 4.0)
    return work


def total_algorithmic_flops(work, iters):
    return (work["kmeans_fused"]["flops"] + work["stage1_summaries"]["flops"]
            + work["stage2_attn"]["flops"])


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
def run_muse(args, w, rank, world, device):
    import clustered_multipole_approximation_b200 as muse

    mode = args.mode or w.mode
    Q, K, V = make_inputs(w, seed=rank_data_seed(w, rank))
    cast = (lambda x: torch.from_numpy(x).to(torch.bfloat16)) if w.dtype == "bf16" else torch.from_numpy
    hq, hk, hv = cast(Q).pin_memory(), cast(K).pin_memory(), cast(V).pin_memory()
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
    _, dbg = fn(q, k, v, debug=True, **kw)
    o_chk = fn(q, k, v, **kw)
    qq = q.float()
    G = w.Hq // w.Hkv
    kk = k.float().repeat_interleave(G, dim=1)
    vv = v.float().repeat_interleave(G, dim=1)
    E = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, is_causal=w.causal,
                                                         scale=w.scale)
    rse_val = float(((o_chk.float() - E) ** 2).sum() / (E ** 2).sum())
    del E, kk, vv, qq
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clk = Clocks(device.index if device.index is not None else 0)
    clk.start()
    muse.profile_enable(True)
    evs = []
    for _ in range(args.steps):
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
    value = whole_job_throughput(tokens, world, args.steps, total_ms)
    ms_per_step = total_ms / args.steps

    # end to end through the public API: host inputs in, host output back
    ho = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    e2e_ms = 0.0
    for i in range(args.warmup + args.steps):
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
        if i >= args.warmup:
            e2e_ms += e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, world, device)
    e2e = {"value": whole_job_throughput(tokens, world, args.steps, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": int(hq.numel() * hq.element_size() * 1 + hk.numel() * hk.element_size()
                                     + hv.numel() * hv.element_size()),
           "d2h_bytes_per_step": int(ho.numel() * ho.element_size())}

    # roofline of the dominant kernel
    pk, how = peaks()
    launches = sum(n for n, _ in prof.values())
    dom = max(prof, key=lambda n: prof[n][1])
    dom_launches, dom_ms = prof[dom]
    avg_ms = dom_ms / dom_launches
    roofline = {"kernel": dom, "bound": "tensor", "achieved": None,
                "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": None,
                "traffic": NCU_TRAFFIC.get((w.name, dom)),
                "peak_source": f"{how} bf16 dense (burst)", "avg_launch_ms": avg_ms}
    if not w.causal:
        work = algorithmic_work(w, mode, {n: t.cpu().numpy() for n, t in dbg.items()})
        if dom in work:
            ach = work[dom]["flops"] / (avg_ms / 1e3) / 1e12
            roofline.update(achieved=ach, frac=ach / pk["bf16_tflops"],
                            frac_of_sustained_peak=ach / pk["bf16_tflops_sustained"],
                            flops_per_launch=work[dom]["flops"])
        f_alg = total_algorithmic_flops(work, w.iters)
        whole = {"algorithmic_tflop": f_alg / 1e12,
                 "achieved_tflops": f_alg / (ms_per_step / 1e3) / 1e12,
                 "frac_of_bf16_peak": f_alg / (ms_per_step / 1e3) / 1e12 / pk["bf16_tflops"],
                 "frac_of_bf16_sustained_peak":
                     f_alg / (ms_per_step / 1e3) / 1e12 / pk["bf16_tflops_sustained"]}
    else:
        whole = None
    kernels = {n: {"launches": c, "ms_total": round(t, 4), "share": round(t / sum(x[1] for x in prof.values()), 4)}
               for n, (c, t) in sorted(prof.items(), key=lambda kv: -kv[1][1])}
    return dict(value=value, ms_per_step=ms_per_step, e2e=e2e, roofline=roofline, clocks=clocks,
                gpu_launches=launches, kernels=kernels, rse=rse_val, mode=mode, whole_op=whole)


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
    r = run_muse(args, w, rank, world, device)
    line = {"metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32",
            "data": "synthetic", "config": config_of(w, r["mode"]),
            "parallelism": f"replicas x{world} (independent layers, no collective)",
            "e2e": r["e2e"], "roofline": r["roofline"], "clocks": r["clocks"],
            "gpu_launches": r["gpu_launches"], "rse_vs_exact": r["rse"], "kernels": r["kernels"],
            "whole_operator": r["whole_op"]}
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
