"""Seeded synthetic inputs for the MuSe forward operator.

This module only draws random numbers: it holds none of the method's
arithmetic, and both the CUDA path and the fp64 oracle read the same bytes it
produces.  The pages measure on trained-model activations (code and science
corpora, Llama layers), which are not available here; clustered Gaussian
mixtures with the pages' layer shapes stand in for them.

Recipe (per (batch, kv-head) a set of `centres` Gaussian centres c_m ~ N(0, I)
shared by the keys of that kv-head and the queries of its q-heads; each token
draws its own component label uniformly, independently for q and k, so token
order carries no cluster information):

    x = r * (c_z + noise * eps) * D**-0.25,   eps ~ N(0, I),
    r = exp(lognormal * N(0, 1)) per token (r = 1 when lognormal = 0),
    v ~ N(0, I).

Scaling q and k by D**-0.25 each splits the usual 1/sqrt(D) softmax scale
between them, so the operator runs with scale = 1.  bf16 inputs are the fp32
draws rounded to nearest-even.
"""
from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    causal: bool
    B: int
    Hq: int
    Hkv: int
    N: int
    D: int
    dtype: str          # "f32" or "bf16"
    C: int              # query and key clusters (per level when causal)
    iters: int
    topk: int
    block: int          # local block L (causal only, else 0)
    centres: int
    noise: float
    lognormal: float
    mode: str = "dipole"
    scale: float = 1.0
    seed_index: int = 0

    @property
    def data_seed(self) -> int:
        return 0x5EED0000 + self.seed_index

    @property
    def cluster_seed(self) -> int:
        return 0xC0FFEE + self.seed_index

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads the operator is specified on.
WORKLOADS = {
    "acausal-f32-n1k": Workload("acausal-f32-n1k", False, 1, 1, 1, 1024, 64, "f32", 16, 10, 2,
                                0, 16, 0.3, 0.0, seed_index=1),
    "acausal-bf16-h8-n8k": Workload("acausal-bf16-h8-n8k", False, 1, 8, 8, 8192, 64, "bf16", 128,
                                    8, 8, 0, 64, 0.3, 0.0, seed_index=2),
    "causal-bf16-b2h8-n16k": Workload("causal-bf16-b2h8-n16k", True, 2, 8, 8, 16384, 64, "bf16",
                                      64, 8, 0, 512, 64, 0.3, 0.0, seed_index=3),
    "causal-gqa32x8-n64k-d64": Workload("causal-gqa32x8-n64k-d64", True, 1, 32, 8, 65536, 64,
                                        "bf16", 256, 8, 16, 1024, 256, 0.25, 0.0, seed_index=4),
    "causal-gqa32x8-n32k-d128": Workload("causal-gqa32x8-n32k-d128", True, 1, 32, 8, 32768, 128,
                                         "bf16", 256, 8, 16, 1024, 256, 0.25, 0.5, seed_index=5),
}
WORKLOAD_ORDER = list(WORKLOADS)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + r) & np.uint32(0xFFFF0000)).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The uint16 bit patterns of bf16-representable float32 values."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def clustered_qkv(B, Hq, Hkv, N, D, centres, noise, lognormal, dtype, seed):
    """Q [B,Hq,N,D], K and V [B,Hkv,N,D] as float32 arrays (bf16-representable
    when dtype == "bf16")."""
    rng = np.random.Generator(np.random.PCG64(seed))
    G = Hq // Hkv
    sc = np.float32(D ** -0.25)
    Q = np.empty((B, Hq, N, D), dtype=np.float32)
    K = np.empty((B, Hkv, N, D), dtype=np.float32)
    V = np.empty((B, Hkv, N, D), dtype=np.float32)

    def draw(cent):
        z = rng.integers(0, centres, size=N)
        x = cent[z] + np.float32(noise) * rng.standard_normal((N, D), dtype=np.float32)
        if lognormal > 0:
            r = np.exp(np.float32(lognormal) * rng.standard_normal(N, dtype=np.float32))
            x *= r[:, None]
        return x * sc

    for b in range(B):
        for h in range(Hkv):
            cent = rng.standard_normal((centres, D), dtype=np.float32)
            K[b, h] = draw(cent)
            for g in range(G):
                Q[b, h * G + g] = draw(cent)
            V[b, h] = rng.standard_normal((N, D), dtype=np.float32)
    if dtype == "bf16":
        Q, K, V = round_bf16(Q), round_bf16(K), round_bf16(V)
    return Q, K, V


def make_inputs(w: Workload, seed: int | None = None):
    """The seeded inputs of a workload: (Q, K, V) float32 numpy arrays."""
    return clustered_qkv(w.B, w.Hq, w.Hkv, w.N, w.D, w.centres, w.noise, w.lognormal, w.dtype,
                         w.data_seed if seed is None else seed)
