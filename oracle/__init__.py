"""fp64 CPU oracle for the MuSe forward operator -- TEST INFRASTRUCTURE ONLY.

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never links, loads or
calls it, and it never calls the CUDA library.  It is a ctypes wrapper around
``muse_oracle.c`` (plain C, fp64), which states the method as the pages of
"Multipole Semantic Attention: A Fast Approximation of Softmax Attention for
Pretraining" describe it; see the header of that file for the sources and the
readings taken where the pages are silent.

All arrays here are float64 numpy arrays in the layouts of the C file:
Q [B,Hq,N,D], K and V [B,Hkv,N,D].
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "muse_oracle.c")
_SO = os.path.join(_HERE, "libmuse_oracle.so")

MODES = {"monopole": 0, "dipole": 1, "tilted": 2, "dipole_q": 3, "tilted_dipole": 4}


def build(force: bool = False) -> str:
    """Compile muse_oracle.c into libmuse_oracle.so (gcc, fp64, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)
_u8p = ctypes.POINTER(ctypes.c_ubyte)
_llp = ctypes.POINTER(ctypes.c_longlong)
_u64p = ctypes.POINTER(ctypes.c_uint64)


def _bind(lib):
    lib.orc_splitmix64_next.restype = ctypes.c_uint64
    lib.orc_splitmix64_next.argtypes = [_u64p]
    lib.orc_stream_state.restype = ctypes.c_uint64
    lib.orc_stream_state.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int]
    lib.orc_init_indices.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                                     ctypes.c_uint64, ctypes.c_int, _ip]
    lib.orc_kmeans_assign.restype = ctypes.c_double
    lib.orc_kmeans_assign.argtypes = [_dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _ip]
    lib.orc_kmeans_update.argtypes = [_dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _ip, _dp, _ip]
    lib.orc_kmeans.argtypes = [_dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                               ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int, _dp, _ip, _dp,
                               _ip, _dp]
    lib.orc_summaries.argtypes = [_dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _ip,
                                  _dp, _dp, _dp]
    lib.orc_muse_acausal.argtypes = [_dp, _dp, _dp] + [ctypes.c_int] * 8 + [
        ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int, ctypes.c_double,
        ctypes.c_int, _u8p, _ip, _ip, _dp, _ip, _ip, _dp, _dp, _ip, _ip, _llp]
    lib.orc_muse_causal.argtypes = [_dp, _dp, _dp] + [ctypes.c_int] * 8 + [
        ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int, ctypes.c_double,
        ctypes.c_int, _u8p, _ip, _ip, _dp, _ip, _ip, _ip, _llp]
    lib.orc_exact_attn.argtypes = [_dp, _dp, _dp] + [ctypes.c_int] * 5 + [
        ctypes.c_double, ctypes.c_int, _u8p, _dp]
    lib.orc_exact_attn_rows.argtypes = [_dp, _dp, _dp] + [ctypes.c_int] * 5 + [
        ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int, _ip, _dp]
    lib.orc_stage1_debug.argtypes = [_dp, _dp, _dp] + [ctypes.c_int] * 4 + [
        _ip, _ip, ctypes.c_int, ctypes.c_double, ctypes.c_int, _dp, _dp, _ip]
    lib.orc_num_threads.restype = ctypes.c_int
    return lib


def _d(a):
    """Contiguous float64 view/copy and its pointer."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(_dp)


def _i(a):
    a = np.ascontiguousarray(a, dtype=np.int32)
    return a, a.ctypes.data_as(_ip)


def _opt(a, kind):
    if a is None:
        return None, None
    if kind == "d":
        return _d(a)
    if kind == "i":
        return _i(a)
    a = np.ascontiguousarray(a, dtype=np.uint8)
    return a, a.ctypes.data_as(_u8p)


class Oracle:
    """The oracle functions bound to one compiled copy of muse_oracle.c
    (the default copy, or a deliberately altered one in the oracle's own
    mutation tests)."""

    def __init__(self, so_path: str):
        self.lib = _bind(ctypes.CDLL(so_path))

    def num_threads(self) -> int:
        return int(self.lib.orc_num_threads())

    def splitmix64(self, state: int, count: int) -> list[int]:
        """`count` successive outputs of splitmix64 started from `state`."""
        st = ctypes.c_uint64(state)
        lib = self.lib
        return [int(lib.orc_splitmix64_next(ctypes.byref(st))) for _ in range(count)]

    def stream_state(self, seed: int, sid: int, role: int) -> int:
        return int(self.lib.orc_stream_state(seed, sid, role))

    def init_indices(self, n: int, C: int, seed: int, sid: int, role: int) -> np.ndarray:
        out = np.zeros(C, dtype=np.int32)
        self.lib.orc_init_indices(n, C, seed, sid, role, out.ctypes.data_as(_ip))
        return out

    def kmeans_assign(self, X, cent):
        X, xp = _d(X)
        cent, cp = _d(cent)
        n, D = X.shape
        a = np.zeros(n, dtype=np.int32)
        inertia = self.lib.orc_kmeans_assign(xp, n, D, cent.shape[0], cp, a.ctypes.data_as(_ip))
        return a, float(inertia)

    def kmeans_update(self, X, assign, cent):
        """One update step from the given assignment; `cent` supplies the centroids
        that empty clusters keep."""
        X, xp = _d(X)
        assign, ap = _i(assign)
        cent = np.array(cent, dtype=np.float64, copy=True)
        counts = np.zeros(cent.shape[0], dtype=np.int32)
        self.lib.orc_kmeans_update(xp, X.shape[0], X.shape[1], cent.shape[0], ap,
                                  cent.ctypes.data_as(_dp), counts.ctypes.data_as(_ip))
        return cent, counts

    def kmeans(self, X, C, iters, seed=0, sid=0, role=0, init=None):
        """Lloyd k-means; returns (assign, centroids, counts, inertia per assign step)."""
        X, xp = _d(X)
        n, D = X.shape
        init_a, init_p = _opt(init, "d")
        a = np.zeros(n, dtype=np.int32)
        cent = np.zeros((C, D))
        counts = np.zeros(C, dtype=np.int32)
        inertia = np.zeros(max(iters, 1))
        self.lib.orc_kmeans(xp, n, D, C, iters, seed, sid, role, init_p, a.ctypes.data_as(_ip),
                           cent.ctypes.data_as(_dp), counts.ctypes.data_as(_ip),
                           inertia.ctypes.data_as(_dp))
        return a, cent, counts, inertia[:iters]

    def summaries(self, K, V, C, assign, mu, with_dipole=True):
        """Monopole sums S [C,D] and dipole moments M [C,D,D] (M[j,e,d])."""
        K, kp = _d(K)
        V, vp = _d(V)
        assign, ap = _i(assign)
        mu, mp = _d(mu)
        n, D = K.shape
        S = np.zeros((C, D))
        M = np.zeros((C, D, D)) if with_dipole else None
        self.lib.orc_summaries(kp, vp, n, D, C, ap, mp, S.ctypes.data_as(_dp),
                              M.ctypes.data_as(_dp) if M is not None else None)
        return S, M

    def muse_acausal(self, Q, K, V, Cq, Ck, iters, seed, topk, scale=1.0, mode="dipole",
                     hq_mask=None, q_assign_in=None, k_assign_in=None, key_stream0=0,
                     query_stream0=0):
        """Acausal MuSe in fp64.  Returns a dict with O, the clusterings, the
        selections R and the number of exactly-attended keys per query."""
        Q, qp = _d(Q)
        K, kp = _d(K)
        V, vp = _d(V)
        B, Hq, N, D = Q.shape
        Hkv = K.shape[1]
        m_a, m_p = _opt(hq_mask, "u8")
        qa_a, qa_p = _opt(q_assign_in, "i")
        ka_a, ka_p = _opt(k_assign_in, "i")
        O = np.zeros_like(Q)
        q_assign = np.zeros((B, Hq, N), dtype=np.int32)
        k_assign = np.zeros((B, Hkv, N), dtype=np.int32)
        q_cent = np.zeros((B, Hq, Cq, D))
        k_cent = np.zeros((B, Hkv, Ck, D))
        k_count = np.zeros((B, Hkv, Ck), dtype=np.int32)
        selected = np.full((B, Hq, Cq, max(topk, 1)), -1, dtype=np.int32)
        n_exact = np.zeros((B, Hq, N), dtype=np.int64)
        self.lib.orc_muse_acausal(
            qp, kp, vp, B, Hq, Hkv, N, D, Cq, Ck, iters, seed, key_stream0, query_stream0, topk,
            float(scale), MODES[mode],
            m_p, qa_p, ka_p, O.ctypes.data_as(_dp), q_assign.ctypes.data_as(_ip),
            k_assign.ctypes.data_as(_ip), q_cent.ctypes.data_as(_dp), k_cent.ctypes.data_as(_dp),
            k_count.ctypes.data_as(_ip), selected.ctypes.data_as(_ip) if topk > 0 else None,
            n_exact.ctypes.data_as(_llp))
        return dict(O=O, q_assign=q_assign, k_assign=k_assign, q_cent=q_cent, k_cent=k_cent,
                    k_count=k_count, selected=selected[..., :topk], n_exact=n_exact)


    def muse_causal(self, Q, K, V, L, C, iters, seed, topk, scale=1.0, mode="dipole", hq_mask=None,
                    q_assign_in=None, k_assign_in=None, key_stream0=0, query_stream0=0):
        """Causal MuSe (hierarchical blocks) in fp64.  Assignment layouts are
        [B,H,levels,N/2] (see the C file)."""
        Q, qp = _d(Q)
        K, kp = _d(K)
        V, vp = _d(V)
        B, Hq, N, D = Q.shape
        Hkv = K.shape[1]
        lv = causal_levels(N, L)
        m_a, m_p = _opt(hq_mask, "u8")
        qa_a, qa_p = _opt(q_assign_in, "i")
        ka_a, ka_p = _opt(k_assign_in, "i")
        O = np.zeros_like(Q)
        q_assign = np.zeros((B, Hq, lv, N // 2), dtype=np.int32)
        k_assign = np.zeros((B, Hkv, lv, N // 2), dtype=np.int32)
        n_exact = np.zeros((B, Hq, N), dtype=np.int64)
        nprob = max(N // L - 1, 1)
        selected = np.full((B, Hq, nprob, C, max(topk, 1)), -1, dtype=np.int32)
        self.lib.orc_muse_causal(
            qp, kp, vp, B, Hq, Hkv, N, D, L, C, iters, seed, key_stream0, query_stream0, topk,
            float(scale), MODES[mode],
            m_p, qa_p, ka_p, O.ctypes.data_as(_dp), q_assign.ctypes.data_as(_ip),
            k_assign.ctypes.data_as(_ip),
            selected.ctypes.data_as(_ip) if topk > 0 and N // L > 1 else None,
            n_exact.ctypes.data_as(_llp))
        out = dict(O=O, q_assign=q_assign, k_assign=k_assign, n_exact=n_exact)
        if topk > 0 and N // L > 1:
            out["selected"] = selected[..., :topk]
        return out

    def exact_attention(self, Q, K, V, scale=1.0, causal=False, hq_mask=None):
        """Plain softmax attention in fp64 (GQA by kv-head = q-head / group)."""
        Q, qp = _d(Q)
        K, kp = _d(K)
        V, vp = _d(V)
        B, Hq, N, D = Q.shape
        m_a, m_p = _opt(hq_mask, "u8")
        E = np.zeros_like(Q)
        self.lib.orc_exact_attn(qp, kp, vp, B, Hq, K.shape[1], N, D, float(scale), int(causal), m_p,
                               E.ctypes.data_as(_dp))
        return E

    def exact_attention_rows(self, Q, K, V, b, hq, rows, scale=1.0, causal=False):
        """Exact attention of the given query rows of (b, q-head hq) only:
        [len(rows), D] (the same arithmetic as exact_attention, row by row)."""
        Q, qp = _d(Q)
        K, kp = _d(K)
        V, vp = _d(V)
        B, Hq, N, D = Q.shape
        rows, rp = _i(rows)
        E = np.zeros((len(rows), D))
        self.lib.orc_exact_attn_rows(qp, kp, vp, B, Hq, K.shape[1], N, D, float(scale),
                                     int(causal), b * Hq + hq, len(rows), rp,
                                     E.ctypes.data_as(_dp))
        return E

    def stage1_debug(self, Qh, Kh, Vh, Cq, Ck, q_assign, k_assign, topk, scale=1.0, mode="dipole"):
        """Stage-1 tables of one acausal (b, q-head) problem for given clusterings:
        (log W [Cq,Ck], U [Cq,Ck,D], R [Cq,topk])."""
        Qh, qp = _d(Qh)
        Kh, kp = _d(Kh)
        Vh, vp = _d(Vh)
        N, D = Qh.shape
        qa, qap = _i(q_assign)
        ka, kap = _i(k_assign)
        logW = np.zeros((Cq, Ck))
        U = np.zeros((Cq, Ck, D))
        R = np.full((Cq, max(topk, 1)), -1, dtype=np.int32)
        self.lib.orc_stage1_debug(qp, kp, vp, N, D, Cq, Ck, qap, kap, topk, float(scale), MODES[mode],
                                 logW.ctypes.data_as(_dp), U.ctypes.data_as(_dp),
                                 R.ctypes.data_as(_ip) if topk > 0 else None)
        return logW, U, R[:, :topk]


def causal_levels(N: int, L: int) -> int:
    """Number of levels of the hierarchical decomposition: log2(N / L)."""
    nblk = N // L
    lv = 0
    while (1 << lv) < nblk:
        lv += 1
    return lv


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def __getattr__(name):
    # module-level access to the default oracle's methods: oracle.kmeans(...)
    if name.startswith("_"):
        raise AttributeError(name)
    return getattr(default(), name)


def rse(O, E) -> float:
    """Relative squared error sum ||O-E||^2 / sum ||E||^2 (global Frobenius)."""
    O = np.asarray(O, dtype=np.float64)
    E = np.asarray(E, dtype=np.float64)
    return float(((O - E) ** 2).sum() / (E ** 2).sum())
