"""MuSe (Multipole Semantic Attention) forward operator on B200.

A thin Python binding over the C ABI of ``libmuse.so`` (declared in
``include/muse.h``): it marshals torch tensors into device pointers and the
current CUDA stream, and nothing else -- every step of the operator runs in the
library's sm_100a kernels.  There is no CPU fallback: without the compiled
library (``python -m clustered_multipole_approximation_b200.build``) every call
raises.

Entry points (same names as the C ABI):
    muse_cluster(x, C, iters, seed, role=0, init=None)
    muse_summarize(k, v, assign, C)
    muse_attn_fwd(q, k, v, Cq=..., Ck=..., iters=..., seed=..., topk=..., ...)
    muse_attn_fwd_causal(q, k, v, C=..., block=..., iters=..., seed=..., topk=..., ...)
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmuse.so")

MODES = {"monopole": 0, "dipole": 1, "tilted": 2, "dipole_q": 3, "tilted_dipole": 4}
STATUS = {0: "MUSE_OK", 1: "MUSE_ERR_INVALID_ARG", 2: "MUSE_ERR_UNSUPPORTED",
          3: "MUSE_ERR_WORKSPACE", 4: "MUSE_ERR_CUDA", 5: "MUSE_ERR_DEVICE_CHECK"}


class MuseError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class muse_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("N", ctypes.c_int), ("D", ctypes.c_int), ("dtype", ctypes.c_int),
                ("out_f32", ctypes.c_int)]


class muse_params(ctypes.Structure):
    _fields_ = [("Cq", ctypes.c_int), ("Ck", ctypes.c_int), ("iters", ctypes.c_int),
                ("seed", ctypes.c_uint64), ("topk", ctypes.c_int), ("block", ctypes.c_int),
                ("scale", ctypes.c_float), ("mode", ctypes.c_int),
                ("key_stream0", ctypes.c_uint64), ("query_stream0", ctypes.c_uint64)]


class muse_debug(ctypes.Structure):
    _fields_ = [("q_assign", ctypes.c_void_p), ("k_assign", ctypes.c_void_p),
                ("selected", ctypes.c_void_p), ("k_counts", ctypes.c_void_p),
                ("q_centroids", ctypes.c_void_p), ("k_centroids", ctypes.c_void_p),
                ("n_exact", ctypes.c_void_p), ("device_error", ctypes.c_void_p)]


class muse_accum_debug(ctypes.Structure):
    _fields_ = [("q_assign", ctypes.c_void_p), ("k_assign", ctypes.c_void_p),
                ("sel1", ctypes.c_void_p), ("sel2", ctypes.c_void_p),
                ("n_exact", ctypes.c_void_p), ("device_error", ctypes.c_void_p)]


EXPORTS = ["muse_workspace_size", "muse_cluster_workspace_size", "muse_cluster", "muse_summarize",
           "muse_attn_fwd", "muse_attn_fwd_causal", "muse_status_string", "muse_last_error",
           "muse_profile_enable", "muse_profile_read", "muse_cluster_static",
           "muse_cluster_static_capacity", "muse_device_status", "muse_debug_inject_barrier_fault",
           "muse_attn_bwd_workspace_size", "muse_attn_bwd", "muse_accum_workspace_size",
           "muse_attn_fwd_causal_accum", "muse_attn_bwd_causal_workspace_size",
           "muse_attn_bwd_causal"]

# Bits of the device error word (include/muse.h MUSE_DEVERR_*).
DEVERR = {1: "MUSE_DEVERR_MMA_WAIT", 2: "MUSE_DEVERR_TEAM_BARRIER", 4: "MUSE_DEVERR_V_RANGE"}

_lib = None


def load_library(path: str = LIB_PATH):
    """Load libmuse.so and declare its signatures (raises if it is missing)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libmuse.so not built ({path}); run "
                          "`python -m clustered_multipole_approximation_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sz, i32, u64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_uint64
    sp, pp = ctypes.POINTER(muse_shape), ctypes.POINTER(muse_params)
    dp = ctypes.POINTER(muse_debug)
    lib.muse_workspace_size.restype = sz
    lib.muse_workspace_size.argtypes = [sp, pp, i32]
    lib.muse_cluster_workspace_size.restype = sz
    lib.muse_cluster_workspace_size.argtypes = [i32] * 5
    lib.muse_cluster.restype = i32
    lib.muse_cluster.argtypes = [vp, i32, i32, i32, i32, i32, i32, i32, u64, i32, vp, vp, vp, vp,
                                 vp, vp, sz, vp]
    lib.muse_summarize.restype = i32
    lib.muse_summarize.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp,
                                   sz, vp]
    for f in ("muse_attn_fwd", "muse_attn_fwd_causal"):
        getattr(lib, f).restype = i32
        getattr(lib, f).argtypes = [vp, vp, vp, vp, sp, pp, dp, vp, sz, vp]
    lib.muse_accum_workspace_size.restype = sz
    lib.muse_accum_workspace_size.argtypes = [sp, pp, i32]
    lib.muse_attn_fwd_causal_accum.restype = i32
    lib.muse_attn_fwd_causal_accum.argtypes = [vp, vp, vp, vp, sp, pp, i32,
                                               ctypes.POINTER(muse_accum_debug), vp, sz, vp]
    lib.muse_attn_bwd_workspace_size.restype = sz
    lib.muse_attn_bwd_workspace_size.argtypes = [sp, pp]
    lib.muse_attn_bwd.restype = i32
    lib.muse_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, sp, pp, vp, sz, vp]
    lib.muse_attn_bwd_causal_workspace_size.restype = sz
    lib.muse_attn_bwd_causal_workspace_size.argtypes = [sp, pp]
    lib.muse_attn_bwd_causal.restype = i32
    lib.muse_attn_bwd_causal.argtypes = [vp, vp, vp, vp, vp, vp, vp, sp, pp, vp, sz, vp]
    lib.muse_status_string.restype = ctypes.c_char_p
    lib.muse_status_string.argtypes = [i32]
    lib.muse_last_error.restype = ctypes.c_char_p
    lib.muse_last_error.argtypes = []
    lib.muse_cluster_static.restype = i32
    lib.muse_cluster_static.argtypes = [vp, i32, i32, i32, i32, i32, i32, i32, u64, i32, vp, vp,
                                        vp, vp, vp, vp]
    lib.muse_device_status.restype = i32
    lib.muse_device_status.argtypes = [vp, vp]
    lib.muse_debug_inject_barrier_fault.restype = None
    lib.muse_debug_inject_barrier_fault.argtypes = [i32, i32]
    lib.muse_cluster_static_capacity.restype = sz
    lib.muse_cluster_static_capacity.argtypes = []
    lib.muse_profile_enable.restype = None
    lib.muse_profile_enable.argtypes = [i32]
    lib.muse_profile_read.restype = i32
    lib.muse_profile_read.argtypes = [ctypes.c_char_p, i32, ctypes.POINTER(ctypes.c_int),
                                      ctypes.POINTER(ctypes.c_double), i32]
    if path == LIB_PATH:
        _lib = lib
    return lib


def _check(lib, st: int):
    if st != 0:
        raise MuseError(st, lib.muse_last_error().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return 0
    if t.dtype == torch.float32:
        return 1
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def make_params(Cq, Ck, iters, seed, topk, block=0, scale=1.0, mode="dipole", key_stream0=0,
                query_stream0=0) -> muse_params:
    return muse_params(int(Cq), int(Ck), int(iters), int(seed) & (2 ** 64 - 1), int(topk),
                       int(block), float(scale), MODES[mode] if isinstance(mode, str) else int(mode),
                       int(key_stream0) & (2 ** 64 - 1), int(query_stream0) & (2 ** 64 - 1))


def make_shape(q, k, out_f32: bool = False) -> muse_shape:
    B, Hq, N, D = q.shape
    return muse_shape(B, Hq, k.shape[1], N, D, _dtype_code(q), int(bool(out_f32)))


def workspace_size(q, k, params: muse_params, causal: bool) -> int:
    lib = load_library()
    sh = make_shape(q, k)
    n = lib.muse_workspace_size(ctypes.byref(sh), ctypes.byref(params), int(causal))
    if n == 0:
        raise MuseError(1, lib.muse_last_error().decode())
    return int(n)


def _debug_buffers(q, k, params, causal):
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    dev = q.device
    i32 = dict(dtype=torch.int32, device=dev)
    if causal:
        from math import log2
        nblk = N // params.block
        lv = int(round(log2(nblk))) if nblk > 1 else 0
        out = dict(q_assign=torch.empty(B, Hq, lv, N // 2, **i32),
                   k_assign=torch.empty(B, Hkv, lv, N // 2, **i32))
        if params.topk > 0 and nblk > 1:
            # one row block per block problem, problems numbered level by level
            out["selected"] = torch.empty(B, Hq, nblk - 1, params.Cq, params.topk, **i32)
    else:
        out = dict(q_assign=torch.empty(B, Hq, N, **i32), k_assign=torch.empty(B, Hkv, N, **i32),
                   k_counts=torch.empty(B, Hkv, params.Ck, **i32),
                   q_centroids=torch.empty(B, Hq, params.Cq, D, dtype=torch.float32, device=dev),
                   k_centroids=torch.empty(B, Hkv, params.Ck, D, dtype=torch.float32, device=dev))
        if params.topk > 0:
            out["selected"] = torch.empty(B, Hq, params.Cq, params.topk, **i32)
    out["n_exact"] = torch.empty(B, Hq, N, dtype=torch.int64, device=dev)
    out["device_error"] = torch.full((1,), -1, dtype=torch.int32, device=dev)
    return out


def _attn(causal, q, k, v, params, out=None, workspace=None, debug=False, stream=None,
          out_dtype=None):
    lib = load_library()
    _need_cuda(q, k, v, out, workspace)
    if k.shape != v.shape or q.dtype != k.dtype or k.dtype != v.dtype:
        raise ValueError("k and v must match in shape; q, k, v must share a dtype")
    if out is not None:
        out_dtype = out.dtype
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if out_dtype not in (q.dtype, torch.float32):
        raise ValueError("the output dtype must be the input dtype or float32")
    sh = make_shape(q, k, out_dtype == torch.float32 and q.dtype != torch.float32)
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    if workspace is None:
        workspace = torch.empty(workspace_size(q, k, params, causal), dtype=torch.uint8,
                                device=q.device)
    dbg = None
    bufs = None
    if debug:
        bufs = _debug_buffers(q, k, params, causal)
        dbg = muse_debug(*[bufs[n].data_ptr() if n in bufs else None for n, _ in muse_debug._fields_])
    f = lib.muse_attn_fwd_causal if causal else lib.muse_attn_fwd
    st = f(_ptr(q), _ptr(k), _ptr(v), _ptr(out), ctypes.byref(sh), ctypes.byref(params),
           ctypes.byref(dbg) if dbg is not None else None, _ptr(workspace),
           workspace.numel(), _stream(stream))
    _check(lib, st)
    return (out, bufs) if debug else out


def muse_attn_fwd(q, k, v, *, Cq, Ck, iters, seed, topk, scale=1.0, mode="dipole", out=None,
                  workspace=None, debug=False, stream=None, out_dtype=None, key_stream0=0,
                  query_stream0=0):
    """Acausal MuSe forward.  q [B,Hq,N,D], k and v [B,Hkv,N,D] (bf16 or fp32,
    contiguous, CUDA).  Returns O (input dtype, or fp32 with out_dtype=float32)
    and, with debug, a dict of inspection tensors.  key_stream0 /
    query_stream0: see muse_params in include/muse.h (shards of a layer)."""
    p = make_params(Cq, Ck, iters, seed, topk, 0, scale, mode, key_stream0, query_stream0)
    return _attn(False, q, k, v, p, out, workspace, debug, stream, out_dtype)


def muse_attn_fwd_causal(q, k, v, *, C, block, iters, seed, topk, scale=1.0, mode="dipole",
                         out=None, workspace=None, debug=False, stream=None, out_dtype=None,
                         key_stream0=0, query_stream0=0):
    """Causal MuSe forward (hierarchical blocks of `block` tokens, C clusters
    per level and role)."""
    p = make_params(C, C, iters, seed, topk, block, scale, mode, key_stream0, query_stream0)
    return _attn(True, q, k, v, p, out, workspace, debug, stream, out_dtype)


def accum_workspace_size(q, k, params: muse_params, topk2: int) -> int:
    """Workspace bytes of muse_attn_fwd_causal_accum."""
    lib = load_library()
    sh = make_shape(q, k)
    n = lib.muse_accum_workspace_size(ctypes.byref(sh), ctypes.byref(params), int(topk2))
    if n == 0:
        raise MuseError(3, lib.muse_last_error().decode())
    return int(n)


def muse_attn_fwd_causal_accum(q, k, v, *, Cq, Ck, block, iters, seed, topk, topk2, scale=1.0,
                               mode="dipole", out=None, workspace=None, debug=False, stream=None,
                               out_dtype=None):
    """Causal MuSe with block-summary accumulation and cluster/block retrieval
    (see muse_attn_fwd_causal_accum in include/muse.h).  Returns O and, with
    debug, a dict of inspection tensors (q_assign, k_assign, sel1, sel2,
    n_exact, device_error)."""
    lib = load_library()
    _need_cuda(q, k, v, out, workspace)
    if k.shape != v.shape or q.dtype != k.dtype or k.dtype != v.dtype:
        raise ValueError("k and v must match in shape; q, k, v must share a dtype")
    if out is not None:
        out_dtype = out.dtype
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if out_dtype not in (q.dtype, torch.float32):
        raise ValueError("the output dtype must be the input dtype or float32")
    p = make_params(Cq, Ck, iters, seed, topk, block, scale, mode)
    sh = make_shape(q, k, out_dtype == torch.float32 and q.dtype != torch.float32)
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    if workspace is None:
        workspace = torch.empty(accum_workspace_size(q, k, p, topk2), dtype=torch.uint8,
                                device=q.device)
    bufs = dbg = None
    if debug:
        B, Hq, N, D = q.shape
        NB = N // block
        i32 = dict(dtype=torch.int32, device=q.device)
        bufs = dict(q_assign=torch.empty(B, Hq, N, **i32),
                    k_assign=torch.empty(B, k.shape[1], N, **i32),
                    sel1=torch.full((B, Hq, NB, Cq, topk), -1, **i32),
                    sel2=torch.full((B, Hq, NB, Cq, topk, topk2), -1, **i32),
                    n_exact=torch.empty(B, Hq, N, dtype=torch.int64, device=q.device),
                    device_error=torch.full((1,), -1, **i32))
        dbg = muse_accum_debug(*[bufs[n].data_ptr() for n, _ in muse_accum_debug._fields_])
    st = lib.muse_attn_fwd_causal_accum(_ptr(q), _ptr(k), _ptr(v), _ptr(out), ctypes.byref(sh),
                                        ctypes.byref(p), int(topk2),
                                        ctypes.byref(dbg) if dbg is not None else None,
                                        _ptr(workspace), workspace.numel(), _stream(stream))
    _check(lib, st)
    return (out, bufs) if debug else out


def backward_workspace_size(q, k, params: muse_params, out_f32: bool = False,
                            causal: bool = False) -> int:
    """Workspace bytes for a forward call followed by its backward call
    (muse_attn_fwd + muse_attn_bwd, or the causal pair)."""
    lib = load_library()
    sh = make_shape(q, k, out_f32)
    f = lib.muse_attn_bwd_causal_workspace_size if causal else lib.muse_attn_bwd_workspace_size
    n = f(ctypes.byref(sh), ctypes.byref(params))
    if n == 0:
        raise MuseError(3, lib.muse_last_error().decode())
    return int(n)


def muse_attn_bwd(q, k, v, do, *, Cq, Ck, iters, seed, topk, scale=1.0, mode="dipole",
                  workspace, stream=None, key_stream0=0, query_stream0=0):
    """Gradients (dq, dk, dv) in fp32 of <do, O> for the acausal forward call
    made with this `workspace` (sized by backward_workspace_size) and these
    parameters; see muse_attn_bwd in include/muse.h."""
    lib = load_library()
    _need_cuda(q, k, v, do, workspace)
    if do.shape != q.shape or do.dtype not in (q.dtype, torch.float32):
        raise ValueError("do must be [B,Hq,N,D] in the input dtype or float32")
    p = make_params(Cq, Ck, iters, seed, topk, 0, scale, mode, key_stream0, query_stream0)
    sh = make_shape(q, k, do.dtype == torch.float32 and q.dtype != torch.float32)
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
    st = lib.muse_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                           ctypes.byref(sh), ctypes.byref(p), _ptr(workspace),
                           workspace.numel(), _stream(stream))
    _check(lib, st)
    return dq, dk, dv


def muse_attn_bwd_causal(q, k, v, do, *, C, block, iters, seed, topk, scale=1.0, mode="dipole",
                         workspace, stream=None, key_stream0=0, query_stream0=0):
    """Gradients (dq, dk, dv) in fp32 of <do, O> for the causal forward call
    made with this `workspace` (sized by backward_workspace_size(...,
    causal=True)) and these parameters; see muse_attn_bwd_causal in
    include/muse.h."""
    lib = load_library()
    _need_cuda(q, k, v, do, workspace)
    if do.shape != q.shape or do.dtype not in (q.dtype, torch.float32):
        raise ValueError("do must be [B,Hq,N,D] in the input dtype or float32")
    p = make_params(C, C, iters, seed, topk, block, scale, mode, key_stream0, query_stream0)
    sh = make_shape(q, k, do.dtype == torch.float32 and q.dtype != torch.float32)
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
    st = lib.muse_attn_bwd_causal(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk),
                                  _ptr(dv), ctypes.byref(sh), ctypes.byref(p), _ptr(workspace),
                                  workspace.numel(), _stream(stream))
    _check(lib, st)
    return dq, dk, dv


class MuseAttention(torch.autograd.Function):
    """Acausal MuSe as a differentiable op: forward and backward both run in
    libmuse (the forward's workspace is kept for the backward)."""

    @staticmethod
    def forward(ctx, q, k, v, Cq, Ck, iters, seed, topk, scale, mode):
        p = make_params(Cq, Ck, iters, seed, topk, 0, scale, mode)
        ws = torch.empty(backward_workspace_size(q, k, p), dtype=torch.uint8, device=q.device)
        o = _attn(False, q, k, v, p, None, ws, False, None, None)
        ctx.save_for_backward(q, k, v, ws)
        ctx.args = dict(Cq=Cq, Ck=Ck, iters=iters, seed=seed, topk=topk, scale=scale, mode=mode)
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, ws = ctx.saved_tensors
        dq, dk, dv = muse_attn_bwd(q, k, v, do.contiguous().to(q.dtype), workspace=ws,
                                   **ctx.args)
        return (dq.to(q.dtype), dk.to(k.dtype), dv.to(v.dtype)) + (None,) * 7


def muse_attention(q, k, v, *, Cq, Ck, iters, seed, topk, scale=1.0, mode="dipole"):
    """Differentiable acausal MuSe (see MuseAttention)."""
    return MuseAttention.apply(q, k, v, Cq, Ck, iters, seed, topk, scale, mode)


def device_status(device_error, stream=None) -> None:
    """Wait for the stream, read a device error word (an int32 CUDA tensor
    written by an entry point) and raise MuseError(MUSE_ERR_DEVICE_CHECK)
    naming its MUSE_DEVERR_* bits if it is not 0."""
    lib = load_library()
    _need_cuda(device_error)
    _check(lib, lib.muse_device_status(_ptr(device_error), _stream(stream)))


def muse_cluster(x, C, iters, seed, role=0, init=None, workspace=None, stream=None,
                 device_error=None):
    """Lloyd k-means of each (b, h) row set of x [B,H,N,D].  Returns
    (assign [B,H,N] int32, centroids [B,H,C,D] fp32, counts [B,H,C] int32).
    `device_error` (optional int32 CUDA tensor of one element) receives the
    device error word."""
    lib = load_library()
    _need_cuda(x, init, workspace, device_error)
    B, H, N, D = x.shape
    if init is not None and (init.dtype != torch.float32 or tuple(init.shape) != (B, H, C, D)):
        raise ValueError("init must be fp32 [B,H,C,D]")
    if workspace is None:
        n = lib.muse_cluster_workspace_size(B, H, N, D, C)
        if n == 0:
            raise MuseError(1, "invalid sizes")
        workspace = torch.empty(n, dtype=torch.uint8, device=x.device)
    assign = torch.empty(B, H, N, dtype=torch.int32, device=x.device)
    cent = torch.empty(B, H, C, D, dtype=torch.float32, device=x.device)
    counts = torch.empty(B, H, C, dtype=torch.int32, device=x.device)
    st = lib.muse_cluster(_ptr(x), _dtype_code(x), B, H, N, D, C, iters, int(seed) & (2 ** 64 - 1),
                          role, _ptr(init), _ptr(assign), _ptr(cent), _ptr(counts),
                          _ptr(device_error), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(lib, st)
    return assign, cent, counts


def muse_cluster_static(x, C, iters, seed, role=0, init=None, stream=None, device_error=None):
    """muse_cluster for callers that cannot allocate a workspace: the scratch
    is the fixed array built into the library (see include/muse.h for its
    limit and its sharing rules).  Returns (assign, centroids, counts)."""
    lib = load_library()
    _need_cuda(x, init, device_error)
    B, H, N, D = x.shape
    assign = torch.empty(B, H, N, dtype=torch.int32, device=x.device)
    cent = torch.empty(B, H, C, D, dtype=torch.float32, device=x.device)
    counts = torch.empty(B, H, C, dtype=torch.int32, device=x.device)
    st = lib.muse_cluster_static(_ptr(x), _dtype_code(x), B, H, N, D, C, iters,
                                 int(seed) & (2 ** 64 - 1), role, _ptr(init), _ptr(assign),
                                 _ptr(cent), _ptr(counts), _ptr(device_error), _stream(stream))
    _check(lib, st)
    return assign, cent, counts


def inject_barrier_fault(rank: int, spin_limit: int = 0) -> None:
    """Failure-path testing: see muse_debug_inject_barrier_fault in
    include/muse.h (rank < 0 switches it off)."""
    load_library().muse_debug_inject_barrier_fault(int(rank), int(spin_limit))


def muse_summarize(k, v, assign, C, with_dipole=True, stream=None):
    """Key-cluster summaries of a given assignment: (counts, mu, S, M)."""
    lib = load_library()
    _need_cuda(k, v, assign)
    B, H, N, D = k.shape
    dev = k.device
    counts = torch.empty(B, H, C, dtype=torch.int32, device=dev)
    mu = torch.empty(B, H, C, D, dtype=torch.float32, device=dev)
    S = torch.empty(B, H, C, D, dtype=torch.float32, device=dev)
    M = torch.empty(B, H, C, D, D, dtype=torch.float32, device=dev) if with_dipole else None
    st = lib.muse_summarize(_ptr(k), _ptr(v), _dtype_code(k), B, H, N, D, C, _ptr(assign),
                            _ptr(counts), _ptr(mu), _ptr(S), _ptr(M), None, 0, _stream(stream))
    _check(lib, st)
    return counts, mu, S, M


def profile_enable(on: bool = True) -> None:
    """Bracket every library kernel launch with CUDA events (benchmarks)."""
    load_library().muse_profile_enable(int(bool(on)))


def profile_read() -> dict:
    """{kernel name: (launches, total ms)} since the last read; clears it."""
    lib = load_library()
    cap, stride = 64, 64
    names = ctypes.create_string_buffer(cap * stride)
    launches = (ctypes.c_int * cap)()
    ms = (ctypes.c_double * cap)()
    n = lib.muse_profile_read(names, stride, launches, ms, cap)
    out = {}
    for i in range(min(n, cap)):
        nm = names.raw[i * stride:(i + 1) * stride].split(b"\0", 1)[0].decode()
        out[nm] = (int(launches[i]), float(ms[i]))
    return out
