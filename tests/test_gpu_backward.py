"""Parity of the CUDA backward pass (muse_attn_bwd, through the C ABI) with the
fp64 gradient oracle (oracle/muse_backward.py).

The oracle is given the GPU forward's clusterings and selections (the forward
parity tests show those equal to the oracle's own), so both sides
differentiate the same function.  Tolerance: the kernels work in fp32 (fp32
sums of at most a few thousand terms, fast exp/log intrinsics of a few ulp), so
every gradient element must lie within 2e-4 of the largest magnitude of its
tensor (and the forward output O within the forward's own tolerance).  The
backward does not read O, so bf16 inputs are held to the same gradient bound
as fp32.
"""
import numpy as np
import pytest
import torch

import clustered_multipole_approximation_b200 as muse
import oracle
from clustered_multipole_approximation_b200 import build
from clustered_multipole_approximation_b200.inputs import WORKLOADS, clustered_qkv, make_inputs
from helpers import TOL, assert_close, to_dev
from oracle.muse_backward import muse_acausal_grads, muse_causal_grads

pytestmark = pytest.mark.gpu

GTOL = 2e-4


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    muse.load_library()


def gpu_fwd_bwd(Q, K, V, dO, dtype, Cq, Ck, iters, seed, topk, scale, mode):
    q, k, v = to_dev(Q, dtype), to_dev(K, dtype), to_dev(V, dtype)
    p = muse.make_params(Cq, Ck, iters, seed, topk, 0, scale, mode)
    ws = torch.empty(muse.backward_workspace_size(q, k, p, out_f32=True), dtype=torch.uint8,
                     device=q.device)
    O, dbg = muse.muse_attn_fwd(q, k, v, Cq=Cq, Ck=Ck, iters=iters, seed=seed, topk=topk,
                                scale=scale, mode=mode, debug=True, out_dtype=torch.float32,
                                workspace=ws)
    do = torch.from_numpy(np.ascontiguousarray(dO, dtype=np.float32)).cuda()
    dq, dk, dv = muse.muse_attn_bwd(q, k, v, do, Cq=Cq, Ck=Ck, iters=iters, seed=seed,
                                    topk=topk, scale=scale, mode=mode, workspace=ws)
    torch.cuda.synchronize()
    assert int(dbg["device_error"].item()) == 0
    g = {n: t.cpu().numpy() for n, t in dbg.items()}
    return O.cpu().numpy(), g, dq.cpu().numpy(), dk.cpu().numpy(), dv.cpu().numpy()


def grad_close(a, r, what):
    err = np.abs(a - r).max()
    ref = np.abs(r).max()
    assert err <= GTOL * ref, f"{what}: max err {err:.3e} vs max |ref| {ref:.3e}"


def check_bwd(Q, K, V, dtype, Cq, Ck, iters, seed, topk, scale, mode, heads=None, dseed=0):
    B, Hq = Q.shape[:2]
    dO = np.random.default_rng(dseed).standard_normal(Q.shape).astype(np.float32)
    O, g, dq, dk, dv = gpu_fwd_bwd(Q, K, V, dO, dtype, Cq, Ck, iters, seed, topk, scale, mode)
    mask = None
    if heads is not None:
        mask = np.zeros((B, Hq), np.uint8)
        for b, h in heads:
            mask[b, h] = 1
    sel = g["selected"] if topk > 0 else np.zeros((B, Hq, Cq, 0), np.int32)
    Or, dQr, dKr, dVr = muse_acausal_grads(Q, K, V, dO, g["q_assign"], g["k_assign"], sel, Cq, Ck,
                                           scale, mode, hq_mask=mask)
    G = Hq // K.shape[1]
    hs = [(b, h) for b in range(B) for h in range(Hq)] if heads is None else heads
    for b, h in hs:
        assert_close(O[b, h], Or[b, h], TOL[dtype], f"O b{b}h{h}")
        grad_close(dq[b, h], dQr[b, h], f"dQ b{b}h{h}")
    if heads is None:  # dK, dV sum over every q-head of the group
        for b in range(B):
            for hk in range(K.shape[1]):
                grad_close(dk[b, hk], dKr[b, hk], f"dK b{b}h{hk}")
                grad_close(dv[b, hk], dVr[b, hk], f"dV b{b}h{hk}")
    return dq, dk, dv, (dQr, dKr, dVr)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("mode", ["monopole", "dipole"])
def test_small_acausal_backward_gqa_ragged(dtype, D, mode):
    Q, K, V = clustered_qkv(2, 4, 2, 1000, D, 12, 0.3, 0.0, dtype, 131 + D)
    check_bwd(Q, K, V, dtype, 11, 13, 5, 77, 3, 0.9, mode, dseed=D)


@pytest.mark.parametrize("mode", ["monopole", "dipole"])
def test_backward_singleton_key_clusters_is_exact_attention_gradient(mode):
    Q, K, V = clustered_qkv(1, 2, 1, 256, 64, 8, 0.3, 0.0, "f32", 132)
    dq, dk, dv, _ = check_bwd(Q, K, V, "f32", 16, 256, 2, 3, 0, 1.0, mode)
    q, k, v = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V))
    kk, vv = k.expand(-1, 2, -1, -1), v.expand(-1, 2, -1, -1)
    o = torch.softmax(q @ kk.transpose(-1, -2), -1) @ vv
    dO = np.random.default_rng(0).standard_normal(Q.shape)
    gq, gk, gv = torch.autograd.grad((o * torch.tensor(dO)).sum(), (q, k, v))
    for a, r, n in ((dq, gq, "dQ"), (dk, gk, "dK"), (dv, gv, "dV")):
        grad_close(a, r.numpy(), n + " vs exact attention")


def test_backward_retrieving_every_cluster_is_exact_attention_gradient():
    Q, K, V = clustered_qkv(1, 1, 1, 512, 64, 8, 0.3, 0.0, "f32", 133)
    check_bwd(Q, K, V, "f32", 8, 8, 4, 9, 8, 1.0, "dipole")


def test_backward_key_and_value_translation_invariants_full_size():
    """The 8-head 8k layer: the key gradient of every head sums to zero over
    its tokens (O is invariant to translating the keys) and the value gradient
    sums to the sum of dO (translating V by c moves O by c)."""
    w = WORKLOADS["acausal-bf16-h8-n8k"]
    Q, K, V = make_inputs(w)
    dO = np.random.default_rng(1).standard_normal(Q.shape).astype(np.float32)
    _, _, _, dk, dv = gpu_fwd_bwd(Q, K, V, dO, w.dtype, w.C, w.C, w.iters, w.cluster_seed, w.topk,
                                  w.scale, "dipole")
    for h in range(w.Hkv):
        scale = np.abs(dk[0, h]).max() * np.sqrt(w.N)
        assert np.abs(dk[0, h].sum(0)).max() <= 1e-4 * scale, h
        want = dO[0, h].astype(np.float64).sum(0)
        assert np.abs(dv[0, h].astype(np.float64).sum(0) - want).max() <= 1e-4 * np.abs(want).max()


@pytest.mark.parametrize("mode", ["monopole", "dipole"])
def test_workload_acausal_bf16_h8_n8k_backward(mode):
    """The 8-head 8k layer, q-heads 2 and 6 against the oracle (dQ), and the
    full dK, dV of their kv-heads against the oracle over all 8 heads."""
    w = WORKLOADS["acausal-bf16-h8-n8k"]
    Q, K, V = make_inputs(w)
    dq, dk, dv, (dQr, dKr, dVr) = check_bwd(Q, K, V, w.dtype, w.C, w.C, w.iters, w.cluster_seed,
                                            w.topk, w.scale, mode, heads=[(0, 2), (0, 6)])
    for h in (2, 6):  # Hq == Hkv: kv-head h is read by q-head h alone
        grad_close(dk[0, h], dKr[0, h], f"dK h{h}")
        grad_close(dv[0, h], dVr[0, h], f"dV h{h}")


def test_workload_acausal_f32_n1k_backward():
    w = WORKLOADS["acausal-f32-n1k"]
    Q, K, V = make_inputs(w)
    check_bwd(Q, K, V, w.dtype, w.C, w.C, w.iters, w.cluster_seed, w.topk, w.scale, w.mode)


def test_autograd_function_matches_the_entry_point():
    Q, K, V = clustered_qkv(1, 2, 2, 512, 64, 8, 0.3, 0.0, "bf16", 134)
    q, k, v = (to_dev(x, "bf16").requires_grad_(True) for x in (Q, K, V))
    o = muse.muse_attention(q, k, v, Cq=8, Ck=8, iters=3, seed=4, topk=2, scale=1.0,
                            mode="dipole")
    do = torch.randn_like(o)
    o.backward(do)
    p = muse.make_params(8, 8, 3, 4, 2, 0, 1.0, "dipole")
    qd, kd, vd = (x.detach() for x in (q, k, v))
    ws = torch.empty(muse.backward_workspace_size(qd, kd, p), dtype=torch.uint8, device="cuda")
    o2 = muse.muse_attn_fwd(qd, kd, vd, Cq=8, Ck=8, iters=3, seed=4, topk=2, workspace=ws)
    assert torch.equal(o.detach(), o2)
    dq, dk, dv = muse.muse_attn_bwd(qd, kd, vd, do, Cq=8, Ck=8, iters=3, seed=4, topk=2,
                                    workspace=ws)
    # fp32 atomic sums make the gradients' last bits order dependent: compare
    # within the bf16 rounding of the autograd path's outputs
    for got, want in ((q.grad, dq), (k.grad, dk), (v.grad, dv)):
        err = (got.float() - want).abs().max().item()
        assert err <= 1e-2 * want.abs().max().item(), err


@pytest.mark.parametrize("mode", ["tilted", "dipole_q"])
def test_backward_unsupported_modes_are_refused(mode):
    Q, K, V = clustered_qkv(1, 1, 1, 256, 64, 4, 0.3, 0.0, "bf16", 135)
    q, k, v = (to_dev(x, "bf16") for x in (Q, K, V))
    p = muse.make_params(4, 4, 2, 1, 1, 0, 1.0, "dipole")
    ws = torch.empty(muse.backward_workspace_size(q, k, p), dtype=torch.uint8, device="cuda")
    with pytest.raises(muse.MuseError):
        muse.muse_attn_bwd(q, k, v, q, Cq=4, Ck=4, iters=2, seed=1, topk=1, mode=mode,
                           workspace=ws)


# ---------------------------------------------------------------------------
# causal
def gpu_causal_fwd_bwd(Q, K, V, dO, dtype, L, C, iters, seed, topk, scale, mode):
    q, k, v = to_dev(Q, dtype), to_dev(K, dtype), to_dev(V, dtype)
    p = muse.make_params(C, C, iters, seed, topk, L, scale, mode)
    ws = torch.empty(muse.backward_workspace_size(q, k, p, out_f32=True, causal=True),
                     dtype=torch.uint8, device=q.device)
    O, dbg = muse.muse_attn_fwd_causal(q, k, v, C=C, block=L, iters=iters, seed=seed, topk=topk,
                                       scale=scale, mode=mode, debug=True,
                                       out_dtype=torch.float32, workspace=ws)
    do = torch.from_numpy(np.ascontiguousarray(dO, dtype=np.float32)).cuda()
    dq, dk, dv = muse.muse_attn_bwd_causal(q, k, v, do, C=C, block=L, iters=iters, seed=seed,
                                           topk=topk, scale=scale, mode=mode, workspace=ws)
    torch.cuda.synchronize()
    assert int(dbg["device_error"].item()) == 0
    g = {n: t.cpu().numpy() for n, t in dbg.items()}
    return O.cpu().numpy(), g, dq.cpu().numpy(), dk.cpu().numpy(), dv.cpu().numpy()


def check_causal_bwd(Q, K, V, dtype, L, C, iters, seed, topk, scale, mode, dseed=0):
    B, Hq = Q.shape[:2]
    dO = np.random.default_rng(dseed).standard_normal(Q.shape).astype(np.float32)
    O, g, dq, dk, dv = gpu_causal_fwd_bwd(Q, K, V, dO, dtype, L, C, iters, seed, topk, scale, mode)
    Or, dQr, dKr, dVr = muse_causal_grads(Q, K, V, dO, g["q_assign"], g["k_assign"],
                                          g.get("selected"), L, C, scale, mode)
    for b in range(B):
        for h in range(Hq):
            assert_close(O[b, h], Or[b, h], TOL[dtype], f"O b{b}h{h}")
            grad_close(dq[b, h], dQr[b, h], f"dQ b{b}h{h}")
        for hk in range(K.shape[1]):
            grad_close(dk[b, hk], dKr[b, hk], f"dK b{b}h{hk}")
            grad_close(dv[b, hk], dVr[b, hk], f"dV b{b}h{hk}")
    return dq, dk, dv


@pytest.mark.parametrize("dtype,D", [("f32", 64), ("bf16", 64), ("bf16", 128)])
@pytest.mark.parametrize("mode", ["monopole", "dipole"])
def test_small_causal_backward_gqa(dtype, D, mode):
    Q, K, V = clustered_qkv(1, 4, 2, 512, D, 8, 0.3, 0.0, dtype, 151 + D)
    check_causal_bwd(Q, K, V, dtype, 64, 12, 4, 21, 2, 0.9, mode, dseed=D)


def test_causal_backward_low_levels_per_key_token():
    # C = 32 with blocks of 128: the forward takes the lowest levels per key
    # token (bf16 DIPOLE); the backward differentiates the same sums
    Q, K, V = clustered_qkv(1, 2, 1, 512, 64, 12, 0.3, 0.0, "bf16", 152)
    check_causal_bwd(Q, K, V, "bf16", 128, 32, 4, 61, 3, 1.0, "dipole")


def test_causal_backward_singletons_is_exact_causal_attention_gradient():
    Q, K, V = clustered_qkv(1, 2, 1, 256, 64, 8, 0.3, 0.0, "f32", 153)
    dq, dk, dv = check_causal_bwd(Q, K, V, "f32", 32, 256, 2, 3, 0, 1.0, "dipole")
    q, k, v = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V))
    o = torch.nn.functional.scaled_dot_product_attention(q, k.expand(-1, 2, -1, -1),
                                                         v.expand(-1, 2, -1, -1), is_causal=True,
                                                         scale=1.0)
    dO = np.random.default_rng(0).standard_normal(Q.shape)
    gq, gk, gv = torch.autograd.grad((o * torch.tensor(dO)).sum(), (q, k, v))
    for a, r, n in ((dq, gq, "dQ"), (dk, gk, "dK"), (dv, gv, "dV")):
        grad_close(a, r.numpy(), n + " vs exact causal attention")


def test_causal_backward_translation_invariants_full_size():
    """The 16k causal layer (B=2, 8 heads, C=64, blocks of 512): every head's
    key gradient sums to zero over its tokens and its value gradient to the
    sum of dO."""
    w = WORKLOADS["causal-bf16-b2h8-n16k"]
    Q, K, V = make_inputs(w)
    dO = np.random.default_rng(2).standard_normal(Q.shape).astype(np.float32)
    _, _, _, dk, dv = gpu_causal_fwd_bwd(Q, K, V, dO, w.dtype, w.block, w.C, w.iters,
                                         w.cluster_seed, w.topk, w.scale, "dipole")
    assert np.isfinite(dk).all() and np.isfinite(dv).all()
    for b in range(w.B):
        for h in range(w.Hkv):
            scale = np.abs(dk[b, h]).max() * np.sqrt(w.N)
            assert np.abs(dk[b, h].sum(0)).max() <= 1e-4 * scale, (b, h)
            want = dO[b, h].astype(np.float64).sum(0)
            got = dv[b, h].astype(np.float64).sum(0)
            assert np.abs(got - want).max() <= 1e-4 * np.abs(want).max(), (b, h)
