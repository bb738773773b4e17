"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/muse.h declares, sizes workspaces, and rejects bad
arguments before launching anything."""
import ctypes
import os
import re

import pytest

import clustered_multipole_approximation_b200 as muse
from clustered_multipole_approximation_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return muse.load_library()


def declared_symbols():
    syms = set()
    for name in os.listdir(os.path.join(ROOT, "include")):
        if name.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", name)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            syms |= set(re.findall(r"\b(muse_[a-z0-9_]+)\s*\(", txt))
    return syms


def test_library_exports_every_declared_symbol(lib):
    syms = declared_symbols()
    assert {"muse_cluster", "muse_summarize", "muse_attn_fwd", "muse_attn_fwd_causal"} <= syms
    for s in syms:
        assert hasattr(lib, s), s
    assert set(muse.EXPORTS) <= syms


def shape(B=1, Hq=2, Hkv=1, N=1024, D=64, dt=0):
    return muse.muse_shape(B, Hq, Hkv, N, D, dt)


def params(Cq=16, Ck=16, iters=3, topk=2, block=0, mode=1):
    return muse.muse_params(Cq, Ck, iters, 1, topk, block, 1.0, mode)


def test_workspace_size_valid_and_invalid(lib):
    ws = lib.muse_workspace_size(ctypes.byref(shape()), ctypes.byref(params()), 0)
    assert ws > 0
    wsc = lib.muse_workspace_size(ctypes.byref(shape()), ctypes.byref(params(block=128)), 1)
    assert wsc > 0
    bad = [(shape(D=96), params(), 0), (shape(Hq=3, Hkv=2), params(), 0),
           (shape(), params(Cq=0), 0), (shape(), params(Ck=2000), 0),
           (shape(N=100), params(Cq=101, Ck=5), 0), (shape(), params(topk=17), 0),
           (shape(), params(iters=0), 0), (shape(), params(mode=7), 0),
           (shape(), params(block=100), 1), (shape(N=768), params(block=128), 1),
           (shape(), params(Cq=8, Ck=16, block=128), 1)]
    for sh, pr, c in bad:
        assert lib.muse_workspace_size(ctypes.byref(sh), ctypes.byref(pr), c) == 0
    assert lib.muse_cluster_workspace_size(1, 2, 1000, 64, 10) > 0
    assert lib.muse_cluster_workspace_size(1, 2, 1000, 80, 10) == 0


def test_invalid_arguments_return_errors_without_launch(lib):
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first
    sh, pr = shape(), params()
    st = lib.muse_attn_fwd(None, fake, fake, fake, ctypes.byref(sh), ctypes.byref(pr), None,
                           fake, 1 << 30, None)
    assert st == 1 and b"NULL" in lib.muse_last_error()
    st = lib.muse_attn_fwd(fake, fake, fake, fake, ctypes.byref(shape(D=80)), ctypes.byref(pr),
                           None, fake, 1 << 30, None)
    assert st == 2
    st = lib.muse_attn_fwd(fake, fake, fake, fake, ctypes.byref(sh), ctypes.byref(pr), None,
                           fake, 16, None)
    assert st == 3 and b"workspace" in lib.muse_last_error()
    st = lib.muse_attn_fwd_causal(fake, fake, fake, fake, ctypes.byref(sh),
                                  ctypes.byref(params(block=100)), None, fake, 1 << 30, None)
    assert st == 1
    st = lib.muse_cluster(fake, 0, 1, 1, 100, 64, 200, 3, 0, 0, None, fake, fake, None, None,
                          fake, 1 << 30, None)
    assert st == 1
    st = lib.muse_cluster(fake, 0, 1, 1, 100, 64, 10, 3, 0, 2, None, fake, fake, None, None, fake,
                          1 << 30, None)
    assert st == 1
    st = lib.muse_summarize(fake, fake, 0, 1, 1, 100, 48, 10, fake, fake, fake, fake, None, None,
                            0, None)
    assert st == 2
    assert lib.muse_status_string(3) == b"workspace too small"


def test_product_path_fails_loudly_without_library(tmp_path):
    with pytest.raises(ImportError):
        muse.load_library(str(tmp_path / "missing.so"))


def test_misaligned_pointers_are_rejected_without_launch(lib):
    """Kernels load 16-byte vectors and carve the workspace in 256-byte
    pieces: misaligned pointers must come back as MUSE_ERR_INVALID_ARG."""
    ok = ctypes.c_void_p(0x10000)    # never dereferenced: validation fails first
    odd = ctypes.c_void_p(0x10008)   # 8-byte aligned only
    ws_odd = ctypes.c_void_p(0x10080)  # 128-byte aligned only
    sh, pr = shape(), params()
    for args in [(odd, ok, ok, ok, ok), (ok, odd, ok, ok, ok), (ok, ok, odd, ok, ok),
                 (ok, ok, ok, odd, ok), (ok, ok, ok, ok, ws_odd)]:
        q, k, v, o, ws = args
        for f in (lib.muse_attn_fwd, lib.muse_attn_fwd_causal):
            p = params(block=128) if f is lib.muse_attn_fwd_causal else pr
            st = f(q, k, v, o, ctypes.byref(sh), ctypes.byref(p), None, ws, 1 << 40, None)
            assert st == 1 and b"aligned" in lib.muse_last_error(), (args, st)
    dbg = muse.muse_debug(None, None, None, None, None, None, ctypes.c_void_p(0x10004), None)
    st = lib.muse_attn_fwd(ok, ok, ok, ok, ctypes.byref(sh), ctypes.byref(pr), ctypes.byref(dbg),
                           ok, 1 << 40, None)
    assert st == 1 and b"aligned" in lib.muse_last_error()
    st = lib.muse_cluster(odd, 0, 1, 1, 100, 64, 10, 3, 0, 0, None, ok, ok, None, None, ok,
                          1 << 30, None)
    assert st == 1 and b"aligned" in lib.muse_last_error()
    st = lib.muse_cluster(ok, 0, 1, 1, 100, 64, 10, 3, 0, 0, None, ok, ok, None, None, ws_odd,
                          1 << 30, None)
    assert st == 1 and b"aligned" in lib.muse_last_error()
    st = lib.muse_summarize(odd, ok, 0, 1, 1, 100, 64, 10, ok, ok, ok, ok, None, None, 0, None)
    assert st == 1 and b"aligned" in lib.muse_last_error()
    st = lib.muse_device_status(None, None)
    assert st == 1


def test_backward_workspace_and_argument_checks(lib):
    """The backward entry point sizes its workspace past the forward's part and
    refuses unsupported modes and sizes, bad pointers and small workspaces
    before launching anything."""
    sh, pr = shape(), params()
    fwd = lib.muse_workspace_size(ctypes.byref(sh), ctypes.byref(pr), 0)
    bwd = lib.muse_attn_bwd_workspace_size(ctypes.byref(sh), ctypes.byref(pr))
    assert bwd > fwd > 0
    mono = lib.muse_attn_bwd_workspace_size(ctypes.byref(sh), ctypes.byref(params(mode=0)))
    assert fwd < mono < bwd  # no M_j or u_ij tables for MONOPOLE
    for bad in (params(mode=2), params(mode=3), params(Ck=512)):  # TILTED, DIPOLE_Q, Ck D > 16384
        assert lib.muse_attn_bwd_workspace_size(ctypes.byref(sh), ctypes.byref(bad)) == 0
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first
    args = [fake] * 7
    st = lib.muse_attn_bwd(*([None] + args[1:]), ctypes.byref(sh), ctypes.byref(pr), fake,
                           1 << 40, None)
    assert st == 1 and b"NULL" in lib.muse_last_error()
    st = lib.muse_attn_bwd(*args, ctypes.byref(sh), ctypes.byref(params(mode=2)), fake, 1 << 40,
                           None)
    assert st == 2
    st = lib.muse_attn_bwd(*args, ctypes.byref(sh), ctypes.byref(pr), fake, fwd, None)
    assert st == 3 and b"backward" in lib.muse_last_error()


def test_accum_workspace_and_argument_checks(lib):
    """The block-accumulation entry point sizes its workspace and refuses
    unsupported modes, sizes and budgets before launching anything."""
    sh = shape()
    ok = lib.muse_accum_workspace_size(ctypes.byref(sh), ctypes.byref(params(block=128)), 2)
    assert ok > 0
    mono = lib.muse_accum_workspace_size(ctypes.byref(sh), ctypes.byref(params(block=128, mode=0)), 2)
    assert 0 < mono < ok  # no A tables for MONOPOLE
    bad = [(params(block=100), 2), (params(block=128), 9), (params(block=128, mode=2), 2),
           (params(block=128, Ck=300), 2), (params(block=0), 0)]
    for pr, k2 in bad:
        assert lib.muse_accum_workspace_size(ctypes.byref(sh), ctypes.byref(pr), k2) == 0
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first
    st = lib.muse_attn_fwd_causal_accum(None, fake, fake, fake, ctypes.byref(sh),
                                        ctypes.byref(params(block=128)), 2, None, fake, 1 << 40,
                                        None)
    assert st == 1 and b"NULL" in lib.muse_last_error()
    st = lib.muse_attn_fwd_causal_accum(fake, fake, fake, fake, ctypes.byref(sh),
                                        ctypes.byref(params(block=128)), 2, None, fake, 16, None)
    assert st == 3


def test_causal_backward_workspace_and_argument_checks(lib):
    """The causal backward sizes its workspace past the causal forward's part,
    and refuses blocks that are not multiples of 32 and unsupported modes
    before launching anything."""
    sh = shape(N=1024)
    pr = params(block=128)
    fwd = lib.muse_workspace_size(ctypes.byref(sh), ctypes.byref(pr), 1)
    bwd = lib.muse_attn_bwd_causal_workspace_size(ctypes.byref(sh), ctypes.byref(pr))
    assert bwd > fwd > 0
    for bad in (params(block=16 * 3), params(block=128, mode=2), params(block=128, mode=4)):
        assert lib.muse_attn_bwd_causal_workspace_size(ctypes.byref(sh), ctypes.byref(bad)) == 0
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first
    st = lib.muse_attn_bwd_causal(*([fake] * 7), ctypes.byref(sh), ctypes.byref(pr), fake, fwd,
                                  None)
    assert st == 3
    st = lib.muse_attn_bwd_causal(*([fake] * 7), ctypes.byref(sh),
                                  ctypes.byref(params(block=96)), fake, 1 << 40, None)
    assert st == 1  # 96 does not divide N = 1024


def test_accuracy_variant_modes_are_accepted_for_sizing(lib):
    """DIPOLE_Q and TILTED_DIPOLE are valid modes (sized like DIPOLE and
    TILTED); mode 5 is not."""
    sh = shape()
    for m in (3, 4):
        assert lib.muse_workspace_size(ctypes.byref(sh), ctypes.byref(params(mode=m)), 0) > 0
    assert lib.muse_workspace_size(ctypes.byref(sh), ctypes.byref(params(mode=5)), 0) == 0
    tilted = lib.muse_workspace_size(ctypes.byref(sh), ctypes.byref(params(mode=2)), 0)
    assert lib.muse_workspace_size(ctypes.byref(sh), ctypes.byref(params(mode=4)), 0) == tilted
