"""muse_cluster_static: k-means for callers that cannot allocate device
memory (no workspace argument; the scratch is an array built into the
library).  Its results must equal those of muse_cluster with a caller-provided
workspace, call after call.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import clustered_multipole_approximation_b200 as muse
from clustered_multipole_approximation_b200 import build
from clustered_multipole_approximation_b200.inputs import clustered_qkv

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_static_scratch_matches_workspace_entry_point(dtype):
    build.build()
    lib = muse.load_library()
    X, _, _ = clustered_qkv(1, 4, 4, 2048, 64, 16, 0.3, 0.0, dtype, 77)
    x = torch.from_numpy(X)
    x = (x.to(torch.bfloat16) if dtype == "bf16" else x).cuda()
    B, H, N, D = x.shape
    C, iters, seed = 48, 5, 123
    ref_a, ref_c, ref_n = muse.muse_cluster(x, C, iters, seed, role=1)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = 0 if dtype == "bf16" else 1
    for _ in range(2):  # the shared scratch keeps the previous call's contents
        a = torch.full_like(ref_a, -1)
        c = torch.full_like(ref_c, float("nan"))
        n = torch.full_like(ref_n, -1)
        err = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        st = lib.muse_cluster_static(_p(x), code, B, H, N, D, C, iters, seed, 1, None, _p(a),
                                     _p(c), _p(n), _p(err), stream)
        assert st == 0, lib.muse_last_error()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert torch.equal(a, ref_a)
        assert torch.equal(n, ref_n)
        np.testing.assert_allclose(c.cpu().numpy(), ref_c.cpu().numpy(), rtol=2e-7, atol=1e-7)


def test_static_scratch_rejects_sizes_beyond_its_capacity():
    lib = muse.load_library()
    cap = lib.muse_cluster_static_capacity()
    assert cap == 16 << 20
    # 64 heads x 32768 tokens x 256 clusters needs far more than the capacity
    assert lib.muse_cluster_workspace_size(1, 64, 32768, 128, 256) > cap
    x = torch.zeros(1, 1, 8, 128, dtype=torch.bfloat16, device="cuda")  # never read
    out = torch.zeros(16, dtype=torch.int32, device="cuda")
    st = lib.muse_cluster_static(_p(x), 0, 1, 64, 32768, 128, 256, 3, 0, 0, None, _p(out),
                                 _p(out), None, None, None)
    assert st == 3
    assert b"scratch" in lib.muse_last_error()
