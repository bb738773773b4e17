"""Shared helpers of the GPU parity tests: device copies of the seeded inputs
and the comparisons against the oracle."""
import numpy as np
import torch

# Output tolerances (max-abs) of the CUDA path against the fp64 oracle, on the
# fp32 output (the computation itself): fp32 inputs are computed in fp32
# throughout; bf16 inputs are exact in fp32 and accumulate in fp32.  The
# bf16-output variant is checked to be that fp32 result rounded once.
TOL = {"f32": 1e-5, "bf16": 2e-3}
# Near-tie band of the k-means assignment (relative distance gap).
TIE_REL = 1e-6


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.cuda()


def assert_assign_match(gpu_a, orc_a, X=None, prev_cent=None, what="assign"):
    """Assignments must be identical; a mismatch is allowed only when the two
    choices are a near tie (relative gap < 1e-6) under the centroids that made
    the decision."""
    gpu_a = np.asarray(gpu_a)
    orc_a = np.asarray(orc_a)
    bad = np.nonzero(gpu_a != orc_a)
    if len(bad[0]) == 0:
        return
    assert X is not None and prev_cent is not None, f"{what}: {len(bad[0])} mismatches"
    for idx in zip(*bad):
        x = X[idx]
        cg, co = prev_cent[gpu_a[idx]], prev_cent[orc_a[idx]]
        dg, do = ((x - cg) ** 2).sum(), ((x - co) ** 2).sum()
        rel = (dg - do) / max(do, 1e-12 * (x ** 2).sum())
        assert rel < TIE_REL, f"{what}: mismatch at {idx} with relative gap {rel}"


def assert_close(gpu, ref, tol, what="O"):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(gpu - ref)
    i = np.unravel_index(np.argmax(err), err.shape)
    assert err.max() <= tol, f"{what}: max abs err {err.max():.3e} at {i} (tol {tol})"


def rse(O, E) -> float:
    O = np.asarray(O, dtype=np.float64)
    E = np.asarray(E, dtype=np.float64)
    return float(((O - E) ** 2).sum() / (E ** 2).sum())
