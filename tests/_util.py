"""Shared helpers of the GPU parity tests: input preparation and tolerances."""
import numpy as np
import torch

# bf16 path: max-abs and relative Frobenius error bounds; fp32 check mode: 1e-4.
TOL_BF16 = dict(maxabs=2e-2, relfro=1e-2)
TOL_F32 = dict(maxabs=1e-4, relfro=1e-4)


def rounded(a, dtype):
    """The values the GPU sees for numpy array a in `dtype` ('bf16' or 'f32'),
    as a (device tensor, exact fp64 numpy copy) pair."""
    t = torch.tensor(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.cuda(), t.double().numpy()


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = got - ref
    maxabs = float(np.abs(diff).max()) if diff.size else 0.0
    den = float(np.linalg.norm(ref))
    relfro = float(np.linalg.norm(diff) / den) if den > 0 else float(np.linalg.norm(diff))
    return maxabs, relfro


def assert_close(got, ref, tol, name=""):
    if isinstance(got, torch.Tensor):
        got = got.detach().double().cpu().numpy()
    maxabs, relfro = errors(got, ref)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    assert maxabs <= tol["maxabs"] and relfro <= tol["relfro"], (
        f"{name}: max-abs {maxabs:.3e} (<= {tol['maxabs']}), rel-Frobenius {relfro:.3e} "
        f"(<= {tol['relfro']})")
    return maxabs, relfro


def as_i32(a):
    return torch.tensor(np.ascontiguousarray(a, dtype=np.int32)).cuda()
