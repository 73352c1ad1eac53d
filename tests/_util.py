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


def assert_close(got, ref, tol, name="", scale_by_ref=False):
    """max-abs and relative-Frobenius bounds.

    The relative measure is skipped when the exact result is zero to rounding
    (||ref||_F below 1e-9 per element, e.g. the gradients of a single-key
    coupling, which vanish identically); max-abs still applies.  With
    scale_by_ref the max-abs bound is multiplied by max(1, max|ref|): bf16
    rounding is relative, so stress inputs with outputs far above the
    workloads' O(1) magnitudes get the same relative allowance."""
    if isinstance(got, torch.Tensor):
        got = got.detach().double().cpu().numpy()
    ref = np.asarray(ref, dtype=np.float64)
    maxabs, relfro = errors(got, ref)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    bound = tol["maxabs"] * (max(1.0, float(np.abs(ref).max())) if scale_by_ref else 1.0)
    degenerate = float(np.linalg.norm(ref)) < 1e-9 * np.sqrt(max(ref.size, 1))
    ok = maxabs <= bound and (degenerate or relfro <= tol["relfro"])
    assert ok, (f"{name}: max-abs {maxabs:.3e} (<= {bound:.3g}), rel-Frobenius {relfro:.3e} "
                f"(<= {tol['relfro']}{', skipped: exact result is zero' if degenerate else ''})")
    return maxabs, relfro


def as_i32(a):
    return torch.tensor(np.ascontiguousarray(a, dtype=np.int32)).cuda()
