"""The dense forward with Q K^T on e4m3 tensor cores: its error against the fp64
oracle, measured next to the bf16 forward's ("Spatial-Spectral Coupling as
Attention", project page, "Spatial-spectral coupling is attention"; Abstract:
accuracy is what the exact coupling preserves, so the lower-precision variant
is measured, not assumed).

Error bound.  e4m3 keeps 3 mantissa bits, so rounding a value changes it by at
most 2^-4 of its magnitude.  A logit S_ij = s sum_c q_c k_c then moves by about
s * 2^-4 * sqrt(2/3) * ||q o k||_2 (independent roundings of q_c and k_c):
with s = 1/sqrt(128), descriptor magnitudes below ~1.5 and 128 channels that is
a few hundredths.  A perturbation of the logits by delta moves O_i by at most
delta times the spread of the V rows under the row's weights, so max-abs
errors of order 1e-2 and relative Frobenius errors of a few 1e-2 are expected;
the test allows 0.1 and 0.05 and asserts that the e4m3 error is above the bf16
one (the e4m3 path is the one that ran)."""
import numpy as np
import pytest
import torch

import oracle
from spatial_spectral_attention_b200 import api, synth

from _util import errors, rounded

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,n", [("dense_10k", None), ("dense_60k", 6000)])
def test_e4m3_forward_error_against_the_oracle(name, n):
    p = synth.make_workload(name, n=n)
    Q, Q64 = rounded(p.F_N, "bf16")
    K, K64 = rounded(p.F_M, "bf16")
    V, V64 = rounded(p.Phi_M, "bf16")
    O8, lse8 = api.ssc_dense_coupling_fwd_e4m3(Q, K, V, p.scale)
    O16, lse16 = api.ssc_dense_coupling_fwd(Q, K, V, p.scale)
    torch.cuda.synchronize()
    assert api.ssc_device_status() == 0
    O64, lse64 = oracle.dense_fwd(Q64, K64, V64, p.scale)
    e8 = errors(O8.double().cpu().numpy(), O64)
    e16 = errors(O16.double().cpu().numpy(), O64)
    l8 = errors(lse8.double().cpu().numpy(), lse64)
    print(f"\n{name} n={p.n}: O e4m3 max-abs {e8[0]:.3e} rel-fro {e8[1]:.3e}; "
          f"bf16 max-abs {e16[0]:.3e} rel-fro {e16[1]:.3e}; lse e4m3 max-abs {l8[0]:.3e}")
    assert np.all(np.isfinite(O8.cpu().numpy()))
    assert e8[0] <= 0.1 and e8[1] <= 0.05
    assert e8[1] > e16[1]
    # rows of the softmax still sum to one: the constant column comes back
    y00 = float(V[0, 0].float())
    assert np.abs(O8[:, 0].cpu().numpy() - y00).max() < 4e-3 * y00


def test_e4m3_forward_rejects_d64():
    Q = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    V = torch.zeros((8, 16), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError):
        api.ssc_dense_coupling_fwd_e4m3(Q, Q, V, 0.125)
