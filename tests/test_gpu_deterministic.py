"""The deterministic dense backward: gradients identical bit for bit from run to
run, and equal to the oracle's within the bf16 tolerances ("Spatial-Spectral
Coupling as Attention", project page, "Spatial-spectral coupling is
attention": the textbook softmax-matmul gradient with Q = F_N, K = F_M,
V = Phi_M)."""
import math

import numpy as np
import pytest
import torch

import oracle
from spatial_spectral_attention_b200 import api, synth

from _util import TOL_BF16, assert_close, rounded

pytestmark = pytest.mark.gpu


def _inputs(Qn, Kn, Vn, dOn):
    Q, Q64 = rounded(Qn, "bf16")
    K, K64 = rounded(Kn, "bf16")
    V, V64 = rounded(Vn, "bf16")
    dO = torch.tensor(np.ascontiguousarray(dOn, np.float32)).cuda()
    dO64 = dO.to(torch.bfloat16).double().cpu().numpy()
    return (Q, K, V, dO), (Q64, K64, V64, dO64)


@pytest.mark.parametrize("nN,nM,d,k", [(1, 1, 128, 196), (129, 300, 64, 25), (513, 77, 128, 16),
                                       (384, 1000, 128, 196), (200, 200, 64, 100),
                                       # k = 256: the dK pass keeps one Q stage
                                       (256, 700, 128, 256),
                                       # more row tiles than SMs: two CTAs share a tile
                                       (300, 40000, 128, 196)])
def test_deterministic_backward_matches_oracle(nN, nM, d, k):
    Qn, Kn, Vn, dOn = synth.random_inputs(nN, nM, d, k, seed=nN * 3 + nM, q_scale=0.5)
    (Q, K, V, dO), (Q64, K64, V64, dO64) = _inputs(Qn, Kn, Vn, dOn)
    s = 1.0 / math.sqrt(d)
    O, lse = api.ssc_dense_coupling_fwd(Q, K, V, s)
    dQ, dK, dV = api.ssc_dense_coupling_bwd(Q, K, V, O, lse, dO, s, need_dV=True, deterministic=True)
    torch.cuda.synchronize()
    assert api.ssc_device_status() == 0
    ref = oracle.dense_bwd(Q64, K64, V64, dO64, s)
    for t, nm in ((dQ, "dQ"), (dK, "dK"), (dV, "dV")):
        assert_close(t, ref[nm], TOL_BF16, nm)


def test_deterministic_backward_is_bit_identical_across_runs():
    p = synth.make_workload("dense_10k")
    (Q, K, V, dO), (Q64, K64, V64, dO64) = _inputs(p.F_N, p.F_M, p.Phi_M, p.dO)
    O, lse = api.ssc_dense_coupling_fwd(Q, K, V, p.scale)
    runs = [api.ssc_dense_coupling_bwd(Q, K, V, O, lse, dO, p.scale, need_dV=True, deterministic=True)
            for _ in range(3)]
    torch.cuda.synchronize()
    assert api.ssc_device_status() == 0
    for other in runs[1:]:
        for a, b in zip(runs[0], other):
            assert torch.equal(a, b)
    ref = oracle.dense_bwd(Q64, K64, V64, dO64, p.scale)
    for t, nm in zip(runs[0], ("dQ", "dK", "dV")):
        assert_close(t, ref[nm], TOL_BF16, nm)


def test_deterministic_backward_at_60k_agrees_with_the_default():
    p = synth.make_workload("dense_60k")
    (Q, K, V, dO), _ = _inputs(p.F_N, p.F_M, p.Phi_M, p.dO)
    O, lse = api.ssc_dense_coupling_fwd(Q, K, V, p.scale)
    a = api.ssc_dense_coupling_bwd(Q, K, V, O, lse, dO, p.scale, need_dV=True, deterministic=True)
    b = api.ssc_dense_coupling_bwd(Q, K, V, O, lse, dO, p.scale, need_dV=True, deterministic=True)
    c = api.ssc_dense_coupling_bwd(Q, K, V, O, lse, dO, p.scale, need_dV=True)
    torch.cuda.synchronize()
    assert api.ssc_device_status() == 0
    for x, y, z, nm in zip(a, b, c, ("dQ", "dK", "dV")):
        assert torch.equal(x, y), nm
        assert_close(x, z.double().cpu().numpy(), TOL_BF16, nm)
