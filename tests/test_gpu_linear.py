"""GPU parity of the linear-attention (ELU) coupling against the fp64 oracle
("Spatial-Spectral Coupling as Attention", project page, Table 1 row "Linear
attention (ELU)"; digest "Interpretation": a low-rank feature map in place of
the softmax).  bf16 tensor-core path, tolerances as for the exact couplings:
max-abs 2e-2 and relative Frobenius 1e-2 on O, den, dQ, dK and dV."""
import numpy as np
import pytest
import torch

from oracle import linear as lin
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


def _status_ok():
    torch.cuda.synchronize()
    assert api.ssc_device_status() == 0


def _case(Qn, Kn, Vn, dOn, need_dV=True):
    (Q, K, V, dO), (Q64, K64, V64, dO64) = _inputs(Qn, Kn, Vn, dOn)
    O, den = api.ssc_linear_coupling_fwd(Q, K, V)
    dQ, dK, dV = api.ssc_linear_coupling_bwd(Q, K, V, O, den, dO, need_dV=need_dV)
    _status_ok()
    ref = lin.linear_bwd(Q64, K64, V64, dO64)
    assert_close(O, ref["O"], TOL_BF16, "O")
    # den grows with nM; its relative error is what bf16 rounding bounds
    assert_close(den.double().cpu().numpy() / ref["den"], np.ones_like(ref["den"]), TOL_BF16, "den")
    assert_close(dQ, ref["dQ"], TOL_BF16, "dQ")
    assert_close(dK, ref["dK"], TOL_BF16, "dK")
    if need_dV:
        assert_close(dV, ref["dV"], TOL_BF16, "dV")


@pytest.mark.parametrize("nN,nM,d,k", [(1, 1, 128, 196), (129, 300, 64, 25), (513, 77, 128, 16),
                                       (256, 1000, 128, 255), (200, 200, 64, 100),
                                       (130, 260, 128, 32), (384, 129, 128, 196),
                                       # k = 192 and 64: the column of ones falls in a box
                                       # that TMA does not load
                                       (300, 4000, 128, 192), (1000, 1000, 128, 64)])
def test_linear_shapes(nN, nM, d, k):
    Qn, Kn, Vn, dOn = synth.random_inputs(nN, nM, d, k, seed=nN * 5 + nM, q_scale=0.5)
    _case(Qn, Kn, Vn, dOn)


def test_linear_10k_workload_full():
    p = synth.make_workload("dense_10k")
    _case(p.F_N, p.F_M, p.Phi_M, p.dO)


def test_linear_60k_workload_sampled():
    p = synth.make_workload("dense_60k")
    (Q, K, V, dO), (Q64, K64, V64, dO64) = _inputs(p.F_N, p.F_M, p.Phi_M, p.dO)
    O, den = api.ssc_linear_coupling_fwd(Q, K, V)
    dQ, dK, dV = api.ssc_linear_coupling_bwd(Q, K, V, O, den, dO, need_dV=True)
    _status_ok()
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(p.n, 512, replace=False))
    cols = np.sort(rng.choice(p.n, 512, replace=False))
    ref = lin.linear_bwd(Q64, K64, V64, dO64, rows=rows, cols=cols)
    assert_close(O.cpu().numpy()[rows], ref["O"], TOL_BF16, "O rows")
    assert_close(dQ.cpu().numpy()[rows], ref["dQ"], TOL_BF16, "dQ rows")
    assert_close(dK.cpu().numpy()[cols], ref["dK"], TOL_BF16, "dK cols")
    assert_close(dV.cpu().numpy()[cols], ref["dV"], TOL_BF16, "dV cols")
    # rows of the normalised weights sum to one: the constant column comes back
    y00 = float(V[0, 0].float())
    assert np.abs(O[:, 0].cpu().numpy() - y00).max() < 4e-3 * y00
    # sum_j dV_j = sum_i dO_i; every dV_j shares the one bf16-rounded dKV, so the
    # rounding does not average out over the rows: relative Frobenius bound
    assert_close(dV.double().sum(0).cpu().numpy(), dO64.sum(0), dict(maxabs=np.inf, relfro=1e-2),
                 "sum_j dV_j")


def test_linear_unaligned_v_and_reused_workspace():
    # k = 25: 50-byte V rows are re-packed by the library; two calls share a workspace
    Qn, Kn, Vn, dOn = synth.random_inputs(700, 650, 64, 25, seed=12, q_scale=0.5)
    (Q, K, V, dO), (Q64, K64, V64, dO64) = _inputs(Qn, Kn, Vn, dOn)
    nb = api.lib().ssc_linear_coupling_workspace_size(700, 650, 64, 25)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    ref = lin.linear_bwd(Q64, K64, V64, dO64)
    for _ in range(2):
        O, den = api.ssc_linear_coupling_fwd(Q, K, V, workspace=ws)
        dQ, dK, dV = api.ssc_linear_coupling_bwd(Q, K, V, O, den, dO, need_dV=True, workspace=ws)
        _status_ok()
        for t, nm in ((O, "O"), (dQ, "dQ"), (dK, "dK"), (dV, "dV")):
            assert_close(t, ref[nm], TOL_BF16, nm)


def test_linear_rejects_k_256():
    Q = torch.zeros((4, 128), dtype=torch.bfloat16, device="cuda")
    V = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError):
        api.ssc_linear_coupling_fwd(Q, Q, V)
