"""GPU parity of the coupling O = softmax(s Q K^T) V and its gradients against
the fp64 oracle, dense and Geo-FlashAttention, bf16 tensor-core path and fp32
check mode ("Spatial-Spectral Coupling as Attention", project page, sections
"Spatial-spectral coupling is attention" and "Geo-FlashAttention")."""
import math

import numpy as np
import pytest
import torch

import oracle
from spatial_spectral_attention_b200 import api, synth

from _util import TOL_BF16, TOL_F32, as_i32, assert_close, rounded

pytestmark = pytest.mark.gpu


def _inputs(Qn, Kn, Vn, dOn, dtype):
    Q, Q64 = rounded(Qn, dtype)
    K, K64 = rounded(Kn, dtype)
    V, V64 = rounded(Vn, dtype)
    # the bf16 path rounds dO once and uses that value throughout
    dO = torch.tensor(np.ascontiguousarray(dOn, np.float32)).cuda()
    dO64 = (dO.to(torch.bfloat16) if dtype == "bf16" else dO).double().cpu().numpy()
    return (Q, K, V, dO), (Q64, K64, V64, dO64)


def _status_ok():
    torch.cuda.synchronize()
    assert api.ssc_device_status() == 0


def _dense_case(Qn, Kn, Vn, dOn, scale, dtype, need_dV=True, scale_by_ref=False):
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    (Q, K, V, dO), (Q64, K64, V64, dO64) = _inputs(Qn, Kn, Vn, dOn, dtype)
    O, lse = api.ssc_dense_coupling_fwd(Q, K, V, scale)
    dQ, dK, dV = api.ssc_dense_coupling_bwd(Q, K, V, O, lse, dO, scale, need_dV=need_dV)
    _status_ok()
    ref = oracle.dense_bwd(Q64, K64, V64, dO64, scale)
    kw = dict(scale_by_ref=scale_by_ref)
    assert_close(O, ref["O"], tol, "O", **kw)
    assert_close(lse, ref["lse"], tol, "lse", **kw)
    assert_close(dQ, ref["dQ"], tol, "dQ", **kw)
    assert_close(dK, ref["dK"], tol, "dK", **kw)
    if need_dV:
        assert_close(dV, ref["dV"], tol, "dV", **kw)


def test_dense_fp32_check_mode_small_workload():
    p = synth.make_workload("small_fp32_2k")
    (Q, K, V, _), (Q64, K64, V64, _) = _inputs(p.F_N, p.F_M, p.Phi_M, p.dO, "f32")
    O, lse = api.ssc_dense_coupling_fwd(Q, K, V, p.scale)
    _status_ok()
    O64, lse64 = oracle.dense_fwd(Q64, K64, V64, p.scale)
    assert_close(O, O64, TOL_F32, "O")
    assert_close(lse, lse64, TOL_F32, "lse")


def test_dense_fp32_check_mode_backward():
    p = synth.make_workload("small_fp32_2k", n=700)
    _dense_case(p.F_N, p.F_M, p.Phi_M, p.dO, p.scale, "f32")


def test_dense_bf16_workload_ragged():
    p = synth.make_workload("dense_10k", n=3000)  # 23 full row tiles + 56 rows
    _dense_case(p.F_N, p.F_M, p.Phi_M, p.dO, p.scale, "bf16")


@pytest.mark.parametrize("nN,nM,d,k", [(1, 1, 128, 196), (129, 300, 64, 25), (513, 77, 128, 16),
                                       (256, 1000, 128, 256), (200, 200, 64, 100),
                                       (130, 260, 128, 32), (384, 129, 128, 196),
                                       # one query tile over 157 key tiles: the dense forward
                                       # splits it between every CTA pair and merges ~74 pieces
                                       (200, 20000, 128, 196),
                                       # two row tiles over 313 key tiles: every CTA of the
                                       # key-stationary dV pass runs through several key tiles
                                       (256, 40000, 128, 196)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_dense_shapes(nN, nM, d, k, dtype):
    Qn, Kn, Vn, dOn = synth.random_inputs(nN, nM, d, k, seed=nN * 7 + nM, q_scale=0.5)
    _dense_case(Qn, Kn, Vn, dOn, 1.0 / math.sqrt(d), dtype)


def test_dense_bf16_unaligned_v_is_repacked():
    # k = 25 gives a 50-byte V row pitch, which the library re-packs itself
    Qn, Kn, Vn, dOn = synth.random_inputs(300, 260, 64, 25, seed=3)
    _dense_case(Qn, Kn, Vn, dOn, 0.125, "bf16")


def test_dense_bf16_peaked_softmax_rescaling():
    # a large scale makes the running max jump often: exercises the O rescale.
    # Gradients here reach |dQ| ~ 10, so the max-abs bound scales with max|ref|.
    Qn, Kn, Vn, dOn = synth.random_inputs(256, 1024, 128, 64, seed=9)
    _dense_case(Qn, Kn, Vn, dOn, 0.6, "bf16", scale_by_ref=True)


def test_dense_bf16_full_size_sampled():
    # the 60k workload the dense metric is quoted on: O, lse and dQ on sampled
    # target rows, dK and dV on sampled source rows, element by element (the
    # oracle's dK/dV columns still sum over all 60k target rows)
    p = synth.make_workload("dense_60k")
    (Q, K, V, dO), (Q64, K64, V64, dO64) = _inputs(p.F_N, p.F_M, p.Phi_M, p.dO, "bf16")
    O, lse = api.ssc_dense_coupling_fwd(Q, K, V, p.scale)
    dQ, dK, dV = api.ssc_dense_coupling_bwd(Q, K, V, O, lse, dO, p.scale, need_dV=True)
    _status_ok()
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(p.n, 384, replace=False))
    cols = np.sort(rng.choice(p.n, 384, replace=False))
    ref = oracle.dense_bwd(Q64, K64, V64, dO64, p.scale, rows=rows, cols=cols)
    assert_close(O.cpu().numpy()[rows], ref["O"], TOL_BF16, "O rows")
    assert_close(lse.cpu().numpy()[rows], ref["lse"], TOL_BF16, "lse rows")
    assert_close(dQ.cpu().numpy()[rows], ref["dQ"], TOL_BF16, "dQ rows")
    assert_close(dK.cpu().numpy()[cols], ref["dK"], TOL_BF16, "dK cols")
    assert_close(dV.cpu().numpy()[cols], ref["dV"], TOL_BF16, "dV cols")
    # properties that hold at any size: sum_j dK_j = 0, sum_j dV_j = sum_i dO_i,
    # sum_i <Q_i, dQ_i> = sum_j <K_j, dK_j>
    dKn, dVn, dQn = (t.double().cpu().numpy() for t in (dK, dV, dQ))
    assert np.abs(dKn.sum(0)).max() <= 1e-2 * np.abs(dKn).sum(0).max()
    np.testing.assert_allclose(dVn.sum(0), dO64.sum(0), atol=0.5, rtol=2e-3)
    a, b = (Q64 * dQn).sum(), (K64 * dKn).sum()
    assert abs(a - b) <= 1e-2 * max(abs(a), abs(b), 1.0)


def test_dense_bf16_10k_workload_full():
    # the 10k forward+backward workload at its full size, every output element
    p = synth.make_workload("dense_10k")
    _dense_case(p.F_N, p.F_M, p.Phi_M, p.dO, p.scale, "bf16")


def _geo_tables(pair, P, R, dtype):
    FN64 = rounded(pair.F_N, dtype)[1]
    FM64 = rounded(pair.F_M, dtype)[1]
    return oracle.patch_pipeline(pair.pts_N, pair.pts_M, FN64, FM64, P, P, R)


def _geo_case(pair, P, R, dtype, need_dV=True):
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    t = _geo_tables(pair, P, R, dtype)
    (Q, K, V, dO), (Q64, K64, V64, dO64) = _inputs(pair.F_N, pair.F_M, pair.Phi_M, pair.dO, dtype)
    tabs = [as_i32(t[x]) for x in ("off_N", "mem_N", "off_M", "mem_M", "topk")]
    O, lse = api.ssc_geo_coupling_fwd(Q, K, V, pair.scale, *tabs)
    dQ, dK, dV = api.ssc_geo_coupling_bwd(Q, K, V, O, lse, dO, pair.scale, *tabs, need_dV=need_dV)
    _status_ok()
    ref = oracle.geo_bwd(Q64, K64, V64, dO64, pair.scale, t["off_N"], t["mem_N"], t["off_M"],
                         t["mem_M"], t["topk"])
    assert_close(O, ref["O"], tol, "O")
    assert_close(lse, ref["lse"], tol, "lse")
    assert_close(dQ, ref["dQ"], tol, "dQ")
    assert_close(dK, ref["dK"], tol, "dK")
    if need_dV:
        assert_close(dV, ref["dV"], tol, "dV")
    return O, lse, dQ, dK, dV


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("n,P,R", [(6000, 48, 8), (2000, 5, 2), (1500, 12, 3), (300, 300, 4)])
def test_geo_matches_oracle(dtype, n, P, R):
    pair = synth.make_workload("geo_60k", n=n)
    _geo_case(pair, P, R, dtype)


def test_geo_all_patches_selected_equals_dense():
    pair = synth.make_workload("geo_60k", n=1200)
    P = 10
    O, lse, dQ, dK, dV = _geo_case(pair, P, P, "bf16")
    (Q, K, V, dO), _ = _inputs(pair.F_N, pair.F_M, pair.Phi_M, pair.dO, "bf16")
    Od, lsed = api.ssc_dense_coupling_fwd(Q, K, V, pair.scale)
    dQd, dKd, dVd = api.ssc_dense_coupling_bwd(Q, K, V, Od, lsed, dO, pair.scale, need_dV=True)
    for a, b, nm in ((O, Od, "O"), (lse, lsed, "lse"), (dQ, dQd, "dQ"), (dK, dKd, "dK"),
                     (dV, dVd, "dV")):
        assert_close(a, b.double().cpu().numpy(), TOL_BF16, nm)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_geo_backward_reusing_the_forward_workspace(dtype):
    # ssc_geo_coupling_bwd_reuse takes the patch-major operands and the schedule
    # from the forward's workspace; the results match the rebuilding call (up to
    # the order of the atomic dK / dQ additions) and the oracle
    pair = synth.make_workload("geo_60k", n=5000)
    P, R = 40, 6
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    t = _geo_tables(pair, P, R, dtype)
    (Q, K, V, dO), (Q64, K64, V64, dO64) = _inputs(pair.F_N, pair.F_M, pair.Phi_M, pair.dO, dtype)
    tabs = [as_i32(t[x]) for x in ("off_N", "mem_N", "off_M", "mem_M", "topk")]
    dt = 0 if dtype == "bf16" else 1
    nb = api.lib().ssc_geo_coupling_workspace_size(pair.n, pair.n, pair.d, pair.k, P, P, R, dt)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    O, lse = api.ssc_geo_coupling_fwd(Q, K, V, pair.scale, *tabs, workspace=ws)
    got = api.ssc_geo_coupling_bwd(Q, K, V, O, lse, dO, pair.scale, *tabs, need_dV=True,
                                   workspace=ws, reuse_forward=True)
    again = api.ssc_geo_coupling_bwd(Q, K, V, O, lse, dO, pair.scale, *tabs, need_dV=True,
                                     workspace=ws, reuse_forward=True)
    plain = api.ssc_geo_coupling_bwd(Q, K, V, O, lse, dO, pair.scale, *tabs, need_dV=True)
    _status_ok()
    ref = oracle.geo_bwd(Q64, K64, V64, dO64, pair.scale, t["off_N"], t["mem_N"], t["off_M"],
                         t["mem_M"], t["topk"])
    for a, b, c, nm in zip(got, again, plain, ("dQ", "dK", "dV")):
        assert_close(a, ref[nm], tol, nm)
        for other in (b, c):
            np.testing.assert_allclose(a.cpu().numpy(), other.cpu().numpy(), rtol=1e-4, atol=1e-6)
    with pytest.raises(ValueError):
        api.ssc_geo_coupling_bwd(Q, K, V, O, lse, dO, pair.scale, *tabs, reuse_forward=True)
    # the workspace holds the fingerprint of the forward that filled it: a reuse
    # call with other operands (here another copy of Q) is reported on the device
    api.ssc_device_status(clear=True)
    Q2 = Q.clone()
    api.ssc_geo_coupling_bwd(Q2, K, V, O, lse, dO, pair.scale, *tabs, workspace=ws,
                             reuse_forward=True)
    assert api.ssc_device_status(clear=True) == 1  # SSC_ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["geo_60k", "geo_160k_warped"])
def test_geo_bf16_full_size(name):
    pair = synth.make_workload(name)
    _geo_case(pair, pair.P, pair.R, "bf16", need_dV=True)


def test_geo_end_to_end_from_gpu_tables():
    pair = synth.make_workload("geo_60k", n=8000)
    (Q, K, V, dO), (Q64, K64, V64, dO64) = _inputs(pair.F_N, pair.F_M, pair.Phi_M, pair.dO, "bf16")
    _, _, offN, memN = api.ssc_fps_patches(torch.tensor(pair.pts_N).cuda(), 64)
    _, _, offM, memM = api.ssc_fps_patches(torch.tensor(pair.pts_M).cuda(), 64)
    topk = api.ssc_patch_scores_topk(Q, K, offN, memN, offM, memM, 8)
    O, lse = api.ssc_geo_coupling_fwd(Q, K, V, pair.scale, offN, memN, offM, memM, topk)
    _status_ok()
    t = oracle.patch_pipeline(pair.pts_N, pair.pts_M, Q64, K64, 64, 64, 8)
    np.testing.assert_array_equal(topk.cpu().numpy(), t["topk"])
    O64, lse64 = oracle.geo_fwd(Q64, K64, V64, pair.scale, t["off_N"], t["mem_N"], t["off_M"],
                                t["mem_M"], t["topk"])
    assert_close(O, O64, TOL_BF16, "O")
    assert_close(lse, lse64, TOL_BF16, "lse")


def test_geo_step_captured_in_a_cuda_graph():
    # scores/top-R + forward + reusing backward, captured once and replayed: the
    # side-stream launches (gather beside the schedule, zeroing beside the row
    # prep) join the capture; a replay after new values are copied into the
    # same input buffers matches the oracle on those values
    pair = synth.make_workload("geo_60k", n=6000)
    P, R = 48, 8
    (Q, K, V, dO), _ = _inputs(pair.F_N, pair.F_M, pair.Phi_M, pair.dO, "bf16")
    t0 = _geo_tables(pair, P, R, "bf16")
    offN, memN, offM, memM = [as_i32(t0[x]) for x in ("off_N", "mem_N", "off_M", "mem_M")]
    nb = api.lib().ssc_geo_coupling_workspace_size(pair.n, pair.n, pair.d, pair.k, P, P, R, 0)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")

    def step():
        topk = api.ssc_patch_scores_topk(Q, K, offN, memN, offM, memM, R)
        O, lse = api.ssc_geo_coupling_fwd(Q, K, V, pair.scale, offN, memN, offM, memM, topk,
                                          workspace=ws)
        dQ, dK, _ = api.ssc_geo_coupling_bwd(Q, K, V, O, lse, dO, pair.scale, offN, memN, offM,
                                             memM, topk, workspace=ws, reuse_forward=True)
        return topk, O, lse, dQ, dK

    eager = step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=cs):
        out = step()
    g.replay()
    _status_ok()
    np.testing.assert_array_equal(out[0].cpu().numpy(), eager[0].cpu().numpy())
    for a, b in zip(out[1:3], eager[1:3]):
        np.testing.assert_array_equal(a.cpu().numpy(), b.cpu().numpy())
    for a, b in zip(out[3:], eager[3:]):
        np.testing.assert_allclose(a.cpu().numpy(), b.cpu().numpy(), rtol=1e-4, atol=1e-6)
    # new operand values in the captured buffers (another seed of the same recipe)
    other = synth.make_workload("geo_60k", n=6000, seed=11)
    (Q2, K2, V2, dO2), (Q64, K64, V64, dO64) = _inputs(other.F_N, other.F_M, other.Phi_M, other.dO,
                                                       "bf16")
    for dst, src in ((Q, Q2), (K, K2), (V, V2), (dO, dO2)):
        dst.copy_(src)
    g.replay()
    _status_ok()
    t = oracle.patch_pipeline(pair.pts_N, pair.pts_M, Q64, K64, P, P, R)
    np.testing.assert_array_equal(out[0].cpu().numpy(), t["topk"])
    ref = oracle.geo_bwd(Q64, K64, V64, dO64, pair.scale, t["off_N"], t["mem_N"], t["off_M"],
                         t["mem_M"], t["topk"])
    for a, nm in zip(out[1:], ("O", "lse", "dQ", "dK")):
        assert_close(a, ref[nm], TOL_BF16, nm)
    del g


def test_constant_eigenfunction_reproduced():
    # rows of Pi sum to one, so the constant column Y_00 of Phi comes back exactly
    # up to the bf16 rounding of P (relative 2^-8 at worst per element)
    p = synth.make_workload("dense_10k", n=2000)
    (Q, K, V, _), _ = _inputs(p.F_N, p.F_M, p.Phi_M, p.dO, "bf16")
    O, _ = api.ssc_dense_coupling_fwd(Q, K, V, p.scale)
    y00 = float(V[0, 0].float())
    assert np.abs(O[:, 0].cpu().numpy() - y00).max() < 4e-3 * y00


def test_wait_timeout_reports_status_without_fault():
    api.ssc_device_status(clear=True)
    api.ssc_debug_wait_timeout(2_000_000)  # 2 ms, nothing ever arrives
    assert api.ssc_device_status(clear=True) == 6
    # the context is still usable
    Qn, Kn, Vn, dOn = synth.random_inputs(130, 140, 64, 16, seed=1)
    _dense_case(Qn, Kn, Vn, dOn, 0.125, "bf16", need_dV=False)


@pytest.mark.parametrize("which", [1, 2])
def test_coupling_kernel_abort_path_leaves_context_usable(which):
    # The library's abort-path hook stalls the MMA issuer of the next forward
    # (1) or dQ/dK backward (2) tensor-core launch on a barrier nothing arrives
    # at.  The bounded wait gives up after the wait limit: the launch ends with
    # the timeout status (every role left its loop, the MMAs drained, TMEM was
    # freed), and the same calls right after it give the oracle's results.
    pair = synth.make_workload("geo_60k", n=3000)
    P, R = 24, 5
    t = _geo_tables(pair, P, R, "bf16")
    (Q, K, V, dO), (Q64, K64, V64, dO64) = _inputs(pair.F_N, pair.F_M, pair.Phi_M, pair.dO, "bf16")
    tabs = [as_i32(t[x]) for x in ("off_N", "mem_N", "off_M", "mem_M", "topk")]
    api.ssc_device_status(clear=True)
    api.ssc_set_wait_limit_ns(50_000_000)  # 50 ms
    try:
        api.ssc_debug_stall_next_launch(which)
        O, lse = api.ssc_geo_coupling_fwd(Q, K, V, pair.scale, *tabs)
        api.ssc_geo_coupling_bwd(Q, K, V, O, lse, dO, pair.scale, *tabs)
        assert api.ssc_device_status(clear=True) == 6
    finally:
        api.ssc_debug_stall_next_launch(0)
        api.ssc_set_wait_limit_ns(0)
    O, lse = api.ssc_geo_coupling_fwd(Q, K, V, pair.scale, *tabs)
    dQ, dK, _ = api.ssc_geo_coupling_bwd(Q, K, V, O, lse, dO, pair.scale, *tabs)
    _status_ok()
    ref = oracle.geo_bwd(Q64, K64, V64, dO64, pair.scale, t["off_N"], t["mem_N"], t["off_M"],
                         t["mem_M"], t["topk"])
    assert_close(O, ref["O"], TOL_BF16, "O")
    assert_close(dQ, ref["dQ"], TOL_BF16, "dQ")
    assert_close(dK, ref["dK"], TOL_BF16, "dK")


def test_profile_record_times_each_coupling_launch():
    torch.manual_seed(0)
    n, d, k = 3000, 128, 196
    Q = torch.randn(n, d).to(torch.bfloat16).cuda()
    K = torch.randn(n, d).to(torch.bfloat16).cuda()
    V = torch.randn(n, k).to(torch.bfloat16).cuda()
    dO = torch.randn(n, k).cuda()
    api.ssc_profile_enable(True)
    for _ in range(2):
        O, lse = api.ssc_dense_coupling_fwd(Q, K, V, 1.0 / math.sqrt(d))
        api.ssc_dense_coupling_bwd(Q, K, V, O, lse, dO, 1.0 / math.sqrt(d))
    api.ssc_profile_enable(False)
    api.ssc_dense_coupling_fwd(Q, K, V, 1.0 / math.sqrt(d))  # not recorded
    fwd_ms, fwd_n = api.ssc_profile_read(api.PROF_DENSE_FWD)
    bwd_ms, bwd_n = api.ssc_profile_read(api.PROF_BWD_DQK)
    assert (fwd_n, bwd_n) == (2, 2)
    assert fwd_ms > 0 and bwd_ms > 0
    assert api.ssc_profile_read(api.PROF_BWD_DV) == (0.0, 0)
