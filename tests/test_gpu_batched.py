"""GPU parity of the batched calls (several shape pairs per launch) and of the
reverse coupling Pi_MN Phi_N, against the fp64 oracle pair by pair ("Spatial-
Spectral Coupling as Attention", project page, Table 1: one training step of a
functional-map pipeline couples every pair of its batch; "Spatial-spectral
coupling is attention" for the definition in either direction)."""
import math

import numpy as np
import pytest
import torch

import oracle
from spatial_spectral_attention_b200 import api, synth

from _util import TOL_BF16, TOL_F32, assert_close

pytestmark = pytest.mark.gpu


def _stack(arrs, dtype):
    t = torch.tensor(np.ascontiguousarray(np.stack(arrs), dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.cuda(), t.double().numpy()


def _status():
    torch.cuda.synchronize()
    return api.ssc_device_status()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_dense_batched_matches_oracle_pair_by_pair(dtype):
    B, nN, nM, d, k = 3, 700, 900, 128, 196
    ins = [synth.random_inputs(nN, nM, d, k, seed=40 + b, q_scale=0.5) for b in range(B)]
    (Q, Q64), (K, K64), (V, V64) = (_stack([x[i] for x in ins], dtype) for i in range(3))
    dO = torch.tensor(np.stack([x[3] for x in ins])).cuda()
    dO64 = (dO.to(torch.bfloat16) if dtype == "bf16" else dO).double().cpu().numpy()
    s = 1.0 / math.sqrt(d)
    O, lse = api.ssc_dense_coupling_fwd_batched(Q, K, V, s)
    dQ, dK, dV = api.ssc_dense_coupling_bwd_batched(Q, K, V, O, lse, dO, s, need_dV=True)
    assert _status() == 0
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    for b in range(B):
        ref = oracle.dense_bwd(Q64[b], K64[b], V64[b], dO64[b], s)
        for t, nm in ((O, "O"), (lse, "lse"), (dQ, "dQ"), (dK, "dK"), (dV, "dV")):
            assert_close(t[b], ref[nm], tol, f"pair {b} {nm}")


def _geo_batch(B, n, P, R, seed0):
    pairs = [synth.make_workload("geo_60k", n=n, seed=seed0 + b) for b in range(B)]
    Q, Q64 = _stack([p.F_N for p in pairs], "bf16")
    K, K64 = _stack([p.F_M for p in pairs], "bf16")
    V, V64 = _stack([p.Phi_M for p in pairs], "bf16")
    dO = torch.tensor(np.stack([p.dO for p in pairs])).cuda()
    dO64 = dO.to(torch.bfloat16).double().cpu().numpy()
    tabs = [oracle.patch_pipeline(p.pts_N, p.pts_M, Q64[b], K64[b], P, P, R)
            for b, p in enumerate(pairs)]
    return pairs, (Q, K, V, dO), (Q64, K64, V64, dO64), tabs


def _i32(arrs):
    return torch.tensor(np.ascontiguousarray(np.stack(arrs), dtype=np.int32)).cuda()


def test_geo_batched_matches_oracle_pair_by_pair():
    B, n, P, R = 3, 3000, 24, 4
    pairs, (Q, K, V, dO), (Q64, K64, V64, dO64), tabs = _geo_batch(B, n, P, R, 70)
    g = [_i32([t[x] for t in tabs]) for x in ("off_N", "mem_N", "off_M", "mem_M", "topk")]
    s = pairs[0].scale
    O, lse = api.ssc_geo_coupling_fwd_batched(Q, K, V, s, *g)
    dQ, dK, dV = api.ssc_geo_coupling_bwd_batched(Q, K, V, O, lse, dO, s, *g, need_dV=True)
    assert _status() == 0
    for b, t in enumerate(tabs):
        ref = oracle.geo_bwd(Q64[b], K64[b], V64[b], dO64[b], s, t["off_N"], t["mem_N"],
                             t["off_M"], t["mem_M"], t["topk"])
        for x, nm in ((O, "O"), (lse, "lse"), (dQ, "dQ"), (dK, "dK"), (dV, "dV")):
            assert_close(x[b], ref[nm], TOL_BF16, f"pair {b} {nm}")


def test_scores_topk_batched_bit_exact():
    B, n, P, R = 4, 2500, 20, 5
    pairs, (Q, K, V, _), (Q64, K64, _, _), tabs = _geo_batch(B, n, P, R, 90)
    g = [_i32([t[x] for t in tabs]) for x in ("off_N", "mem_N", "off_M", "mem_M")]
    topk, sc = api.ssc_patch_scores_topk_batched(Q, K, *g, R, return_scores=True)
    assert _status() == 0
    for b, t in enumerate(tabs):
        np.testing.assert_array_equal(topk[b].cpu().numpy(), t["topk"])
        np.testing.assert_array_equal(sc[b].cpu().numpy(), t["scores"])


def test_reverse_coupling_in_one_batch_with_the_forward_direction():
    # pair 0: Pi_NM Phi_M (Q = F_N, K = F_M); pair 1: Pi_MN Phi_N (Q = F_M,
    # K = F_N, V = the target eigenbasis)
    p = synth.make_workload("dense_10k", n=1500)
    Phi_N = synth.real_sph_harm(p.pts_N.astype(np.float64), p.meta["L"]).astype(np.float32)
    Q, Q64 = _stack([p.F_N, p.F_M], "bf16")
    K, K64 = _stack([p.F_M, p.F_N], "bf16")
    V, V64 = _stack([p.Phi_M, Phi_N], "bf16")
    dO = torch.tensor(np.stack([p.dO, p.dO[::-1].copy()])).cuda()
    dO64 = dO.to(torch.bfloat16).double().cpu().numpy()
    O, lse = api.ssc_dense_coupling_fwd_batched(Q, K, V, p.scale)
    dQ, dK, _ = api.ssc_dense_coupling_bwd_batched(Q, K, V, O, lse, dO, p.scale)
    assert _status() == 0
    for b in range(2):
        ref = oracle.dense_bwd(Q64[b], K64[b], V64[b], dO64[b], p.scale)
        for x, nm in ((O, "O"), (lse, "lse"), (dQ, "dQ"), (dK, "dK")):
            assert_close(x[b], ref[nm], TOL_BF16, f"direction {b} {nm}")
    # the reverse Geo coupling: M tables as the target tables, top-R scored from F_M
    P, R = 12, 3
    t = oracle.patch_pipeline(p.pts_M, p.pts_N, Q64[1], K64[1], P, P, R)
    tabs = [torch.tensor(t[x], dtype=torch.int32).cuda()
            for x in ("off_N", "mem_N", "off_M", "mem_M")]
    topk = api.ssc_patch_scores_topk(Q[1], K[1], *tabs, R)
    np.testing.assert_array_equal(topk.cpu().numpy(), t["topk"])
    Og, lseg = api.ssc_geo_coupling_fwd(Q[1], K[1], V[1], p.scale, *tabs, topk)
    assert _status() == 0
    Or, lser = oracle.geo_fwd(Q64[1], K64[1], V64[1], p.scale, t["off_N"], t["mem_N"], t["off_M"],
                              t["mem_M"], t["topk"])
    assert_close(Og, Or, TOL_BF16, "reverse Geo O")
    assert_close(lseg, lser, TOL_BF16, "reverse Geo lse")


def test_bad_entry_of_one_pair_stays_in_that_pair():
    B, n, P, R = 2, 2000, 16, 3
    pairs, (Q, K, V, _), (Q64, K64, V64, _), tabs = _geo_batch(B, n, P, R, 110)
    topk = np.stack([t["topk"] for t in tabs])
    topk[1, 0, 0] = P  # one past the last source patch of pair 1
    g = [_i32([t[x] for t in tabs]) for x in ("off_N", "mem_N", "off_M", "mem_M")]
    api.ssc_device_status(clear=True)
    O, lse = api.ssc_geo_coupling_fwd_batched(Q, K, V, pairs[0].scale, *g, _i32(list(topk)))
    assert _status() == 1  # SSC_ERR_INVALID_ARG reported, nothing faulted
    t = tabs[0]
    Or, lser = oracle.geo_fwd(Q64[0], K64[0], V64[0], pairs[0].scale, t["off_N"], t["mem_N"],
                              t["off_M"], t["mem_M"], t["topk"])
    assert_close(O[0], Or, TOL_BF16, "pair 0 O")
    assert_close(lse[0], lser, TOL_BF16, "pair 0 lse")
