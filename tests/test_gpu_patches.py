"""GPU parity of the patch pipeline: FPS, patch assignment, patch tables,
pooling, scores and top-R, bit-exact against the fp64 oracle (project page of
"Spatial-Spectral Coupling as Attention", section Geo-FlashAttention)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from spatial_spectral_attention_b200 import api, synth

from _util import as_i32, rounded

pytestmark = pytest.mark.gpu
GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gpu_fps(pts, P, seed=0):
    c, o, off, mem = api.ssc_fps_patches(torch.tensor(pts).cuda(), P, seed)
    torch.cuda.synchronize()
    assert api.ssc_device_status() == 0
    return [t.cpu().numpy() for t in (c, o, off, mem)]


def _check_fps(pts, P, seed=0):
    c, o, off, mem = _gpu_fps(pts, P, seed)
    rc, ro, _ = oracle.fps(pts, P, seed)
    roff, rmem = oracle.csr(ro, P)
    np.testing.assert_array_equal(c, rc)
    np.testing.assert_array_equal(o, ro)
    np.testing.assert_array_equal(off, roff)
    np.testing.assert_array_equal(mem, rmem)


@pytest.mark.parametrize("name", ["fps_octahedron.json", "fps_cube.json"])
def test_fps_golden(name):
    g = json.load(open(os.path.join(GOLD, name)))
    if "points" in g:
        pts = np.array(g["points"], np.float32)
    else:
        pts = (np.array(g["signs"], np.float32) * np.float32(1 / np.sqrt(3))).astype(np.float32)
    for case in g["cases"]:
        c, o, _, _ = _gpu_fps(pts, case["P"], g["seed"])
        assert c.tolist() == case["centers"]
        assert o.tolist() == case["owner"]


@pytest.mark.parametrize("n,P,seed", [(1, 1, 0), (300, 300, 0), (1000, 37, 5), (5000, 100, 0),
                                      (20000, 1, 0), (33000, 257, 11)])
def test_fps_matches_oracle(n, P, seed):
    pts = synth.sphere_points(n, np.random.default_rng(n + P)).astype(np.float32)
    _check_fps(pts, P, seed)


def test_fps_workload_sizes():
    for name in ("geo_60k", "geo_160k_warped"):
        pair = synth.make_workload(name)
        _check_fps(pair.pts_M, pair.P)
        _check_fps(pair.pts_N, pair.P)


def test_fps_beyond_on_chip_capacity_uses_memory_path():
    # more points than a 16-CTA cluster holds on chip (262144)
    pts = synth.sphere_points(300000, np.random.default_rng(1)).astype(np.float32)
    _check_fps(pts, 40)


def _tables(pair, P):
    _, oN, _ = oracle.fps(pair.pts_N, P)
    _, oM, _ = oracle.fps(pair.pts_M, P)
    return oracle.csr(oN, P), oracle.csr(oM, P)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("n,P,R", [(6000, 48, 8), (2000, 16, 16), (3000, 30, 1)])
def test_scores_topk_match_oracle(dtype, n, P, R):
    pair = synth.make_workload("geo_60k", n=n)
    (offN, memN), (offM, memM) = _tables(pair, P)
    FN, FN64 = rounded(pair.F_N, dtype)
    FM, FM64 = rounded(pair.F_M, dtype)
    topk, sc = api.ssc_patch_scores_topk(FN, FM, as_i32(offN), as_i32(memN), as_i32(offM),
                                         as_i32(memM), R, return_scores=True)
    rsc = oracle.scores(oracle.pool(FN64, offN, memN), oracle.pool(FM64, offM, memM))
    np.testing.assert_array_equal(sc.cpu().numpy(), rsc)  # bit-exact fp64
    np.testing.assert_array_equal(topk.cpu().numpy(), oracle.topk(rsc, R))


def test_scores_topk_ties_go_to_lower_patch():
    # patches 1 and 3 get identical member descriptors, so identical means and scores
    n, d, P = 40, 64, 5
    owner = np.repeat(np.arange(P), n // P).astype(np.int32)
    off, mem = oracle.csr(owner, P)
    rng = np.random.default_rng(0)
    F = rng.standard_normal((n, d)).astype(np.float32)
    F[mem[off[3]:off[4]]] = F[mem[off[1]:off[2]]]
    FN, _ = rounded(F, "f32")
    topk, sc = api.ssc_patch_scores_topk(FN, FN, as_i32(off), as_i32(mem), as_i32(off),
                                         as_i32(mem), P, return_scores=True)
    sc = sc.cpu().numpy()
    assert np.all(sc[:, 1] == sc[:, 3])
    rsc = oracle.scores(oracle.pool(F.astype(np.float64), off, mem),
                        oracle.pool(F.astype(np.float64), off, mem))
    ref = oracle.topk(rsc, P)
    np.testing.assert_array_equal(topk.cpu().numpy(), ref)
    for row in ref:
        assert list(row).index(1) < list(row).index(3)


@pytest.mark.parametrize("name", ["geo_60k", "geo_160k_warped"])
def test_pipeline_workload_sizes_bit_exact(name):
    pair = synth.make_workload(name)
    FN, FN64 = rounded(pair.F_N, "bf16")
    FM, FM64 = rounded(pair.F_M, "bf16")
    _, _, offN, memN = api.ssc_fps_patches(torch.tensor(pair.pts_N).cuda(), pair.P)
    _, _, offM, memM = api.ssc_fps_patches(torch.tensor(pair.pts_M).cuda(), pair.P)
    topk = api.ssc_patch_scores_topk(FN, FM, offN, memN, offM, memM, pair.R)
    ref = oracle.patch_pipeline(pair.pts_N, pair.pts_M, FN64, FM64, pair.P, pair.P, pair.R)
    np.testing.assert_array_equal(offN.cpu().numpy(), ref["off_N"])
    np.testing.assert_array_equal(memM.cpu().numpy(), ref["mem_M"])
    np.testing.assert_array_equal(topk.cpu().numpy(), ref["topk"])
