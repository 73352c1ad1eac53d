"""Pins of the oracle's patch pipeline (CPU only).

Each check ties the oracle to something other than itself: hand-worked golden
cases, brute force on the geodesic (arccos) distance, numpy's stable sort and
lexsort, numpy's mean and dot within their rounding bounds, and invariants of
farthest-point sampling.  Definitions: project page of "Spatial-Spectral
Coupling as Attention", section Geo-FlashAttention; digest, Interpretation.
"""
import json
import os

import numpy as np
import pytest

import oracle
from spatial_spectral_attention_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def test_fps_octahedron_golden():
    g = _gold("fps_octahedron.json")
    pts = np.array(g["points"], np.float32)
    for c in g["cases"]:
        centers, owner, _ = oracle.fps(pts, c["P"], g["seed"])
        assert centers.tolist() == c["centers"], c
        assert owner.tolist() == c["owner"], c


def test_fps_cube_golden():
    g = _gold("fps_cube.json")
    a = np.float32(1.0 / np.sqrt(3.0))
    pts = (np.array(g["signs"], np.float32) * a).astype(np.float32)
    for c in g["cases"]:
        centers, owner, _ = oracle.fps(pts, c["P"], g["seed"])
        assert centers.tolist() == c["centers"], c
        assert owner.tolist() == c["owner"], c


def _brute_fps_geodesic(pts, P, seed):
    """FPS on great-circle distance arccos(<x,y>) with a full distance matrix."""
    x = pts.astype(np.float64)
    G = np.clip(x @ x.T, -1.0, 1.0)
    dist = np.arccos(G)
    centers = [seed]
    mind = dist[seed].copy()
    mind[seed] = -1.0
    for _ in range(1, P):
        cand = np.where(np.isin(np.arange(len(x)), centers), -np.inf, mind)
        c = int(np.argmax(cand))           # first maximum = lowest index
        centers.append(c)
        mind = np.minimum(mind, dist[c])
    own = np.argmin(dist[:, centers], axis=1)  # first minimum = lowest patch
    own[centers] = np.arange(P)
    return np.array(centers), own


@pytest.mark.parametrize("n,P,seed", [(50, 7, 0), (200, 25, 0), (200, 200, 3), (97, 1, 5)])
def test_fps_matches_geodesic_brute_force(n, P, seed):
    rng = np.random.default_rng(n * 31 + P)
    pts = synth.sphere_points(n, rng).astype(np.float32)
    centers, owner, _ = oracle.fps(pts, P, seed)
    bc, bo = _brute_fps_geodesic(pts, P, seed)
    assert centers.tolist() == bc.tolist()
    assert owner.tolist() == bo.tolist()


def test_fps_invariants():
    rng = np.random.default_rng(7)
    pts = synth.sphere_points(3000, rng).astype(np.float32)
    P = 120
    centers, owner, maxdot = oracle.fps(pts, P, 0)
    assert len(set(centers.tolist())) == P
    assert centers[0] == 0
    # every patch non-empty and each centre in its own patch
    assert np.all(np.bincount(owner, minlength=P) >= 1)
    assert np.all(owner[centers] == np.arange(P))
    x = pts.astype(np.float64)
    # covering radius (largest distance to the nearest centre) never grows
    radius = []
    best = np.full(len(x), -np.inf)
    for t in range(P):
        best = np.maximum(best, x @ x[centers[t]])
        radius.append(np.arccos(np.clip(best.min(), -1, 1)))
    assert all(radius[i + 1] <= radius[i] + 1e-15 for i in range(P - 1))
    # each new centre was the farthest point from the previous ones
    best = np.full(len(x), -np.inf)
    for t in range(P - 1):
        best = np.maximum(best, x @ x[centers[t]])
        cand = best.copy()
        cand[centers[:t + 1]] = np.inf
        assert abs(cand.min() - best[centers[t + 1]]) < 1e-12


def test_csr_matches_stable_sort():
    rng = np.random.default_rng(3)
    owner = rng.integers(0, 37, size=5000).astype(np.int32)
    owner[:37] = np.arange(37)
    off, mem = oracle.csr(owner, 37)
    assert off.tolist() == np.concatenate([[0], np.cumsum(np.bincount(owner, minlength=37))]).tolist()
    assert mem.tolist() == np.argsort(owner, kind="stable").tolist()


def test_pool_matches_mean_and_is_exact_on_dyadic_values():
    rng = np.random.default_rng(11)
    n, d, P = 4000, 16, 30
    owner = rng.integers(0, P, size=n).astype(np.int32)
    owner[:P] = np.arange(P)
    off, mem = oracle.csr(owner, P)
    F = rng.standard_normal((n, d)).astype(np.float32)
    mu = oracle.pool(F, off, mem)
    for p in range(P):
        ref = F[mem[off[p]:off[p + 1]]].astype(np.float64).mean(axis=0)
        np.testing.assert_allclose(mu[p], ref, rtol=1e-13, atol=1e-15)
    # small integers: every partial sum is exact; mean of a power-of-two count is exact
    Fi = rng.integers(-8, 9, size=(n, d)).astype(np.float32)
    mu_i = oracle.pool(Fi, off, mem)
    for p in range(P):
        rows = mem[off[p]:off[p + 1]]
        assert np.array_equal(mu_i[p], Fi[rows].astype(np.float64).sum(0) / len(rows))


def test_scores_match_numpy_dot():
    rng = np.random.default_rng(5)
    muN = rng.standard_normal((40, 128))
    muM = rng.standard_normal((33, 128))
    sc = oracle.scores(muN, muM)
    np.testing.assert_allclose(sc, muN @ muM.T, rtol=1e-12, atol=1e-12)
    # dyadic inputs: exact
    a = rng.integers(-4, 5, size=(6, 8)).astype(np.float64) / 4
    b = rng.integers(-4, 5, size=(5, 8)).astype(np.float64) / 8
    assert np.array_equal(oracle.scores(a, b), a @ b.T)


def test_topk_golden_ties():
    g = _gold("topk_ties.json")
    sc = np.array(g["scores"], np.float64)
    for c in g["cases"]:
        assert oracle.topk(sc, c["R"]).tolist() == c["topk"], c


def _lexsort_topk(sc, R):
    q = np.arange(sc.shape[1])
    return np.stack([np.lexsort((q, -row))[:R] for row in sc])


@pytest.mark.parametrize("R", [1, 3, 8, 50])
def test_topk_matches_lexsort_with_ties(R):
    rng = np.random.default_rng(R)
    sc = rng.integers(-5, 6, size=(64, 50)).astype(np.float64)  # many exact ties
    assert oracle.topk(sc, R).tolist() == _lexsort_topk(sc, R).tolist()
    sc2 = rng.standard_normal((64, 50))
    assert oracle.topk(sc2, R).tolist() == _lexsort_topk(sc2, R).tolist()


def test_duplicate_patch_means_tie_to_lower_index():
    # two source patches with identical members' descriptors give equal scores
    F = np.array([[1, 0], [1, 0], [0, 1], [1, 0]], np.float32)
    owner = np.array([0, 1, 2, 1], np.int32)
    off, mem = oracle.csr(owner, 3)
    mu = oracle.pool(F, off, mem)
    sc = oracle.scores(np.array([[2.0, 0.0]]), mu)
    assert sc[0, 0] == sc[0, 1]
    assert oracle.topk(sc, 2).tolist() == [[0, 1]]


def test_pipeline_on_workload_shapes_are_consistent():
    pair = synth.make_workload("geo_60k", n=6000)
    out = oracle.patch_pipeline(pair.pts_N, pair.pts_M, pair.F_N, pair.F_M,
                                pair.P, pair.P, pair.R)
    for side in "NM":
        off, mem = out["off_" + side], out["mem_" + side]
        assert off[-1] == pair.n and np.all(np.diff(off) >= 1)
        assert sorted(mem.tolist()) == list(range(pair.n))
    t = out["topk"]
    assert t.shape == (pair.P, pair.R)
    assert all(len(set(r)) == pair.R for r in t.tolist())
