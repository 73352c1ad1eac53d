"""Pins of the oracle's mesh-geodesic FPS (CPU only).

Definition: ai4snews digest of "Spatial-Spectral Coupling as Attention",
"Interpretation" (geodesic farthest-point sampling) and project page,
"Geo-FlashAttention" (geodesic patches); distances read as shortest paths
along mesh edges.

The oracle is tied to: hand-worked golden graphs with ties
(tests/golden/fps_mesh_graphs.json), Floyd-Warshall on small graphs with
integer edge lengths (every sum exact, so FPS from the all-pairs matrix must
agree bit for bit), scipy's Dijkstra (a library route to the distances), the
chord lower bound on sphere meshes, disconnected graphs, and the prefix
property of farthest-point sampling.
"""
import json
import os

import numpy as np
import pytest
from scipy.sparse import csr_matrix
from scipy.sparse.csgraph import dijkstra

import oracle
from spatial_spectral_attention_b200 import synth

HERE = os.path.dirname(os.path.abspath(__file__))


def _csr(n, edges, w=None):
    e = np.asarray(edges, dtype=np.int64)
    wts = np.ones(len(e)) if w is None else np.asarray(w, dtype=np.float64)
    e2 = np.concatenate([e, e[:, ::-1]])
    w2 = np.concatenate([wts, wts])
    order = np.lexsort((e2[:, 1], e2[:, 0]))
    e2, w2 = e2[order], w2[order]
    off = np.zeros(n + 1, np.int64)
    np.add.at(off, e2[:, 0] + 1, 1)
    return np.cumsum(off).astype(np.int32), e2[:, 1].astype(np.int32), w2


def test_golden_graphs():
    g = json.load(open(os.path.join(HERE, "golden", "fps_mesh_graphs.json")))
    for graph in g["graphs"]:
        off, adj, w = _csr(graph["n"], graph["edges"])
        for case in graph["cases"]:
            c, o, _ = oracle.fps_mesh(off, adj, w, case["P"], graph["seed"])
            assert c.tolist() == case["centers"], graph["name"]
            assert o.tolist() == case["owner"], graph["name"]


def _fps_from_apsp(D, P, seed):
    """FPS and nearest-centre patches straight from an all-pairs matrix."""
    n = D.shape[0]
    best = np.full(n, np.inf)
    owner = np.full(n, -1)
    centers = []
    c = seed
    for t in range(P):
        centers.append(c)
        better = D[c] < best
        best[better] = D[c][better]
        owner[better] = t
        c = int(np.argmax(best))  # first maximum = lowest index
    return np.array(centers), owner


@pytest.mark.parametrize("seed", [1, 2, 3, 4])
def test_floyd_warshall_integer_lengths(seed):
    rng = np.random.default_rng(seed)
    n = 40
    edges = [(i, i + 1) for i in range(n - 1)]  # connected
    extra = rng.integers(0, n, size=(60, 2))
    edges += [(int(a), int(b)) for a, b in extra if a != b]
    edges = sorted({(min(a, b), max(a, b)) for a, b in edges})
    w = rng.integers(1, 9, size=len(edges)).astype(np.float64)
    off, adj, ww = _csr(n, edges, w)
    D = np.full((n, n), np.inf)
    np.fill_diagonal(D, 0.0)
    for (a, b), x in zip(edges, w):
        D[a, b] = D[b, a] = min(D[a, b], x)
    for k in range(n):
        D = np.minimum(D, D[:, k:k + 1] + D[k:k + 1, :])
    for P in (1, 7, n):
        c, o, dist = oracle.fps_mesh(off, adj, ww, P, seed % n)
        c2, o2 = _fps_from_apsp(D, P, seed % n)
        np.testing.assert_array_equal(c, c2)
        np.testing.assert_array_equal(o, o2)
        np.testing.assert_array_equal(dist, D[c].min(axis=0))


def test_single_source_matches_scipy_dijkstra():
    pts = synth.sphere_points(2000, np.random.default_rng(5)).astype(np.float32)
    off, adj, w = synth.sphere_mesh(pts)
    A = csr_matrix((w, adj, off), shape=(2000, 2000))
    for s in (0, 17, 1999):
        ref = dijkstra(A, directed=True, indices=s)
        np.testing.assert_allclose(oracle.sssp(off, adj, w, s), ref, rtol=1e-14, atol=0)


def test_sphere_mesh_distances_bound_the_chord_from_above():
    pts = synth.sphere_points(3000, np.random.default_rng(6)).astype(np.float32)
    off, adj, w = synth.sphere_mesh(pts)
    d = oracle.sssp(off, adj, w, 0)
    p = pts.astype(np.float64)
    chord = np.sqrt(((p - p[0]) ** 2).sum(axis=1))
    assert np.all(d >= chord * (1 - 1e-12))
    assert np.all(np.isfinite(d))  # a sphere mesh is connected


def test_disconnected_parts_each_receive_a_centre_first():
    off, adj, w = _csr(6, [(0, 1), (1, 2), (2, 0), (3, 4), (4, 5), (5, 3)])
    c, o, dist = oracle.fps_mesh(off, adj, w, 2, 0)
    assert c.tolist() == [0, 3]
    assert o.tolist() == [0, 0, 0, 1, 1, 1]
    c, _, _ = oracle.fps_mesh(off, adj, w, 1, 4)
    assert c.tolist() == [4]


def test_fps_is_a_prefix_and_the_covering_radius_shrinks():
    pts = synth.sphere_points(1500, np.random.default_rng(8)).astype(np.float32)
    off, adj, w = synth.sphere_mesh(pts)
    c40, _, d40 = oracle.fps_mesh(off, adj, w, 40)
    radius = []
    for P in (5, 10, 20, 39):
        c, _, d = oracle.fps_mesh(off, adj, w, P)
        np.testing.assert_array_equal(c, c40[:P])
        radius.append(d.max())
    assert all(a >= b for a, b in zip(radius, radius[1:])) and radius[-1] >= d40.max()
