"""GPU parity of geodesic FPS on a mesh graph against the oracle: centres,
owners and patch tables bit-exact (ai4snews digest of "Spatial-Spectral
Coupling as Attention", "Interpretation": geodesic farthest-point sampling;
project page, "Geo-FlashAttention": geodesic patches; distances are shortest
paths along mesh edges)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from spatial_spectral_attention_b200 import api, synth

pytestmark = pytest.mark.gpu

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


def _gpu(off, adj, w, P, seed=0):
    t = (torch.tensor(off, dtype=torch.int32).cuda(), torch.tensor(adj, dtype=torch.int32).cuda(),
         torch.tensor(w, dtype=torch.float64).cuda())
    out = api.ssc_fps_patches_mesh(*t, P, seed)
    torch.cuda.synchronize()
    return [x.cpu().numpy() for x in out]


def _tables(owner, P):
    """Patch tables of an owner array; vertices without a patch (-1) after the
    last patch, ascending."""
    key = np.where(owner < 0, P, owner)
    mem = np.lexsort((np.arange(owner.shape[0]), key)).astype(np.int32)
    off = np.searchsorted(key[mem], np.arange(P + 1), side="left").astype(np.int32)
    return off, mem


def _check(off, adj, w, P, seed=0):
    c, o, offs, mem = _gpu(off, adj, w, P, seed)
    assert api.ssc_device_status() == 0
    rc, ro, _ = oracle.fps_mesh(off, adj, w, P, seed)
    roff, rmem = _tables(ro, P)
    np.testing.assert_array_equal(c, rc)
    np.testing.assert_array_equal(o, ro)
    np.testing.assert_array_equal(offs, roff)
    np.testing.assert_array_equal(mem, rmem)


def test_golden_graphs():
    g = json.load(open(os.path.join(HERE, "golden", "fps_mesh_graphs.json")))
    for graph in g["graphs"]:
        off, adj, w = _csr(graph["n"], graph["edges"])
        for case in graph["cases"]:
            c, o, _, _ = _gpu(off, adj, w, case["P"], graph["seed"])
            assert c.tolist() == case["centers"], graph["name"]
            assert o.tolist() == case["owner"], graph["name"]


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_random_graphs_with_integer_lengths(seed):
    rng = np.random.default_rng(seed)
    n = 3000
    edges = [(i, i + 1) for i in range(n - 1)]
    extra = rng.integers(0, n, size=(4 * n, 2))
    edges += [(int(a), int(b)) for a, b in extra if a != b]
    edges = sorted({(min(a, b), max(a, b)) for a, b in edges})
    w = rng.integers(1, 9, size=len(edges)).astype(np.float64)
    off, adj, ww = _csr(n, edges, w)
    for P in (1, 37, 500):
        _check(off, adj, ww, P, seed)


@pytest.mark.parametrize("n,P", [(2000, 16), (20000, 160)])
def test_sphere_meshes(n, P):
    pts = synth.sphere_points(n, np.random.default_rng(n)).astype(np.float32)
    off, adj, w = synth.sphere_mesh(pts)
    _check(off, adj, w, P)


def test_sphere_mesh_60k_workload():
    p = synth.make_workload("geo_60k")
    off, adj, w = synth.sphere_mesh(p.pts_N)
    _check(off, adj, w, p.P)


def test_disconnected_parts_and_zero_length_edges():
    off, adj, w = _csr(9, [(0, 1), (1, 2), (2, 0), (3, 4), (4, 5), (5, 3), (6, 7), (7, 8)],
                       [1, 2, 3, 0.5, 0.0, 0.25, 1, 1])
    for P in (1, 2, 3, 9):
        _check(off, adj, w, P, seed=4)


def test_bad_edge_is_reported_without_fault():
    off, adj, w = _csr(5, [(0, 1), (1, 2), (2, 3), (3, 4)])
    w = w.copy()
    w[0] = -1.0
    api.ssc_device_status(clear=True)
    _gpu(off, adj, w, 2)
    assert api.ssc_device_status() == 1
