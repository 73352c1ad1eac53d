"""ctypes front end of the oracle's mesh-geodesic FPS (mesh.c), test infrastructure.

Follows the ai4snews digest of "Spatial-Spectral Coupling as Attention",
"Interpretation" (geodesic farthest-point sampling partitions the surface) and
the project page, "Geo-FlashAttention" (geodesic patches).  Distances are
shortest paths along the mesh edges; the readings taken where the pages are
silent are listed at the top of mesh.c.
"""
from __future__ import annotations

import ctypes

import numpy as np

from .build import build_mesh

_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build_mesh())
        P = ctypes.c_void_p
        I = ctypes.c_int
        _lib.oracle_fps_mesh.argtypes = [P, P, P, I, I, I, P, P, P]
        _lib.oracle_fps_mesh.restype = ctypes.c_long
        _lib.oracle_sssp.argtypes = [P, P, P, I, I, P]
        _lib.oracle_sssp.restype = ctypes.c_long
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _graph(off, adj, w):
    return (np.ascontiguousarray(off, np.int32), np.ascontiguousarray(adj, np.int32),
            np.ascontiguousarray(w, np.float64))


def fps_mesh(off, adj, w, P: int, seed: int = 0):
    """Geodesic FPS + nearest-centre patches on the graph (CSR off [n+1], adj
    [nnz], edge lengths w [nnz]).  Returns (centers int32 [P], owner int32 [n],
    dist fp64 [n]: each vertex's distance to its nearest centre)."""
    off, adj, w = _graph(off, adj, w)
    n = off.shape[0] - 1
    centers = np.zeros(P, np.int32)
    owner = np.zeros(n, np.int32)
    dist = np.zeros(n, np.float64)
    rc = _L().oracle_fps_mesh(_p(off), _p(adj), _p(w), n, P, seed, _p(centers), _p(owner), _p(dist))
    if rc < 0:
        raise ValueError("oracle_fps_mesh: invalid arguments")
    if rc > 0:
        raise ValueError("oracle_fps_mesh: the graph holds invalid edges")
    return centers, owner, dist


def sssp(off, adj, w, s: int):
    """Shortest-path distances fp64 [n] from vertex s (+inf where unreachable)."""
    off, adj, w = _graph(off, adj, w)
    n = off.shape[0] - 1
    dist = np.zeros(n, np.float64)
    if _L().oracle_sssp(_p(off), _p(adj), _p(w), n, s, _p(dist)) != 0:
        raise ValueError("oracle_sssp: invalid arguments or edges")
    return dist
