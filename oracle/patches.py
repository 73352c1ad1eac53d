"""ctypes front end of the oracle's patch pipeline (patches.c), test infrastructure.

Follows "Spatial-Spectral Coupling as Attention", project page, section
"Geo-FlashAttention": partition both shapes into geodesic patches (farthest-point
sampling, digest "Interpretation"), pool source keys, score source patches and
keep the top R per target patch.  The readings taken where the pages are silent
are listed at the top of patches.c.
"""
from __future__ import annotations

import ctypes
import numpy as np

from .build import build

_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        _lib.oracle_fps.argtypes = [P, I, I, I, P, P, P]
        _lib.oracle_fps.restype = I
        _lib.oracle_csr.argtypes = [P, I, I, P, P]
        _lib.oracle_csr.restype = I
        _lib.oracle_pool.argtypes = [P, I, I, P, P, I, P]
        _lib.oracle_pool.restype = I
        _lib.oracle_scores.argtypes = [P, I, P, I, I, P]
        _lib.oracle_scores.restype = None
        _lib.oracle_topk.argtypes = [P, I, I, I, P]
        _lib.oracle_topk.restype = I
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def fps(pts: np.ndarray, P: int, seed: int = 0):
    """Farthest-point sampling on the sphere plus nearest-centre assignment.

    Returns (centers int32 [P], owner int32 [n], maxdot fp64 [n])."""
    pts = np.ascontiguousarray(pts, dtype=np.float32)
    n = pts.shape[0]
    centers = np.zeros(P, np.int32)
    owner = np.zeros(n, np.int32)
    maxdot = np.zeros(n, np.float64)
    rc = _L().oracle_fps(_p(pts), n, P, seed, _p(centers), _p(owner), _p(maxdot))
    if rc != 0:
        raise ValueError("oracle_fps: invalid arguments")
    return centers, owner, maxdot


def csr(owner: np.ndarray, P: int):
    """Patch offsets int32 [P+1] and members int32 [n] (per patch, ascending)."""
    owner = np.ascontiguousarray(owner, dtype=np.int32)
    n = owner.shape[0]
    off = np.zeros(P + 1, np.int32)
    mem = np.zeros(n, np.int32)
    if _L().oracle_csr(_p(owner), n, P, _p(off), _p(mem)) != 0:
        raise ValueError("oracle_csr: owner out of range")
    return off, mem


def pool(F: np.ndarray, off: np.ndarray, mem: np.ndarray):
    """Mean descriptor per patch, fp64 [P,d]; F is widened exactly to fp64."""
    F64 = np.ascontiguousarray(F, dtype=np.float64)
    n, d = F64.shape
    P = off.shape[0] - 1
    mu = np.zeros((P, d), np.float64)
    off = np.ascontiguousarray(off, np.int32)
    mem = np.ascontiguousarray(mem, np.int32)
    if _L().oracle_pool(_p(F64), n, d, _p(off), _p(mem), P, _p(mu)) != 0:
        raise ValueError("oracle_pool: empty patch or bad member index")
    return mu


def scores(muN: np.ndarray, muM: np.ndarray):
    """Patch score matrix fp64 [PN,PM] = <mu_N(p), mu_M(q)>."""
    muN = np.ascontiguousarray(muN, np.float64)
    muM = np.ascontiguousarray(muM, np.float64)
    PN, d = muN.shape
    PM = muM.shape[0]
    s = np.zeros((PN, PM), np.float64)
    _L().oracle_scores(_p(muN), PN, _p(muM), PM, d, _p(s))
    return s


def topk(sc: np.ndarray, R: int):
    """int32 [PN,R]: best R source patches per target patch (score desc, index asc)."""
    sc = np.ascontiguousarray(sc, np.float64)
    PN, PM = sc.shape
    t = np.zeros((PN, R), np.int32)
    if _L().oracle_topk(_p(sc), PN, PM, R, _p(t)) != 0:
        raise ValueError("oracle_topk: need 1 <= R <= PM")
    return t


def patch_pipeline(pts_N, pts_M, F_N, F_M, P_N: int, P_M: int, R: int, seed: int = 0):
    """Whole selection: FPS + assignment on both shapes, pooling, scores, top R."""
    cN, ownN, _ = fps(pts_N, P_N, seed)
    cM, ownM, _ = fps(pts_M, P_M, seed)
    offN, memN = csr(ownN, P_N)
    offM, memM = csr(ownM, P_M)
    sc = scores(pool(F_N, offN, memN), pool(F_M, offM, memM))
    return dict(centers_N=cN, owner_N=ownN, off_N=offN, mem_N=memN,
                centers_M=cM, owner_M=ownM, off_M=offM, mem_M=memM,
                scores=sc, topk=topk(sc, R))
