"""Seeded synthetic inputs for the spatial-spectral coupling.

This module only draws data: points on the unit sphere, a random rotation,
random-Fourier-feature descriptors, the real spherical-harmonic basis that plays
the role of the source Laplace-Beltrami eigenbasis, and the upstream gradient.
It holds none of the coupling's arithmetic; both the CUDA path and the oracle
consume what it returns.

Workloads (the pages' meshes and trained descriptor networks are not available,
so these sphere workloads stand in for them at the same vertex scales):

  small_fp32_2k     n=2048,   d=64,  l<=4  (k=25),  target = rotated copy of the
                    source points, F_N = F(source) + noise(var 0.05), fp32
  dense_10k         n=10000,  d=128, l<=13 (k=196), independent target draw,
                    rotated; noise var 0.05; bf16
  dense_60k         n=60000,  d=128, k=196, noise var 0.1; bf16
  geo_60k           as dense_60k, P=480 patches, R=8 selected source patches
  geo_160k_warped   n=160000, d=128, k=196, P=1280, R=8; target descriptors are
                    taken at x -> normalize(x + 0.3 sin(3x)) (non-isometric pair)

Descriptor recipe: F(x) = sin(W x + b), W ~ N(0, 4^2) (d x 3), b ~ U(0, 2 pi);
W and b are shared by both shapes.  The noise N(0, v) is read with v a
variance, matching the N(0, 4^2) notation of the same recipe.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

WORKLOADS = {
    "small_fp32_2k": dict(n=2048, d=64, L=4, noise_var=0.05, same_points=True,
                          warp=False, P=16, R=4, dtype="f32", seed=1000),
    "dense_10k": dict(n=10000, d=128, L=13, noise_var=0.05, same_points=False,
                      warp=False, P=80, R=8, dtype="bf16", seed=1001),
    "dense_60k": dict(n=60000, d=128, L=13, noise_var=0.1, same_points=False,
                      warp=False, P=480, R=8, dtype="bf16", seed=1002),
    "geo_60k": dict(n=60000, d=128, L=13, noise_var=0.1, same_points=False,
                    warp=False, P=480, R=8, dtype="bf16", seed=1003),
    "geo_160k_warped": dict(n=160000, d=128, L=13, noise_var=0.1, same_points=False,
                            warp=True, P=1280, R=8, dtype="bf16", seed=1004),
}


def sphere_points(n: int, rng: np.random.Generator) -> np.ndarray:
    """n points uniform on the unit sphere: normalised N(0, I3) draws (fp64)."""
    x = rng.standard_normal((n, 3))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def random_rotation(rng: np.random.Generator) -> np.ndarray:
    """Haar-random rotation: QR of a 3x3 Gaussian with the sign fix, det = +1."""
    a = rng.standard_normal((3, 3))
    q, r = np.linalg.qr(a)
    q = q * np.sign(np.diag(r))[None, :]
    if np.linalg.det(q) < 0:
        q[:, 0] = -q[:, 0]
    return q


def rff_params(d: int, rng: np.random.Generator):
    w = rng.normal(0.0, 4.0, size=(d, 3))
    b = rng.uniform(0.0, 2.0 * math.pi, size=(d,))
    return w, b


def rff(x: np.ndarray, w: np.ndarray, b: np.ndarray) -> np.ndarray:
    return np.sin(x @ w.T + b[None, :])


def warp_points(x: np.ndarray) -> np.ndarray:
    y = x + 0.3 * np.sin(3.0 * x)
    return y / np.linalg.norm(y, axis=1, keepdims=True)


def real_sph_harm(x: np.ndarray, L: int) -> np.ndarray:
    """Orthonormal real spherical harmonics Y_lm(x) for l <= L at unit vectors x.

    Columns are ordered (l ascending, m = -l..l), so column 0 is the constant
    Y_00 = 1/(2 sqrt(pi)).  The normalised associated Legendre functions are built
    with the standard three-term recurrence in l (no Condon-Shortley phase):
      p_mm      = sqrt((2m+1)/(2m)) sin(theta) p_{m-1,m-1},  p_00 = 1/sqrt(4 pi)
      p_{m+1,m} = sqrt(2m+3) cos(theta) p_mm
      p_lm      = a_lm (cos(theta) p_{l-1,m} - b_lm p_{l-2,m})
    with a_lm = sqrt((4l^2-1)/(l^2-m^2)), b_lm = sqrt(((l-1)^2-m^2)/(4(l-1)^2-1)).
    Y_l0 = p_l0, Y_lm = sqrt(2) p_lm cos(m phi), Y_l,-m = sqrt(2) p_lm sin(m phi).
    """
    x = np.asarray(x, dtype=np.float64)
    ct = np.clip(x[:, 2], -1.0, 1.0)
    st = np.sqrt(np.maximum(0.0, 1.0 - ct * ct))
    phi = np.arctan2(x[:, 1], x[:, 0])
    n = x.shape[0]
    p = {}
    p[(0, 0)] = np.full(n, 1.0 / math.sqrt(4.0 * math.pi))
    for m in range(1, L + 1):
        p[(m, m)] = math.sqrt((2 * m + 1) / (2.0 * m)) * st * p[(m - 1, m - 1)]
    for m in range(0, L):
        p[(m + 1, m)] = math.sqrt(2 * m + 3) * ct * p[(m, m)]
    for m in range(0, L + 1):
        for l in range(m + 2, L + 1):
            a = math.sqrt((4.0 * l * l - 1.0) / (l * l - m * m))
            bb = math.sqrt(((l - 1.0) ** 2 - m * m) / (4.0 * (l - 1.0) ** 2 - 1.0))
            p[(l, m)] = a * (ct * p[(l - 1, m)] - bb * p[(l - 2, m)])
    cols = []
    for l in range(L + 1):
        for m in range(-l, l + 1):
            if m == 0:
                cols.append(p[(l, 0)])
            elif m > 0:
                cols.append(math.sqrt(2.0) * p[(l, m)] * np.cos(m * phi))
            else:
                cols.append(math.sqrt(2.0) * p[(l, -m)] * np.sin(-m * phi))
    return np.stack(cols, axis=1)


@dataclass
class ShapePair:
    name: str
    n: int
    d: int
    k: int
    P: int
    R: int
    dtype: str
    scale: float
    pts_M: np.ndarray      # fp32 [n,3] source geometry
    pts_N: np.ndarray      # fp32 [n,3] target geometry
    F_M: np.ndarray        # fp32 [n,d] source descriptors (K)
    F_N: np.ndarray        # fp32 [n,d] target descriptors (Q)
    Phi_M: np.ndarray      # fp32 [n,k] source eigenbasis (V)
    dO: np.ndarray         # fp32 [n,k] upstream gradient of the coupling
    meta: dict = field(default_factory=dict)


def make_pair(n: int, d: int, L: int, noise_var: float, same_points: bool,
              warp: bool, P: int, R: int, dtype: str, seed: int,
              name: str = "custom") -> ShapePair:
    """Draw one synthetic source/target pair (numpy PCG64 seeded with `seed`)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x_m = sphere_points(n, rng)
    rot = random_rotation(rng)
    z = x_m.copy() if same_points else sphere_points(n, rng)
    x_n = z @ rot.T
    w, b = rff_params(d, rng)
    f_m = rff(x_m, w, b)
    zf = warp_points(z) if warp else z
    f_n = rff(zf, w, b) + rng.normal(0.0, math.sqrt(noise_var), size=(n, d))
    phi = real_sph_harm(x_m, L)
    dout = rng.standard_normal((n, phi.shape[1]))
    return ShapePair(
        name=name, n=n, d=d, k=phi.shape[1], P=P, R=R, dtype=dtype,
        scale=1.0 / math.sqrt(d),
        pts_M=x_m.astype(np.float32), pts_N=x_n.astype(np.float32),
        F_M=f_m.astype(np.float32), F_N=f_n.astype(np.float32),
        Phi_M=phi.astype(np.float32), dO=dout.astype(np.float32),
        meta=dict(seed=seed, noise_sigma=math.sqrt(noise_var), L=L, warp=warp,
                  same_points=same_points))


def make_workload(name: str, n: int | None = None, seed: int | None = None) -> ShapePair:
    """The named workload, optionally at another size n (P scaled to keep n/P)."""
    cfg = dict(WORKLOADS[name])
    if n is not None and n != cfg["n"]:
        cfg["P"] = max(1, int(round(cfg["P"] * n / cfg["n"])))
        cfg["n"] = n
    if seed is not None:
        cfg["seed"] = seed
    return make_pair(name=name, **cfg)


def sphere_mesh(pts: np.ndarray):
    """Triangle mesh of points on the unit sphere as an edge graph.

    The convex hull of points on a sphere is their spherical Delaunay
    triangulation, so its triangles mesh the surface.  Returns the undirected
    edge graph in CSR form: off int32 [n+1], adj int32 [nnz] (each vertex's
    neighbours ascending, every edge listed from both ends) and the edge
    lengths w fp64 [nnz] (Euclidean distance between the fp32 coordinates,
    the length of the mesh edge)."""
    from scipy.spatial import ConvexHull

    p32 = np.ascontiguousarray(pts, dtype=np.float32)
    n = p32.shape[0]
    tri = ConvexHull(p32.astype(np.float64)).simplices
    e = np.concatenate([tri[:, [0, 1]], tri[:, [1, 2]], tri[:, [2, 0]]])
    e = np.concatenate([e, e[:, ::-1]])
    e = np.unique(e, axis=0)  # sorted by (vertex, neighbour)
    off = np.zeros(n + 1, np.int64)
    np.add.at(off, e[:, 0] + 1, 1)
    off = np.cumsum(off).astype(np.int32)
    p64 = p32.astype(np.float64)
    w = np.sqrt(((p64[e[:, 0]] - p64[e[:, 1]]) ** 2).sum(axis=1))
    return off, e[:, 1].astype(np.int32), w


def random_inputs(nN: int, nM: int, d: int, k: int, seed: int, q_scale: float = 1.0):
    """Plain Gaussian Q, K, V, dO (fp32) for shape-edge parity cases."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = (rng.standard_normal((nN, d)) * q_scale).astype(np.float32)
    kk = rng.standard_normal((nM, d)).astype(np.float32)
    v = rng.standard_normal((nM, k)).astype(np.float32)
    do = rng.standard_normal((nN, k)).astype(np.float32)
    return q, kk, v, do
