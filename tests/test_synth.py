"""The seeded input generator: determinism and the spherical-harmonic basis."""
import math

import numpy as np

from spatial_spectral_attention_b200 import synth


def test_spherical_harmonics_orthonormal_on_fibonacci_grid():
    # quasi-uniform Fibonacci points integrate low-degree polynomials well
    n = 200000
    i = np.arange(n) + 0.5
    z = 1 - 2 * i / n
    phi = math.pi * (1 + 5 ** 0.5) * i
    r = np.sqrt(1 - z * z)
    x = np.stack([r * np.cos(phi), r * np.sin(phi), z], 1)
    Y = synth.real_sph_harm(x, 6)
    assert Y.shape[1] == 49
    G = (Y.T @ Y) * (4 * math.pi / n)
    np.testing.assert_allclose(G, np.eye(49), atol=2e-3)
    np.testing.assert_allclose(Y[:, 0], 1 / (2 * math.sqrt(math.pi)), rtol=0, atol=1e-15)


def test_workloads_are_seeded_and_shaped():
    a = synth.make_workload("dense_10k", n=500)
    b = synth.make_workload("dense_10k", n=500)
    assert a.k == 196 and a.d == 128 and a.F_N.shape == (500, 128)
    for f in ("pts_M", "pts_N", "F_M", "F_N", "Phi_M", "dO"):
        assert np.array_equal(getattr(a, f), getattr(b, f))
    c = synth.make_workload("small_fp32_2k")
    assert c.k == 25 and c.d == 64 and c.n == 2048
    # target geometry is the rotated source in the small workload
    g = c.pts_N.astype(np.float64) @ c.pts_N.astype(np.float64).T
    h = c.pts_M.astype(np.float64) @ c.pts_M.astype(np.float64).T
    np.testing.assert_allclose(g[:50, :50], h[:50, :50], atol=1e-6)
