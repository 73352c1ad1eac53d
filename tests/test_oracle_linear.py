"""Pins of the oracle's linear-attention (ELU) coupling (CPU only, fp64).

Definition: project page of "Spatial-Spectral Coupling as Attention", Table 1
row "Linear attention (ELU)", and the digest's "Interpretation" (a low-rank
feature map in place of the softmax); the feature map read as elu(x) + 1.

The oracle is tied to: torch's elu (a library route to the feature map and its
derivative), central finite differences of <dO, O>, closed forms (equal keys
give the column mean of V for every row; a single key gives that key's row of
V and zero descriptor gradients), the constant eigenfunction reproduced
exactly (normalised weights), the factored evaluation that makes the coupling
linear (associativity of the products), and the gradient invariant
sum_j dV_j = sum_i dO_i.
"""
import numpy as np
import pytest
import torch

from oracle import linear as lin
from spatial_spectral_attention_b200 import synth


def _rand(nN, nM, d, k, seed, qs=1.0):
    q, kk, v, do = synth.random_inputs(nN, nM, d, k, seed, q_scale=qs)
    return [a.astype(np.float64) for a in (q, kk, v, do)]


def test_feature_map_is_elu_plus_one():
    x = np.concatenate([np.linspace(-30, 30, 2001), [0.0, -0.0, 1e-300, -1e-300, 5e-324]])
    t = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    y = torch.nn.functional.elu(t, alpha=1.0) + 1.0
    y.sum().backward()
    # torch forms expm1(x) + 1 for x <= 0, exact to one rounding of the sum
    np.testing.assert_allclose(lin.phi(x), y.detach().numpy(), rtol=1e-15, atol=2.3e-16)
    np.testing.assert_allclose(lin.dphi(x), t.grad.numpy(), rtol=1e-15, atol=0)
    assert lin.phi(np.array([0.0]))[0] == 1.0 and np.all(lin.phi(x) > 0)


def test_equal_keys_give_the_column_mean_of_v():
    Q, K, V, _ = _rand(40, 25, 8, 5, seed=3)
    K[:] = K[0]
    O, den = lin.linear_fwd(Q, K, V)
    np.testing.assert_allclose(O, np.broadcast_to(V.mean(axis=0), O.shape), rtol=0, atol=1e-13)
    np.testing.assert_allclose(den, 25 * (lin.phi(Q) @ lin.phi(K[0])), rtol=1e-14)


def test_single_key_gives_its_row_and_zero_descriptor_gradients():
    Q, K, V, dO = _rand(9, 1, 6, 4, seed=5)
    g = lin.linear_bwd(Q, K, V, dO)
    np.testing.assert_allclose(g["O"], np.broadcast_to(V[0], g["O"].shape), rtol=0, atol=1e-14)
    assert np.abs(g["dQ"]).max() < 1e-14 and np.abs(g["dK"]).max() < 1e-12
    np.testing.assert_allclose(g["dV"][0], dO.sum(axis=0), rtol=1e-13, atol=1e-13)


def test_constant_eigenfunction_is_reproduced():
    p = synth.make_workload("small_fp32_2k", n=600)
    O, _ = lin.linear_fwd(p.F_N, p.F_M, p.Phi_M)
    y00 = float(np.float64(p.Phi_M[0, 0]))
    assert np.all(p.Phi_M[:, 0] == p.Phi_M[0, 0])
    np.testing.assert_allclose(O[:, 0], y00, rtol=1e-13, atol=0)


def test_factored_evaluation_is_linear_attention():
    # (phi(Q) phi(K)^T) V = phi(Q) (phi(K)^T V): the form whose cost is linear
    Q, K, V, _ = _rand(70, 90, 16, 7, seed=11, qs=0.5)
    pQ, pK = lin.phi(Q), lin.phi(K)
    O_f = (pQ @ (pK.T @ V)) / (pQ @ pK.sum(axis=0))[:, None]
    O, den = lin.linear_fwd(Q, K, V)
    np.testing.assert_allclose(O, O_f, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(den, pQ @ pK.sum(axis=0), rtol=1e-13)


def test_backward_finite_differences():
    Q, K, V, dO = _rand(6, 7, 4, 3, seed=2)
    g = lin.linear_bwd(Q, K, V, dO)

    def loss(Q_, K_, V_):
        O, _ = lin.linear_fwd(Q_, K_, V_)
        return float((O * dO).sum())

    h = 1e-6
    for name, X, grad in (("Q", Q, g["dQ"]), ("K", K, g["dK"]), ("V", V, g["dV"])):
        num = np.zeros_like(X)
        for idx in np.ndindex(*X.shape):
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += h
            Xm[idx] -= h
            args_p = {"Q": (Xp, K, V), "K": (Q, Xp, V), "V": (Q, K, Xp)}[name]
            args_m = {"Q": (Xm, K, V), "K": (Q, Xm, V), "V": (Q, K, Xm)}[name]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-9, err_msg=name)


@pytest.mark.parametrize("seed", [1, 4])
def test_dv_sums_to_the_upstream_gradient(seed):
    Q, K, V, dO = _rand(50, 33, 8, 6, seed=seed)
    g = lin.linear_bwd(Q, K, V, dO)
    np.testing.assert_allclose(g["dV"].sum(axis=0), dO.sum(axis=0), rtol=1e-12, atol=1e-12)


def test_row_and_column_samples_match_the_full_result():
    Q, K, V, dO = _rand(2100, 300, 8, 5, seed=7)
    full = lin.linear_bwd(Q, K, V, dO)
    rows, cols = np.array([0, 5, 1024, 2099]), np.array([3, 0, 299])
    part = lin.linear_bwd(Q, K, V, dO, rows=rows, cols=cols)
    for nm, idx in (("O", rows), ("den", rows), ("dQ", rows), ("dK", cols), ("dV", cols)):
        np.testing.assert_allclose(part[nm], full[nm][idx], rtol=1e-13, atol=1e-15, err_msg=nm)
