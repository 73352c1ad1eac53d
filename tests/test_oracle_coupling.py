"""Pins of the oracle's coupling (CPU only, fp64).

The oracle is tied to: torch's scaled_dot_product_attention and autograd in
fp64 (a library route to the same attention, with a boolean mask for Geo),
central finite differences, closed forms (n_M = 1, s = 0, the constant
eigenfunction), permutation recovery at large scale, and invariants of the
gradients.  Definition: project page of "Spatial-Spectral Coupling as
Attention", section "Spatial-spectral coupling is attention" (Q = F_N,
K = F_M, V = Phi_M) and section Geo-FlashAttention (exact softmax within the
selected support).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from spatial_spectral_attention_b200 import synth


def _rand(nN, nM, d, k, seed, qs=1.0):
    q, kk, v, do = synth.random_inputs(nN, nM, d, k, seed, q_scale=qs)
    return [a.astype(np.float64) for a in (q, kk, v, do)]


def _sdpa(Q, K, V, dO, s, mask=None):
    t = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (Q, K, V)]
    m = None if mask is None else torch.tensor(mask)
    O = torch.nn.functional.scaled_dot_product_attention(
        t[0][None], t[1][None], t[2][None], attn_mask=m, scale=s)[0]
    (O * torch.tensor(dO)).sum().backward()
    S = s * (t[0] @ t[1].T)
    if m is not None:
        S = S.masked_fill(~m, -math.inf)
    lse = torch.logsumexp(S, dim=-1)
    return (O.detach().numpy(), lse.detach().numpy(),
            t[0].grad.numpy(), t[1].grad.numpy(), t[2].grad.numpy())


@pytest.mark.parametrize("nN,nM,d,k", [(37, 53, 16, 9), (130, 70, 64, 25), (5, 1, 8, 3)])
def test_dense_matches_torch_sdpa_fp64(nN, nM, d, k):
    Q, K, V, dO = _rand(nN, nM, d, k, seed=nN + nM)
    s = 1.0 / math.sqrt(d)
    O, lse, dQ, dK, dV = _sdpa(Q, K, V, dO, s)
    g = oracle.dense_bwd(Q, K, V, dO, s)
    np.testing.assert_allclose(g["O"], O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["lse"], lse, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dQ"], dQ, rtol=0, atol=1e-11)
    np.testing.assert_allclose(g["dK"], dK, rtol=0, atol=1e-11)
    np.testing.assert_allclose(g["dV"], dV, rtol=0, atol=1e-11)
    O2, lse2 = oracle.dense_fwd(Q, K, V, s)
    np.testing.assert_allclose(O2, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-12)


def test_dense_bwd_finite_differences():
    Q, K, V, dO = _rand(6, 7, 4, 3, seed=2)
    s = 0.7
    g = oracle.dense_bwd(Q, K, V, dO, s)

    def loss(Q_, K_, V_):
        O, _ = oracle.dense_fwd(Q_, K_, V_, s)
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
        np.testing.assert_allclose(grad, num, rtol=1e-7, atol=1e-8, err_msg=name)


def test_row_stochastic_reproduces_constant_eigenfunction():
    pair = synth.make_workload("small_fp32_2k", n=700)
    Q, K, V = (a.astype(np.float64) for a in (pair.F_N, pair.F_M, pair.Phi_M))
    O, _ = oracle.dense_fwd(Q, K, V, pair.scale)
    y00 = 1.0 / (2.0 * math.sqrt(math.pi))
    # the generator's Y_00 column is fp32-rounded; rows of Pi sum to one
    np.testing.assert_allclose(O[:, 0], V[0, 0], rtol=0, atol=1e-15)
    assert abs(V[0, 0] - y00) < 1e-7


def test_closed_forms_single_key_and_zero_scale():
    Q, K, V, _ = _rand(9, 1, 8, 5, seed=4)
    O, lse = oracle.dense_fwd(Q, K, V, 0.3)
    np.testing.assert_array_equal(O, np.repeat(V, 9, axis=0))
    np.testing.assert_allclose(lse, 0.3 * (Q @ K[0]), rtol=0, atol=1e-14)
    Q, K, V, _ = _rand(9, 40, 8, 5, seed=5)
    O, lse = oracle.dense_fwd(Q, K, V, 0.0)
    np.testing.assert_allclose(O, np.repeat(V.mean(0, keepdims=True), 9, 0), atol=1e-15)
    np.testing.assert_allclose(lse, math.log(40), atol=1e-14)


def test_lse_bounds():
    Q, K, V, _ = _rand(50, 80, 16, 4, seed=6)
    s = 0.25
    _, lse = oracle.dense_fwd(Q, K, V, s)
    smax = (s * (Q @ K.T)).max(1)
    assert np.all(lse >= smax - 1e-13)
    assert np.all(lse <= smax + math.log(80) + 1e-13)


def test_permutation_recovery_at_large_scale():
    rng = np.random.default_rng(0)
    n, d = 300, 32
    K = rng.standard_normal((n, d))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    perm = rng.permutation(n)
    Q = K[perm]
    V = rng.standard_normal((n, 7))
    G = Q @ K.T
    assert np.all(np.argmax(G, axis=1) == perm)
    gap = np.min(np.sort(G, axis=1)[:, -1] - np.sort(G, axis=1)[:, -2])
    s = 200.0
    O, _ = oracle.dense_fwd(Q, K, V, s)
    bound = n * math.exp(-s * gap) * np.abs(V).max() * 2
    np.testing.assert_allclose(O, V[perm], rtol=0, atol=max(bound, 1e-12))


def test_gradient_invariants():
    Q, K, V, dO = _rand(60, 45, 16, 6, seed=8)
    s = 0.3
    g = oracle.dense_bwd(Q, K, V, dO, s)
    np.testing.assert_allclose(g["dK"].sum(0), 0.0, atol=1e-12)
    np.testing.assert_allclose(g["dV"].sum(0), dO.sum(0), atol=1e-12)
    assert abs((Q * g["dQ"]).sum() - (K * g["dK"]).sum()) < 1e-11


def test_bwd_row_and_column_subsets_match_full():
    Q, K, V, dO = _rand(40, 30, 8, 5, seed=9)
    full = oracle.dense_bwd(Q, K, V, dO, 0.4)
    rows = np.array([3, 17, 39])
    cols = np.array([0, 29, 11])
    sub = oracle.dense_bwd(Q, K, V, dO, 0.4, rows=rows, cols=cols)
    for key in ("O", "lse", "D", "dQ"):
        np.testing.assert_allclose(sub[key], full[key][rows], atol=1e-13)
    for key in ("dK", "dV"):
        np.testing.assert_allclose(sub[key], full[key][cols], atol=1e-13)


def _patches(n, P, R, seed, d=16, k=9):
    rng = np.random.default_rng(seed)
    ptsN = synth.sphere_points(n, rng).astype(np.float32)
    ptsM = synth.sphere_points(n + 7, rng).astype(np.float32)
    Q, K, V, dO = _rand(n, n + 7, d, k, seed=seed)
    _, ownN, _ = oracle.fps(ptsN, P, 0)
    _, ownM, _ = oracle.fps(ptsM, P + 1, 0)
    offN, memN = oracle.csr(ownN, P)
    offM, memM = oracle.csr(ownM, P + 1)
    sc = oracle.scores(oracle.pool(Q, offN, memN), oracle.pool(K, offM, memM))
    topk = oracle.topk(sc, R)
    return Q, K, V, dO, ownN, ownM, offN, memN, offM, memM, topk


def test_geo_matches_masked_sdpa_fp64():
    Q, K, V, dO, ownN, ownM, offN, memN, offM, memM, topk = _patches(120, 9, 3, seed=1)
    s = 0.25
    # brute-force support: vertex j is visible to row i iff owner_M(j) is among
    # the patches selected by owner_N(i)
    mask = np.zeros((Q.shape[0], K.shape[0]), bool)
    for i in range(Q.shape[0]):
        mask[i] = np.isin(ownM, topk[ownN[i]])
    O, lse, dQ, dK, dV = _sdpa(Q, K, V, dO, s, mask)
    g = oracle.geo_bwd(Q, K, V, dO, s, offN, memN, offM, memM, topk)
    np.testing.assert_allclose(g["O"], O, atol=1e-12)
    np.testing.assert_allclose(g["lse"], lse, atol=1e-12)
    np.testing.assert_allclose(g["dQ"], dQ, atol=1e-11)
    np.testing.assert_allclose(g["dK"], dK, atol=1e-11)
    np.testing.assert_allclose(g["dV"], dV, atol=1e-11)
    O2, lse2 = oracle.geo_fwd(Q, K, V, s, offN, memN, offM, memM, topk)
    np.testing.assert_allclose(O2, O, atol=1e-12)


def test_geo_with_every_patch_selected_equals_dense():
    Q, K, V, dO, *_rest = _patches(90, 6, 7, seed=2)
    ownN, ownM, offN, memN, offM, memM, topk = _rest
    assert topk.shape[1] == offM.shape[0] - 1
    s = 0.3
    g = oracle.geo_bwd(Q, K, V, dO, s, offN, memN, offM, memM, topk)
    d = oracle.dense_bwd(Q, K, V, dO, s)
    for key in ("O", "lse", "dQ", "dK", "dV"):
        np.testing.assert_allclose(g[key], d[key], rtol=1e-13, atol=1e-13, err_msg=key)


def test_geo_singleton_patches_all_selected_is_dense():
    Q, K, V, dO = _rand(12, 10, 4, 3, seed=3)
    offN, memN = np.arange(13, dtype=np.int32), np.arange(12, dtype=np.int32)
    offM, memM = np.arange(11, dtype=np.int32), np.random.default_rng(0).permutation(10).astype(np.int32)
    topk = np.tile(np.arange(10, dtype=np.int32), (12, 1))
    g = oracle.geo_bwd(Q, K, V, dO, 0.5, offN, memN, offM, memM, topk)
    d = oracle.dense_bwd(Q, K, V, dO, 0.5)
    for key in ("O", "dQ", "dK", "dV"):
        np.testing.assert_allclose(g[key], d[key], rtol=1e-13, atol=1e-13)


def test_geo_invariants_and_support_bound():
    Q, K, V, dO, ownN, ownM, offN, memN, offM, memM, topk = _patches(150, 10, 2, seed=4)
    s = 0.4
    g = oracle.geo_bwd(Q, K, V, dO, s, offN, memN, offM, memM, topk)
    np.testing.assert_allclose(g["dK"].sum(0), 0.0, atol=1e-12)
    np.testing.assert_allclose(g["dV"].sum(0), dO.sum(0), atol=1e-12)
    assert abs((Q * g["dQ"]).sum() - (K * g["dK"]).sum()) < 1e-11
    for i in range(Q.shape[0]):
        U = oracle.geo_support(offM, memM, topk[ownN[i]])
        smax = (s * (K[U] @ Q[i])).max()
        assert smax - 1e-13 <= g["lse"][i] <= smax + math.log(len(U)) + 1e-13
