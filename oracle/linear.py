"""Oracle (test infrastructure only): the linear-attention (ELU) coupling in
plain fp64.

Source: "Spatial-Spectral Coupling as Attention", project page, Table 1, row
"Linear attention (ELU)" (the approximate coupling that the exact ones are
compared with), and the ai4snews digest of the paper, "Interpretation":
linear attention replaces the softmax with a low-rank feature map.  The pages
print neither the map nor the normalisation.  Reading taken here (the common
ELU form): phi(x) = elu(x) + 1, i.e. x + 1 for x > 0 and exp(x) otherwise,
applied entry-wise to the descriptors; the weight of a pair is
W_ij = <phi(Q_i), phi(K_j)> and each target row is normalised by its sum.

Definitions written out (weights materialised row block by row block; no
factored evaluation):
  W_ij  = <phi(Q_i), phi(K_j)>,  s_i = sum_j W_ij (the row normaliser "den")
  O_i   = sum_j W_ij V_j / s_i
Backward of a scalar loss L with dL/dO = dO, differentiating that definition:
  D_i    = <dO_i, O_i>
  dW_ij  = (<dO_i, V_j> - D_i) / s_i
  dQ_i   = phi'(Q_i) * sum_j dW_ij phi(K_j)
  dK_j   = phi'(K_j) * sum_i dW_ij phi(Q_i)
  dV_j   = sum_i (W_ij / s_i) dO_i
with phi'(x) = 1 for x > 0 and exp(x) otherwise.
"""
from __future__ import annotations

import numpy as np

_CHUNK = 1024


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def phi(x):
    """ELU feature map plus one: x + 1 where x > 0, exp(x) elsewhere."""
    x = _f64(x)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def dphi(x):
    """Derivative of phi: 1 where x > 0, exp(x) elsewhere."""
    x = _f64(x)
    return np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))


def linear_fwd(Q, K, V, rows=None):
    """O [len(rows), k] and den [len(rows)] of the linear coupling."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    rows = np.arange(Q.shape[0]) if rows is None else np.asarray(rows)
    pK = phi(K)
    O = np.zeros((rows.shape[0], V.shape[1]))
    den = np.zeros(rows.shape[0])
    for a in range(0, rows.shape[0], _CHUNK):
        r = rows[a:a + _CHUNK]
        W = phi(Q[r]) @ pK.T
        s = W.sum(axis=1)
        O[a:a + _CHUNK] = (W @ V) / s[:, None]
        den[a:a + _CHUNK] = s
    return O, den


def linear_bwd(Q, K, V, dO, rows=None, cols=None):
    """Gradients of the linear coupling for upstream gradient dO.

    Returns dict(O, den, D, dQ, dK, dV).  `rows` restricts O/den/D/dQ to a
    subset of target rows; `cols` restricts dK/dV to a subset of source rows
    (they still sum over every target row)."""
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    nN = Q.shape[0]
    O, den = linear_fwd(Q, K, V)
    D = (dO * O).sum(axis=1)
    rows = np.arange(nN) if rows is None else np.asarray(rows)
    cols = np.arange(K.shape[0]) if cols is None else np.asarray(cols)
    pK = phi(K)
    dQ = np.zeros((rows.shape[0], Q.shape[1]))
    for a in range(0, rows.shape[0], _CHUNK):
        r = rows[a:a + _CHUNK]
        dW = (dO[r] @ V.T - D[r][:, None]) / den[r][:, None]
        dQ[a:a + _CHUNK] = dphi(Q[r]) * (dW @ pK)
    pKc, Vc = pK[cols], V[cols]
    dphiK = np.zeros((cols.shape[0], K.shape[1]))
    dV = np.zeros((cols.shape[0], V.shape[1]))
    for a in range(0, nN, _CHUNK):
        r = slice(a, a + _CHUNK)
        pQ = phi(Q[r])
        W = pQ @ pKc.T
        dW = (dO[r] @ Vc.T - D[r][:, None]) / den[r][:, None]
        dphiK += dW.T @ pQ
        dV += (W / den[r][:, None]).T @ dO[r]
    dK = dphi(K[cols]) * dphiK
    return dict(O=O[rows], den=den[rows], D=D[rows], dQ=dQ, dK=dK, dV=dV)
