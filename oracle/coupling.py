"""Oracle (test infrastructure only): the spatial-spectral coupling in plain fp64.

Source: "Spatial-Spectral Coupling as Attention", project page, section
"Spatial-spectral coupling is attention": the coupled functional-map pipeline
consumes only the product Pi_NM Phi_M, which is scaled dot-product attention
with Q = F_N (target descriptors), K = F_M (source descriptors) and
V = Phi_M (source Laplace-Beltrami eigenbasis).  Section "Geo-FlashAttention":
the exact softmax is evaluated within the selected support only.

Definitions written out (no tiling, no online softmax):
  S_ij  = s * <Q_i, K_j>
  Pi_ij = exp(S_ij - max_j S_ij) / sum_j exp(S_ij - max_j S_ij)   (rows sum to 1)
  O_i   = sum_j Pi_ij V_j,   lse_i = max_j S_ij + ln sum_j exp(S_ij - max_j S_ij)
Backward of a scalar loss L with dL/dO = dO (textbook softmax-matmul gradient):
  D_i = <dO_i, O_i>,  dP_ij = <dO_i, V_j>,  dS_ij = Pi_ij (dP_ij - D_i)
  dQ_i = s sum_j dS_ij K_j,  dK_j = s sum_i dS_ij Q_i,  dV_j = sum_i Pi_ij dO_i
Geo: j runs over U(i) = union of the members of the source patches selected by
the target patch of i; the softmax is normalised over U(i) only.

Readings (the pages give no scale, axis or gradient list): s is an argument
(1/sqrt(d) in every workload); the softmax runs over source vertices, so each
row of Pi sums to one; natural log for lse.

Rows are evaluated in independent chunks only to bound memory; matrix
products are numpy's (a library primitive), so results differ from a
row-by-row loop only in rounding order.
"""
from __future__ import annotations

import numpy as np

_CHUNK = 1024


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _softmax_rows(S):
    m = S.max(axis=1)
    E = np.exp(S - m[:, None])
    l = E.sum(axis=1)
    return E / l[:, None], m + np.log(l)


def dense_fwd(Q, K, V, scale, rows=None):
    """O [len(rows),k] and lse [len(rows)] of the dense coupling (all rows by default)."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    rows = np.arange(Q.shape[0]) if rows is None else np.asarray(rows)
    O = np.zeros((rows.shape[0], V.shape[1]))
    lse = np.zeros(rows.shape[0])
    for a in range(0, rows.shape[0], _CHUNK):
        r = rows[a:a + _CHUNK]
        Pi, lse[a:a + _CHUNK] = _softmax_rows(scale * (Q[r] @ K.T))
        O[a:a + _CHUNK] = Pi @ V
    return O, lse


def dense_bwd(Q, K, V, dO, scale, rows=None, cols=None):
    """Gradients of the dense coupling for upstream gradient dO.

    Returns dict(O, lse, D, dQ, dK, dV).  `rows` restricts dQ/O/lse/D to a subset
    of target rows; `cols` restricts dK/dV to a subset of source rows (they still
    sum over every target row)."""
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    nN = Q.shape[0]
    O, lse = dense_fwd(Q, K, V, scale)
    D = (dO * O).sum(axis=1)
    rows = np.arange(nN) if rows is None else np.asarray(rows)
    cols = np.arange(K.shape[0]) if cols is None else np.asarray(cols)
    dQ = np.zeros((rows.shape[0], Q.shape[1]))
    for a in range(0, rows.shape[0], _CHUNK):
        r = rows[a:a + _CHUNK]
        Pi, _ = _softmax_rows(scale * (Q[r] @ K.T))
        dS = Pi * (dO[r] @ V.T - D[r][:, None])
        dQ[a:a + _CHUNK] = scale * (dS @ K)
    dK = np.zeros((cols.shape[0], K.shape[1]))
    dV = np.zeros((cols.shape[0], V.shape[1]))
    Kc, Vc = K[cols], V[cols]
    for a in range(0, nN, _CHUNK):
        r = slice(a, a + _CHUNK)
        Pi = np.exp(scale * (Q[r] @ Kc.T) - lse[r][:, None])
        dS = Pi * (dO[r] @ Vc.T - D[r][:, None])
        dK += scale * (dS.T @ Q[r])
        dV += Pi.T @ dO[r]
    return dict(O=O[rows], lse=lse[rows], D=D[rows], dQ=dQ, dK=dK, dV=dV)


def geo_support(off_M, mem_M, topk_row):
    """U for one target patch: the members of its selected source patches."""
    return np.concatenate([mem_M[off_M[q]:off_M[q + 1]] for q in topk_row])


def geo_fwd(Q, K, V, scale, off_N, mem_N, off_M, mem_M, topk):
    """O [nN,k], lse [nN] of Geo-FlashAttention in vertex order."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    O = np.zeros((Q.shape[0], V.shape[1]))
    lse = np.zeros(Q.shape[0])
    for p in range(off_N.shape[0] - 1):
        rows = mem_N[off_N[p]:off_N[p + 1]]
        U = geo_support(off_M, mem_M, topk[p])
        Pi, lse[rows] = _softmax_rows(scale * (Q[rows] @ K[U].T))
        O[rows] = Pi @ V[U]
    return O, lse


def geo_bwd(Q, K, V, dO, scale, off_N, mem_N, off_M, mem_M, topk):
    """Gradients of Geo-FlashAttention: dict(O, lse, D, dQ, dK, dV), vertex order."""
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    O, lse = geo_fwd(Q, K, V, scale, off_N, mem_N, off_M, mem_M, topk)
    D = (dO * O).sum(axis=1)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for p in range(off_N.shape[0] - 1):
        rows = mem_N[off_N[p]:off_N[p + 1]]
        U = geo_support(off_M, mem_M, topk[p])
        Pi, _ = _softmax_rows(scale * (Q[rows] @ K[U].T))
        dS = Pi * (dO[rows] @ V[U].T - D[rows][:, None])
        dQ[rows] = scale * (dS @ K[U])
        dK[U] += scale * (dS.T @ Q[rows])
        dV[U] += Pi.T @ dO[rows]
    return dict(O=O, lse=lse, D=D, dQ=dQ, dK=dK, dV=dV)
