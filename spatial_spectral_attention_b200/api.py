"""Python binding of libssc: the C calls of include/ssc.h under the same names.

Argument marshalling only: every step of the computation runs in libssc's CUDA
kernels.  PyTorch provides device memory (outputs and workspaces are allocated
with torch) and the current CUDA stream.  Inputs must be CUDA tensors; nothing
here falls back to a CPU computation.
"""
from __future__ import annotations

import ctypes

import torch

from ._abi import check, lib

SSC_BF16 = 0
SSC_F32 = 1


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libssc calls take CUDA tensors")


def _rowmajor(t):
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D row-major tensor (unit column stride)")
    return t.stride(0)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return SSC_BF16
    if t.dtype == torch.float32:
        return SSC_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def _workspace(nbytes, device):
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def ssc_version():
    return lib().ssc_version()


def ssc_kernel_launches():
    """Running count of the kernels libssc has enqueued."""
    return int(lib().ssc_kernel_launches())


PROF_DENSE_FWD, PROF_FWD, PROF_BWD_DQK, PROF_BWD_DV = 0, 1, 2, 3
PROF_FPS, PROF_POOL, PROF_SCORES, PROF_TOPK, PROF_GATHER = 4, 5, 6, 7, 8
PROF_LIN_REDUCE, PROF_LIN_ROWS, PROF_BWD_DK = 9, 10, 11


def ssc_profile_enable(on=True, clear=True):
    """Start (clearing the record unless clear=False) or stop recording the
    device time of every coupling kernel launch with CUDA events on its stream."""
    check("ssc_profile_enable", lib().ssc_profile_enable((1 if clear else 2) if on else 0))


def ssc_profile_read(kernel):
    """(summed milliseconds, launches) of one tracked kernel in the record."""
    ms = ctypes.c_double(0.0)
    n = ctypes.c_int(0)
    check("ssc_profile_read", lib().ssc_profile_read(int(kernel), ctypes.byref(ms), ctypes.byref(n)))
    return ms.value, n.value


def ssc_device_status(clear=True):
    """Synchronises the current stream and returns the device status word as a
    status code (0 ok, 6 a bounded wait ran out, 1 a bad index table entry)."""
    out = ctypes.c_int(0)
    check("ssc_device_status", lib().ssc_device_status(_stream(), int(clear), ctypes.byref(out)))
    return out.value


def ssc_set_wait_limit_ns(ns):
    check("ssc_set_wait_limit_ns", lib().ssc_set_wait_limit_ns(int(ns)))


def ssc_debug_wait_timeout(limit_ns):
    check("ssc_debug_wait_timeout", lib().ssc_debug_wait_timeout(int(limit_ns), _stream()))


def ssc_debug_stall_next_launch(which):
    """Abort-path test hook: 1 = next forward kernel launch, 2 = next dQ/dK
    backward kernel launch, 0 = disarm."""
    check("ssc_debug_stall_next_launch", lib().ssc_debug_stall_next_launch(int(which)))


def ssc_fps_patches(pts, P, seed_vertex=0):
    """Geodesic FPS + Voronoi patches.  pts: fp32 [n,3] CUDA tensor.
    Returns (centers [P], owner [n], offsets [P+1], members [n]) int32."""
    _cuda(pts)
    pts = pts.contiguous()
    n = pts.shape[0]
    dev = pts.device
    centers = torch.empty(P, dtype=torch.int32, device=dev)
    owner = torch.empty(n, dtype=torch.int32, device=dev)
    offsets = torch.empty(P + 1, dtype=torch.int32, device=dev)
    members = torch.empty(n, dtype=torch.int32, device=dev)
    nb = lib().ssc_fps_patches_workspace_size(n, P)
    ws = _workspace(nb, dev)
    check("ssc_fps_patches", lib().ssc_fps_patches(
        _ptr(pts), n, P, seed_vertex, _ptr(centers), _ptr(owner), _ptr(offsets), _ptr(members),
        _ptr(ws), ws.numel(), _stream()))
    return centers, owner, offsets, members


def ssc_fps_patches_noalloc(pts, P, seed_vertex=0):
    """ssc_fps_patches without a workspace: the library's fixed device scratch
    is used instead (n <= 262144, P <= 65535; concurrent calls must not overlap)."""
    _cuda(pts)
    pts = pts.contiguous()
    n = pts.shape[0]
    dev = pts.device
    centers = torch.empty(P, dtype=torch.int32, device=dev)
    owner = torch.empty(n, dtype=torch.int32, device=dev)
    offsets = torch.empty(P + 1, dtype=torch.int32, device=dev)
    members = torch.empty(n, dtype=torch.int32, device=dev)
    check("ssc_fps_patches_noalloc", lib().ssc_fps_patches_noalloc(
        _ptr(pts), n, P, seed_vertex, _ptr(centers), _ptr(owner), _ptr(offsets), _ptr(members),
        _stream()))
    return centers, owner, offsets, members


def ssc_fps_patches_mesh(adj_off, adj, edge_len, P, seed_vertex=0):
    """Geodesic FPS + patches on a mesh graph: adj_off int32 [n+1], adj int32 [nnz],
    edge_len fp64 [nnz] (CUDA tensors).  Returns (centers, owner, offsets, members)."""
    _cuda(adj_off, adj, edge_len)
    if adj_off.dtype != torch.int32 or adj.dtype != torch.int32 or edge_len.dtype != torch.float64:
        raise ValueError("adj_off/adj must be int32 and edge_len fp64")
    adj_off, adj, edge_len = adj_off.contiguous(), adj.contiguous(), edge_len.contiguous()
    n = adj_off.numel() - 1
    nnz = adj.numel()
    dev = adj_off.device
    centers = torch.empty(P, dtype=torch.int32, device=dev)
    owner = torch.empty(n, dtype=torch.int32, device=dev)
    offsets = torch.empty(P + 1, dtype=torch.int32, device=dev)
    members = torch.empty(n, dtype=torch.int32, device=dev)
    ws = _workspace(lib().ssc_fps_patches_mesh_workspace_size(n, P), dev)
    check("ssc_fps_patches_mesh", lib().ssc_fps_patches_mesh(
        _ptr(adj_off), _ptr(adj), _ptr(edge_len), n, nnz, P, seed_vertex, _ptr(centers),
        _ptr(owner), _ptr(offsets), _ptr(members), _ptr(ws), ws.numel(), _stream()))
    return centers, owner, offsets, members


def ssc_patch_scores_topk(FN, FM, offN, memN, offM, memM, R, return_scores=False):
    """Patch-mean scores and the top-R source patches of every target patch."""
    _cuda(FN, FM, offN, memN, offM, memM)
    d = FN.shape[1]
    PN, PM = offN.numel() - 1, offM.numel() - 1
    dev = FN.device
    topk = torch.empty((PN, R), dtype=torch.int32, device=dev)
    scores = torch.empty((PN, PM), dtype=torch.float64, device=dev) if return_scores else None
    ws = _workspace(lib().ssc_patch_scores_topk_workspace_size(PN, PM, d), dev)
    check("ssc_patch_scores_topk", lib().ssc_patch_scores_topk(
        _ptr(FN), _rowmajor(FN), FN.shape[0], _ptr(FM), _rowmajor(FM), FM.shape[0], d,
        _dtype_code(FN), _ptr(offN), _ptr(memN), PN, _ptr(offM), _ptr(memM), PM, R,
        _ptr(topk), _ptr(scores), _ptr(ws), ws.numel(), _stream()))
    return (topk, scores) if return_scores else topk


def _qkv(Q, K, V):
    _cuda(Q, K, V)
    if not (Q.dtype == K.dtype == V.dtype):
        raise ValueError("Q, K and V must share one dtype")
    return _rowmajor(Q), _rowmajor(K), _rowmajor(V), _dtype_code(Q)


def ssc_dense_coupling_fwd(Q, K, V, scale, workspace=None):
    """Dense coupling: O = softmax(scale Q K^T) V (fp32 [nN,k]) and lse (fp32 [nN])."""
    ldq, ldk, ldv, dt = _qkv(Q, K, V)
    nN, d = Q.shape
    nM, k = V.shape
    O = torch.empty((nN, k), dtype=torch.float32, device=Q.device)
    lse = torch.empty(nN, dtype=torch.float32, device=Q.device)
    nb = lib().ssc_dense_coupling_workspace_size(nN, nM, d, k, dt)
    ws = workspace if workspace is not None and workspace.numel() >= nb else _workspace(nb, Q.device)
    check("ssc_dense_coupling_fwd", lib().ssc_dense_coupling_fwd(
        _ptr(Q), ldq, _ptr(K), ldk, _ptr(V), ldv, nN, nM, d, k, float(scale), dt,
        _ptr(O), k, _ptr(lse), _ptr(ws), ws.numel(), _stream()))
    return O, lse


def ssc_dense_coupling_fwd_e4m3(Q, K, V, scale, workspace=None):
    """Dense forward with Q K^T on e4m3 tensor cores (bf16 Q, K, V; d = 128):
    O (fp32 [nN,k]) and lse (fp32 [nN])."""
    ldq, ldk, ldv, dt = _qkv(Q, K, V)
    nN, d = Q.shape
    nM, k = V.shape
    O = torch.empty((nN, k), dtype=torch.float32, device=Q.device)
    lse = torch.empty(nN, dtype=torch.float32, device=Q.device)
    nb = lib().ssc_dense_coupling_fwd_e4m3_workspace_size(nN, nM, d, k)
    ws = workspace if workspace is not None and workspace.numel() >= nb else _workspace(nb, Q.device)
    check("ssc_dense_coupling_fwd_e4m3", lib().ssc_dense_coupling_fwd_e4m3(
        _ptr(Q), ldq, _ptr(K), ldk, _ptr(V), ldv, nN, nM, d, k, float(scale),
        _ptr(O), k, _ptr(lse), _ptr(ws), ws.numel(), _stream()))
    return O, lse


def ssc_dense_coupling_bwd(Q, K, V, O, lse, dO, scale, need_dV=False, workspace=None,
                           deterministic=False):
    """Gradients (dQ, dK, dV or None) of the dense coupling for upstream dO (fp32)."""
    ldq, ldk, ldv, dt = _qkv(Q, K, V)
    _cuda(O, lse, dO)
    nN, d = Q.shape
    nM, k = V.shape
    dev = Q.device
    dQ = torch.empty((nN, d), dtype=torch.float32, device=dev)
    dK = torch.empty((nM, d), dtype=torch.float32, device=dev)
    dV = torch.empty((nM, k), dtype=torch.float32, device=dev) if need_dV else None
    O, dO, lse = O.contiguous(), dO.contiguous(), lse.contiguous()
    nb = lib().ssc_dense_coupling_workspace_size(nN, nM, d, k, dt)
    ws = workspace if workspace is not None and workspace.numel() >= nb else _workspace(nb, dev)
    fn = "ssc_dense_coupling_bwd_deterministic" if deterministic else "ssc_dense_coupling_bwd"
    check(fn, getattr(lib(), fn)(
        _ptr(Q), ldq, _ptr(K), ldk, _ptr(V), ldv, nN, nM, d, k, float(scale), dt,
        _ptr(O), O.stride(0), _ptr(lse), _ptr(dO), dO.stride(0),
        _ptr(dQ), d, _ptr(dK), d, _ptr(dV), k, _ptr(ws), ws.numel(), _stream()))
    return dQ, dK, dV


def _patches(offN, memN, offM, memM, topk):
    _cuda(offN, memN, offM, memM, topk)
    for t in (offN, memN, offM, memM, topk):
        if t.dtype != torch.int32:
            raise ValueError("patch tables must be int32")
    return offN.numel() - 1, offM.numel() - 1, topk.shape[1]


def ssc_geo_coupling_fwd(Q, K, V, scale, offN, memN, offM, memM, topk, workspace=None):
    """Geo-FlashAttention forward: (O fp32 [nN,k], lse fp32 [nN]) in vertex order."""
    ldq, ldk, ldv, dt = _qkv(Q, K, V)
    PN, PM, R = _patches(offN, memN, offM, memM, topk)
    nN, d = Q.shape
    nM, k = V.shape
    O = torch.empty((nN, k), dtype=torch.float32, device=Q.device)
    lse = torch.empty(nN, dtype=torch.float32, device=Q.device)
    nb = lib().ssc_geo_coupling_workspace_size(nN, nM, d, k, PN, PM, R, dt)
    ws = workspace if workspace is not None and workspace.numel() >= nb else _workspace(nb, Q.device)
    topk = topk.contiguous()
    check("ssc_geo_coupling_fwd", lib().ssc_geo_coupling_fwd(
        _ptr(Q), ldq, _ptr(K), ldk, _ptr(V), ldv, nN, nM, d, k, float(scale), dt,
        _ptr(offN), _ptr(memN), PN, _ptr(offM), _ptr(memM), PM, _ptr(topk), R,
        _ptr(O), k, _ptr(lse), _ptr(ws), ws.numel(), _stream()))
    return O, lse


def ssc_geo_coupling_bwd(Q, K, V, O, lse, dO, scale, offN, memN, offM, memM, topk,
                         need_dV=False, workspace=None, reuse_forward=False):
    """Geo-FlashAttention backward: (dQ, dK, dV or None) in vertex order.

    reuse_forward=True calls ssc_geo_coupling_bwd_reuse: the patch-major
    operands and the tile schedule are taken from `workspace`, which must be the
    workspace the matching ssc_geo_coupling_fwd call used (same inputs and
    tables, not written since)."""
    ldq, ldk, ldv, dt = _qkv(Q, K, V)
    PN, PM, R = _patches(offN, memN, offM, memM, topk)
    _cuda(O, lse, dO)
    nN, d = Q.shape
    nM, k = V.shape
    dev = Q.device
    dQ = torch.empty((nN, d), dtype=torch.float32, device=dev)
    dK = torch.empty((nM, d), dtype=torch.float32, device=dev)
    dV = torch.empty((nM, k), dtype=torch.float32, device=dev) if need_dV else None
    O, dO, lse, topk = O.contiguous(), dO.contiguous(), lse.contiguous(), topk.contiguous()
    nb = lib().ssc_geo_coupling_workspace_size(nN, nM, d, k, PN, PM, R, dt)
    if reuse_forward:
        if workspace is None or workspace.numel() < nb:
            raise ValueError("reuse_forward needs the forward's workspace")
        name = "ssc_geo_coupling_bwd_reuse"
    else:
        name = "ssc_geo_coupling_bwd"
    ws = workspace if workspace is not None and workspace.numel() >= nb else _workspace(nb, dev)
    check(name, getattr(lib(), name)(
        _ptr(Q), ldq, _ptr(K), ldk, _ptr(V), ldv, nN, nM, d, k, float(scale), dt,
        _ptr(offN), _ptr(memN), PN, _ptr(offM), _ptr(memM), PM, _ptr(topk), R,
        _ptr(O), O.stride(0), _ptr(lse), _ptr(dO), dO.stride(0),
        _ptr(dQ), d, _ptr(dK), d, _ptr(dV), k, _ptr(ws), ws.numel(), _stream()))
    return dQ, dK, dV


def _bf16_qkv(Q, K, V):
    _cuda(Q, K, V)
    if not (Q.dtype == K.dtype == V.dtype == torch.bfloat16):
        raise ValueError("the linear coupling takes bf16 Q, K and V")
    return _rowmajor(Q), _rowmajor(K), _rowmajor(V)


def ssc_linear_coupling_fwd(Q, K, V, workspace=None):
    """Linear-attention (ELU) coupling: O (fp32 [nN,k]) and den (fp32 [nN])."""
    ldq, ldk, ldv = _bf16_qkv(Q, K, V)
    nN, d = Q.shape
    nM, k = V.shape
    O = torch.empty((nN, k), dtype=torch.float32, device=Q.device)
    den = torch.empty(nN, dtype=torch.float32, device=Q.device)
    nb = lib().ssc_linear_coupling_workspace_size(nN, nM, d, k)
    ws = workspace if workspace is not None and workspace.numel() >= nb else _workspace(nb, Q.device)
    check("ssc_linear_coupling_fwd", lib().ssc_linear_coupling_fwd(
        _ptr(Q), ldq, _ptr(K), ldk, _ptr(V), ldv, nN, nM, d, k, _ptr(O), k, _ptr(den),
        _ptr(ws), ws.numel(), _stream()))
    return O, den


def ssc_linear_coupling_bwd(Q, K, V, O, den, dO, need_dV=False, workspace=None):
    """Gradients (dQ, dK, dV or None) of the linear coupling for upstream dO (fp32)."""
    ldq, ldk, ldv = _bf16_qkv(Q, K, V)
    _cuda(O, den, dO)
    nN, d = Q.shape
    nM, k = V.shape
    dev = Q.device
    dQ = torch.empty((nN, d), dtype=torch.float32, device=dev)
    dK = torch.empty((nM, d), dtype=torch.float32, device=dev)
    dV = torch.empty((nM, k), dtype=torch.float32, device=dev) if need_dV else None
    O, dO, den = O.contiguous(), dO.contiguous(), den.contiguous()
    nb = lib().ssc_linear_coupling_workspace_size(nN, nM, d, k)
    ws = workspace if workspace is not None and workspace.numel() >= nb else _workspace(nb, dev)
    check("ssc_linear_coupling_bwd", lib().ssc_linear_coupling_bwd(
        _ptr(Q), ldq, _ptr(K), ldk, _ptr(V), ldv, nN, nM, d, k, _ptr(O), O.stride(0), _ptr(den),
        _ptr(dO), dO.stride(0), _ptr(dQ), d, _ptr(dK), d, _ptr(dV), k, _ptr(ws), ws.numel(),
        _stream()))
    return dQ, dK, dV


# ---------------------------------------------------------------- batches of pairs
def _batched(t):
    """Leading dimension of a [batch, rows, cols] tensor whose pairs are stored
    back to back (unit column stride, batch stride = rows x leading dimension)."""
    if t.dim() != 3 or t.stride(2) != 1 or t.stride(0) != t.shape[1] * t.stride(1):
        raise ValueError("expected a [batch, rows, cols] tensor with pairs stored back to back")
    return t.stride(1)


def _bqkv(Q, K, V):
    _cuda(Q, K, V)
    if not (Q.dtype == K.dtype == V.dtype):
        raise ValueError("Q, K and V must share one dtype")
    if not (Q.shape[0] == K.shape[0] == V.shape[0]) or K.shape[1] != V.shape[1]:
        raise ValueError("Q [B,nN,d], K [B,nM,d] and V [B,nM,k] must agree")
    return _batched(Q), _batched(K), _batched(V), _dtype_code(Q)


def ssc_dense_coupling_fwd_batched(Q, K, V, scale, workspace=None):
    """Dense coupling of B pairs in one call: O [B,nN,k] fp32 and lse [B,nN]."""
    ldq, ldk, ldv, dt = _bqkv(Q, K, V)
    B, nN, d = Q.shape
    nM, k = V.shape[1], V.shape[2]
    O = torch.empty((B, nN, k), dtype=torch.float32, device=Q.device)
    lse = torch.empty((B, nN), dtype=torch.float32, device=Q.device)
    nb = lib().ssc_dense_coupling_batched_workspace_size(B, nN, nM, d, k, dt)
    ws = workspace if workspace is not None and workspace.numel() >= nb else _workspace(nb, Q.device)
    check("ssc_dense_coupling_fwd_batched", lib().ssc_dense_coupling_fwd_batched(
        B, _ptr(Q), ldq, _ptr(K), ldk, _ptr(V), ldv, nN, nM, d, k, float(scale), dt,
        _ptr(O), k, _ptr(lse), _ptr(ws), ws.numel(), _stream()))
    return O, lse


def ssc_dense_coupling_bwd_batched(Q, K, V, O, lse, dO, scale, need_dV=False, workspace=None):
    """Gradients (dQ [B,nN,d], dK [B,nM,d], dV [B,nM,k] or None) of B dense couplings."""
    ldq, ldk, ldv, dt = _bqkv(Q, K, V)
    _cuda(O, lse, dO)
    B, nN, d = Q.shape
    nM, k = V.shape[1], V.shape[2]
    dev = Q.device
    dQ = torch.empty((B, nN, d), dtype=torch.float32, device=dev)
    dK = torch.empty((B, nM, d), dtype=torch.float32, device=dev)
    dV = torch.empty((B, nM, k), dtype=torch.float32, device=dev) if need_dV else None
    O, dO, lse = O.contiguous(), dO.contiguous(), lse.contiguous()
    nb = lib().ssc_dense_coupling_batched_workspace_size(B, nN, nM, d, k, dt)
    ws = workspace if workspace is not None and workspace.numel() >= nb else _workspace(nb, dev)
    check("ssc_dense_coupling_bwd_batched", lib().ssc_dense_coupling_bwd_batched(
        B, _ptr(Q), ldq, _ptr(K), ldk, _ptr(V), ldv, nN, nM, d, k, float(scale), dt,
        _ptr(O), k, _ptr(lse), _ptr(dO), k, _ptr(dQ), d, _ptr(dK), d, _ptr(dV), k,
        _ptr(ws), ws.numel(), _stream()))
    return dQ, dK, dV


def _btables(offN, memN, offM, memM, topk):
    _cuda(offN, memN, offM, memM, topk)
    for t in (offN, memN, offM, memM, topk):
        if t.dtype != torch.int32:
            raise ValueError("patch tables must be int32")
    return (offN.contiguous(), memN.contiguous(), offM.contiguous(), memM.contiguous(),
            topk.contiguous())


def ssc_geo_coupling_fwd_batched(Q, K, V, scale, offN, memN, offM, memM, topk, workspace=None):
    """Geo-FlashAttention for B pairs: tables offN [B,PN+1], memN [B,nN], offM [B,PM+1],
    memM [B,nM], topk [B,PN,R] (local indices).  Returns O [B,nN,k], lse [B,nN]."""
    ldq, ldk, ldv, dt = _bqkv(Q, K, V)
    offN, memN, offM, memM, topk = _btables(offN, memN, offM, memM, topk)
    B, nN, d = Q.shape
    nM, k = V.shape[1], V.shape[2]
    PN, PM, R = offN.shape[1] - 1, offM.shape[1] - 1, topk.shape[2]
    O = torch.empty((B, nN, k), dtype=torch.float32, device=Q.device)
    lse = torch.empty((B, nN), dtype=torch.float32, device=Q.device)
    nb = lib().ssc_geo_coupling_batched_workspace_size(B, nN, nM, d, k, PN, PM, R, dt)
    ws = workspace if workspace is not None and workspace.numel() >= nb else _workspace(nb, Q.device)
    check("ssc_geo_coupling_fwd_batched", lib().ssc_geo_coupling_fwd_batched(
        B, _ptr(Q), ldq, _ptr(K), ldk, _ptr(V), ldv, nN, nM, d, k, float(scale), dt,
        _ptr(offN), _ptr(memN), PN, _ptr(offM), _ptr(memM), PM, _ptr(topk), R,
        _ptr(O), k, _ptr(lse), _ptr(ws), ws.numel(), _stream()))
    return O, lse


def ssc_geo_coupling_bwd_batched(Q, K, V, O, lse, dO, scale, offN, memN, offM, memM, topk,
                                 need_dV=False, workspace=None):
    """Gradients of B Geo couplings (dQ, dK, dV or None), tables as for the forward."""
    ldq, ldk, ldv, dt = _bqkv(Q, K, V)
    offN, memN, offM, memM, topk = _btables(offN, memN, offM, memM, topk)
    _cuda(O, lse, dO)
    B, nN, d = Q.shape
    nM, k = V.shape[1], V.shape[2]
    PN, PM, R = offN.shape[1] - 1, offM.shape[1] - 1, topk.shape[2]
    dev = Q.device
    dQ = torch.empty((B, nN, d), dtype=torch.float32, device=dev)
    dK = torch.empty((B, nM, d), dtype=torch.float32, device=dev)
    dV = torch.empty((B, nM, k), dtype=torch.float32, device=dev) if need_dV else None
    O, dO, lse = O.contiguous(), dO.contiguous(), lse.contiguous()
    nb = lib().ssc_geo_coupling_batched_workspace_size(B, nN, nM, d, k, PN, PM, R, dt)
    ws = workspace if workspace is not None and workspace.numel() >= nb else _workspace(nb, dev)
    check("ssc_geo_coupling_bwd_batched", lib().ssc_geo_coupling_bwd_batched(
        B, _ptr(Q), ldq, _ptr(K), ldk, _ptr(V), ldv, nN, nM, d, k, float(scale), dt,
        _ptr(offN), _ptr(memN), PN, _ptr(offM), _ptr(memM), PM, _ptr(topk), R,
        _ptr(O), k, _ptr(lse), _ptr(dO), k, _ptr(dQ), d, _ptr(dK), d, _ptr(dV), k,
        _ptr(ws), ws.numel(), _stream()))
    return dQ, dK, dV


def ssc_patch_scores_topk_batched(FN, FM, offN, memN, offM, memM, R, return_scores=False):
    """Patch scores and top-R for B pairs: FN [B,nN,d], FM [B,nM,d]; topk [B,PN,R]."""
    _cuda(FN, FM, offN, memN, offM, memM)
    ldn, ldm = _batched(FN), _batched(FM)
    B, nN, d = FN.shape
    nM = FM.shape[1]
    PN, PM = offN.shape[1] - 1, offM.shape[1] - 1
    dev = FN.device
    topk = torch.empty((B, PN, R), dtype=torch.int32, device=dev)
    scores = torch.empty((B, PN, PM), dtype=torch.float64, device=dev) if return_scores else None
    ws = _workspace(lib().ssc_patch_scores_topk_batched_workspace_size(B, nN, nM, PN, PM, d), dev)
    check("ssc_patch_scores_topk_batched", lib().ssc_patch_scores_topk_batched(
        B, _ptr(FN), ldn, nN, _ptr(FM), ldm, nM, d, _dtype_code(FN), _ptr(offN.contiguous()),
        _ptr(memN.contiguous()), PN, _ptr(offM.contiguous()), _ptr(memM.contiguous()), PM, R,
        _ptr(topk), _ptr(scores), _ptr(ws), ws.numel(), _stream()))
    return (topk, scores) if return_scores else topk
