"""ctypes declarations of libssc (include/ssc.h).  Loading fails loudly when the
library has not been built: there is no fallback implementation."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssc.so")

P = ctypes.c_void_p
I = ctypes.c_int
F = ctypes.c_float
Z = ctypes.c_size_t
U64 = ctypes.c_ulonglong

# name -> (restype, argtypes)
SIGNATURES = {
    "ssc_status_string": (ctypes.c_char_p, [I]),
    "ssc_version": (I, []),
    "ssc_kernel_launches": (U64, []),
    "ssc_profile_enable": (I, [I]),
    "ssc_profile_read": (I, [I, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int)]),
    "ssc_device_status": (I, [P, I, ctypes.POINTER(I)]),
    "ssc_set_wait_limit_ns": (I, [U64]),
    "ssc_debug_wait_timeout": (I, [U64, P]),
    "ssc_debug_stall_next_launch": (I, [I]),
    "ssc_debug_fps_cluster_size": (I, [I]),
    "ssc_fps_patches_workspace_size": (Z, [I, I]),
    "ssc_fps_patches": (I, [P, I, I, I, P, P, P, P, P, Z, P]),
    "ssc_fps_patches_noalloc": (I, [P, I, I, I, P, P, P, P, P]),
    "ssc_fps_patches_mesh_workspace_size": (Z, [I, I]),
    "ssc_fps_patches_mesh": (I, [P, P, P, I, I, I, I, P, P, P, P, P, Z, P]),
    "ssc_patch_scores_topk_workspace_size": (Z, [I, I, I]),
    "ssc_patch_scores_topk": (I, [P, I, I, P, I, I, I, I, P, P, I, P, P, I, I, P, P, P, Z, P]),
    "ssc_dense_coupling_workspace_size": (Z, [I, I, I, I, I]),
    "ssc_dense_coupling_fwd": (I, [P, I, P, I, P, I, I, I, I, I, F, I, P, I, P, P, Z, P]),
    "ssc_dense_coupling_bwd": (I, [P, I, P, I, P, I, I, I, I, I, F, I, P, I, P, P, I,
                                   P, I, P, I, P, I, P, Z, P]),
    "ssc_dense_coupling_fwd_e4m3_workspace_size": (Z, [I, I, I, I]),
    "ssc_dense_coupling_fwd_e4m3": (I, [P, I, P, I, P, I, I, I, I, I, F, P, I, P, P, Z, P]),
    "ssc_dense_coupling_bwd_deterministic": (I, [P, I, P, I, P, I, I, I, I, I, F, I, P, I, P, P, I,
                                                 P, I, P, I, P, I, P, Z, P]),
    "ssc_geo_coupling_workspace_size": (Z, [I, I, I, I, I, I, I, I]),
    "ssc_geo_coupling_fwd": (I, [P, I, P, I, P, I, I, I, I, I, F, I,
                                 P, P, I, P, P, I, P, I, P, I, P, P, Z, P]),
    "ssc_geo_coupling_bwd": (I, [P, I, P, I, P, I, I, I, I, I, F, I,
                                 P, P, I, P, P, I, P, I, P, I, P, P, I,
                                 P, I, P, I, P, I, P, Z, P]),
    "ssc_geo_coupling_bwd_reuse": (I, [P, I, P, I, P, I, I, I, I, I, F, I,
                                       P, P, I, P, P, I, P, I, P, I, P, P, I,
                                       P, I, P, I, P, I, P, Z, P]),
    "ssc_dense_coupling_batched_workspace_size": (Z, [I, I, I, I, I, I]),
    "ssc_dense_coupling_fwd_batched": (I, [I, P, I, P, I, P, I, I, I, I, I, F, I, P, I, P, P, Z, P]),
    "ssc_dense_coupling_bwd_batched": (I, [I, P, I, P, I, P, I, I, I, I, I, F, I, P, I, P, P, I,
                                           P, I, P, I, P, I, P, Z, P]),
    "ssc_geo_coupling_batched_workspace_size": (Z, [I, I, I, I, I, I, I, I, I]),
    "ssc_geo_coupling_fwd_batched": (I, [I, P, I, P, I, P, I, I, I, I, I, F, I,
                                         P, P, I, P, P, I, P, I, P, I, P, P, Z, P]),
    "ssc_geo_coupling_bwd_batched": (I, [I, P, I, P, I, P, I, I, I, I, I, F, I,
                                         P, P, I, P, P, I, P, I, P, I, P, P, I,
                                         P, I, P, I, P, I, P, Z, P]),
    "ssc_patch_scores_topk_batched_workspace_size": (Z, [I, I, I, I, I, I]),
    "ssc_patch_scores_topk_batched": (I, [I, P, I, I, P, I, I, I, I, P, P, I, P, P, I, I, P, P, P,
                                          Z, P]),
    "ssc_linear_coupling_workspace_size": (Z, [I, I, I, I]),
    "ssc_linear_coupling_fwd": (I, [P, I, P, I, P, I, I, I, I, I, P, I, P, P, Z, P]),
    "ssc_linear_coupling_bwd": (I, [P, I, P, I, P, I, I, I, I, I, P, I, P, P, I,
                                    P, I, P, I, P, I, P, Z, P]),
}

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libssc.so not found at {LIB_PATH}; build it with "
                "`python -m spatial_spectral_attention_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


class SSCError(RuntimeError):
    def __init__(self, fn: str, code: int):
        msg = lib().ssc_status_string(code).decode()
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


def check(fn: str, code: int) -> None:
    if code != 0:
        raise SSCError(fn, code)
