"""The C ABI without a GPU: the library loads, exports every call include/ssc.h
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

from spatial_spectral_attention_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssc.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ssc_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary_calls():
    names = _declared()
    for must in ("ssc_fps_patches", "ssc_patch_scores_topk", "ssc_dense_coupling_fwd",
                 "ssc_dense_coupling_bwd", "ssc_geo_coupling_fwd", "ssc_geo_coupling_bwd"):
        assert must in names


def test_library_exports_every_declared_symbol():
    L = _abi.lib()
    for name in _declared():
        assert hasattr(L, name), name
        assert name in _abi.SIGNATURES, name


def test_status_strings_and_version():
    L = _abi.lib()
    for code in range(7):
        assert L.ssc_status_string(code)
    assert L.ssc_version() >= 1


def test_workspace_queries_are_host_only():
    L = _abi.lib()
    assert L.ssc_fps_patches_workspace_size(160000, 1280) > 160000 * 8
    assert L.ssc_patch_scores_topk_workspace_size(1280, 1280, 128) >= 1280 * 1280 * 8
    assert L.ssc_dense_coupling_workspace_size(60000, 60000, 128, 196, 0) > 60000 * 208 * 2
    assert L.ssc_geo_coupling_workspace_size(60000, 60000, 128, 196, 480, 480, 8, 0) > 0
    assert L.ssc_dense_coupling_workspace_size(0, 10, 128, 196, 0) == 0


P0 = ctypes.c_void_p(16)  # a non-null, aligned dummy address that is never dereferenced


def _dense_fwd(nN=10, nM=10, d=128, k=16, scale=0.1, dtype=0, ldq=128, ldk=128, ldv=16,
               ws=None, wsb=1 << 20):
    L = _abi.lib()
    return L.ssc_dense_coupling_fwd(P0, ldq, P0, ldk, P0, ldv, nN, nM, d, k, scale, dtype,
                                    P0, k, P0, ws if ws is not None else ctypes.c_void_p(256),
                                    wsb, None)


def test_argument_checks_return_before_any_device_work():
    assert _dense_fwd(nN=0) == 1                  # invalid size
    assert _dense_fwd(d=96, ldq=96, ldk=96) == 2  # unsupported d
    assert _dense_fwd(k=300, ldv=300) == 2        # unsupported k
    assert _dense_fwd(scale=float("nan")) == 1
    assert _dense_fwd(scale=-1.0) == 1
    assert _dense_fwd(ldq=127, d=128) == 1        # ld < d
    assert _dense_fwd(ldq=132) == 3               # bf16 row pitch not a multiple of 8
    assert _dense_fwd(dtype=5) == 1
    assert _dense_fwd(ws=ctypes.c_void_p(0)) == 4  # no workspace
    assert _dense_fwd(wsb=16) == 4                 # workspace too small
    L = _abi.lib()
    assert L.ssc_fps_patches(P0, 10, 11, 0, P0, P0, P0, P0, ctypes.c_void_p(256), 1 << 20, None) == 1
    assert L.ssc_fps_patches(P0, 10, 3, 10, P0, P0, P0, P0, ctypes.c_void_p(256), 1 << 20, None) == 1
    assert L.ssc_patch_scores_topk(P0, 128, 100, P0, 128, 100, 128, 0, P0, P0, 10, P0, P0, 10,
                                   11, P0, None, ctypes.c_void_p(256), 1 << 20, None) == 1


def test_profile_record_arguments_are_checked_on_the_host():
    L = _abi.lib()
    ms, n = ctypes.c_double(-1.0), ctypes.c_int(-1)
    assert L.ssc_profile_enable(3) == 1  # SSC_ERR_INVALID_ARG
    assert L.ssc_profile_read(1000, ctypes.byref(ms), ctypes.byref(n)) == 1
    assert L.ssc_profile_read(-1, ctypes.byref(ms), ctypes.byref(n)) == 1
    assert L.ssc_profile_read(0, None, ctypes.byref(n)) == 1
    # an empty record reads as zero launches without touching the device
    assert L.ssc_profile_enable(1) == 0 and L.ssc_profile_enable(0) == 0
    assert L.ssc_profile_read(2, ctypes.byref(ms), ctypes.byref(n)) == 0
    assert n.value == 0 and ms.value == 0.0


def test_fps_cluster_size_hook_checks_its_argument():
    L = _abi.lib()
    assert L.ssc_debug_fps_cluster_size(5) == 1
    assert L.ssc_debug_fps_cluster_size(8) == 0
    assert L.ssc_debug_fps_cluster_size(0) == 0


def test_abort_path_hook_checks_its_argument():
    L = _abi.lib()
    assert L.ssc_debug_stall_next_launch(3) == 1   # SSC_ERR_INVALID_ARG
    assert L.ssc_debug_stall_next_launch(-1) == 1
    assert L.ssc_debug_stall_next_launch(2) == 0   # armed (host-side flag only)
    assert L.ssc_debug_stall_next_launch(0) == 0   # and disarmed
