"""ssc_fps_patches_noalloc: the patch call for callers that cannot allocate any
device memory (not even a workspace), which uses the library's fixed device
scratch instead.  Called through the C ABI directly and compared with the
workspace-taking ssc_fps_patches on two calls in a row (the second call finds
the shared scratch dirty from the first).  Results are integer tables, so the
comparison is bit-exact, as for every FPS test.  Collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from spatial_spectral_attention_b200 import _abi, api, synth

pytestmark = pytest.mark.gpu


def _raw_noalloc(pts, P):
    n = pts.shape[0]
    outs = [torch.empty(m, dtype=torch.int32, device="cuda") for m in (P, n, P + 1, n)]
    rc = _abi.lib().ssc_fps_patches_noalloc(
        ctypes.c_void_p(pts.data_ptr()), n, P, 0, *[ctypes.c_void_p(t.data_ptr()) for t in outs],
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, _abi.lib().ssc_status_string(rc)
    return outs


def test_noalloc_matches_workspace_call_twice():
    for n, P, seed in ((40000, 320, 1), (7000, 61, 2)):
        pts = torch.tensor(synth.sphere_points(n, np.random.default_rng(seed)).astype(np.float32)).cuda()
        got = _raw_noalloc(pts, P)
        ref = api.ssc_fps_patches(pts, P)
        torch.cuda.synchronize()
        for g, r in zip(got, ref):
            assert torch.equal(g, r)


def test_noalloc_memory_resident_path_near_its_limit():
    # with 8-CTA clusters, n > 131072 keeps the running distances in the
    # scratch array instead of on chip; n close to the 262144 limit fills
    # most of the array
    L = _abi.lib()
    assert L.ssc_debug_fps_cluster_size(8) == 0
    try:
        n, P = 250000, 40
        pts = torch.tensor(synth.sphere_points(n, np.random.default_rng(3)).astype(np.float32)).cuda()
        for _ in range(2):
            got = _raw_noalloc(pts, P)
            ref = api.ssc_fps_patches(pts, P)
            torch.cuda.synchronize()
            for g, r in zip(got, ref):
                assert torch.equal(g, r)
    finally:
        assert L.ssc_debug_fps_cluster_size(0) == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = _abi.lib()
    big = 262145
    rc = L.ssc_fps_patches_noalloc(ctypes.c_void_p(16), big, 10, 0, ctypes.c_void_p(16),
                                   ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16),
                                   None)
    assert rc == 2  # SSC_ERR_UNSUPPORTED, nothing enqueued
