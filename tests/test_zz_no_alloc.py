"""qwm_build_centroids_noalloc: the centroid build for callers that cannot
allocate device memory (hosts that own the GPU memory budget and forbid
cudaMalloc/cudaFree inside plugins).  Its scratch is a fixed array inside the
library; it must write exactly the tables qwm_build_centroids writes with the
cache's WORKSPACE buffer, call after call, although every call reuses the
array.  Collected last so that a failure here stops a -x run only after every
other test has run."""
import numpy as np
import pytest
import torch

import bit_kv_cache_23_b200 as q
import qwm_synth as syn

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def _tables(g):
    torch.cuda.synchronize()
    return (g.view("cent_k").cpu().numpy().copy(), g.view("cent_v").cpu().numpy().copy())


def _cache(c):
    return q.QuantKVCache(c.heads, c.head_dim, c.n_centroids, c.group, c.n_cand, c.rank,
                          c.total_tokens, max_versions=4)


def test_noalloc_matches_workspace_build_on_two_calls():
    c = syn.get_config("small")
    src = syn.FrameSource(c)
    g_ref = _cache(c)
    g_na = _cache(c)
    for f in (0, 1):  # two calls in a row, different inputs, one shared scratch
        K, V = _dev(src.keys(f)), _dev(src.values(f))
        g_ref.build_centroids(K, V, iters=c.kmeans_iters)
        q.qwm_build_centroids_noalloc(g_na.c, K, V, c.kmeans_iters)
        ref_k, ref_v = _tables(g_ref)
        na_k, na_v = _tables(g_na)
        assert np.array_equal(ref_k, na_k) and np.array_equal(ref_v, na_v), f
    assert g_na.c.has_centroids == 1


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # fp32 centroids 4 H C d + assignments 4 H n must fit the 16 MiB array.
    # 32 heads x 512 x 128: 8 MiB of centroids, so n = 65536 tokens fill the
    # array exactly and one more token does not fit.
    H, C, d = 32, 512, 128
    n_fit = (q.QWM_NOALLOC_SCRATCH_BYTES - 4 * H * C * d) // (4 * H)
    assert n_fit == 65536
    g = q.QuantKVCache(H, d, C, 32, 4, 8, n_fit + 1, max_versions=2)
    K = torch.zeros((n_fit + 1, H, d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(q.QwmError) as ei:
        q.qwm_build_centroids_noalloc(g.c, K, K, 1)
    assert ei.value.status == 3  # QWM_ERR_CAPACITY
    assert g.c.has_centroids == 0
    q.qwm_build_centroids_noalloc(g.c, K[:n_fit], K[:n_fit], 1)   # exactly the array
    torch.cuda.synchronize()
    assert g.c.has_centroids == 1 and q.qwm_device_status() == 0
    # the centroid part alone beyond the array: 64 heads x 512 x 128 x 4 B = 16 MiB
    g2 = q.QuantKVCache(64, d, C, 32, 4, 8, 1024, max_versions=2)
    K2 = torch.zeros((600, 64, d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(q.QwmError) as ei:
        q.qwm_build_centroids_noalloc(g2.c, K2, K2, 1)
    assert ei.value.status == 3
