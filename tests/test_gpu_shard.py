"""Head-sharded caches on the GPU: the split that `bench.py --shard heads`
uses across ranks, checked on one GPU.

The path has no exchange between heads: statistics, basis refresh, centroid
tables, append and attention are all per head.  So caches built for the head
blocks [0, 6) and [6, 12) of the small layer must hold exactly what the
whole-layer cache holds for those heads, and give the same outputs bit for bit.
"""
import numpy as np
import pytest
import torch

import qwm_synth as syn
from parity_util import to_dev

pytestmark = pytest.mark.gpu

FIELDS = ["k_codes", "k_params", "k_idx", "k_coef", "k_cscale", "v_codes", "v_params", "v_idx",
          "cent_k", "cent_v", "qstats", "sens", "wgroup"]


def test_head_blocks_equal_whole_layer():
    q = pytest.importorskip("bit_kv_cache_23_b200")
    from bit_kv_cache_23_b200 import shard

    c = syn.get_config("small")
    src = syn.FrameSource(c)
    world = 2
    blocks = [shard.head_range(r, world, c.heads) for r in range(world)]
    assert blocks == [(0, 6), (6, 12)]

    def cache(H):
        return q.QuantKVCache(H, c.head_dim, c.n_centroids, c.group, c.n_cand, c.rank,
                              c.total_tokens, max_versions=c.frames + 2)

    full = cache(c.heads)
    parts = [cache(h1 - h0) for h0, h1 in blocks]
    outs_full, outs_part = [], [[] for _ in blocks]
    for f in range(c.frames):
        Q, K, V = src.frame(f)
        if f == 0:
            full.build_centroids(to_dev(K), to_dev(V), iters=c.kmeans_iters)
        full.update_query_stats(to_dev(Q))
        full.append_kv(to_dev(K), to_dev(V))
        outs_full.append(full.attention(to_dev(Q)))
        for i, (h0, h1) in enumerate(blocks):
            Qb, Kb, Vb = (np.ascontiguousarray(a[:, h0:h1]) for a in (Q, K, V))
            g = parts[i]
            if f == 0:
                g.build_centroids(to_dev(Kb), to_dev(Vb), iters=c.kmeans_iters)
            g.update_query_stats(to_dev(Qb))
            g.append_kv(to_dev(Kb), to_dev(Vb))
            outs_part[i].append(g.attention(to_dev(Qb)))
    torch.cuda.synchronize()
    assert q.qwm_device_status() == 0
    T = full.len
    for i, (h0, h1) in enumerate(blocks):
        g = parts[i]
        for name in FIELDS:
            a = full.view(name)[h0:h1]
            b = g.view(name)
            if a.dim() >= 2 and name not in ("cent_k", "cent_v", "qstats", "sens", "wgroup"):
                a, b = a[:, :T], b[:, :T]
            assert torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8)), name
        # the basis version in force, and the per-token versions
        bf = full.view("basis")[full.version, h0:h1]
        bp = g.view("basis")[g.version]
        assert torch.equal(bf.contiguous().view(torch.int32), bp.contiguous().view(torch.int32))
        assert torch.equal(full.view("tokver")[:T], g.view("tokver")[:T])
        assert torch.equal(full.view("centver")[:T], g.view("centver")[:T])
        for f in range(c.frames):
            a = outs_full[f][:, h0:h1].contiguous().view(torch.int16)
            assert torch.equal(a, outs_part[i][f].view(torch.int16)), (i, f)
