"""Centroid refresh under Key drift on the CUDA path, against the oracle.

The 1-minute streaming layer's Key distribution drifts (a random walk of the
channel means), so tables built on the first frame go stale.  The pages say
only that each Key is assigned to a cluster centre kept at higher precision
("Flickering after quantization?" (SynthePulse), QSAC paragraph) and are silent
on refreshing the centres; the reading taken here: a rebuild runs the same
k-means on the newest frame and writes a new table version, later appends
encode against it, and every cached token keeps decoding with the version it
was encoded with.

Checked bit for bit: every table version, every packed field of every token and
each token's table version; the reconstruction of tokens cached before a
rebuild is unchanged by it.  Attention is checked within tolerance over a cache
whose version boundaries fall inside 64-key tiles.
"""
import numpy as np
import pytest
import torch

import oracle
import qwm_synth as syn
from parity_util import (ATOL_MAX, ATOL_MEAN, attention_error, compare_packed,
                         new_state_report, refresh_from_oracle, stack_state, to_dev, u16)

pytestmark = pytest.mark.gpu


def _layer(heads, n, frames, rebuild_every, refresh_every):
    q = pytest.importorskip("bit_kv_cache_23_b200")
    c = syn.get_config("1min")
    src = syn.FrameSource(c)
    H, d, C = len(heads), c.head_dim, c.n_centroids
    nver = frames // rebuild_every + 1
    g = q.QuantKVCache(H, d, C, c.group, c.n_cand, c.rank, frames * n,
                       max_versions=frames + 2, max_cent_versions=nver, max_queries=n)
    oc = oracle.OracleCache(H, d, C, c.group, c.n_cand, c.rank, frames * n)
    Mref = {h: np.zeros((d, d)) for h in range(H)}
    rep = new_state_report()
    out = dict(tables=[], packed={}, cver_ok=True, attn=[], old_tokens_same=True, g=g, oc=oc)
    nq = 0
    snapshot = None
    for f in range(frames):
        Q, K, V = src.frame(f, heads=heads)
        Q, K, V = Q[:n], K[:n], V[:n]
        Qd, Kd, Vd = to_dev(Q), to_dev(K), to_dev(V)
        if f % rebuild_every == 0:
            g.build_centroids(Kd, Vd, iters=c.kmeans_iters)
            if f == 0:
                oc.build_centroids(K, V, iters=c.kmeans_iters)
            else:
                oc.rebuild_centroids(K, V, iters=c.kmeans_iters)
            torch.cuda.synchronize()
            ck = g.view("cent_k").cpu().numpy().view(np.uint16)
            cv = g.view("cent_v").cpu().numpy().view(np.uint16)
            out["tables"].append((g.cent_version, oc.cent_version,
                                  bool(np.array_equal(ck, oc.CK) and np.array_equal(cv, oc.CV))))
            if snapshot is not None:
                # tokens cached before the rebuild reconstruct exactly as before it
                Kp, Vp = g.reconstruct(0, snapshot[0])
                out["old_tokens_same"] &= bool(torch.equal(Kp, snapshot[1])
                                               and torch.equal(Vp, snapshot[2]))
        refresh = (f % refresh_every) == 0
        g.update_query_stats(Qd, refresh_basis=refresh)
        for h in range(H):
            oracle.stats_accumulate(Q[:, h, :], Mref[h])
        nq += n
        if refresh:
            st = refresh_from_oracle(g, Mref, nq, range(H), c.rank, c.group, rep)
            s, w, U = stack_state(st, H)
            oc.set_state(s=s, w=w, U=U)
        t0 = g.len
        g.append_kv(Kd, Vd)
        oc.append_kv(K, V)
        for k, v in compare_packed(g, oc, t0, g.len).items():
            out["packed"][k] = out["packed"].get(k, 0) + v
        torch.cuda.synchronize()
        cvg = g.view("centver")[t0:g.len].cpu().numpy().view(np.uint16)
        out["cver_ok"] &= bool(np.array_equal(cvg, oc.tok_cver[t0:g.len]))
        if (f + 1) % rebuild_every == 0 and f + 1 < frames:
            Kp, Vp = g.reconstruct(0, g.len)
            snapshot = (g.len, Kp.clone(), Vp.clone())
        if f in (rebuild_every, frames - 1):
            Od = g.attention(Qd)
            torch.cuda.synchronize()
            assert q.qwm_device_status() == 0
            rows = np.arange(0, n, 7)
            Oref = oc.attention(Q, rows=rows)
            out["attn"].append((f,) + attention_error(syn.bf16_bits_to_f32(u16(Od))[rows], Oref))
    out["rep"] = rep
    return out


def test_centroid_rebuilds_match_oracle():
    """1-minute layer, 3 heads, 9 frames of 600 tokens (600 = 9 x 64 + 24, so each
    frame boundary, and with it each table-version boundary, falls inside a key
    tile), C = 512, tables rebuilt every 3 frames, basis every 2."""
    out = _layer(heads=[0, 17, 39], n=600, frames=9, rebuild_every=3, refresh_every=2)
    assert [t[:2] for t in out["tables"]] == [(0, 0), (1, 1), (2, 2)]
    assert all(t[2] for t in out["tables"]), "a rebuilt table differs from the oracle's"
    assert out["packed"] == {}, out["packed"]
    assert out["cver_ok"], "per-token table versions differ"
    assert out["old_tokens_same"], "a rebuild changed the reconstruction of cached tokens"
    rep = out["rep"]
    assert rep["stats_mismatch"] == 0 and rep["sw_mismatch"] == 0, rep
    for f, mx, mean in out["attn"]:
        assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (f, mx, mean)


def test_rebuild_on_empty_cache_and_capacity():
    """A rebuild before any token rewrites the version in force; once tokens are
    cached every rebuild takes a new slot, and with none left the call fails
    with QWM_ERR_CAPACITY and changes nothing."""
    q = pytest.importorskip("bit_kv_cache_23_b200")
    c = syn.get_config("small")
    src = syn.FrameSource(c)
    g = q.QuantKVCache(2, 128, 256, 32, 4, 8, 4 * 880, max_versions=8, max_cent_versions=2)
    _, K0, V0 = src.frame(0, heads=[0, 1])
    _, K1, V1 = src.frame(1, heads=[0, 1])
    g.build_centroids(to_dev(K0), to_dev(V0), iters=3)
    g.build_centroids(to_dev(K1), to_dev(V1), iters=3)      # empty cache: same slot
    assert (g.c.n_cent_versions, g.cent_version) == (1, 0)
    g.append_kv(to_dev(K0), to_dev(V0))
    g.build_centroids(to_dev(K0), to_dev(V0), iters=3)      # second slot
    assert (g.c.n_cent_versions, g.cent_version) == (2, 1)
    g.append_kv(to_dev(K1), to_dev(V1))
    with pytest.raises(q.QwmError) as ei:
        g.build_centroids(to_dev(K1), to_dev(V1), iters=3)
    assert ei.value.status == 3
    assert (g.c.n_cent_versions, g.cent_version) == (2, 1)
    torch.cuda.synchronize()
    cv = g.view("centver")[:2 * 880].cpu().numpy()
    assert np.all(cv[:880] == 0) and np.all(cv[880:] == 1)
    # the first table is the k-means of frame 1 (the rewrite), the second of frame 0
    ck0 = np.stack([oracle.kmeans(K1[:, h, :], 256, 3)[0] for h in range(2)])
    ck1 = np.stack([oracle.kmeans(K0[:, h, :], 256, 3)[0] for h in range(2)])
    assert np.array_equal(g.view("cent_k", 0).cpu().numpy().view(np.uint16), ck0)
    assert np.array_equal(g.view("cent_k", 1).cpu().numpy().view(np.uint16), ck1)
