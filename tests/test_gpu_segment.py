"""Attention over the packed history followed by a bf16 segment (qwm_attention_ext),
and its log-sum-exp output, against the CPU oracle.

The oracle attends over its own reconstruction of the packed cache concatenated
with the exact segment (fp64), and gives ln sum exp of the scaled scores over the
same keys.  Cases: head_dim 128 (tensor-core kernel) and 64 (CUDA-core kernel),
ragged packed and segment lengths, an empty cache (plain bf16 attention over
the segment), an empty segment, and the merge of two disjoint key sets through
the log-sum-exp weights.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import qwm_synth as syn
from parity_util import (ATOL_MAX, ATOL_MEAN, compare_packed, new_state_report,
                         refresh_from_oracle, stack_state, to_dev, u16)

pytestmark = pytest.mark.gpu

# |lse_gpu - lse_oracle|: the scores differ by the bf16 rounding of the
# reconstructed keys and the fp32 accumulation, which the log-sum-exp averages
LSE_MAX, LSE_MEAN = 2e-2, 2e-3


def _bf(x):
    return syn.f32_to_bf16_bits(np.asarray(x, np.float32))


def _filled_cache(H, d, C, G, M, r, frames, n, seed, max_queries=0):
    """GPU cache and oracle cache, filled with the same frames, both encoding with
    the oracle's own state; returns (g, oc, frames of (Q, K, V))."""
    q = pytest.importorskip("bit_kv_cache_23_b200")
    rng = np.random.default_rng(seed)
    T = frames * n
    g = q.QuantKVCache(H, d, C, G, M, r, T, max_versions=frames + 2, max_queries=max_queries)
    oc = oracle.OracleCache(H, d, C, G, M, r, T)
    w = np.ones(d)
    w[rng.permutation(d)[:4]] = 6.0
    basis = np.linalg.qr(rng.standard_normal((d, 8)))[0]
    data = []
    Mref = {h: np.zeros((d, d)) for h in range(H)}
    rep = new_state_report()
    for f in range(frames):
        K = _bf((rng.standard_normal((n, H, d)) + 0.3 * rng.standard_normal(d)) * w)
        V = _bf(rng.standard_normal((n, H, d)))
        Q = _bf(3.0 * rng.standard_normal((n, H, 8)) @ basis.T + 0.5 * rng.standard_normal((n, H, d)))
        if f == 0:
            g.build_centroids(to_dev(K), to_dev(V), iters=3)
            ck = np.stack([oracle.kmeans(K[:, h, :], C, 3)[0] for h in range(H)])
            cv = np.stack([oracle.kmeans(V[:, h, :], C, 3)[0] for h in range(H)])
            torch.cuda.synchronize()
            assert np.array_equal(ck, g.view("cent_k").cpu().numpy().view(np.uint16))
            assert np.array_equal(cv, g.view("cent_v").cpu().numpy().view(np.uint16))
            oc.set_state(CK=ck, CV=cv)
        g.update_query_stats(to_dev(Q), refresh_basis=True)
        for h in range(H):
            oracle.stats_accumulate(Q[:, h, :], Mref[h])
        st = refresh_from_oracle(g, Mref, n * (f + 1), range(H), r, G, rep, check_basis=False)
        s, wg, U = stack_state(st, H)
        oc.set_state(s=s, w=wg, U=U if r else None)
        t0 = g.len
        g.append_kv(to_dev(K), to_dev(V))
        oc.append_kv(K, V)
        assert compare_packed(g, oc, t0, g.len) == {}
        data.append((Q, K, V))
    assert rep["stats_mismatch"] == 0 and rep["sw_mismatch"] == 0, rep
    return g, oc, data


def _oracle_ext(oc, Q, Kseg, Vseg, heads, scale):
    """Oracle attention and lse over [reconstructed cache ; segment] per head."""
    nq, H, d = Q.shape
    O = np.zeros((nq, len(heads), d))
    L = np.zeros((nq, len(heads)))
    for i, h in enumerate(heads):
        if oc.len > 0:
            Kp, Vp = oc.reconstruct(h)
            Kp, Vp = Kp[:oc.len], Vp[:oc.len]
        else:
            Kp = np.zeros((0, d), np.uint16)
            Vp = np.zeros((0, d), np.uint16)
        Kall = np.concatenate([Kp, Kseg[:, h, :]]) if Kseg is not None else Kp
        Vall = np.concatenate([Vp, Vseg[:, h, :]]) if Vseg is not None else Vp
        O[:, i, :] = oracle.attention_head(Q[:, h, :], Kall, Vall, scale)
        L[:, i] = oracle.attention_lse(Q[:, h, :], Kall, scale)
    return O, L


def _check(Og, Lg, Oo, Lo):
    e = np.abs(syn.bf16_bits_to_f32(Og).astype(np.float64) - Oo)
    assert e.max() <= ATOL_MAX and e.mean() <= ATOL_MEAN, (e.max(), e.mean())
    el = np.abs(Lg.astype(np.float64) - Lo)
    assert el.max() <= LSE_MAX and el.mean() <= LSE_MEAN, (el.max(), el.mean())


def _run_ext(g, Q, Kseg, Vseg):
    q = pytest.importorskip("bit_kv_cache_23_b200")
    nq, H, _ = Q.shape
    lse = torch.empty((nq, H), dtype=torch.float32, device="cuda")
    O = g.attention_ext(to_dev(Q), None if Kseg is None else to_dev(Kseg),
                        None if Vseg is None else to_dev(Vseg), lse=lse)
    torch.cuda.synchronize()
    assert q.qwm_device_status() == 0, "a bounded device wait timed out"
    return u16(O), lse.cpu().numpy()


@pytest.mark.parametrize("d,C,G,M,r,n,nseg,nq,split", [
    (128, 64, 32, 4, 8, 700, 300, 300, False),   # tensor-core kernel, ragged tiles, one pair
    (128, 64, 32, 4, 8, 700, 300, 300, True),    # the same with the key range split across pairs
    (128, 64, 16, 1, 0, 650, 64, 130, True),     # no compensation (rank 0), one full segment tile
    (64, 16, 16, 4, 4, 300, 77, 70, False),      # CUDA-core kernel
])
def test_history_plus_segment(d, C, G, M, r, n, nseg, nq, split):
    H = 3 if d == 128 else 2
    g, oc, data = _filled_cache(H, d, C, G, M, r, 2, n, seed=500 + d + r,
                                max_queries=nq if split else 0)
    rng = np.random.default_rng(600 + d)
    Kseg = _bf(rng.standard_normal((nseg, H, d)) * 1.5)
    Vseg = _bf(rng.standard_normal((nseg, H, d)))
    Q = data[-1][0][:nq]
    Og, Lg = _run_ext(g, Q, Kseg, Vseg)
    Oo, Lo = _oracle_ext(oc, Q, Kseg, Vseg, range(H), 1.0 / math.sqrt(d))
    _check(Og, Lg, Oo, Lo)
    # no segment: the packed history alone, with its lse
    Og0, Lg0 = _run_ext(g, Q, None, None)
    Oo0, Lo0 = _oracle_ext(oc, Q, None, None, range(H), 1.0 / math.sqrt(d))
    _check(Og0, Lg0, Oo0, Lo0)
    assert np.array_equal(Og0, u16(g.attention(to_dev(Q))))


@pytest.mark.parametrize("d,nseg,nq", [(128, 1000, 260), (128, 5, 17), (64, 200, 64)])
def test_empty_cache_is_plain_attention(d, nseg, nq):
    """With no packed tokens the call is plain bf16 attention over the segment."""
    q = pytest.importorskip("bit_kv_cache_23_b200")
    H = 2
    g = q.QuantKVCache(H, d, 16, 16, 4, 4, 64, max_versions=2)   # never filled
    rng = np.random.default_rng(700 + nseg)
    Kseg = _bf(rng.standard_normal((nseg, H, d)) * 2.0)
    Vseg = _bf(rng.standard_normal((nseg, H, d)))
    Q = _bf(rng.standard_normal((nq, H, d)))
    Og, Lg = _run_ext(g, Q, Kseg, Vseg)
    Oo, Lo = _oracle_ext(oracle.OracleCache(H, d, 16, 16, 4, 4, 64), Q, Kseg, Vseg, range(H),
                         1.0 / math.sqrt(d))
    _check(Og, Lg, Oo, Lo)


def test_merge_of_history_and_segment():
    """Attention over [history ; segment] equals the lse-weighted merge of the
    attention over the history alone and over the segment alone (an empty cache),
    on the small layer (12 heads, 7920 cached tokens, an 880-token segment)."""
    q = pytest.importorskip("bit_kv_cache_23_b200")
    from parity_util import make_gpu_cache
    c = syn.get_config("small")
    src = syn.FrameSource(c)
    g = make_gpu_cache(c)
    for f in range(c.frames):
        Q, K, V = src.frame(f)
        if f == 0:
            g.build_centroids(to_dev(K), to_dev(V), iters=c.kmeans_iters)
        g.update_query_stats(to_dev(Q), refresh_basis=True)
        g.append_kv(to_dev(K), to_dev(V))
    Q, Kseg, Vseg = src.frame(c.frames)            # the frame being generated
    empty = q.QuantKVCache(c.heads, c.head_dim, c.n_centroids, c.group, c.n_cand, c.rank, 16)
    O, L = _run_ext(g, Q, Kseg, Vseg)
    O1, L1 = _run_ext(g, Q, None, None)
    O2, L2 = _run_ext(empty, Q, Kseg, Vseg)
    Lm = np.logaddexp(L1.astype(np.float64), L2.astype(np.float64))
    assert np.abs(Lm - L).max() <= 1e-4 * max(1.0, np.abs(L).max())
    w1 = np.exp(L1 - Lm)[..., None]
    w2 = np.exp(L2 - Lm)[..., None]
    f = lambda a: syn.bf16_bits_to_f32(a).astype(np.float64)
    merged = w1 * f(O1) + w2 * f(O2)
    e = np.abs(merged - f(O))
    # each side is rounded to bf16 once: two half-ulps of |O| <= ~4
    assert e.max() <= 2e-2 and e.mean() <= 2e-3, (e.max(), e.mean())
