"""GPU path (C ABI through the binding) against the CPU oracle.

Bit-exact: centroid tables, the Query statistics matrix, s and w, centroid
indices, INT2 codes, fp16 group parameters, INT8 coefficients and scales.
Tolerance: the basis against the oracle's Jacobi basis (which both sides then
encode with), and attention output within max-abs 2e-2 and mean-abs 2e-3 of the
oracle's fp64 attention over its own reconstructed cache.
"""
import numpy as np
import pytest
import torch

import oracle
import qwm_synth as syn
from parity_util import (ATOL_MAX, ATOL_MEAN, compare_packed, new_state_report,
                         refresh_from_oracle, run_layer, stack_state, to_dev, u16)

pytestmark = pytest.mark.gpu


def _assert_common(out, proj_tol=1e-4):
    assert out["cent_k_equal"] and out["cent_v_equal"], "k-means centroids differ"
    assert out["packed_mismatch"] == {}, out["packed_mismatch"]
    assert out["stats_mismatch"] == 0, out["stats_mismatch"]
    assert out["sw_mismatch"] == 0, out["sw_mismatch"]
    assert out["orth_err"] < 1e-5, out["orth_err"]
    assert out["proj_err"] < proj_tol, out["proj_err"]
    for f, mx, mean in out["attn"]:
        assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (f, mx, mean)


def test_tiny_full():
    out = run_layer("tiny")
    _assert_common(out)
    # reconstruction: GPU fp32 sum vs oracle fp64 sum, both rounded to bf16
    g, oc = out["gpu"], out["oracle"]
    Kp, Vp = g.reconstruct()
    Ko, Vo = oc.reconstruct(0)
    kg = syn.bf16_bits_to_f32(u16(Kp[0])).astype(np.float64)
    ko = syn.bf16_bits_to_f32(Ko).astype(np.float64)
    # one bf16 ulp (8 significant bits) of the larger magnitude: the two sums may
    # straddle a bf16 rounding boundary; that must stay rare
    big = np.maximum(np.abs(kg), np.abs(ko))
    ulp = np.where(big > 0, 2.0 ** (np.floor(np.log2(np.where(big > 0, big, 1.0))) - 7), 0.0)
    diff = np.abs(kg - ko)
    assert np.all(diff <= ulp), float((diff / np.maximum(ulp, 1e-300)).max())
    assert np.count_nonzero(diff) <= 1e-3 * diff.size, np.count_nonzero(diff)
    assert np.array_equal(u16(Vp[0]), Vo)


def test_small_full():
    out = run_layer("small", attn_rows=24, attn_frames={0, 4, 8})
    _assert_common(out)


def test_top1_shift_tiny():
    out = run_layer("tiny")
    g, oc, src, c = out["gpu"], out["oracle"], out["src"], out["cfg"]
    Kall = np.concatenate([src.keys(f) for f in range(c.frames)], axis=0)
    Q = src.queries(c.frames - 1)
    ie, iq = g.top1_shift(to_dev(Q), to_dev(Kall))
    ie, iq = ie.cpu().numpy(), iq.cpu().numpy()
    Ko, _ = oc.reconstruct(0)
    ref_e = oracle.top1(Q[:, 0, :], Kall[:, 0, :])
    ref_q = oracle.top1(Q[:, 0, :], Ko)
    qf = syn.bf16_bits_to_f32(Q[:, 0, :]).astype(np.float64)
    for ref, got, K in ((ref_e, ie[:, 0], Kall[:, 0, :]), (ref_q, iq[:, 0], Ko)):
        sc = qf @ syn.bf16_bits_to_f32(K).astype(np.float64).T
        best = sc[np.arange(len(ref)), ref]
        mine = sc[np.arange(len(ref)), got]
        assert np.all(best - mine <= 1e-4 * np.abs(best) + 1e-4)


def test_qvg_mode_without_statistics():
    """QVG reading (M = 1, s = 1, r = 0): no Query statistics are ever taken, so
    every key goes to its plain nearest centroid; head_dim 128 and 64."""
    q = pytest.importorskip("bit_kv_cache_23_b200")
    for (H, d, C, G, n) in [(3, 128, 256, 32, 900), (2, 64, 16, 16, 300)]:
        g = q.QuantKVCache(H, d, C, G, 1, 0, 2 * n, max_versions=2)
        oc = oracle.OracleCache(H, d, C, G, 1, 0, 2 * n)
        rng = np.random.default_rng(4000 + d)
        w = np.ones(d)
        w[rng.permutation(d)[:4]] = 6.0
        K = [syn.f32_to_bf16_bits((rng.standard_normal((n, H, d)) * w).astype(np.float32))
             for _ in range(2)]
        V = [syn.f32_to_bf16_bits(rng.standard_normal((n, H, d)).astype(np.float32))
             for _ in range(2)]
        g.build_centroids(to_dev(K[0]), to_dev(V[0]), iters=3)
        ck = np.stack([oracle.kmeans(K[0][:, h, :], C, 3)[0] for h in range(H)])
        cv = np.stack([oracle.kmeans(V[0][:, h, :], C, 3)[0] for h in range(H)])
        oc.set_state(CK=ck, CV=cv)
        for f in range(2):
            t0 = g.len
            g.append_kv(to_dev(K[f]), to_dev(V[f]))
            oc.append_kv(K[f], V[f])
            assert compare_packed(g, oc, t0, g.len) == {}, (d, f)
        Q = syn.f32_to_bf16_bits(rng.standard_normal((150, H, d)).astype(np.float32))
        O = g.attention(to_dev(Q))
        torch.cuda.synchronize()
        assert q.qwm_device_status() == 0
        Oref = oc.attention(Q)
        err = np.abs(syn.bf16_bits_to_f32(u16(O)) - Oref)
        assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN, (d, err.max(), err.mean())


@pytest.mark.parametrize("d,C,G,M,r,n,nqa", [(128, 64, 32, 4, 8, 300, 300),
                                              (128, 64, 32, 4, 8, 700, 200),
                                              (64, 16, 16, 4, 4, 700, 200)])
def test_full_quadratic_qsac(d, C, G, M, r, n, nqa):
    """QSAC stage 2 by e^T A e (the full-quadratic option, CUDA-core append): the
    GPU's snapshot A = fp32(M / n) equals the oracle's bit for bit, and every
    packed field matches the oracle's encoding with the same option.  The first
    case (900 cached keys, 300 queries of norm ~10, outlier channels, a peaky
    softmax) is the one where attention is most sensitive to how each K' element
    is rounded: the attention must read exactly the bf16 reconstruction."""
    q = pytest.importorskip("bit_kv_cache_23_b200")
    H, F = 2, 3
    g = q.QuantKVCache(H, d, C, G, M, r, F * n, max_versions=F + 2, qsac_full=True)
    oc = oracle.OracleCache(H, d, C, G, M, r, F * n, qsac_full=True)
    rng = np.random.default_rng(5000 + d)
    w = np.ones(d)
    w[rng.permutation(d)[:4]] = 6.0
    basis = np.linalg.qr(rng.standard_normal((d, 8)))[0]
    Mref = {h: np.zeros((d, d)) for h in range(H)}
    rep = new_state_report()
    for f in range(F):
        K = syn.f32_to_bf16_bits(((rng.standard_normal((n, H, d)) + 0.3 * rng.standard_normal(d))
                                  * w).astype(np.float32))
        V = syn.f32_to_bf16_bits(rng.standard_normal((n, H, d)).astype(np.float32))
        Q = syn.f32_to_bf16_bits((3.0 * rng.standard_normal((n, H, 8)) @ basis.T
                                  + 0.5 * rng.standard_normal((n, H, d))).astype(np.float32))
        if f == 0:
            g.build_centroids(to_dev(K), to_dev(V), iters=3)
            oc.set_state(CK=np.stack([oracle.kmeans(K[:, h, :], C, 3)[0] for h in range(H)]),
                         CV=np.stack([oracle.kmeans(V[:, h, :], C, 3)[0] for h in range(H)]))
        g.update_query_stats(to_dev(Q), refresh_basis=True)
        for h in range(H):
            oracle.stats_accumulate(Q[:, h, :], Mref[h])
        st = refresh_from_oracle(g, Mref, n * (f + 1), range(H), r, G, rep, check_basis=False)
        s, wg, U = stack_state(st, H)
        A = np.stack([oracle.full_quadratic_matrix(Mref[h], n * (f + 1)) for h in range(H)])
        eig = g.view("eigvec").cpu().numpy()
        for h in range(H):
            blk = eig[h * d * d:(h + 1) * d * d].view(np.float32)[64 * d:64 * d + d * d]
            assert np.array_equal(blk.view(np.uint32), A[h].reshape(-1).view(np.uint32)), (f, h)
        oc.set_state(s=s, w=wg, U=U, A=A)
        t0 = g.len
        g.append_kv(to_dev(K), to_dev(V))
        oc.append_kv(K, V)
        assert compare_packed(g, oc, t0, g.len) == {}, f
    assert rep["stats_mismatch"] == 0 and rep["sw_mismatch"] == 0, rep
    Qa = np.ascontiguousarray(Q[:nqa])
    O = g.attention(to_dev(Qa))
    torch.cuda.synchronize()
    assert q.qwm_device_status() == 0
    Oref = oc.attention(Qa)
    err = np.abs(syn.bf16_bits_to_f32(u16(O)) - Oref)
    assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN, (err.max(), err.mean())


def test_degenerate_inputs():
    """Constant keys (zero residual groups), repeated tokens, one-token appends,
    a ragged tail and zero-variance channels."""
    c = syn.get_config("tiny")
    H, d, C = 1, 64, 16
    g = pytest.importorskip("bit_kv_cache_23_b200").QuantKVCache(H, d, C, 16, 4, 4, 300,
                                                                 max_versions=8)
    oc = oracle.OracleCache(H, d, C, 16, 4, 4, 300)
    rng = np.random.default_rng(77)
    base = rng.standard_normal((40, H, d)).astype(np.float32)
    base[:, :, :16] = 0.25       # a constant group
    base[5:15] = base[5]         # repeated tokens
    K = syn.f32_to_bf16_bits(base)
    V = syn.f32_to_bf16_bits(rng.standard_normal((40, H, d)).astype(np.float32))
    g.build_centroids(to_dev(K), to_dev(V), iters=3)
    torch.cuda.synchronize()
    CK = g.view("cent_k").cpu().numpy().view(np.uint16).copy()
    CV = g.view("cent_v").cpu().numpy().view(np.uint16).copy()
    ck, _ = oracle.kmeans(K[:, 0, :], C, 3)
    cv, _ = oracle.kmeans(V[:, 0, :], C, 3)
    assert np.array_equal(ck, CK[0]) and np.array_equal(cv, CV[0])
    oc.set_state(CK=ck[None], CV=cv[None])
    # appends before any query statistics: s = 1, U = 0
    for n in (1, 7, 32):
        t0 = g.len
        g.append_kv(to_dev(K[:n]), to_dev(V[:n]))
        oc.append_kv(K[:n], V[:n])
        assert compare_packed(g, oc, t0, g.len) == {}
    Q = syn.f32_to_bf16_bits(rng.standard_normal((3, H, d)).astype(np.float32))
    g.update_query_stats(to_dev(Q), refresh_basis=True)   # fewer queries than rank
    Mref = {0: np.zeros((d, d))}
    oracle.stats_accumulate(Q[:, 0, :], Mref[0])
    rep = new_state_report()
    # rank-deficient statistics: the basis is not unique, so only the oracle's is used
    st = refresh_from_oracle(g, Mref, 3, [0], 4, 16, rep, check_basis=False)
    assert rep["stats_mismatch"] == 0 and rep["sw_mismatch"] == 0, rep
    s, w, U = stack_state(st, H)
    oc.set_state(s=s, w=w, U=U)
    t0 = g.len
    g.append_kv(to_dev(K), to_dev(V))
    oc.append_kv(K, V)
    assert compare_packed(g, oc, t0, g.len) == {}
    O = g.attention(to_dev(Q))
    torch.cuda.synchronize()
    Oref = oc.attention(Q)
    err = np.abs(syn.bf16_bits_to_f32(u16(O)) - Oref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3


@pytest.mark.parametrize("G,C,M,r", [(16, 64, 4, 8), (32, 48, 3, 16), (16, 512, 8, 5),
                                     (32, 256, 1, 0), (32, 256, 4, 0), (32, 256, 1, 8),
                                     (32, 256, 4, 2), (16, 128, 4, 4)])
def test_head128_shapes(G, C, M, r):
    """head_dim 128 with groups of 16, C not a power of two, C = 512 (two MMA
    chunks), M up to 8 and ranks other than 8: every packed field bit for bit,
    attention within tolerance; keys with outlier channels and frame drift.
    Also the ablation settings: M = 1 and r = 0 (plain nearest centroid with the
    sensitivity weights, no compensation), QSAC alone (r = 0), PSAC alone
    (M = 1), and ranks 2 and 4."""
    H, d, n = 3, 128, 700
    q = pytest.importorskip("bit_kv_cache_23_b200")
    # workspace for split-key attention (the key range is split across pairs)
    g = q.QuantKVCache(H, d, C, G, M, r, 3 * n, max_versions=8, max_queries=200)
    oc = oracle.OracleCache(H, d, C, G, M, r, 3 * n)
    rng = np.random.default_rng(1000 + G + C + r)
    w = np.ones(d)
    w[rng.permutation(d)[:6]] = 6.0
    Kf = [((rng.standard_normal((n, H, d)) + 0.3 * rng.standard_normal(d)) * w).astype(np.float32)
          for _ in range(3)]
    K = [syn.f32_to_bf16_bits(x) for x in Kf]
    V = [syn.f32_to_bf16_bits(rng.standard_normal((n, H, d)).astype(np.float32)) for _ in range(3)]
    basis = np.linalg.qr(rng.standard_normal((d, 8)))[0]
    g.build_centroids(to_dev(K[0]), to_dev(V[0]), iters=4)
    torch.cuda.synchronize()
    CK = g.view("cent_k").cpu().numpy().view(np.uint16).copy()
    CV = g.view("cent_v").cpu().numpy().view(np.uint16).copy()
    ck = np.stack([oracle.kmeans(K[0][:, h, :], C, 4)[0] for h in range(H)])
    cv = np.stack([oracle.kmeans(V[0][:, h, :], C, 4)[0] for h in range(H)])
    assert np.array_equal(ck, CK) and np.array_equal(cv, CV)
    oc.set_state(CK=ck, CV=cv)
    Mref = {h: np.zeros((d, d)) for h in range(H)}
    rep = new_state_report()
    for f in range(3):
        Q = syn.f32_to_bf16_bits((3.3 * rng.standard_normal((200, H, 8)) @ basis.T
                                  + 0.5 * rng.standard_normal((200, H, d))).astype(np.float32))
        g.update_query_stats(to_dev(Q), refresh_basis=True)
        for h in range(H):
            oracle.stats_accumulate(Q[:, h, :], Mref[h])
        st = refresh_from_oracle(g, Mref, 200 * (f + 1), range(H), r, G, rep,
                                 check_basis=(r <= 8))
        s, w, U = stack_state(st, H)
        oc.set_state(s=s, w=w, U=U if r else None)
        t0 = g.len
        g.append_kv(to_dev(K[f]), to_dev(V[f]))
        oc.append_kv(K[f], V[f])
        assert compare_packed(g, oc, t0, g.len) == {}, f
    assert rep["stats_mismatch"] == 0 and rep["sw_mismatch"] == 0, rep
    assert rep["orth_err"] < 1e-5 and rep["proj_err"] < 1e-3, rep
    O = g.attention(to_dev(Q))
    torch.cuda.synchronize()
    assert q.qwm_device_status() == 0
    rows = np.arange(0, 200, 13)
    Oref = oc.attention(Q, rows=rows)
    err = np.abs(syn.bf16_bits_to_f32(u16(O))[rows] - Oref)
    assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN, (err.max(), err.mean())


def _edge_tables(rng, C, d):
    """Centroid tables built to hit the append's corner cases: rows 0..63 are
    sign flips of one vector (a zero key is equally far from all 64, so far more
    than 16 centroids survive the tensor-core prefilter and the full exact
    rescoring runs), rows 64..66 are one row repeated (exact distance ties,
    which go to the lower index), row 67 is all zero, the rest Gaussian with
    outlier channels."""
    base = 1.0 + np.arange(d) / d
    signs = np.where(rng.integers(0, 2, (64, d)) == 1, 1.0, -1.0)
    T = rng.standard_normal((C, d)) * np.where(np.arange(d) % 17 == 0, 6.0, 1.0)
    T[:64] = signs * base
    T[65] = T[64]
    T[66] = T[64]
    T[67] = 0.0
    return _bf_rows(T)


def _bf_rows(x):
    return syn.f32_to_bf16_bits(np.asarray(x, np.float32))


def _edge_tokens(rng, tab, n, d):
    """n rows mixing: zero rows, rows equal to a centroid (incl. the repeated
    one), rows with constant and all-zero 32-channel groups, rows with channels
    scaled by 100, rows next to the repeated centroid, and Gaussian rows."""
    X = rng.standard_normal((n, d)) * np.where(np.arange(d) % 17 == 0, 6.0, 1.0)
    tf = syn.bf16_bits_to_f32(tab).astype(np.float64)
    kinds = np.arange(n) % 8
    for i in range(n):
        k = kinds[i]
        if k == 0:
            X[i] = 0.0
        elif k == 1:
            X[i] = tf[rng.integers(0, tab.shape[0])]
        elif k == 2:
            X[i] = tf[64]
        elif k == 3:
            X[i, :32] = 0.25
            X[i, 64:96] = 0.0
        elif k == 4:
            X[i, rng.permutation(d)[:5]] *= 100.0
        elif k == 5:
            X[i] = tf[64] + 0.01 * rng.standard_normal(d)
    return _bf_rows(X)


@pytest.mark.parametrize("C", [256, 512])
def test_append_tc_edge_cases(C):
    """head_dim 128 (the tensor-core append): exact distance ties between
    distinct centroid rows, keys equal to a centroid, zero and constant groups,
    outlier channels scaled by 100 against the prefilter's error bound, and the
    more-than-16-survivors fallback (zero keys against 64 equidistant rows):
    every packed field bit for bit against the oracle."""
    q = pytest.importorskip("bit_kv_cache_23_b200")
    H, d, G, M, r, n = 2, 128, 32, 4, 8, 640
    rng = np.random.default_rng(9000 + C)
    g = q.QuantKVCache(H, d, C, G, M, r, 2 * n, max_versions=4)
    oc = oracle.OracleCache(H, d, C, G, M, r, 2 * n)
    K0 = _bf_rows(rng.standard_normal((C, H, d)))
    g.build_centroids(to_dev(K0), to_dev(K0), iters=1)      # sets the state; tables replaced
    CK = np.stack([_edge_tables(rng, C, d) for _ in range(H)])
    CV = np.stack([_edge_tables(rng, C, d) for _ in range(H)])
    g.view("cent_k").copy_(torch.from_numpy(CK.view(np.int16)))
    g.view("cent_v").copy_(torch.from_numpy(CV.view(np.int16)))
    oc.set_state(CK=CK, CV=CV)
    basis = np.linalg.qr(rng.standard_normal((d, 8)))[0]
    Mref = {h: np.zeros((d, d)) for h in range(H)}
    rep = new_state_report()
    for f in range(2):
        Q = _bf_rows(3.0 * rng.standard_normal((300, H, 8)) @ basis.T
                     + 0.5 * rng.standard_normal((300, H, d)))
        g.update_query_stats(to_dev(Q), refresh_basis=True)
        for h in range(H):
            oracle.stats_accumulate(Q[:, h, :], Mref[h])
        st = refresh_from_oracle(g, Mref, 300 * (f + 1), range(H), r, G, rep)
        s, w, U = stack_state(st, H)
        oc.set_state(s=s, w=w, U=U)
        K = np.stack([_edge_tokens(rng, CK[h], n, d) for h in range(H)], axis=1)
        V = np.stack([_edge_tokens(rng, CV[h], n, d) for h in range(H)], axis=1)
        t0 = g.len
        g.append_kv(to_dev(K), to_dev(V))
        oc.append_kv(K, V)
        assert compare_packed(g, oc, t0, g.len) == {}, f
        assert q.qwm_device_status() == 0
    assert rep["stats_mismatch"] == 0 and rep["sw_mismatch"] == 0, rep
    # the zero keys really did meet 64 equidistant centroids
    kz = np.zeros(d, np.uint16)
    _, D = oracle.qsac_shortlist(kz, CK[0], s[0], M)
    assert np.count_nonzero(D[:64] == D[:64].min()) == 64
