"""Pins for the CPU oracle: each test checks it against something other than
itself (number-format definitions via numpy/torch, closed forms, library
routines, brute force, hand-worked fixtures)."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import qwm_synth as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _bf(x):
    return syn.f32_to_bf16_bits(np.asarray(x, np.float32))


# ----------------------------------------------------------------- number formats
def test_f16_decode_all_patterns():
    """Every binary16 bit pattern decodes like numpy's float16."""
    L = oracle.lib()
    for h in range(0, 65536):
        ref = np.array([h], np.uint16).view(np.float16).astype(np.float32)[0]
        got = L.qo_f16_to_f32(h)
        if np.isnan(ref):
            assert math.isnan(got)
        else:
            assert got == ref, hex(h)


def test_f16_round_modes_against_numpy():
    """RN matches numpy's float16 cast; RD/RU bracket the value and sit on
    adjacent binary16 values (or coincide when the value is representable)."""
    rng = np.random.default_rng(5)
    xs = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * np.float32(10.0) ** rng.integers(-9, 5, 4000),
        np.array([0.0, -0.0, 65504.0, 65519.0, 65520.0, 70000.0, -70000.0, 2.0 ** -24,
                  2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14, 1.0 / 3.0, -1.0 / 3.0], np.float32)])
    for x in xs:
        x = np.float32(x)
        rn = oracle.f32_to_f16(x, oracle.RN)
        assert rn == int(np.array([x]).astype(np.float16).view(np.uint16)[0]), x
        rd = np.array([oracle.f32_to_f16(x, oracle.RD)], np.uint16).view(np.float16)[0]
        ru = np.array([oracle.f32_to_f16(x, oracle.RU)], np.uint16).view(np.float16)[0]
        if abs(x) <= 65504:
            assert float(rd) <= float(x) <= float(ru), x
            if float(rd) == float(x):
                assert float(ru) == float(x)
            else:
                assert np.nextafter(rd, np.float16(np.inf)) == ru, x


def test_bf16_rounding_against_torch():
    rng = np.random.default_rng(6)
    xs = (rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000)).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.lib().qo_f32_to_bf16(float(x)) for x in xs], np.uint16)
    assert np.array_equal(got, ref)
    # the generator's independent bit-level rounding agrees too
    assert np.array_equal(syn.f32_to_bf16_bits(xs), ref)


# ----------------------------------------------------------------- INT2 residual
def test_int2_hand_worked_cases():
    with open(os.path.join(GOLDEN, "int2_hand_worked.json")) as f:
        gold = json.load(f)
    G = gold["group"]
    for case in gold["cases"]:
        rho = np.array(case["rho"], np.float32)
        codes, params = oracle.int2_encode(rho, G)
        assert list(params) == case["params"], case["derivation"]
        assert list(codes) == case["codes"], case["derivation"]
        deq = oracle.int2_decode(codes, params, len(rho), G)
        assert np.allclose(deq, case["deq"], rtol=0, atol=1e-6), case["derivation"]


@pytest.mark.parametrize("cfg", ["tiny", "small"])
def test_int2_round_trip_bound(cfg):
    """|rho - deq| <= sc/2 (+1 fp32 ulp) on every channel of real residuals."""
    c = syn.get_config(cfg)
    src = syn.FrameSource(c)
    K = src.keys(0)[:, 0, :]
    Kf = syn.bf16_bits_to_f32(K)
    G, d = c.group, c.head_dim
    rng = np.random.default_rng(1)
    n = K.shape[0] if cfg == "tiny" else 200
    for t in range(n):
        cen = Kf[rng.integers(0, K.shape[0])]
        rho = (Kf[t] - cen).astype(np.float32)
        codes, params = oracle.int2_encode(rho, G)
        deq = oracle.int2_decode(codes, params, d, G)
        for g in range(d // G):
            mn = oracle.f16_bits_to_f32(params[2 * g])
            sc = oracle.f16_bits_to_f32(params[2 * g + 1])
            seg = slice(g * G, (g + 1) * G)
            assert mn <= rho[seg].min()
            assert mn + 3 * np.float64(sc) >= rho[seg].max() - 1e-6 * abs(rho[seg].max())
            err = np.abs(rho[seg].astype(np.float64) - deq[seg].astype(np.float64))
            ulp = np.spacing(np.abs(rho[seg]).max() + np.abs(mn) + 3 * sc)
            assert np.all(err <= sc / 2 + 2 * ulp), (t, g)


# ----------------------------------------------------------------- QSAC
def _literal_score(k, c, s, G):
    """The stated score, fp64: sum_g sum_{j in g} s_j step_g^2 / 12, step = range/3."""
    rho = k.astype(np.float64) - c.astype(np.float64)
    tot = 0.0
    for g in range(len(k) // G):
        seg = slice(g * G, (g + 1) * G)
        step = (rho[seg].max() - rho[seg].min()) / 3.0
        tot += float(np.sum(s[seg].astype(np.float64)) * step * step / 12.0)
    return tot


def test_qsac_full_shortlist_is_bruteforce_argmin():
    """With M = C the two-stage choice is the argmin of the stated score over
    all centroids (ties: the chosen score equals the minimum to rounding)."""
    rng = np.random.default_rng(2)
    d, C, G = 16, 8, 4
    for _ in range(3000):
        k = _bf(rng.standard_normal(d) * 2)
        CK = _bf(rng.standard_normal((C, d)) * 2)
        s = rng.uniform(0.05, 3.0, d).astype(np.float32)
        enc = oracle.encode_key(k, CK, G, C, s, _group_sums(s, G), np.zeros((d, 0), np.float32))
        kf, Cf = syn.bf16_bits_to_f32(k), syn.bf16_bits_to_f32(CK)
        scores = np.array([_literal_score(kf, Cf[i], s, G) for i in range(C)])
        best = scores.min()
        assert scores[enc["idx"]] <= best * (1 + 1e-5) + 1e-30


def _group_sums(s, G):
    out = []
    for g in range(len(s) // G):
        acc = np.float32(0.0)
        for j in range(g * G, (g + 1) * G):
            acc = np.float32(acc + s[j])
        out.append(acc)
    return np.array(out, np.float32)


def test_qsac_shortlist_is_smallest_weighted_distances():
    """Stage 1 keeps the M smallest sum_j s_j (k_j - c_j)^2 (checked by a full
    fp64 sort; near-ties may swap only within rounding)."""
    rng = np.random.default_rng(3)
    d, C, M = 16, 8, 4
    for _ in range(3000):
        k = _bf(rng.standard_normal(d) * 2)
        CK = _bf(rng.standard_normal((C, d)) * 2)
        s = rng.uniform(0.05, 3.0, d).astype(np.float32)
        cand, D = oracle.qsac_shortlist(k, CK, s, M)
        kf, Cf = syn.bf16_bits_to_f32(k).astype(np.float64), syn.bf16_bits_to_f32(CK).astype(np.float64)
        Dx = ((kf[None, :] - Cf) ** 2 * s.astype(np.float64)).sum(1)
        order = np.argsort(Dx, kind="stable")
        thr = Dx[order[M - 1]]
        assert np.all(Dx[cand] <= thr * (1 + 1e-5))
        assert len(set(cand.tolist())) == M
        assert list(cand) == sorted(cand, key=lambda i: (D[i], i))
        assert np.allclose(D, Dx, rtol=1e-5)


def test_qsac_reduces_to_nearest_centroid():
    """QVG special case: s = 1 and M = 1 pick the plain nearest centroid."""
    rng = np.random.default_rng(4)
    d, C, G = 64, 16, 16
    for _ in range(500):
        k = _bf(rng.standard_normal(d))
        CK = _bf(rng.standard_normal((C, d)))
        s = np.ones(d, np.float32)
        enc = oracle.encode_key(k, CK, G, 1, s, _group_sums(s, G), np.zeros((d, 0), np.float32))
        dist = ((syn.bf16_bits_to_f32(k).astype(np.float64) - syn.bf16_bits_to_f32(CK)) ** 2).sum(1)
        assert dist[enc["idx"]] <= dist.min() * (1 + 1e-6)


def test_qsac_score_is_expected_logit_perturbation():
    """Eq. 7 with the diagonal of M: for queries with independent channels of
    second moment s_j and INT2 rounding noise uniform on [-step/2, step/2],
    E[(q^T e)^2] = sum_g sum_{j in g} s_j step_g^2 / 12.  The oracle's score
    (the same quantity without the constant 1/108) times 1/108 matches a
    Monte-Carlo estimate."""
    rng = np.random.default_rng(9)
    d, G = 64, 16
    k = _bf(rng.standard_normal(d) * 3)
    c = _bf(rng.standard_normal(d) * 3)
    s = rng.uniform(0.1, 4.0, d).astype(np.float32)
    score = oracle.qsac_score(k, c, _group_sums(s, G), G) / 108.0
    rho = syn.bf16_bits_to_f32(k).astype(np.float64) - syn.bf16_bits_to_f32(c)
    steps = np.repeat([(rho[g * G:(g + 1) * G].max() - rho[g * G:(g + 1) * G].min()) / 3.0
                       for g in range(d // G)], G)
    n = 400000
    q = rng.standard_normal((n, d)) * np.sqrt(s.astype(np.float64))
    e = (rng.random((n, d)) - 0.5) * steps
    mc = np.mean(np.sum(q * e, axis=1) ** 2)
    assert abs(mc - score) / score < 0.02


# ----------------------------------------------------------------- stats, eigen, PSAC
def test_jacobi_matches_numpy_eigh():
    rng = np.random.default_rng(7)
    for d in (16, 64, 128):
        A = rng.standard_normal((d, d))
        A = A @ A.T / d + np.diag(np.arange(d) * 0.01)
        ev, V, _ = oracle.eigh_jacobi(A)
        ref_w, ref_v = np.linalg.eigh(A)
        assert np.allclose(ev, ref_w[::-1], rtol=1e-10, atol=1e-12)
        assert np.allclose(V.T @ V, np.eye(d), atol=1e-12)
        assert np.allclose(A @ V, V * ev, atol=1e-10)
        for kk in range(d):  # eigenvalues here are distinct: vectors equal up to sign
            v, rv = V[:, kk], ref_v[:, d - 1 - kk]
            assert min(np.abs(v - rv).max(), np.abs(v + rv).max()) < 1e-8
            assert v[np.argmax(np.abs(v))] > 0


def test_stats_and_basis_match_planted_query_subspace():
    """Synthetic queries have M = alpha^2 W W^T + beta^2 I in expectation: the
    oracle's statistics recover 0.70 of the energy in the top 8 directions
    (the pages report about 71 %), and U spans W."""
    c = syn.get_config("small")
    src = syn.FrameSource(c)
    Q = src.queries(0, heads=[0], rows=4000)[:, 0, :]
    M = np.zeros((c.head_dim, c.head_dim))
    oracle.stats_accumulate(Q, M)
    s, w, U, ev = oracle.refresh(M, Q.shape[0], 8, c.group)
    share = ev[:8].sum() / ev.sum()
    assert abs(share - 0.70) < 0.02
    W = src.query_basis(0)
    P1, P2 = U.astype(np.float64) @ U.T.astype(np.float64), W @ W.T
    assert np.linalg.norm(P1 - P2, 2) < 0.1
    Mf = M / Q.shape[0]
    assert np.allclose(s, np.diag(Mf), rtol=1e-6)
    # sample second moment: mean of (q^T e)^2 equals e^T M e for any e (Eq. 7)
    qf = syn.bf16_bits_to_f32(Q).astype(np.float64)
    rng = np.random.default_rng(0)
    for _ in range(5):
        e = rng.standard_normal(c.head_dim)
        assert abs(np.mean((qf @ e) ** 2) - e @ Mf @ e) < 1e-9 * (e @ Mf @ e)


def _int2_error(k, c, G):
    """Key error e = k - (c + deq(INT2(k - c))) in fp64, from the pinned INT2 codec."""
    kf = syn.bf16_bits_to_f32(k).astype(np.float64)
    cf = syn.bf16_bits_to_f32(c).astype(np.float64)
    rho = (syn.bf16_bits_to_f32(k) - syn.bf16_bits_to_f32(c)).astype(np.float32)
    codes, params = oracle.int2_encode(rho, G)
    deq = oracle.int2_decode(codes, params, k.shape[0], G).astype(np.float64)
    return kf - (cf + deq)


def test_full_quadratic_score_is_mean_squared_logit_error():
    """Eq. 7 with all of M: for A = (sum_t q_t q_t^T) / n the score equals the mean
    of (q_t . e)^2 over the same queries (exact identity; fp32 rounding only).
    With A = I it is |e|^2, with a rank-one A = q q^T it is (q . e)^2."""
    rng = np.random.default_rng(21)
    d, G, n = 64, 16, 300
    basis = np.linalg.qr(rng.standard_normal((d, 4)))[0]
    Q = _bf(3.0 * rng.standard_normal((n, 4)) @ basis.T + 0.3 * rng.standard_normal((n, d)))
    M = np.zeros((d, d))
    oracle.stats_accumulate(Q, M)
    A = oracle.full_quadratic_matrix(M, n)
    qf = syn.bf16_bits_to_f32(Q).astype(np.float64)
    for _ in range(20):
        k = _bf(rng.standard_normal(d) * 1.5)
        c = _bf(rng.standard_normal(d))
        e = _int2_error(k, c, G)
        ref = np.mean((qf @ e) ** 2)
        assert abs(oracle.qsac_score_full(k, c, A, G) - ref) <= 1e-4 * ref
        assert abs(oracle.qsac_score_full(k, c, np.eye(d, dtype=np.float32), G) - e @ e) \
            <= 1e-5 * (e @ e)
        q1 = qf[0].astype(np.float32)
        A1 = np.outer(q1, q1).astype(np.float32)
        assert abs(oracle.qsac_score_full(k, c, A1, G) - (q1.astype(np.float64) @ e) ** 2) \
            <= 1e-4 * (np.abs(q1) @ np.abs(e)) ** 2
    assert np.array_equal(oracle.full_quadratic_matrix(M, 0), np.zeros((d, d), np.float32))


def test_full_quadratic_choice_minimizes_its_score():
    """With the full-quadratic option the chosen centroid is the shortlist member
    with the smallest e^T A e (ties to the earlier position), and the shortlist
    itself (stage 1) is unchanged."""
    rng = np.random.default_rng(22)
    d, G, C, Mc = 64, 16, 32, 4
    CK = _bf(rng.standard_normal((C, d)))
    s = rng.uniform(0.2, 2.0, d).astype(np.float32)
    X = rng.standard_normal((d, d))
    A = (X @ X.T / d).astype(np.float32)
    U = np.zeros((d, 0), np.float32)
    changed = 0
    for _ in range(100):
        k = _bf(rng.standard_normal(d) * 1.5)
        diag = oracle.encode_key(k, CK, G, Mc, s, _group_sums(s, G), U)
        full = oracle.encode_key(k, CK, G, Mc, s, _group_sums(s, G), U, Afull=A)
        assert np.array_equal(diag["shortlist"], full["shortlist"])
        scores = [oracle.qsac_score_full(k, CK[i], A, G) for i in full["shortlist"]]
        assert full["idx"] == full["shortlist"][int(np.argmin(scores))]
        changed += full["idx"] != diag["idx"]
    assert changed > 0     # the two scores do disagree on some keys


def test_refresh_without_history_is_identity():
    s, w, U, _ = oracle.refresh(np.zeros((64, 64)), 0, 4, 16)
    assert np.all(s == 1.0) and np.all(U == 0.0) and np.all(w == 16.0)


def _psac_case(d, G, r, U, seed):
    rng = np.random.default_rng(seed)
    C = 16
    CK = _bf(rng.standard_normal((C, d)))
    s = rng.uniform(0.2, 2.0, d).astype(np.float32)
    out = []
    for _ in range(200):
        k = _bf(rng.standard_normal(d) * 1.5)
        enc = oracle.encode_key(k, CK, G, 4, s, _group_sums(s, G), U)
        kp = oracle.reconstruct_key_f64(CK[enc["idx"]], enc["codes"], enc["params"],
                                        enc["coef"], enc["cscale"], U, G)
        cs = float(oracle.f16_bits_to_f32(enc["cscale"]))
        out.append((syn.bf16_bits_to_f32(k).astype(np.float64), kp, cs))
    return out


def test_psac_error_on_subspace_is_int8_rounding():
    """|U^T (K - K')|_inf <= cs/2 (+ fp32 rounding) for orthonormal U."""
    d, G, r = 64, 16, 4
    rng = np.random.default_rng(11)
    U = np.linalg.qr(rng.standard_normal((d, r)))[0].astype(np.float32)
    for k, kp, cs in _psac_case(d, G, r, U, 12):
        proj = U.astype(np.float64).T @ (k - kp)
        assert np.abs(proj).max() <= cs / 2 + 1e-5 * (cs + 1e-3)


def test_psac_full_rank_identity_recovers_key():
    """r = d with U = I: the correction carries the whole residual error, so
    K' = K up to the INT8 step (cs/2 per channel)."""
    d, G = 64, 16
    U = np.eye(d, dtype=np.float32)
    for k, kp, cs in _psac_case(d, G, d, U, 13):
        assert np.abs(k - kp).max() <= cs / 2 + 1e-6


def test_psac_logit_error_bound_for_queries_in_span():
    """For q in span(U): |q.(K - K')| <= |q| sqrt(r) cs / 2."""
    d, G, r = 64, 16, 4
    rng = np.random.default_rng(14)
    U = np.linalg.qr(rng.standard_normal((d, r)))[0].astype(np.float32)
    for k, kp, cs in _psac_case(d, G, r, U, 15):
        q = U.astype(np.float64) @ rng.standard_normal(r)
        assert abs(q @ (k - kp)) <= np.linalg.norm(q) * math.sqrt(r) * cs / 2 + 1e-5


# ----------------------------------------------------------------- k-means
def test_kmeans_fixed_point_and_sklearn():
    from sklearn.cluster import KMeans
    c = syn.get_config("tiny")
    X = syn.FrameSource(c).keys(0)[:, 0, :]
    C, it = c.n_centroids, 10
    cent, asg = oracle.kmeans(X, C, it)
    Xf = syn.bf16_bits_to_f32(X).astype(np.float64)
    n = X.shape[0]
    init = Xf[[(i * n) // C for i in range(C)]]
    km = KMeans(n_clusters=C, init=init, n_init=1, max_iter=it, tol=0.0, algorithm="lloyd")
    km.fit(Xf)
    cf = syn.bf16_bits_to_f32(cent).astype(np.float64)
    inertia = ((Xf - cf[asg]) ** 2).sum()
    ref_inertia = ((Xf - syn.bf16_bits_to_f32(syn.f32_to_bf16_bits(
        km.cluster_centers_.astype(np.float32))).astype(np.float64)[km.predict(Xf)]) ** 2).sum()
    assert abs(inertia - ref_inertia) / ref_inertia < 1e-3
    assert np.bincount(asg, minlength=C).sum() == n


def test_kmeans_bruteforce_tiny():
    """Lloyd on a tiny set against a direct fp64 numpy transcription of the
    textbook iteration (assign to nearest, move to the mean)."""
    rng = np.random.default_rng(21)
    for trial in range(20):
        n, d, C = 40, 8, 5
        X = _bf(rng.standard_normal((n, d)))
        cent, asg = oracle.kmeans(X, C, 6)
        Xf = syn.bf16_bits_to_f32(X).astype(np.float64)
        ce = Xf[[(i * n) // C for i in range(C)]].copy()
        for _ in range(6):
            a = np.argmin(((Xf[:, None, :] - ce[None]) ** 2).sum(-1), axis=1)
            for i in range(C):
                if np.any(a == i):
                    ce[i] = Xf[a == i].mean(0)
        assert np.array_equal(a, asg)
        assert np.allclose(syn.bf16_bits_to_f32(cent), ce, rtol=1e-2, atol=1e-2)


# ----------------------------------------------------------------- Values
def _grid_rows(rng, shape, step=0.25, lim=2.0):
    """bf16 rows on a coarse grid: differences, squares and sums of up to 128
    of them are exact in fp32, so the oracle's fp32 fold equals the exact
    distance and every tie it meets is a real tie."""
    k = int(round(lim / step))
    return _bf(rng.integers(-k, k + 1, shape).astype(np.float64) * step)


def test_value_choice_is_bruteforce_nearest_centroid():
    """qo_encode_value picks argmin_i sum_j (v_j - c_ij)^2 over all C centroids
    (numpy fp64 brute force), ties to the lower index, and codes the fp32
    residual v - c of that centroid with the INT2 rule.  3000 grid cases (exact
    arithmetic; half of them with a duplicated nearest row, an exact tie that
    must go to the lower index) plus 1000 Gaussian cases checked against the
    fp32 fold's error bound."""
    rng = np.random.default_rng(41)
    ties = 0
    for case in range(3000):
        d = (16, 32, 64, 128)[case % 4]
        G = 16 if d == 16 else (16, 32)[case % 2]
        C = int(rng.integers(2, 40))
        CV = _grid_rows(rng, (C, d))
        v = _grid_rows(rng, d)
        if case % 2:
            i, j = sorted(rng.choice(C, 2, replace=False))
            CV[j] = CV[i]
            # v one grid step from the duplicated row: the pair is nearest
            v = CV[i].copy()
            v[int(rng.integers(d))] = _bf([syn.bf16_bits_to_f32(v[:1])[0] + 0.25])[0]
        enc = oracle.encode_value(v, CV, G)
        dist = ((syn.bf16_bits_to_f32(CV).astype(np.float64)
                 - syn.bf16_bits_to_f32(v).astype(np.float64)) ** 2).sum(1)
        want = int(np.argmin(dist))            # first index among equal minima
        ties += int(np.count_nonzero(dist == dist.min()) > 1)
        assert enc["idx"] == want, (case, enc["idx"], want)
        rho = (syn.bf16_bits_to_f32(v) - syn.bf16_bits_to_f32(CV[want])).astype(np.float32)
        codes, params = oracle.int2_encode(rho, G)
        assert np.array_equal(enc["codes"], codes) and np.array_equal(enc["params"], params)
    assert ties >= 1500            # the duplicated rows did produce exact ties
    for case in range(1000):
        d, G, C = 128, 32, 64
        CV = _bf(rng.standard_normal((C, d)))
        v = _bf(rng.standard_normal(d) * 1.3)
        enc = oracle.encode_value(v, CV, G)
        dist = ((syn.bf16_bits_to_f32(CV).astype(np.float64)
                 - syn.bf16_bits_to_f32(v).astype(np.float64)) ** 2).sum(1)
        # a left-to-right fp32 fold of d non-negative terms is within
        # (d + 2) 2^-24 of the exact sum, relatively
        tol = (d + 2) * 2.0 ** -24 * dist
        assert dist[enc["idx"]] <= dist.min() + tol[enc["idx"]] + tol.min()
        order = np.argsort(dist, kind="stable")
        if dist[order[1]] - dist[order[0]] > 2 * tol[order[1]]:
            assert enc["idx"] == order[0], case


def test_value_reconstruction_hand_worked_cases():
    """V' = bf16(c + mn_g + code_j sc_g) on fixtures worked out by hand: a
    nonzero centroid with distinct group parameters (a dropped centroid or a
    wrong group index changes every entry) and the single round-to-nearest-even
    of the sum at exact bf16 midpoints."""
    with open(os.path.join(GOLDEN, "value_reconstruct_hand_worked.json")) as f:
        gold = json.load(f)
    G = gold["group"]
    for case in gold["cases"]:
        c = _bf(case["centroid"])
        assert np.array_equal(syn.bf16_bits_to_f32(c), np.array(case["centroid"], np.float32))
        out = oracle.reconstruct_value(c, np.array(case["codes"], np.uint8),
                                       np.array(case["params"], np.uint16), G)
        got = syn.bf16_bits_to_f32(out)
        assert np.array_equal(got, np.array(case["expected"], np.float32)), case["derivation"]


@pytest.mark.parametrize("d,G,C", [(64, 16, 16), (128, 32, 256)])
def test_value_round_trip_bound(d, G, C):
    """Encoding then reconstructing a Value leaves |v - V'| <= sc_g / 2 plus half
    a bf16 ulp of V' on every channel: the INT2 step bound of the residual and
    the one rounding of the sum."""
    rng = np.random.default_rng(43 + d)
    CV = _bf(rng.standard_normal((C, d)))
    for _ in range(300):
        v = _bf(rng.standard_normal(d) * rng.uniform(0.2, 4.0))
        enc = oracle.encode_value(v, CV, G)
        out = oracle.reconstruct_value(CV[enc["idx"]], enc["codes"], enc["params"], G)
        vf = syn.bf16_bits_to_f32(v).astype(np.float64)
        of = syn.bf16_bits_to_f32(out).astype(np.float64)
        sc = np.repeat(oracle.f16_bits_to_f32(enc["params"][1::2]).astype(np.float64), G)
        half_ulp = np.where(of != 0, 2.0 ** (np.floor(np.log2(np.abs(of) + 1e-300)) - 8), 2.0 ** -134)
        slack = 4 * 2.0 ** -24 * (np.abs(vf) + np.abs(of))      # fp32 residual and decode
        assert np.all(np.abs(vf - of) <= sc / 2 + half_ulp + slack)


# ----------------------------------------------------------------- attention, compression
def test_attention_unquantized_matches_sdpa_fp64():
    rng = np.random.default_rng(31)
    for (nq, T, d) in [(5, 1, 64), (17, 300, 64), (9, 129, 128)]:
        Q = _bf(rng.standard_normal((nq, d)))
        K = _bf(rng.standard_normal((T, d)) * 2)
        V = _bf(rng.standard_normal((T, d)))
        O = oracle.attention_head(Q, K, V, 1.0 / math.sqrt(d))
        t = lambda a: torch.from_numpy(syn.bf16_bits_to_f32(a).astype(np.float64))
        ref = torch.nn.functional.scaled_dot_product_attention(t(Q)[None], t(K)[None], t(V)[None])[0]
        assert np.abs(O - ref.numpy()).max() <= 1e-5


def test_attention_lse_brute_force_and_invariants():
    """ln sum exp against math.fsum over Python floats on small cases; equal keys
    give s + ln T; a key set split in two merges through the log-sum-exp weights
    into the attention over the union."""
    rng = np.random.default_rng(33)
    for (nq, T, d) in [(3, 1, 64), (4, 37, 64), (2, 130, 128)]:
        Q = _bf(rng.standard_normal((nq, d)))
        K = _bf(rng.standard_normal((T, d)) * 3)
        sc = 1.0 / math.sqrt(d)
        got = oracle.attention_lse(Q, K, sc)
        qf = syn.bf16_bits_to_f32(Q).astype(np.float64)
        kf = syn.bf16_bits_to_f32(K).astype(np.float64)
        for i in range(nq):
            s = [sc * math.fsum(float(a) * float(b) for a, b in zip(qf[i], kf[t])) for t in range(T)]
            m = max(s)
            ref = m + math.log(math.fsum(math.exp(x - m) for x in s))
            assert abs(got[i] - ref) <= 1e-12 * max(1.0, abs(ref))
    Q = _bf(rng.standard_normal((3, 64)))
    k = _bf(rng.standard_normal((1, 64)))
    K = np.repeat(k, 50, axis=0)
    s0 = (syn.bf16_bits_to_f32(Q).astype(np.float64) @ syn.bf16_bits_to_f32(k[0]).astype(np.float64)) * 0.125
    assert np.allclose(oracle.attention_lse(Q, K, 0.125), s0 + math.log(50), rtol=0, atol=1e-12)
    K = _bf(rng.standard_normal((90, 64)))
    V = _bf(rng.standard_normal((90, 64)))
    Q = _bf(rng.standard_normal((5, 64)))
    O = oracle.attention_head(Q, K, V, 0.125)
    O1, O2 = oracle.attention_head(Q, K[:40], V[:40], 0.125), oracle.attention_head(Q, K[40:], V[40:], 0.125)
    l1, l2 = oracle.attention_lse(Q, K[:40], 0.125), oracle.attention_lse(Q, K[40:], 0.125)
    l = oracle.attention_lse(Q, K, 0.125)
    w1, w2 = np.exp(l1 - l)[:, None], np.exp(l2 - l)[:, None]
    assert np.allclose(w1 + w2, 1.0, atol=1e-12)
    assert np.allclose(w1 * O1 + w2 * O2, O, atol=1e-12)


def test_top1_matches_numpy_argmax():
    rng = np.random.default_rng(32)
    Q = _bf(rng.standard_normal((20, 64)))
    K = _bf(rng.standard_normal((500, 64)))
    idx = oracle.top1(Q, K)
    ref = np.argmax(syn.bf16_bits_to_f32(Q).astype(np.float64) @ syn.bf16_bits_to_f32(K).astype(np.float64).T, axis=1)
    assert np.array_equal(idx, ref)


def test_packed_bytes_follow_compression_formula():
    c = syn.get_config("tiny")
    src = syn.FrameSource(c)
    oc = oracle.OracleCache(c.heads, c.head_dim, c.n_centroids, c.group, c.n_cand, c.rank,
                            c.total_tokens)
    Q, K, V = src.frame(0)
    oc.build_centroids(K, V)
    oc.update_query_stats(Q)
    oc.append_kv(K, V)
    per = oracle.bytes_per_token_head(c.head_dim, c.n_centroids, c.group, c.rank)
    assert per == 2 * (64 // 4 + 4 * (64 // 16) + 1) + 4 + 2
    assert oc.packed_bytes() == per * c.heads * oc.len
    for (d, C, G, r, want) in [(128, 256, 32, 8, 108), (128, 512, 32, 8, 110)]:
        assert oracle.bytes_per_token_head(d, C, G, r) == want


# ----------------------------------------------------------------------------- centroid refresh
def _drift_cache(rebuild_every, frames=12, n=192, sigma=0.4, seed=31):
    import dataclasses
    c = dataclasses.replace(syn.get_config("1min"), heads=1, tokens_per_frame=n, q_rows=n,
                            frames=frames, n_centroids=32, drift_sigma=sigma)
    src = syn.FrameSource(c, seed)
    oc = oracle.OracleCache(1, c.head_dim, c.n_centroids, c.group, c.n_cand, c.rank,
                            frames * n)
    Ks = []
    for f in range(frames):
        Q, K, V = src.frame(f)
        if f == 0:
            oc.build_centroids(K, V, iters=5)
        elif rebuild_every and f % rebuild_every == 0:
            oc.rebuild_centroids(K, V, iters=5)
        oc.update_query_stats(Q, refresh_basis=True)
        oc.append_kv(K, V)
        Ks.append(K[:, 0, :])
    return oc, np.concatenate(Ks), n


def test_ranged_reconstruction_equals_whole_head():
    """One table version: the per-run reconstruction equals the whole-head routine."""
    oc, _, _ = _drift_cache(0, frames=3)
    Kp, Vp = oc.reconstruct(0)
    T = oc.len
    Kh = np.zeros((T, oc.d), np.uint16); Vh = np.zeros((T, oc.d), np.uint16)
    Uall = np.ascontiguousarray(np.stack(oc.U), np.float32)
    P = oracle._p
    oracle.lib().qo_reconstruct_head(0, 1, oc.d, oc.C, oc.G, oc.r, oc.Tcap, T, P(oc.CK), P(oc.CV),
                                     P(Uall), P(oc.tok_ver), P(oc.k_codes), P(oc.k_params),
                                     P(oc.k_idx), P(oc.k_coef), P(oc.k_cscale), P(oc.v_codes),
                                     P(oc.v_params), P(oc.v_idx), P(Kh), P(Vh))
    assert np.array_equal(Kp, Kh) and np.array_equal(Vp, Vh)


def test_centroid_rebuild_keeps_old_tokens():
    """Tokens appended before a centroid rebuild reconstruct bit for bit as before."""
    import dataclasses
    c = dataclasses.replace(syn.get_config("1min"), heads=1, tokens_per_frame=160, q_rows=160,
                            frames=4, n_centroids=32, drift_sigma=0.4)
    src = syn.FrameSource(c, 5)
    oc = oracle.OracleCache(1, c.head_dim, c.n_centroids, c.group, c.n_cand, c.rank, 4 * 160)
    for f in range(2):
        Q, K, V = src.frame(f)
        if f == 0:
            oc.build_centroids(K, V, iters=4)
        oc.update_query_stats(Q, True)
        oc.append_kv(K, V)
    before = oc.reconstruct(0)
    Q, K, V = src.frame(2)
    oc.rebuild_centroids(K, V, iters=4)
    assert oc.cent_version == 1 and not np.array_equal(oc.cent_versions[0][0], oc.CK)
    oc.update_query_stats(Q, True)
    oc.append_kv(K, V)
    after = oc.reconstruct(0)
    assert np.array_equal(after[0][:320], before[0]) and np.array_equal(after[1][:320], before[1])
    assert np.all(oc.tok_cver[:320] == 0) and np.all(oc.tok_cver[320:480] == 1)
    # rebuilding from the first frame's data gives the first tables again (determinism)
    _, K0, V0 = src.frame(0)
    oc.rebuild_centroids(K0, V0, iters=4)
    assert np.array_equal(oc.CK, oc.cent_versions[0][0])
    assert np.array_equal(oc.CV, oc.cent_versions[0][1])


def test_centroid_rebuild_tracks_key_drift():
    """Under a drifting Key mean, tables rebuilt every 4 frames from the newest
    frame leave a smaller reconstruction error on the late frames than the
    frame-0 tables do."""
    stale, K, n = _drift_cache(0)
    fresh, _, _ = _drift_cache(4)
    kf = syn.bf16_bits_to_f32(K).astype(np.float64)
    late = slice(len(kf) - 4 * n, len(kf))
    err = {}
    for name, oc in (("stale", stale), ("fresh", fresh)):
        Kp, _ = oc.reconstruct(0)
        err[name] = float(np.mean((syn.bf16_bits_to_f32(Kp).astype(np.float64)[late] - kf[late]) ** 2))
    assert err["fresh"] < 0.9 * err["stale"], err

