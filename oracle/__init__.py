"""CPU oracle for the QuantWM KV-cache path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (the CUDA library in
``bit_kv_cache_23_b200``) never imports it, and the two share no code.

The arithmetic lives in ``qwm_oracle.c`` (plain C, built with gcc
``-O2 -ffp-contract=off``); this module loads it through ctypes and adds the
bookkeeping of a cache (frame-by-frame append, basis versions, statistics)
with numpy arrays.  Every function names the passage of the QuantWM pages it
follows in the C source.

Parity status: every oracle function is pinned by a ``-m "not gpu"`` test
(closed forms, library routines, brute force), except attention over the
*quantized* cache, whose value the pages do not fix: parity unpinned there
beyond the pinned pieces it is built from (reconstruction and exact attention).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qwm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

P = ctypes.c_void_p
I32 = ctypes.c_int32
I64 = ctypes.c_int64
F32 = ctypes.c_float
F64 = ctypes.c_double
U16 = ctypes.c_uint16


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (no GPU needed)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=gnu11", "-Wall",
               "-shared", "-fPIC", "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        sig = {
            "qo_f16_to_f32": (F32, [U16]),
            "qo_f32_to_f16": (U16, [F32, I32]),
            "qo_bf16_to_f32": (F32, [U16]),
            "qo_f64_to_bf16": (U16, [F64]),
            "qo_f32_to_bf16": (U16, [F32]),
            "qo_weighted_dist": (F32, [P, P, P, I32]),
            "qo_sq_dist_f32c": (F32, [P, P, I32]),
            "qo_kmeans": (I32, [P, I64, I32, I64, I32, I32, P, P]),
            "qo_stats_accumulate": (None, [P, I64, I32, I64, P]),
            "qo_eigh_jacobi": (I32, [P, I32, P, P]),
            "qo_refresh": (None, [P, I64, I32, I32, I32, P, P, P, P]),
            "qo_int2_encode": (None, [P, I32, I32, P, P]),
            "qo_int2_decode": (None, [P, P, I32, I32, P]),
            "qo_qsac_shortlist": (None, [P, P, I32, I32, P, I32, P, P]),
            "qo_qsac_score": (F32, [P, P, P, I32, I32]),
            "qo_qsac_score_full": (F32, [P, P, P, I32, I32]),
            "qo_encode_key": (None, [P, P, I32, I32, I32, I32, P, P, P, I32, P, P, P, P, P, P,
                                     P]),
            "qo_encode_value": (None, [P, P, I32, I32, I32, P, P, P]),
            "qo_append_frame": (None, [I32, I32, I32, I32, I32, I32, I64, I64, P, P, I64, P, P,
                                       P, P, P, P, P, P, P, P, P, P, P, P]),
            "qo_reconstruct_key": (None, [P, P, P, P, U16, P, I32, I32, I32, P, P]),
            "qo_reconstruct_value": (None, [P, P, P, I32, I32, P]),
            "qo_reconstruct_head": (None, [I32, I32, I32, I32, I32, I32, I64, I64, P, P, P, P,
                                           P, P, P, P, P, P, P, P, P, P]),
            "qo_reconstruct_range": (None, [I32, I32, I32, I32, I32, I32, I64, I64, I64, P, P, P,
                                            P, P, P, P, P, P, P, P, P, P, P]),
            "qo_attention_head": (None, [P, I64, I64, P, P, I64, I32, F64, P]),
            "qo_attention_lse": (None, [P, I64, I64, P, I64, I32, F64, P]),
            "qo_top1": (None, [P, I64, I64, P, I64, I64, I32, P]),
            "qo_bytes_per_token_head": (I64, [I32, I32, I32, I32]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


RN, RD, RU = 0, 1, 2


# ----------------------------------------------------------------------------- formats
def f32_to_f16(x: float, mode: int) -> int:
    return int(lib().qo_f32_to_f16(F32(x), mode))


def f16_to_f32(h: int) -> float:
    return float(lib().qo_f16_to_f32(h))


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f64_to_bf16(x: float) -> int:
    return int(lib().qo_f64_to_bf16(float(x)))


def f16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return np.asarray(h, dtype=np.uint16).view(np.float16).astype(np.float32)


# ----------------------------------------------------------------------------- pieces
def weighted_dist(k: np.ndarray, c: np.ndarray, s: np.ndarray) -> float:
    k = np.ascontiguousarray(k, np.uint16); c = np.ascontiguousarray(c, np.uint16)
    s = np.ascontiguousarray(s, np.float32)
    return float(lib().qo_weighted_dist(_p(k), _p(c), _p(s), k.shape[-1]))


def kmeans(X: np.ndarray, C: int, iters: int):
    """X [n][d] bf16 bits -> (centroids [C][d] bf16 bits, final assignment [n])."""
    X = np.ascontiguousarray(X, np.uint16)
    n, d = X.shape
    cent = np.zeros((C, d), np.uint16)
    asg = np.zeros(n, np.int32)
    rc = lib().qo_kmeans(_p(X), n, d, d, C, iters, _p(cent), _p(asg))
    assert rc == 0
    return cent, asg


def stats_accumulate(Q: np.ndarray, M: np.ndarray) -> None:
    Q = np.ascontiguousarray(Q, np.uint16)
    n, d = Q.shape
    assert M.dtype == np.float64 and M.shape == (d, d)
    lib().qo_stats_accumulate(_p(Q), n, d, d, _p(M))


def eigh_jacobi(A: np.ndarray):
    A = np.ascontiguousarray(A, np.float64)
    d = A.shape[0]
    ev = np.zeros(d, np.float64)
    V = np.zeros((d, d), np.float64)
    sweeps = lib().qo_eigh_jacobi(_p(A), d, _p(ev), _p(V))
    return ev, V, sweeps


def refresh(M: np.ndarray, n: int, r: int, G: int):
    d = M.shape[0]
    M = np.ascontiguousarray(M, np.float64)
    s = np.zeros(d, np.float32); w = np.zeros(d // G, np.float32)
    U = np.zeros((d, r), np.float32); ev = np.zeros(d, np.float64)
    lib().qo_refresh(_p(M), int(n), d, r, G, _p(s), _p(w), _p(U), _p(ev))
    return s, w, U, ev


def int2_encode(rho: np.ndarray, G: int):
    rho = np.ascontiguousarray(rho, np.float32)
    d = rho.shape[0]
    codes = np.zeros(d // 4, np.uint8); params = np.zeros(2 * (d // G), np.uint16)
    lib().qo_int2_encode(_p(rho), d, G, _p(codes), _p(params))
    return codes, params


def int2_decode(codes: np.ndarray, params: np.ndarray, d: int, G: int) -> np.ndarray:
    out = np.zeros(d, np.float32)
    lib().qo_int2_decode(_p(np.ascontiguousarray(codes, np.uint8)),
                         _p(np.ascontiguousarray(params, np.uint16)), d, G, _p(out))
    return out


def qsac_shortlist(k, CK, s, M):
    k = np.ascontiguousarray(k, np.uint16); CK = np.ascontiguousarray(CK, np.uint16)
    s = np.ascontiguousarray(s, np.float32)
    C, d = CK.shape
    cand = np.zeros(M, np.int32); D = np.zeros(C, np.float32)
    lib().qo_qsac_shortlist(_p(k), _p(CK), C, d, _p(s), M, _p(cand), _p(D))
    return cand, D


def qsac_score(k, c, w, G) -> float:
    k = np.ascontiguousarray(k, np.uint16); c = np.ascontiguousarray(c, np.uint16)
    w = np.ascontiguousarray(w, np.float32)
    return float(lib().qo_qsac_score(_p(k), _p(c), _p(w), k.shape[0], G))


def encode_key(k, CK, G, M, s, w, U, Afull=None):
    """One key row -> dict(idx, codes, params, coef, cscale, shortlist).  With
    Afull ([d][d] fp32) QSAC stage 2 scores by the full quadratic form."""
    k = np.ascontiguousarray(k, np.uint16); CK = np.ascontiguousarray(CK, np.uint16)
    s = np.ascontiguousarray(s, np.float32); w = np.ascontiguousarray(w, np.float32)
    U = np.ascontiguousarray(U, np.float32)
    C, d = CK.shape
    r = U.shape[1] if U.ndim == 2 else 0
    if r == 0:
        U = np.zeros((d, 1), np.float32)
    idx = np.zeros(1, np.int32); codes = np.zeros(d // 4, np.uint8)
    params = np.zeros(2 * (d // G), np.uint16); coef = np.zeros(max(r, 1), np.int8)
    cs = np.zeros(1, np.uint16); sl = np.zeros(M, np.int32)
    Af = None if Afull is None else np.ascontiguousarray(Afull, np.float32)
    lib().qo_encode_key(_p(k), _p(CK), C, d, G, M, _p(s), _p(w), _p(U), r, _p(idx), _p(codes),
                        _p(params), _p(coef), _p(cs), _p(sl), None if Af is None else _p(Af))
    return dict(idx=int(idx[0]), codes=codes, params=params, coef=coef[:r], cscale=int(cs[0]),
                shortlist=sl)


def qsac_score_full(k, c, A, G):
    """e^T A e for the Key error e that centroid c leaves after INT2 (fp32 folds)."""
    k = np.ascontiguousarray(k, np.uint16); c = np.ascontiguousarray(c, np.uint16)
    A = np.ascontiguousarray(A, np.float32)
    return float(lib().qo_qsac_score_full(_p(k), _p(c), _p(A), k.shape[0], G))


def full_quadratic_matrix(M: np.ndarray, n: int) -> np.ndarray:
    """A = fp32(M / n) (fp64 division, rounded once), the matrix the full-quadratic
    QSAC score reads; zero before any query."""
    if n <= 0:
        return np.zeros(M.shape, np.float32)
    return (np.asarray(M, np.float64) / float(n)).astype(np.float32)


def encode_value(v, CV, G):
    v = np.ascontiguousarray(v, np.uint16); CV = np.ascontiguousarray(CV, np.uint16)
    C, d = CV.shape
    idx = np.zeros(1, np.int32); codes = np.zeros(d // 4, np.uint8)
    params = np.zeros(2 * (d // G), np.uint16)
    lib().qo_encode_value(_p(v), _p(CV), C, d, G, _p(idx), _p(codes), _p(params))
    return dict(idx=int(idx[0]), codes=codes, params=params)


def reconstruct_key_f64(c, codes, params, coef, cscale, U, G) -> np.ndarray:
    d = c.shape[0]
    U = np.ascontiguousarray(U, np.float32)
    r = U.shape[1]
    out = np.zeros(d, np.float64)
    coef = np.ascontiguousarray(coef, np.int8)
    lib().qo_reconstruct_key(_p(np.ascontiguousarray(c, np.uint16)),
                             _p(np.ascontiguousarray(codes, np.uint8)),
                             _p(np.ascontiguousarray(params, np.uint16)), _p(coef), int(cscale),
                             _p(U), d, G, r, None, _p(out))
    return out


def reconstruct_value(c, codes, params, G) -> np.ndarray:
    """V' = bf16(c + deq(codes, params)) of one Value row, as bf16 bits."""
    c = np.ascontiguousarray(c, np.uint16)
    d = c.shape[0]
    out = np.zeros(d, np.uint16)
    lib().qo_reconstruct_value(_p(c), _p(np.ascontiguousarray(codes, np.uint8)),
                               _p(np.ascontiguousarray(params, np.uint16)), d, G, _p(out))
    return out


def attention_head(Q, Kp, Vp, scale):
    """Q [nq][d], K', V' [T][d] (bf16 bits) -> O [nq][d] fp64."""
    Q = np.ascontiguousarray(Q, np.uint16); Kp = np.ascontiguousarray(Kp, np.uint16)
    Vp = np.ascontiguousarray(Vp, np.uint16)
    nq, d = Q.shape
    T = Kp.shape[0]
    O = np.zeros((nq, d), np.float64)
    lib().qo_attention_head(_p(Q), nq, d, _p(Kp), _p(Vp), T, d, float(scale), _p(O))
    return O


def attention_lse(Q, K, scale):
    """Q [nq][d], K [T][d] (bf16 bits) -> ln sum_t exp(scale q . k_t) per row, fp64."""
    Q = np.ascontiguousarray(Q, np.uint16); K = np.ascontiguousarray(K, np.uint16)
    nq, d = Q.shape
    out = np.zeros(nq, np.float64)
    lib().qo_attention_lse(_p(Q), nq, d, _p(K), K.shape[0], d, float(scale), _p(out))
    return out


def top1(Q, K):
    Q = np.ascontiguousarray(Q, np.uint16); K = np.ascontiguousarray(K, np.uint16)
    nq, d = Q.shape
    idx = np.zeros(nq, np.int32)
    lib().qo_top1(_p(Q), nq, d, _p(K), K.shape[0], d, d, _p(idx))
    return idx


def bytes_per_token_head(d, C, G, r) -> int:
    return int(lib().qo_bytes_per_token_head(d, C, G, r))


# ----------------------------------------------------------------------------- cache
class OracleCache:
    """The whole cache in numpy, driven frame by frame like the C-ABI library.

    Per frame: ``update_query_stats(Q_f, refresh)``, then ``append_kv(K_f, V_f)``,
    then ``attention(Q_f)``; the basis version in force at append time
    reconstructs a token forever after.
    """

    def __init__(self, H, d, C, G, M, r, Tcap, max_versions=256, qsac_full=False):
        self.H, self.d, self.C, self.G, self.n_cand, self.r = H, d, C, G, M, r
        # full-quadratic QSAC: A = fp32(M / n) in force, per head
        self.A = np.zeros((H, d, d), np.float32) if qsac_full else None
        self.Tcap = int(Tcap)
        ng = d // G
        idt = np.uint8 if C <= 256 else np.uint16
        self.k_codes = np.zeros((H, self.Tcap, d // 4), np.uint8)
        self.k_params = np.zeros((H, self.Tcap, ng, 2), np.uint16)
        self.k_idx = np.zeros((H, self.Tcap), idt)
        self.k_coef = np.zeros((H, self.Tcap, max(r, 0)), np.int8)
        self.k_cscale = np.zeros((H, self.Tcap), np.uint16)
        self.v_codes = np.zeros((H, self.Tcap, d // 4), np.uint8)
        self.v_params = np.zeros((H, self.Tcap, ng, 2), np.uint16)
        self.v_idx = np.zeros((H, self.Tcap), idt)
        self.tok_ver = np.zeros(self.Tcap, np.uint16)
        # centroid tables: one (CK, CV) pair per build; each token keeps the
        # version in force at its append (tok_cver), like the basis versions
        self.cent_versions = []
        self.tok_cver = np.zeros(self.Tcap, np.uint16)
        self.M = np.zeros((H, d, d), np.float64)
        self.nq = 0
        self.s = np.ones((H, d), np.float32)
        self.w = np.full((H, ng), float(G), np.float32)
        self.U = [np.zeros((H, d, max(r, 1)), np.float32)]
        self.len = 0

    @property
    def version(self):
        return len(self.U) - 1

    # the tables in force (the latest version)
    @property
    def CK(self):
        return self.cent_versions[-1][0] if self.cent_versions else None

    @CK.setter
    def CK(self, v):
        self._set_current(0, v)

    @property
    def CV(self):
        return self.cent_versions[-1][1] if self.cent_versions else None

    @CV.setter
    def CV(self, v):
        self._set_current(1, v)

    def _set_current(self, i, v):
        v = np.ascontiguousarray(v, np.uint16)
        if not self.cent_versions:
            self.cent_versions.append([None, None])
        self.cent_versions[-1][i] = v

    @property
    def cent_version(self):
        return len(self.cent_versions) - 1

    def _kmeans_tables(self, K, V, iters):
        H, d, C = self.H, self.d, self.C
        CK = np.zeros((H, C, d), np.uint16)
        CV = np.zeros((H, C, d), np.uint16)
        for h in range(H):
            CK[h], _ = kmeans(K[:, h, :], C, iters)
            CV[h], _ = kmeans(V[:, h, :], C, iters)
        return CK, CV

    def build_centroids(self, K, V, iters=10):
        """K, V [n][H][d] bf16 bits (frame 0): the first centroid tables."""
        self.cent_versions = [list(self._kmeans_tables(K, V, iters))]

    def rebuild_centroids(self, K, V, iters=10):
        """Centroid refresh under drift: k-means on a recent frame K, V gives a new
        version of the tables; later appends encode against it, while tokens
        already cached keep the tables they were encoded with."""
        self.cent_versions.append(list(self._kmeans_tables(K, V, iters)))

    def update_query_stats(self, Q, refresh_basis=True):
        for h in range(self.H):
            stats_accumulate(Q[:, h, :], self.M[h])
        self.nq += Q.shape[0]
        if refresh_basis:
            U = np.zeros((self.H, self.d, max(self.r, 1)), np.float32)
            for h in range(self.H):
                s, w, Uh, _ = refresh(self.M[h], self.nq, self.r, self.G)
                self.s[h], self.w[h] = s, w
                if self.A is not None:
                    self.A[h] = full_quadratic_matrix(self.M[h], self.nq)
                if self.r:
                    U[h] = Uh
            self.U.append(U)

    def set_state(self, s=None, w=None, U=None, CK=None, CV=None, A=None):
        """Install a state: the tests install the oracle's own refresh and k-means
        results computed outside this object."""
        if A is not None:
            self.A = np.ascontiguousarray(A, np.float32)
        if s is not None:
            self.s = np.ascontiguousarray(s, np.float32)
        if w is not None:
            self.w = np.ascontiguousarray(w, np.float32)
        if U is not None:
            self.U.append(np.ascontiguousarray(U, np.float32).reshape(self.H, self.d, -1))
        if CK is not None:
            self.CK = CK
        if CV is not None:
            self.CV = CV

    def append_kv(self, K, V):
        n = K.shape[0]
        assert self.len + n <= self.Tcap
        K = np.ascontiguousarray(K, np.uint16); V = np.ascontiguousarray(V, np.uint16)
        U = np.ascontiguousarray(self.U[-1], np.float32)
        if self.r == 0:
            U = np.zeros((self.H, self.d, 1), np.float32)
        lib().qo_append_frame(self.H, self.d, self.C, self.G, self.n_cand, self.r, self.Tcap,
                              self.len, _p(K), _p(V), n, _p(self.CK), _p(self.CV), _p(self.s),
                              _p(self.w), _p(U), _p(self.k_codes), _p(self.k_params),
                              _p(self.k_idx), _p(self.k_coef), _p(self.k_cscale),
                              _p(self.v_codes), _p(self.v_params), _p(self.v_idx),
                              None if self.A is None else _p(self.A))
        self.tok_ver[self.len:self.len + n] = self.version
        self.tok_cver[self.len:self.len + n] = self.cent_version
        self.len += n

    def reconstruct(self, h):
        """K', V' of head h as [T][d] bf16 bits."""
        T = self.len
        Kp = np.zeros((T, self.d), np.uint16); Vp = np.zeros((T, self.d), np.uint16)
        Uall = np.ascontiguousarray(np.stack(self.U), np.float32)
        r = self.r
        if r == 0:
            Uall = np.zeros((len(self.U), self.H, self.d, 1), np.float32)
        # runs of tokens sharing one centroid-table version (versions only grow)
        t0 = 0
        while t0 < T:
            cv = int(self.tok_cver[t0])
            t1 = t0
            while t1 < T and self.tok_cver[t1] == cv:
                t1 += 1
            CK, CV = self.cent_versions[cv]
            lib().qo_reconstruct_range(h, self.H, self.d, self.C, self.G, r, self.Tcap, t0, t1,
                                       _p(CK), _p(CV), _p(Uall), _p(self.tok_ver),
                                       _p(self.k_codes), _p(self.k_params), _p(self.k_idx),
                                       _p(self.k_coef), _p(self.k_cscale), _p(self.v_codes),
                                       _p(self.v_params), _p(self.v_idx), _p(Kp[t0:]),
                                       _p(Vp[t0:]))
            t0 = t1
        return Kp, Vp

    def attention(self, Q, rows=None, heads=None, scale=None):
        """O[rows][heads][d] in fp64 for the given query rows (default all)."""
        scale = 1.0 / math.sqrt(self.d) if scale is None else scale
        rows = np.arange(Q.shape[0]) if rows is None else np.asarray(rows)
        heads = list(range(self.H) if heads is None else heads)
        out = np.zeros((len(rows), len(heads), self.d), np.float64)
        for i, h in enumerate(heads):
            Kp, Vp = self.reconstruct(h)
            out[:, i, :] = attention_head(Q[rows, h, :], Kp, Vp, scale)
        return out

    def packed_bytes(self) -> int:
        """Bytes the packed tokens occupy (all per-token fields, len tokens)."""
        T = self.len
        arrs = [self.k_codes, self.k_params, self.k_idx, self.k_coef, self.k_cscale,
                self.v_codes, self.v_params, self.v_idx]
        return sum(a[:, :T].nbytes for a in arrs)

    def fixed_bytes(self) -> int:
        """Centroid tables (bf16) plus the fp32 bases in use."""
        nver = len(set(int(v) for v in self.tok_ver[: self.len])) if self.len else 1
        return 2 * self.H * self.C * self.d * 2 + nver * self.H * self.d * self.r * 4
