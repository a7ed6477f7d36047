"""Shared driver for the GPU-vs-oracle parity tests.

Runs a synthetic layer frame by frame through the CUDA library (C ABI via the
Python binding) and, on the same inputs, through the CPU oracle; compares what
must be identical bit for bit and what is compared within tolerance.

The oracle only ever runs on its own state: its own k-means tables, its own
fp64 Query statistics and its own refresh (s, w and the Jacobi basis U).  The
GPU's centroid tables, statistics matrix, s and w must equal the oracle's bit
for bit; its basis (block subspace iteration, a different eigen-solver) is
compared within tolerance and then overwritten with the oracle's U, so that
both sides encode every later token with the same basis.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import bit_kv_cache_23_b200 as q
import oracle
import qwm_synth as syn

ATOL_MAX = 2e-2   # attention: max |O_gpu - O_oracle|
ATOL_MEAN = 2e-3  # attention: mean |O_gpu - O_oracle|


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def make_gpu_cache(c: syn.LayerConfig, max_tokens=None, max_versions=None) -> q.QuantKVCache:
    """The layer's cache as the benchmark makes it: workspace for split-key
    attention partials of one frame's query chunk."""
    T = c.total_tokens if max_tokens is None else max_tokens
    nv = (c.frames // c.refresh_every + 2) if max_versions is None else max_versions
    return q.QuantKVCache(c.heads, c.head_dim, c.n_centroids, c.group, c.n_cand, c.rank, T,
                          max_versions=nv, max_queries=c.q_rows)


def make_oracle_cache(c: syn.LayerConfig) -> oracle.OracleCache:
    return oracle.OracleCache(c.heads, c.head_dim, c.n_centroids, c.group, c.n_cand, c.rank,
                              c.total_tokens)


def new_state_report():
    return dict(stats_mismatch=0, sw_mismatch=0, orth_err=0.0, proj_err=0.0)


def refresh_from_oracle(g: q.QuantKVCache, Mref: dict, nq: int, heads, rank: int, group: int,
                        rep: dict, check_basis=True):
    """The oracle's refresh of `heads` from its own statistics `Mref[h]` over `nq`
    queries.  Counts the GPU's statistics, s and w entries that differ from the
    oracle's in any bit, measures the GPU basis against the oracle's (orthonormality
    and projector distance), then installs the oracle's U into the GPU basis slot
    now in force.  Returns {h: (s, w, U)}, the oracle's state."""
    torch.cuda.synchronize()
    Mg, Ub = g.view("qstats"), g.view("basis")[g.version]
    sg, wg = g.view("sens").cpu().numpy(), g.view("wgroup").cpu().numpy()
    st = {}
    for h in heads:
        so, wo, Uo, _ = oracle.refresh(Mref[h], nq, rank, group)
        Mh = Mg[h].cpu().numpy()
        rep["stats_mismatch"] += int(np.count_nonzero(Mh.view(np.uint64)
                                                      != Mref[h].view(np.uint64)))
        rep["sw_mismatch"] += int(np.count_nonzero(sg[h].view(np.uint32) != so.view(np.uint32)))
        rep["sw_mismatch"] += int(np.count_nonzero(wg[h].view(np.uint32) != wo.view(np.uint32)))
        if rank:
            Ug = Ub[h].cpu().numpy().astype(np.float64)[:, :rank]
            assert np.all(np.isfinite(Ug))
            if check_basis:
                rep["orth_err"] = max(rep["orth_err"],
                                      float(np.abs(Ug.T @ Ug - np.eye(rank)).max()))
                P1 = Ug @ Ug.T
                P2 = Uo.astype(np.float64) @ Uo.T.astype(np.float64)
                rep["proj_err"] = max(rep["proj_err"], float(np.linalg.norm(P1 - P2, 2)))
            Ub[h].copy_(torch.from_numpy(np.ascontiguousarray(Uo, np.float32)))
        st[h] = (so, wo, Uo)
    torch.cuda.synchronize()
    return st


def stack_state(st: dict, H: int):
    """(s [H][d], w [H][ng], U [H][d][r]) from a per-head state dict."""
    return tuple(np.stack([st[h][i] for h in range(H)]) for i in range(3))


def compare_packed(g: q.QuantKVCache, oc: oracle.OracleCache, t0: int, t1: int, heads=None):
    """Bit-exact comparison of every packed field for tokens [t0, t1)."""
    torch.cuda.synchronize()
    hs = slice(None) if heads is None else heads
    fields = ["k_codes", "k_params", "k_idx", "k_cscale", "v_codes", "v_params", "v_idx"]
    if oc.r > 0:
        fields.append("k_coef")
    bad = {}
    for f in fields:
        gv = g.view(f)[hs, t0:t1].cpu().numpy()
        ov = getattr(oc, f)[hs, t0:t1]
        gv = gv.view(ov.dtype) if gv.dtype.itemsize == ov.dtype.itemsize else gv.astype(ov.dtype)
        ne = int(np.count_nonzero(gv != ov))
        if ne:
            bad[f] = ne
    return bad


def attention_error(O_gpu: np.ndarray, O_ref: np.ndarray):
    err = np.abs(O_gpu.astype(np.float64) - O_ref)
    return float(err.max()), float(err.mean())


def run_layer(name: str, frames=None, attn_rows=None, attn_frames=None, check_every=1,
              seed=None, heads_check=None):
    """Drive the layer; returns a dict of measured discrepancies (all must be 0
    or within tolerance, which the calling test asserts)."""
    c = syn.get_config(name)
    src = syn.FrameSource(c, seed)
    F = c.frames if frames is None else frames
    g = make_gpu_cache(c)
    oc = make_oracle_cache(c)
    out = dict(packed_mismatch={}, attn=[], cent_k_equal=None, cent_v_equal=None, top1=None)
    out.update(new_state_report())
    Mref = {h: np.zeros((c.head_dim, c.head_dim)) for h in range(c.heads)}
    nq = 0
    rng = np.random.default_rng(123)
    for f in range(F):
        Q, K, V = src.frame(f)
        Qd, Kd, Vd = to_dev(Q), to_dev(K), to_dev(V)
        if f == 0:
            g.build_centroids(Kd, Vd, iters=c.kmeans_iters)
            torch.cuda.synchronize()
            CKg = g.view("cent_k").cpu().numpy().view(np.uint16).copy()
            CVg = g.view("cent_v").cpu().numpy().view(np.uint16).copy()
            CK, CV = np.zeros_like(CKg), np.zeros_like(CVg)
            for h in range(c.heads):
                CK[h], _ = oracle.kmeans(K[:, h, :], c.n_centroids, c.kmeans_iters)
                CV[h], _ = oracle.kmeans(V[:, h, :], c.n_centroids, c.kmeans_iters)
            out["cent_k_equal"] = bool(np.array_equal(CK, CKg))
            out["cent_v_equal"] = bool(np.array_equal(CV, CVg))
            oc.set_state(CK=CK, CV=CV)
        refresh = (f % c.refresh_every) == 0
        g.update_query_stats(Qd, refresh_basis=refresh)
        for h in range(c.heads):
            oracle.stats_accumulate(Q[:, h, :], Mref[h])
        nq += Q.shape[0]
        if refresh:
            st = refresh_from_oracle(g, Mref, nq, range(c.heads), c.rank, c.group, out)
            s, w, U = stack_state(st, c.heads)
            oc.set_state(s=s, w=w, U=U)
        t0 = g.len
        g.append_kv(Kd, Vd)
        oc.append_kv(K, V)
        if f % check_every == 0 or f == F - 1:
            bad = compare_packed(g, oc, t0, g.len, heads_check)
            for k, v in bad.items():
                out["packed_mismatch"][k] = out["packed_mismatch"].get(k, 0) + v
        if attn_frames is None or f in attn_frames:
            Od = g.attention(Qd)
            torch.cuda.synchronize()
            assert q.qwm_device_status() == 0, "a bounded device wait timed out"
            Og = syn.bf16_bits_to_f32(u16(Od))
            rows = (np.arange(Q.shape[0]) if attn_rows is None
                    else np.sort(rng.choice(Q.shape[0], size=min(attn_rows, Q.shape[0]),
                                            replace=False)))
            heads = list(range(c.heads)) if heads_check is None else list(heads_check)
            Oref = oc.attention(Q, rows=rows, heads=heads)
            mx, mean = attention_error(Og[rows][:, heads, :], Oref)
            out["attn"].append((f, mx, mean))
    out["gpu"], out["oracle"], out["src"], out["cfg"] = g, oc, src, c
    return out
