"""Full-size parity driver: every frame of a layer configuration through the CUDA
library (all heads), and for a few sampled heads every token re-encoded by the
CPU oracle and compared bit for bit, plus attention on sampled query rows.

The oracle work is spread over a process pool started with ``spawn`` (safe next
to a live CUDA context).  Each worker draws its own inputs for one head from the
seeded generator, so no large array crosses a process boundary.

Token encodings depend only on the frame's inputs and the state in force at
append time (centroid tables, sensitivities s, group weights w, basis U).  The
centroids are compared bit for bit first; s, w and U are compared with the
oracle's own fp64 refresh within tolerance and then the GPU's values are
installed, as in the small-config parity tests, so that the codes can be
compared exactly.
"""
from __future__ import annotations

import math
import multiprocessing as mp
import os

import numpy as np

import oracle
import qwm_synth as syn


def pool(n=None):
    n = n or max(1, min(16, (os.cpu_count() or 2)))
    return mp.get_context("spawn").Pool(n)


# ----------------------------------------------------------------- worker tasks
def gen_frame(args):
    """(name, seed, f) -> (Q, K, V) of frame f, all heads."""
    name, seed, f = args
    return syn.FrameSource(syn.get_config(name), seed).frame(f)


def kmeans_head(args):
    """Oracle centroid tables of head h from frame 0."""
    name, seed, h = args
    c = syn.get_config(name)
    _, K, V = syn.FrameSource(c, seed).frame(0, heads=[h])
    ck, _ = oracle.kmeans(K[:, 0, :], c.n_centroids, c.kmeans_iters)
    cv, _ = oracle.kmeans(V[:, 0, :], c.n_centroids, c.kmeans_iters)
    return ck, cv


def encode_frames(args):
    """Oracle encoding of frames [f0, f1) of head h with the given per-frame state.

    states: list over frames of (s[d], w[ng], U[d][r]) in force at append time.
    Returns the packed per-token fields of those frames.
    """
    name, seed, h, f0, f1, CK, CV, states = args
    c = syn.get_config(name)
    src = syn.FrameSource(c, seed)
    n = (f1 - f0) * c.tokens_per_frame
    oc = oracle.OracleCache(1, c.head_dim, c.n_centroids, c.group, c.n_cand, c.rank, n,
                            max_versions=f1 - f0 + 2)
    oc.set_state(CK=CK[None], CV=CV[None])
    for i, f in enumerate(range(f0, f1)):
        s, w, U = states[i]
        oc.set_state(s=s[None], w=w[None], U=U[None])
        _, K, V = src.frame(f, heads=[h])
        oc.append_kv(K, V)
    fields = ["k_codes", "k_params", "k_idx", "k_coef", "k_cscale", "v_codes", "v_params",
              "v_idx"]
    return {k: getattr(oc, k)[0, :n].copy() for k in fields}


def stats_head(args):
    """Oracle fp64 Query second-moment matrix of head h over frames [0, f1)."""
    name, seed, h, f1 = args
    c = syn.get_config(name)
    src = syn.FrameSource(c, seed)
    M = np.zeros((c.head_dim, c.head_dim))
    for f in range(f1):
        oracle.stats_accumulate(src.queries(f, heads=[h])[:, 0, :], M)
    return M


# ----------------------------------------------------------------- driver
def run_full(name, heads, attn_frames, attn_rows, seed=None, check_refresh=3):
    """Run configuration `name` at full size; returns measured discrepancies."""
    import torch

    import bit_kv_cache_23_b200 as q
    from parity_util import attention_error, make_gpu_cache, to_dev, u16

    c = syn.get_config(name)
    seed = c.seed if seed is None else seed
    F = c.frames
    out = dict(packed_mismatch={}, cent_equal=True, attn=[], stats_rel=0.0, orth_err=0.0,
               proj_err=0.0, frames=F)
    rng = np.random.default_rng(2024)
    g = make_gpu_cache(c)
    with pool() as P:
        # centroids of the sampled heads (oracle) while the GPU runs
        km = P.map_async(kmeans_head, [(name, seed, h) for h in heads])
        frames = P.imap(gen_frame, [(name, seed, f) for f in range(F)], chunksize=1)
        states = {h: [] for h in heads}        # per frame: (s, w, U) in force at append
        refreshes = []                         # (frame, n_queries) of each refresh
        ver_state = None
        attn_out = {}
        nq = 0
        for f, (Q, K, V) in enumerate(frames):
            Qd, Kd, Vd = to_dev(Q), to_dev(K), to_dev(V)
            if f == 0:
                g.build_centroids(Kd, Vd, iters=c.kmeans_iters)
            refresh = (f % c.refresh_every) == 0
            g.update_query_stats(Qd, refresh_basis=refresh)
            nq += Q.shape[0]
            if refresh:
                torch.cuda.synchronize()
                s = g.view("sens").cpu().numpy()
                w = g.view("wgroup").cpu().numpy()
                U = g.view("basis")[g.version].cpu().numpy()
                ver_state = {h: (s[h].copy(), w[h].copy(), U[h].copy()) for h in heads}
                refreshes.append((f, nq))
            for h in heads:
                states[h].append(ver_state[h])
            g.append_kv(Kd, Vd)
            if f in attn_frames:
                rows = np.sort(rng.choice(Q.shape[0], size=min(attn_rows, Q.shape[0]),
                                          replace=False))
                Od = g.attention(Qd)
                torch.cuda.synchronize()
                assert q.qwm_device_status() == 0, "a bounded device wait timed out"
                Og = syn.bf16_bits_to_f32(u16(Od))
                attn_out[f] = (rows, Q[rows][:, heads, :].copy(), Og[rows][:, heads, :].copy(),
                               g.len)
        torch.cuda.synchronize()
        CKg = g.view("cent_k").cpu().numpy().view(np.uint16)
        CVg = g.view("cent_v").cpu().numpy().view(np.uint16)
        for h, (ck, cv) in zip(heads, km.get()):
            out["cent_equal"] &= bool(np.array_equal(ck, CKg[h]) and np.array_equal(cv, CVg[h]))

        # every token of the sampled heads, re-encoded by the oracle
        ncpu = os.cpu_count() or 2
        chunk = max(1, math.ceil(F * len(heads) / (2 * ncpu)))
        tasks, keys = [], []
        for h in heads:
            for f0 in range(0, F, chunk):
                f1 = min(F, f0 + chunk)
                tasks.append((name, seed, h, f0, f1, CKg[h].copy(), CVg[h].copy(),
                              states[h][f0:f1]))
                keys.append((h, f0, f1))
        enc = P.map(encode_frames, tasks, chunksize=1)
        N = c.tokens_per_frame
        ofields = {h: {} for h in heads}
        for (h, f0, f1), e in zip(keys, enc):
            for k, v in e.items():
                ofields[h].setdefault(k, [None] * F)
                ofields[h][k][f0] = v
        for h in heads:
            for k in list(ofields[h]):
                ofields[h][k] = np.concatenate([a for a in ofields[h][k] if a is not None])
            for k, ov in ofields[h].items():
                if k == "k_coef" and c.rank == 0:
                    continue
                gv = g.view(k)[h, :F * N].cpu().numpy()
                gv = gv.view(ov.dtype) if gv.dtype.itemsize == ov.dtype.itemsize \
                    else gv.astype(ov.dtype)
                ne = int(np.count_nonzero(gv != ov))
                if ne:
                    out["packed_mismatch"][(h, k)] = ne

        # statistics and basis at a few refreshes, against the oracle's fp64 refresh
        picks = [refreshes[i] for i in sorted(set(
            np.linspace(0, len(refreshes) - 1, min(check_refresh, len(refreshes))).astype(int)))]
        Ms = P.map(stats_head, [(name, seed, h, f + 1) for (f, _) in picks for h in heads])
        i = 0
        for (f, nqf) in picks:
            for h in heads:
                so, wo, Uo, _ = oracle.refresh(Ms[i], nqf, c.rank, c.group)
                s, w, U = states[h][f]
                out["stats_rel"] = max(out["stats_rel"],
                                       float(np.abs(s - so).max() / np.abs(so).max()))
                if c.rank:
                    Ug = U.astype(np.float64)[:, :c.rank]
                    out["orth_err"] = max(out["orth_err"],
                                          float(np.abs(Ug.T @ Ug - np.eye(c.rank)).max()))
                    P1 = Ug @ Ug.T
                    P2 = Uo.astype(np.float64) @ Uo.T.astype(np.float64)
                    out["proj_err"] = max(out["proj_err"], float(np.linalg.norm(P1 - P2, 2)))
                i += 1

    # attention on sampled rows, over the oracle's own reconstruction
    for hi, h in enumerate(heads):
        oc = oracle.OracleCache(1, c.head_dim, c.n_centroids, c.group, c.n_cand, c.rank,
                                F * N, max_versions=len(refreshes) + 2)
        oc.set_state(CK=CKg[h][None], CV=CVg[h][None])
        for k, v in ofields[h].items():
            getattr(oc, k)[0, :F * N] = v
        # versions: 0 = the zero basis before any refresh, then one per refresh
        oc.U = [np.zeros((1, c.head_dim, max(c.rank, 1)), np.float32)]
        ver_of_frame = []
        for f in range(F):
            if f % c.refresh_every == 0:
                oc.U.append(states[h][f][2][None].astype(np.float32))
            ver_of_frame.append(len(oc.U) - 1)
        oc.tok_ver[:F * N] = np.repeat(np.asarray(ver_of_frame, np.uint16), N)
        for f, (rows, Qs, Og, T) in sorted(attn_out.items()):
            oc.len = T
            Oref = oc.attention(Qs[:, hi:hi + 1, :])
            mx, mean = attention_error(Og[:, hi:hi + 1, :], Oref)
            out["attn"].append((f, h, mx, mean))
    return out
