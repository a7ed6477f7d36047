"""Full-size parity driver: every frame of a layer configuration through the CUDA
library (all heads), and for a few sampled heads every token re-encoded by the
CPU oracle and compared bit for bit, plus attention on sampled query rows.

The oracle work is spread over a process pool started with ``spawn`` (safe next
to a live CUDA context).  Each worker draws its own inputs for one head from the
seeded generator, so no large array crosses a process boundary.

Token encodings depend only on the frame's inputs and the state in force at
append time (centroid tables, sensitivities s, group weights w, basis U).  The
oracle runs on its own state throughout: its own k-means tables, its own fp64
statistics of the sampled heads (accumulated here frame by frame) and its own
refresh.  At every refresh the GPU's statistics matrix, s and w must equal the
oracle's bit for bit, its basis is compared within tolerance, and the oracle's U
is installed as the GPU's basis of the sampled heads, so that both sides encode
with the same state and the codes can be compared exactly.
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


def attention_rows(args):
    """Oracle fp64 attention of query rows Qs [n][d] over K', V' [T][d]."""
    Qs, Kp, Vp, scale = args
    return oracle.attention_head(Qs, Kp, Vp, scale)


# ----------------------------------------------------------------- driver
def run_full(name, heads, attn_frames, attn_rows, seed=None, full_rows_head=None):
    """Run configuration `name` at full size; returns measured discrepancies.
    With `full_rows_head` (one of `heads`), every query row of that head is also
    compared at the last frame (which includes the last, partial, CTA of rows)."""
    import torch

    import bit_kv_cache_23_b200 as q
    from parity_util import (attention_error, make_gpu_cache, new_state_report,
                             refresh_from_oracle, to_dev, u16)

    c = syn.get_config(name)
    seed = c.seed if seed is None else seed
    F = c.frames
    out = dict(packed_mismatch={}, cent_equal=True, attn=[], frames=F, refreshes=0)
    out.update(new_state_report())
    Mref = {h: np.zeros((c.head_dim, c.head_dim)) for h in heads}
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
            for h in heads:
                oracle.stats_accumulate(Q[:, h, :], Mref[h])
            nq += Q.shape[0]
            if refresh:
                ver_state = refresh_from_oracle(g, Mref, nq, heads, c.rank, c.group, out)
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
            if full_rows_head is not None and f == F - 1:
                if f not in attn_frames:
                    Od = g.attention(Qd)
                    torch.cuda.synchronize()
                    assert q.qwm_device_status() == 0, "a bounded device wait timed out"
                    Og = syn.bf16_bits_to_f32(u16(Od))
                full_rows = (Q[:, full_rows_head, :].copy(), Og[:, full_rows_head, :].copy())
        torch.cuda.synchronize()
        out["refreshes"] = len(refreshes)
        CKg = g.view("cent_k").cpu().numpy().view(np.uint16)
        CVg = g.view("cent_v").cpu().numpy().view(np.uint16)
        cents = dict(zip(heads, km.get()))     # the oracle's own tables
        for h, (ck, cv) in cents.items():
            out["cent_equal"] &= bool(np.array_equal(ck, CKg[h]) and np.array_equal(cv, CVg[h]))

        # every token of the sampled heads, re-encoded by the oracle
        ncpu = os.cpu_count() or 2
        chunk = max(1, math.ceil(F * len(heads) / (2 * ncpu)))
        tasks, keys = [], []
        for h in heads:
            for f0 in range(0, F, chunk):
                f1 = min(F, f0 + chunk)
                tasks.append((name, seed, h, f0, f1, cents[h][0], cents[h][1],
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


    # attention on sampled rows, over the oracle's own reconstruction
    for hi, h in enumerate(heads):
        oc = oracle.OracleCache(1, c.head_dim, c.n_centroids, c.group, c.n_cand, c.rank,
                                F * N, max_versions=len(refreshes) + 2)
        oc.set_state(CK=cents[h][0][None], CV=cents[h][1][None])
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
        if h == full_rows_head:
            oc.len = F * N
            Kp, Vp = oc.reconstruct(0)
            Qh, Oh = full_rows
            step = 64
            tasks = [(np.ascontiguousarray(Qh[i:i + step]), Kp, Vp, 1.0 / math.sqrt(c.head_dim))
                     for i in range(0, Qh.shape[0], step)]
            with pool() as P:
                Oref = np.concatenate(P.map(attention_rows, tasks, chunksize=1))
            mx, mean = attention_error(Oh, Oref)
            out["attn"].append(("all rows", h, mx, mean))
            out["full_rows"] = Qh.shape[0]
    return out
