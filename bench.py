#!/usr/bin/env python
"""Benchmark of the QuantWM 2-bit KV-cache hot path on B200.

One step = one pass of the whole hot path for one new frame of the 480p
93-frame layer (40 heads x 128, 1560 tokens per latent frame, cache of 24
latent frames = 37 440 tokens, C = 256, G = 32, M = 4, r = 8):

    qwm_update_query_stats(Q_f, refresh)   query second moment + basis refresh
    qwm_append_kv(K_f, V_f)                QSAC + INT2 + PSAC keys, INT2 values
    qwm_attention(Q_f)                     1560 queries over the full packed cache

The cache is filled with the 24 frames before timing; each timed step
re-appends the newest frame slot (the host length is rewound by one frame), so
every step attends over the full 37 440-token cache.  Step inputs rotate over a
pool of frames resident in HBM; together with the 161 MB packed cache every
step touches more than the 126 MB L2.

Prints one JSON line (rank 0).  `value` is query tokens per second for the
whole job (all ranks); each rank runs its own replica (weak scaling).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import qwm_synth as syn  # noqa: E402

METRIC = "quantized-KV attention query-tok/s & append GB/s; % of roofline"
UNIT = "query-tok/s"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons sampled during the timed region.

    Reads NVML from a background thread every 5 ms (read-only queries; nothing
    is changed on the GPU), so that even a timed region of a few tens of
    milliseconds is covered; reports None when NVML is not available.
    """

    REASONS = [("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap")]

    def __init__(self, device: torch.device):
        self.device = device
        self.samples = []
        self.thread = None
        self.stop_flag = threading.Event()
        self.handle = None
        self.nv = None
        self.error = None

    def _open(self):
        import pynvml as nv
        nv.nvmlInit()
        props = torch.cuda.get_device_properties(self.device)
        want = str(getattr(props, "uuid", "")).lower().replace("gpu-", "")
        bus = getattr(props, "pci_bus_id", None)
        for i in range(nv.nvmlDeviceGetCount()):
            h = nv.nvmlDeviceGetHandleByIndex(i)
            u = nv.nvmlDeviceGetUUID(h)
            u = (u.decode() if isinstance(u, bytes) else u).lower().replace("gpu-", "")
            if want and u == want:
                self.handle = h
                break
            if bus is not None and nv.nvmlDeviceGetPciInfo(h).bus == bus:
                self.handle = h
        if self.handle is None:
            raise RuntimeError("no NVML device matches the CUDA device")
        self.nv = nv

    def _run(self):
        nv, h = self.nv, self.handle
        while not self.stop_flag.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, mx, rs))
            except Exception as e:  # noqa: BLE001 - reported when no sample succeeds
                self.error = f"{type(e).__name__}: {e}"
            self.stop_flag.wait(0.005)

    def start(self):
        try:
            self._open()
        except Exception as e:  # noqa: BLE001 - reported in the JSON line
            self.handle = None
            self.error = f"{type(e).__name__}: {e}"
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.samples and time.time() - t0 < 2.0:  # sampling is live before timing
            time.sleep(0.001)
        self.samples.clear()

    def stop(self):
        if self.thread is None:
            return {"error": self.error} if self.error else None
        self.stop_flag.set()
        self.thread.join(timeout=2)
        if not self.samples:
            return {"error": self.error or "no sample during the timed region"}
        nv = self.nv
        reasons = sorted({name for _, _, rs in self.samples for name, attr in self.REASONS
                          if hasattr(nv, attr) and rs & getattr(nv, attr)})
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": max(s[1] for s in self.samples), "reasons": reasons,
                "samples": len(self.samples), "source": "nvml, 5 ms"}


# DRAM bytes (read + write) per attention launch on the 480p workload (24 cached
# frames), from one ncu capture of dram__bytes_read.sum + dram__bytes_write.sum
# at that size: 187.3 MB read (the 161.7 MB packed cache, Q, the centroid
# tables) and 147.5 MB written (the split key ranges' fp32 partials, which the
# merge kernel reads back, and O).  Valid only for the kernel sources it was
# taken on (hash of attention_tc.cu, dequant.cuh and tc.cuh below).
ATTN_TRAFFIC = {"sha256_16": "b194f56ffdbd9d07", "config": "480p", "frames": 24,
                "bytes_per_launch": 187332864 + 147464448}


def attention_traffic(cfg) -> float | None:
    import hashlib

    src = os.path.join(os.path.dirname(os.path.abspath(__file__)), "bit_kv_cache_23_b200", "csrc")
    h = hashlib.sha256()
    try:
        for f in ("attention_tc.cu", "dequant.cuh", "tc.cuh"):
            h.update(open(os.path.join(src, f), "rb").read())
    except OSError:
        return None
    if (h.hexdigest()[:16] != ATTN_TRAFFIC["sha256_16"] or cfg.name != ATTN_TRAFFIC["config"]
            or cfg.frames != ATTN_TRAFFIC["frames"]):
        return None
    return ATTN_TRAFFIC["bytes_per_launch"]


def attention_splits(cfg, heads: int, device) -> bool:
    """Whether qwm_attention splits the key range for this workload (the
    library's rule: more than one range when the pairs of CTAs of one pass
    would leave the last round of SM pairs partly empty; the cache here has
    workspace for one frame's query chunk)."""
    if cfg.head_dim != 128:
        return False
    ntile = (cfg.total_tokens + 63) // 64
    if ntile < 16:
        return False
    npairs = (cfg.q_rows + 511) // 512
    units = npairs * heads
    slots = torch.cuda.get_device_properties(device).multi_processor_count // 2
    best, bestc = 1, float("inf")
    for sp in range(1, min(6, ntile // 8) + 1):
        c = -(-units * sp // slots) * (ntile / sp + 4.0)
        if c < bestc * 0.98:
            best, bestc = sp, c
    return best > 1


# ----------------------------------------------------------------------------- workload
def packed_bytes_per_token_head(c: syn.LayerConfig) -> int:
    """Stored bytes of one token of one head: K and V codes, group parameters and
    centroid index, plus the Key's INT8 coefficients and their fp16 scale."""
    idx = 1 if c.n_centroids <= 256 else 2
    return 2 * (c.head_dim // 4 + 4 * (c.head_dim // c.group) + idx) + c.rank + 2


def config_dict(c: syn.LayerConfig, workload_name: str, world: int, shard_mode: str,
                nh: int) -> dict:
    """The `config` object of the JSON line (the same for both arms)."""
    cache = c.total_tokens * nh * packed_bytes_per_token_head(c)
    return {"workload": workload_name,
            "l2": (f"packed cache of {cache / 1e6:.0f} MB read per step "
                   f"({'larger' if cache > 126e6 else 'smaller'} than "
                   "the 126 MB L2), step inputs rotate over 4 HBM-resident frames"),
            "parallelism": (f"heads split over {world} ranks ({nh} on rank 0)"
                            if shard_mode == "heads" else f"replicas x{world}")}


def dev_bf16(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)


class Workload:
    """The layer (or this rank's block of its heads) filled with all its frames."""

    def __init__(self, cfg: syn.LayerConfig, device, extra_versions: int, pool: int = 4,
                 heads=None, rebuild_every: int = 0):
        import bit_kv_cache_23_b200 as q

        self.cfg = cfg
        self.device = device
        c = cfg
        self.heads = list(range(c.heads)) if heads is None else list(heads)
        nrb = (c.frames - 1) // rebuild_every if rebuild_every > 0 else 0
        self.cache = q.QuantKVCache(len(self.heads), c.head_dim, c.n_centroids, c.group,
                                    c.n_cand, c.rank, c.total_tokens,
                                    max_versions=c.frames // c.refresh_every + extra_versions + 4,
                                    device=device, max_queries=c.q_rows,
                                    max_cent_versions=nrb + 1)
        self.rebuilds = 0
        src = syn.FrameSource(c)
        self.src = src
        self.pool = []
        self.host_pool = []
        hs = None if heads is None else self.heads
        for f in range(c.frames):
            Q, K, V = src.frame(f, hs)
            Qd, Kd, Vd = dev_bf16(Q, device), dev_bf16(K, device), dev_bf16(V, device)
            if f == 0 or (rebuild_every > 0 and f % rebuild_every == 0):
                # the first tables, then (with rebuild_every) a new table version
                # from the newest frame under Key drift
                self.cache.build_centroids(Kd, Vd, iters=c.kmeans_iters)
                self.rebuilds += f > 0
            self.cache.update_query_stats(Qd, refresh_basis=(f % c.refresh_every) == 0)
            self.cache.append_kv(Kd, Vd)
            if f >= c.frames - pool:
                self.pool.append((Qd, Kd, Vd))
                self.host_pool.append(tuple(torch.from_numpy(a.view(np.int16)).pin_memory()
                                            for a in (Q, K, V)))
        torch.cuda.synchronize(device)
        self.t_last = self.cache.len - c.tokens_per_frame
        self.O = torch.empty_like(self.pool[0][0])
        self.nstep = 0

    def step(self, i: int, ev=None):
        """One hot-path pass; `ev` = 4 events to record around the three calls."""
        Qd, Kd, Vd = self.pool[i % len(self.pool)]
        c = self.cache
        c.c.len = self.t_last
        if ev:
            ev[0].record()
        c.update_query_stats(Qd, refresh_basis=(self.nstep % self.cfg.refresh_every) == 0)
        if ev:
            ev[1].record()
        c.append_kv(Kd, Vd)
        if ev:
            ev[2].record()
        c.attention(Qd, self.O)
        if ev:
            ev[3].record()
        self.nstep += 1

    def host_sets(self):
        """Two device buffer sets (Q, K, V, O) and a pinned host output per set."""
        Qh, Kh, Vh = self.host_pool[0]
        sets = []
        for _ in range(2):
            sets.append(dict(Q=torch.empty_like(Qh, device=self.device),
                             K=torch.empty_like(Kh, device=self.device),
                             V=torch.empty_like(Vh, device=self.device),
                             O=torch.empty_like(self.O), Oh=torch.empty_like(Qh).pin_memory(),
                             h2d=torch.cuda.Event(), done=torch.cuda.Event(),
                             d2h=torch.cuda.Event(), used=False))
        return sets

    def run_host(self, n: int, sets, cs, first: int = 0):
        """n passes through the public API from pinned host buffers.  Every pass
        copies its own Q, K, V to the device and reads its O back; the copies run
        on the stream `cs`, the upload of pass i + 1 and the read-back of pass i
        overlapping the kernels of pass i (two buffer sets alternate)."""
        comp = torch.cuda.current_stream(self.device)

        def upload(i):
            b = sets[i % 2]
            Qh, Kh, Vh = self.host_pool[(first + i) % len(self.host_pool)]
            if b["used"]:
                cs.wait_event(b["done"])            # the kernels of pass i - 2 read this set
            with torch.cuda.stream(cs):
                b["Q"].copy_(Qh, non_blocking=True)
                b["K"].copy_(Kh, non_blocking=True)
                b["V"].copy_(Vh, non_blocking=True)
            b["h2d"].record(cs)

        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload(i + 1)
            b = sets[i % 2]
            comp.wait_event(b["h2d"])
            if b["used"]:
                comp.wait_event(b["d2h"])           # O of pass i - 2 has been read back
            c = self.cache
            c.c.len = self.t_last
            q16 = b["Q"].view(torch.bfloat16)
            c.update_query_stats(q16, refresh_basis=(self.nstep % self.cfg.refresh_every) == 0)
            c.append_kv(b["K"].view(torch.bfloat16), b["V"].view(torch.bfloat16))
            c.attention(q16, b["O"])
            b["done"].record(comp)
            cs.wait_event(b["done"])
            with torch.cuda.stream(cs):
                b["Oh"].copy_(b["O"].view(torch.int16), non_blocking=True)
            b["d2h"].record(cs)
            b["used"] = True
            self.nstep += 1


# ----------------------------------------------------------------------------- ablations
# (name, M, r, Query statistics taken, tensors quantized, full-quadratic QSAC);
# None = the layer's own.
ABLATIONS = [
    ("quantwm", None, None, True, "kv", False),     # QSAC + PSAC, both tensors
    ("qvg", 1, 0, False, "kv", False),              # nearest centroid: M = 1, s = 1, r = 0
    ("qsac_only", None, 0, True, "kv", False),      # no compensation (rank 0)
    ("rank2", None, 2, True, "kv", False),
    ("rank4", None, 4, True, "kv", False),
    ("rank16", None, 16, True, "kv", False),
    ("qsac_full_quadratic", None, None, True, "kv", True),  # stage 2 by e^T A e
    ("k_only", None, None, True, "k", False),       # Keys quantized, Values exact
    ("v_only", None, None, True, "v", False),       # Values quantized, Keys exact
]


def run_ablation(cfg: syn.LayerConfig, device, frames: int) -> list:
    """Quality of each quantization setting on a synthetic layer: top-1 key
    selection shift (fraction of query rows and heads whose highest-scoring key
    changes), K / V reconstruction error relative to the mean square of the exact
    tensors, error of the attention output against exact bf16 attention (absolute,
    and relative to the mean square of the exact output, which is small here: the
    synthetic keys carry no structure, so attention is spread over many keys),
    and the compression ratio.
    Every step runs in the library's kernels (append, reconstruction, top-1, the
    fused attention, and attention over exact or reconstructed bf16 segments on an
    empty cache); torch only reduces the differences to means."""
    import bit_kv_cache_23_b200 as q

    c = dataclasses.replace(cfg, frames=frames)
    src = syn.FrameSource(c)
    data = [src.frame(f) for f in range(c.frames)]
    Kx = torch.cat([dev_bf16(K, device) for _, K, _ in data], 0)
    Vx = torch.cat([dev_bf16(V, device) for _, _, V in data], 0)
    Qd = dev_bf16(data[-1][0], device)
    T = Kx.shape[0]
    empty = q.QuantKVCache(c.heads, c.head_dim, c.n_centroids, c.group, c.n_cand, c.rank, 16,
                           device=device)
    Oexact = empty.attention_ext(Qd, Kx, Vx).float()
    e_o = Oexact.pow(2).mean().item()
    e_k, e_v = Kx.float().pow(2).mean().item(), Vx.float().pow(2).mean().item()
    out = []
    for name, M, r, stats, which, full in ABLATIONS:
        M = c.n_cand if M is None else M
        r = c.rank if r is None else r
        g = q.QuantKVCache(c.heads, c.head_dim, c.n_centroids, c.group, M, r, T,
                           max_versions=c.frames + 2, device=device, qsac_full=full)
        for f, (Q, K, V) in enumerate(data):
            Kd, Vd = dev_bf16(K, device), dev_bf16(V, device)
            if f == 0:
                g.build_centroids(Kd, Vd, iters=c.kmeans_iters)
            if stats:
                g.update_query_stats(dev_bf16(Q, device),
                                     refresh_basis=(f % c.refresh_every) == 0)
            g.append_kv(Kd, Vd)
        Kp, Vp = g.reconstruct()                       # [H][T][d]
        Kp = Kp.permute(1, 0, 2).contiguous()
        Vp = Vp.permute(1, 0, 2).contiguous()
        k_err = (Kp.float() - Kx.float()).pow(2).mean().item() / e_k
        v_err = (Vp.float() - Vx.float()).pow(2).mean().item() / e_v
        if which == "kv":
            O = g.attention(Qd)
        elif which == "k":
            O = empty.attention_ext(Qd, Kp, Vx)
        else:
            O = empty.attention_ext(Qd, Kx, Vp)
        o_mse = (O.float() - Oexact).pow(2).mean().item()
        shift = 0.0
        if which != "v":
            ie, iq = g.top1_shift(Qd, Kx)
            shift = float((ie != iq).float().mean().item())
        d, G = c.head_dim, c.group
        # stored bytes per token-head and tensor (the layout keeps the coefficient
        # scale even at rank 0)
        packed = d // 4 + 4 * (d // G) + (1 if c.n_centroids <= 256 else 2)
        k_bytes = packed + r + 2 if which != "v" else 2 * d
        v_bytes = packed if which != "k" else 2 * d
        fixed = (c.heads * c.n_centroids * d * 2 * ((which != "v") + (which != "k"))
                 + (c.frames // c.refresh_every) * c.heads * d * r * 4 * (which != "v"))
        ratio = 4.0 * d * T * c.heads / (T * c.heads * (k_bytes + v_bytes) + fixed)
        out.append({"ablation": name, "M": M, "r": r, "query_stats": stats, "quantized": which,
                    "qsac_full_quadratic": full,
                    "top1_shift": shift, "k_rel_mse": k_err, "v_rel_mse": v_err,
                    "out_mse": o_mse, "out_rel_mse": o_mse / e_o, "compression_ratio": ratio,
                    "workload": f"{c.name} layer, {c.frames} frames x {c.tokens_per_frame} "
                                f"tokens, {c.heads} heads, queries of the last frame"})
        del g, Kp, Vp, O
        torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- segment
def run_segment(cfg: syn.LayerConfig, device, reps: int = 10) -> list:
    """Times attention of the newest frame's queries over (a) the packed history,
    (b) the packed history followed by the frame's own keys and values as an exact
    bf16 segment, and (c) the same kernel over all keys as bf16 (an empty cache),
    which isolates what decoding the packed cache costs.  CUDA events on the
    launching stream, median of `reps` after 3 warm-ups; every input set is
    larger than the L2."""
    import bit_kv_cache_23_b200 as q

    c = cfg
    wl = Workload(c, device, extra_versions=4)
    src = wl.src
    # the frame being generated: the next one, not yet in the cache
    Qd, Kd, Vd = (dev_bf16(a, device) for a in src.frame(c.frames))
    Kall = torch.cat([dev_bf16(src.keys(f), device) for f in range(c.frames)] + [Kd], 0)
    Vall = torch.cat([dev_bf16(src.values(f), device) for f in range(c.frames)] + [Vd], 0)
    empty = q.QuantKVCache(c.heads, c.head_dim, c.n_centroids, c.group, c.n_cand, c.rank, 16,
                           device=device)
    O = torch.empty_like(Qd)
    T, nseg = wl.cache.len, Kd.shape[0]
    cases = [
        ("packed history", T, lambda: wl.cache.attention(Qd, O)),
        ("packed history + bf16 segment", T + nseg,
         lambda: wl.cache.attention_ext(Qd, Kd, Vd, O=O)),
        ("all keys bf16 (no decode)", Kall.shape[0],
         lambda: empty.attention_ext(Qd, Kall, Vall, O=O)),
    ]
    out = []
    for name, keys, fn in cases:
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize(device)
            ts.append(a.elapsed_time(b))
        ms = statistics.median(ts)
        flop = 4.0 * c.q_rows * keys * c.head_dim * c.heads
        out.append({"attention": name, "keys": int(keys), "ms": ms,
                    "TFLOP_per_s": flop / (ms * 1e-3) / 1e12,
                    "workload": f"{c.name} layer, {c.q_rows} queries x {c.heads} heads"})
    return out


# ----------------------------------------------------------------------------- oracle arm
def _oracle_head_step(args):
    """One head's share of a step, timed on the oracle (a worker of the process
    pool): statistics of n_s query rows, the append of n_s tokens, the
    reconstruction of the head's whole cache and the attention of a few query
    rows over it, each scaled to the full step of that head.  The oracle runs on
    its own state (its own k-means tables from a sample of the frame;
    reconstruction and attention cost the same whatever the packed values are)."""
    name, frames, h, n_s, n_rows = args
    import oracle

    c = dataclasses.replace(syn.get_config(name), frames=frames)
    Q, K, V = syn.FrameSource(c).frame(c.frames - 1, heads=[h])
    oc = oracle.OracleCache(1, c.head_dim, c.n_centroids, c.group, c.n_cand, c.rank,
                            c.total_tokens)
    nk = max(c.n_centroids, 64)
    oc.build_centroids(K[:nk], V[:nk], iters=1)
    t0 = time.perf_counter()
    M = np.zeros((c.head_dim, c.head_dim))
    oracle.stats_accumulate(Q[:n_s, 0, :], M)
    t_stats = (time.perf_counter() - t0) * c.q_rows / n_s
    oc.len = c.total_tokens - c.tokens_per_frame
    t0 = time.perf_counter()
    oc.append_kv(K[:n_s], V[:n_s])
    t_app = (time.perf_counter() - t0) * c.tokens_per_frame / n_s
    oc.len = c.total_tokens
    t0 = time.perf_counter()
    Kp, Vp = oc.reconstruct(0)
    t_rec = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.attention_head(np.ascontiguousarray(Q[:n_rows, 0, :]), Kp, Vp,
                          1.0 / math.sqrt(c.head_dim))
    t_rows = (time.perf_counter() - t0) * c.q_rows / n_rows
    return dict(stats_s=t_stats, append_s=t_app, reconstruct_s=t_rec, attention_rows_s=t_rows)


def host_cpu():
    """(usable cores, CPU model) of this host."""
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return cores, model


def oracle_throughput(cfg: syn.LayerConfig, n_s: int = 16, n_rows: int = 4):
    """The CPU oracle, as it stands, on a bounded sample of one step of the
    workload, on this host's cores: one process per core (spawned), each taking
    whole heads; every head's sample (statistics and append of n_s tokens, the
    reconstruction of its cache, attention of n_rows query rows) is scaled to
    that head's full step, and the step takes as long as the busiest core's
    heads (longest-first assignment).  Also reported: the same per-head times
    summed, i.e. the step on one core.  Returns a dict."""
    import multiprocessing as mp

    cores, model = host_cpu()
    workers = max(1, min(cores, cfg.heads))
    args = [(cfg.name, cfg.frames, h, n_s, n_rows) for h in range(cfg.heads)]
    t0 = time.perf_counter()
    with mp.get_context("spawn").Pool(workers) as pool:
        per_head = pool.map(_oracle_head_step, args, chunksize=1)
    wall = time.perf_counter() - t0
    totals = sorted((sum(d.values()) for d in per_head), reverse=True)
    load = [0.0] * workers
    for t in totals:                      # longest-first onto the least loaded core
        i = load.index(min(load))
        load[i] += t
    t_par, t_one = max(load), sum(totals)
    parts = {k: sum(d[k] for d in per_head) for k in per_head[0]}
    note = (f"oracle (plain C via ctypes) on {workers} of {cores} cores ({model}), one spawned "
            f"process per core taking whole heads; per head: statistics of {n_s} query rows, "
            f"append of {n_s} tokens, reconstruction of its {cfg.total_tokens}-token cache and "
            f"attention of {n_rows} query rows, each scaled to the head's share of one "
            f"{cfg.q_rows}-query step; sample wall time {wall:.1f} s")
    return dict(value=cfg.q_rows / t_par, single_thread=cfg.q_rows / t_one, cores=workers,
                host_cores=cores, cpu_model=model, note=note, parts_s=parts, sample_wall_s=wall)


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="480p", choices=sorted(syn.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-top1", action="store_true")
    ap.add_argument("--cache-frames", type=int, default=0,
                    help="cache length in frames (default: the configuration's); smaller "
                         "values give the short runs used for ncu captures")
    ap.add_argument("--shard", default="replica", choices=["replica", "heads"],
                    help="with several ranks: a whole layer per rank (weak scaling), or the "
                         "layer's heads split over the ranks (strong scaling); neither "
                         "exchanges data between ranks")
    ap.add_argument("--ablation", action="store_true",
                    help="instead of timing, print one JSON line per quantization setting "
                         "(QVG, QSAC only, rank sweep, K-only, V-only) with its quality")
    ap.add_argument("--rebuild-every", type=int, default=0,
                    help="while filling the cache, rebuild the centroid tables from the newest "
                         "frame every N frames (a new table version each time; the 1-minute "
                         "layer's Key distribution drifts)")
    ap.add_argument("--segment", action="store_true",
                    help="instead of the step, time attention over the packed history, over "
                         "history + the frame's bf16 segment, and over all keys in bf16")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = syn.get_config(args.config)
    if args.cache_frames > 0:
        cfg = dataclasses.replace(cfg, frames=args.cache_frames)
    workload_name = (f"{cfg.name} layer: {cfg.heads} heads x {cfg.head_dim}, cache "
                     f"{cfg.frames} latent frames x {cfg.tokens_per_frame} tokens, "
                     f"{cfg.q_rows}-query chunk, C={cfg.n_centroids}, G={cfg.group}, "
                     f"M={cfg.n_cand}, r={cfg.rank}")
    if args.rebuild_every > 0:
        workload_name += (f", centroid tables rebuilt every {args.rebuild_every} frames "
                          "(one table version per rebuild)")

    if args.segment:
        if rank == 0:
            device = torch.device("cuda", local)
            torch.cuda.set_device(device)
            for line in run_segment(cfg, device):
                print(json.dumps(line), flush=True)
        return

    if args.ablation:
        if rank == 0:
            device = torch.device("cuda", local)
            torch.cuda.set_device(device)
            frames = args.cache_frames if args.cache_frames > 0 else cfg.frames
            for line in run_ablation(syn.get_config(args.config), device, frames):
                print(json.dumps(line), flush=True)
        return

    if args.impl == "reference":
        if rank != 0:
            return
        t0 = time.time()
        runs = []
        for _ in range(max(1, args.steps)):
            runs.append(oracle_throughput(cfg))
            if time.time() - t0 > 120:
                break
        v = statistics.median(r["value"] for r in runs)
        r0 = runs[0]
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": len(runs), "warmup": 0, "ms_per_step": 1e3 * cfg.q_rows / v,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            # rank 0's heads under --shard heads: the first heads % world ranks
            # hold one more (the partition the ours arm uses)
            "config": config_dict(cfg, workload_name, world, args.shard,
                                  cfg.heads if args.shard != "heads"
                                  else -(-cfg.heads // world)),
            "cpu_baseline": {"kind": "oracle", "cores": r0["cores"], "host_cores": r0["host_cores"],
                             "cpu_model": r0["cpu_model"], "sample": r0["note"], "value": v,
                             "unit": UNIT, "single_thread": statistics.median(
                                 r["single_thread"] for r in runs)},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }))
        return

    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    peaks = load_peaks()
    W, K = max(3, args.warmup), args.steps
    from bit_kv_cache_23_b200 import shard

    if args.shard == "heads":
        h0, h1 = shard.head_range(rank, world, cfg.heads)
        heads = list(range(h0, h1))
    else:
        heads = None
    wl = Workload(cfg, device, extra_versions=2 * (W + K) + 8, heads=heads,
                  rebuild_every=args.rebuild_every)
    nh = len(wl.heads)
    # query tokens of the whole layer this rank serves per step (a fraction of a
    # layer when the heads are split)
    units = cfg.q_rows * nh / cfg.heads

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    def max_over_ranks(x: float) -> float:
        return shard.max_over_ranks(x, device)

    for i in range(W):
        wl.step(i)
    torch.cuda.synchronize(device)
    # ---- timed region (device time, CUDA events on the launching stream)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(device)
    clocks.start()
    barrier()
    torch.cuda.synchronize(device)
    nstep0 = wl.nstep
    start.record()
    for i in range(K):
        wl.step(i, evs[i])
    end.record()
    torch.cuda.synchronize(device)
    barrier()
    clk = clocks.stop()
    total_ms = max_over_ranks(start.elapsed_time(end))
    seg = np.array([[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3])]
                    for e in evs])
    stats_ms, app_ms, att_ms = (float(x) for x in seg.mean(0))
    ms_step = total_ms / K
    value = shard.throughput(units, ms_step * 1e-3, device)
    # our kernels in the timed region: per step statistics, the append (Keys and
    # Values in one launch) and the attention (plus its merge kernel when the key
    # range is split), and the refresh kernel on the steps that refresh the basis
    n_launches = (3 + (1 if attention_splits(cfg, nh, device) else 0)) * K + sum(
        1 for n in range(nstep0, nstep0 + K) if n % cfg.refresh_every == 0)

    # ---- end to end through the public API from pinned host memory
    e2e = None
    if not args.no_e2e:
        Qh, Kh, Vh = wl.host_pool[0]
        sets = wl.host_sets()
        cs = torch.cuda.Stream(device)
        wl.run_host(W, sets, cs)
        torch.cuda.synchronize(device)
        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(cs)                     # before the first upload, on the copy stream
        wl.run_host(K, sets, cs, first=W)
        e2.record(cs)                     # after the last read-back
        torch.cuda.synchronize(device)
        barrier()
        e2e_ms = max_over_ranks(s2.elapsed_time(e2)) / K
        e2e = {"value": shard.throughput(units, e2e_ms * 1e-3, device), "unit": UNIT,
               "h2d_bytes_per_step": int(Qh.numel() * 2 + Kh.numel() * 2 + Vh.numel() * 2),
               "d2h_bytes_per_step": int(Qh.numel() * 2),
               "copies": "per step: Q, K, V uploaded from pinned host memory and O read back, "
                         "on a copy stream overlapping the neighbouring steps' kernels"}

    # ---- derived figures
    c = cfg
    T = c.total_tokens
    # per launch on this rank (its heads)
    att_flop = 4.0 * c.q_rows * T * c.head_dim * nh
    att_tflops = att_flop / (att_ms * 1e-3) / 1e12
    per_tok = packed_bytes_per_token_head(c)
    app_bytes = c.tokens_per_frame * nh * (4 * c.head_dim + per_tok)
    app_gbs = app_bytes / (app_ms * 1e-3) / 1e9
    # fixed bytes: every centroid-table version in use and every basis version
    fixed = ((1 + wl.rebuilds) * 2 * c.heads * c.n_centroids * c.head_dim * 2
             + (c.frames // c.refresh_every) * c.heads * c.head_dim * c.rank * 4)
    compression = (4.0 * c.head_dim * T * c.heads) / (T * c.heads * per_tok + fixed)

    top1 = None
    if not args.no_top1 and rank == 0:
        hs = None if heads is None else wl.heads
        Kall = torch.cat([dev_bf16(wl.src.keys(f, hs), device) for f in range(c.frames - 1)]
                         + [wl.pool[(wl.nstep - 1) % len(wl.pool)][1]], 0)
        ie, iq = wl.cache.top1_shift(wl.pool[(wl.nstep - 1) % len(wl.pool)][0], Kall)
        top1 = float((ie != iq).float().mean().item())
        del Kall

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if args.shard == "heads" else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict(c, workload_name, world, args.shard, nh),
        "gpu_launches": n_launches,
        "roofline": {"bound": "tensor", "achieved": att_tflops, "peak": peaks["bf16"],
                     "unit": "TFLOP/s", "frac": att_tflops / peaks["bf16"],
                     "traffic": attention_traffic(cfg), "traffic_unit": "bytes per launch",
                     "kernel": "qwm_attention", "peak_source": f"{peaks['source']} bf16 burst"},
        "append": {"ms": app_ms, "tokens_per_s": c.tokens_per_frame / (app_ms * 1e-3),
                   "GB_per_s": app_gbs, "frac_hbm": app_gbs / peaks["hbm"],
                   "bytes_per_frame": app_bytes},
        "attention": {"ms": att_ms, "TFLOP_per_s": att_tflops, "flop_per_call": att_flop,
                      "frac_bf16": att_tflops / peaks["bf16"]},
        "stats_refresh_ms": stats_ms,
        "top1_shift": top1, "compression_ratio": compression,
        "clocks": clk, "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ob = oracle_throughput(cfg)
        line["cpu_baseline"] = {"value": ob["value"], "unit": UNIT, "cores": ob["cores"],
                                "host_cores": ob["host_cores"], "cpu_model": ob["cpu_model"],
                                "kind": "oracle", "sample": ob["note"],
                                "single_thread": ob["single_thread"], "parts_s": ob["parts_s"]}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
