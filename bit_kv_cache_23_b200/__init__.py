"""Python binding of libqwm.so, the B200 QuantWM 2-bit KV-cache library.

Argument marshalling only: every function forwards to the C entry point of the
same name declared in ``include/qwm.h``; every step of the computation runs in
the library's CUDA kernels.  PyTorch provides device memory and streams.  There
is no CPU fallback: a missing library or a tensor that is not on a CUDA device
raises.

Tensors Q, K, V, O are token-major ``[n][heads][head_dim]`` ``torch.bfloat16``
(contiguous, CUDA).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "QwmError", "qwm_config", "qwm_sizes", "qwm_buffers", "qwm_cache", "BUFFER_NAMES",
    "lib", "qwm_abi_version", "qwm_status_string", "qwm_cache_sizes", "qwm_cache_init",
    "qwm_build_centroids", "qwm_build_centroids_noalloc", "qwm_update_query_stats", "qwm_append_kv", "qwm_attention",
    "qwm_attention_ext", "qwm_reconstruct", "qwm_top1_shift", "qwm_device_status", "QuantKVCache",
    "QWM_FLAG_QSAC_FULL", "QWM_NOALLOC_SCRATCH_BYTES", "QWM_ATTN_MAX_SPLIT",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqwm.so")

QWM_FLAG_QSAC_FULL = 1   # QSAC stage 2 by the full quadratic form e^T A e
QWM_NOALLOC_SCRATCH_BYTES = 16 << 20   # fixed scratch of qwm_build_centroids_noalloc
QWM_ATTN_MAX_SPLIT = 6                 # key ranges an attention call may be split into

BUFFER_NAMES = ["k_codes", "k_params", "k_idx", "k_coef", "k_cscale", "v_codes", "v_params",
                "v_idx", "cent_k", "cent_v", "qstats", "sens", "wgroup", "basis", "tokver",
                "centver", "eigvec", "workspace"]
NBUF = len(BUFFER_NAMES)

STATUS = {0: "QWM_OK", 1: "QWM_ERR_INVALID_ARG", 2: "QWM_ERR_ALIGNMENT", 3: "QWM_ERR_CAPACITY",
          4: "QWM_ERR_STATE", 5: "QWM_ERR_CUDA", 6: "QWM_ERR_TIMEOUT", 7: "QWM_ERR_UNSUPPORTED"}


class qwm_config(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("n_centroids", ctypes.c_int32), ("group", ctypes.c_int32),
                ("n_cand", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("max_versions", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("max_cent_versions", ctypes.c_int32), ("max_queries", ctypes.c_int32),
                ("max_tokens", ctypes.c_int64)]


class qwm_sizes(ctypes.Structure):
    _fields_ = [("bytes", ctypes.c_uint64 * NBUF), ("tcap", ctypes.c_int64),
                ("bytes_per_token_head", ctypes.c_int64)]


class qwm_buffers(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p * NBUF)]


class qwm_cache(ctypes.Structure):
    _fields_ = [("cfg", qwm_config), ("buf", qwm_buffers), ("tcap", ctypes.c_int64),
                ("len", ctypes.c_int64), ("n_queries", ctypes.c_int64),
                ("frames", ctypes.c_int32), ("n_versions", ctypes.c_int32),
                ("cur_version", ctypes.c_int32), ("has_centroids", ctypes.c_int32),
                ("has_eigvec", ctypes.c_int32), ("magic", ctypes.c_int32),
                ("n_cent_versions", ctypes.c_int32), ("cur_cent_version", ctypes.c_int32)]


class QwmError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")


_lib = None
_P = ctypes.c_void_p


def lib():
    """Load libqwm.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libqwm.so not built ({LIB_PATH}); run "
                              "python -m bit_kv_cache_23_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        I32, I64, F32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float
        pc = ctypes.POINTER(qwm_cache)
        sig = {
            "qwm_abi_version": (I32, []),
            "qwm_status_string": (ctypes.c_char_p, [I32]),
            "qwm_cache_sizes": (I32, [ctypes.POINTER(qwm_config), ctypes.POINTER(qwm_sizes)]),
            "qwm_cache_init": (I32, [pc, ctypes.POINTER(qwm_config), ctypes.POINTER(qwm_buffers), _P]),
            "qwm_build_centroids": (I32, [pc, _P, _P, I64, I32, _P]),
            "qwm_update_query_stats": (I32, [pc, _P, I64, I32, _P]),
            "qwm_append_kv": (I32, [pc, _P, _P, I64, _P]),
            "qwm_attention": (I32, [pc, _P, I64, F32, _P, _P]),
            "qwm_attention_ext": (I32, [pc, _P, I64, _P, _P, I64, F32, _P, _P, _P]),
            "qwm_reconstruct": (I32, [pc, I64, I64, _P, _P, _P]),
            "qwm_top1_shift": (I32, [pc, _P, I64, _P, _P, _P, _P]),
            "qwm_device_status": (I32, [ctypes.POINTER(ctypes.c_int32)]),
            "qwm_build_centroids_noalloc": (I32, [pc, _P, _P, I64, I32, _P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(fn: str, st: int) -> None:
    if st != 0:
        raise QwmError(fn, st)


def _stream(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev_ptr(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


# ----------------------------------------------------------------- thin entry points
def qwm_abi_version() -> int:
    return int(lib().qwm_abi_version())


def qwm_status_string(status: int) -> str:
    return lib().qwm_status_string(status).decode()


def qwm_cache_sizes(cfg: qwm_config) -> qwm_sizes:
    out = qwm_sizes()
    _check("qwm_cache_sizes", lib().qwm_cache_sizes(ctypes.byref(cfg), ctypes.byref(out)))
    return out


def qwm_cache_init(cache: qwm_cache, cfg: qwm_config, bufs: qwm_buffers, stream=None,
                   device=None) -> None:
    _check("qwm_cache_init", lib().qwm_cache_init(ctypes.byref(cache), ctypes.byref(cfg),
                                                  ctypes.byref(bufs), _stream(stream, device)))


def qwm_build_centroids(cache: qwm_cache, K: torch.Tensor, V: torch.Tensor, iters: int = 10,
                        stream=None) -> None:
    _check("qwm_build_centroids", lib().qwm_build_centroids(
        ctypes.byref(cache), _dev_ptr(K, "K", torch.bfloat16), _dev_ptr(V, "V", torch.bfloat16),
        K.shape[0], iters, _stream(stream, K.device)))


def qwm_build_centroids_noalloc(cache: qwm_cache, K: torch.Tensor, V: torch.Tensor,
                                iters: int = 10, stream=None) -> None:
    """Same result as qwm_build_centroids, with the scratch taken from a fixed
    device array inside the library (for callers that cannot allocate)."""
    _check("qwm_build_centroids_noalloc", lib().qwm_build_centroids_noalloc(
        ctypes.byref(cache), _dev_ptr(K, "K", torch.bfloat16), _dev_ptr(V, "V", torch.bfloat16),
        K.shape[0], iters, _stream(stream, K.device)))


def qwm_update_query_stats(cache: qwm_cache, Q: torch.Tensor, refresh_basis: bool = True,
                           stream=None) -> None:
    _check("qwm_update_query_stats", lib().qwm_update_query_stats(
        ctypes.byref(cache), _dev_ptr(Q, "Q", torch.bfloat16), Q.shape[0], int(refresh_basis),
        _stream(stream, Q.device)))


def qwm_append_kv(cache: qwm_cache, K: torch.Tensor, V: torch.Tensor, stream=None) -> None:
    _check("qwm_append_kv", lib().qwm_append_kv(
        ctypes.byref(cache), _dev_ptr(K, "K", torch.bfloat16), _dev_ptr(V, "V", torch.bfloat16),
        K.shape[0], _stream(stream, K.device)))


def qwm_attention(cache: qwm_cache, Q: torch.Tensor, O: torch.Tensor | None = None,
                  scale: float = 0.0, stream=None) -> torch.Tensor:
    if O is None:
        O = torch.empty_like(Q)
    _check("qwm_attention", lib().qwm_attention(
        ctypes.byref(cache), _dev_ptr(Q, "Q", torch.bfloat16), Q.shape[0], float(scale),
        _dev_ptr(O, "O", torch.bfloat16), _stream(stream, Q.device)))
    return O


def qwm_attention_ext(cache: qwm_cache, Q: torch.Tensor, K_seg: torch.Tensor | None = None,
                      V_seg: torch.Tensor | None = None, O: torch.Tensor | None = None,
                      lse: torch.Tensor | None = None, scale: float = 0.0,
                      stream=None) -> torch.Tensor:
    """Attention over the packed cache followed by the bf16 segment (K_seg, V_seg),
    [n_seg][H][d]; lse, if given, is a [n_q][H] float32 tensor that receives the
    natural-log softmax denominators."""
    if O is None:
        O = torch.empty_like(Q)
    n_seg = 0 if K_seg is None else K_seg.shape[0]
    if (K_seg is None) != (V_seg is None) or (V_seg is not None and V_seg.shape != K_seg.shape):
        raise ValueError("K_seg and V_seg must be given together, with equal shapes")
    kp = _dev_ptr(K_seg, "K_seg", torch.bfloat16) if n_seg else None
    vp = _dev_ptr(V_seg, "V_seg", torch.bfloat16) if n_seg else None
    lp = _dev_ptr(lse, "lse", torch.float32) if lse is not None else None
    _check("qwm_attention_ext", lib().qwm_attention_ext(
        ctypes.byref(cache), _dev_ptr(Q, "Q", torch.bfloat16), Q.shape[0], kp, vp, n_seg,
        float(scale), _dev_ptr(O, "O", torch.bfloat16), lp, _stream(stream, Q.device)))
    return O


def qwm_reconstruct(cache: qwm_cache, t0: int, n: int, device, stream=None):
    H, d = cache.cfg.heads, cache.cfg.head_dim
    Kp = torch.empty((H, n, d), dtype=torch.bfloat16, device=device)
    Vp = torch.empty((H, n, d), dtype=torch.bfloat16, device=device)
    _check("qwm_reconstruct", lib().qwm_reconstruct(
        ctypes.byref(cache), int(t0), int(n), _dev_ptr(Kp, "Kp"), _dev_ptr(Vp, "Vp"),
        _stream(stream, device)))
    return Kp, Vp


def qwm_top1_shift(cache: qwm_cache, Q: torch.Tensor, K_exact: torch.Tensor, stream=None):
    H = cache.cfg.heads
    ie = torch.empty((Q.shape[0], H), dtype=torch.int32, device=Q.device)
    iq = torch.empty_like(ie)
    _check("qwm_top1_shift", lib().qwm_top1_shift(
        ctypes.byref(cache), _dev_ptr(Q, "Q", torch.bfloat16), Q.shape[0],
        _dev_ptr(K_exact, "K_exact", torch.bfloat16), _dev_ptr(ie, "idx_exact"),
        _dev_ptr(iq, "idx_quant"), _stream(stream, Q.device)))
    return ie, iq


def qwm_device_status() -> int:
    """Synchronize and return 1 if a bounded device wait timed out since the
    last call (the flag is cleared), else 0."""
    f = ctypes.c_int32(0)
    st = lib().qwm_device_status(ctypes.byref(f))
    if st not in (0, 6):
        raise QwmError("qwm_device_status", st)
    return int(f.value)


# ----------------------------------------------------------------- convenience owner
class QuantKVCache:
    """Allocates the caller-owned device buffers with torch and holds the host
    state; every method is one C-ABI call."""

    def __init__(self, heads: int, head_dim: int, n_centroids: int, group: int, n_cand: int,
                 rank: int, max_tokens: int, max_versions: int = 1024, device="cuda",
                 stream=None, qsac_full: bool = False, max_cent_versions: int = 1,
                 max_queries: int = 0):
        self.device = torch.device(device)
        if self.device.type != "cuda":
            raise ValueError("QuantKVCache lives on a CUDA device")
        flags = QWM_FLAG_QSAC_FULL if qsac_full else 0
        self.cfg = qwm_config(heads, head_dim, n_centroids, group, n_cand, rank, max_versions,
                              flags, max_cent_versions, max_queries, max_tokens)
        self.sizes = qwm_cache_sizes(self.cfg)
        self.buffers = {}
        bufs = qwm_buffers()
        for i, name in enumerate(BUFFER_NAMES):
            nb = int(self.sizes.bytes[i])
            t = torch.empty(max(nb, 256), dtype=torch.uint8, device=self.device)
            self.buffers[name] = t
            bufs.ptr[i] = t.data_ptr()
        self.bufs = bufs
        self.c = qwm_cache()
        qwm_cache_init(self.c, self.cfg, bufs, stream, self.device)

    # host state
    @property
    def len(self) -> int:
        return int(self.c.len)

    @property
    def tcap(self) -> int:
        return int(self.sizes.tcap)

    @property
    def version(self) -> int:
        return int(self.c.cur_version)

    @property
    def cent_version(self) -> int:
        return int(self.c.cur_cent_version)

    def build_centroids(self, K, V, iters=10, stream=None):
        qwm_build_centroids(self.c, K, V, iters, stream)

    def update_query_stats(self, Q, refresh_basis=True, stream=None):
        qwm_update_query_stats(self.c, Q, refresh_basis, stream)

    def append_kv(self, K, V, stream=None):
        qwm_append_kv(self.c, K, V, stream)

    def attention(self, Q, O=None, scale=0.0, stream=None):
        return qwm_attention(self.c, Q, O, scale, stream)

    def attention_ext(self, Q, K_seg=None, V_seg=None, O=None, lse=None, scale=0.0,
                      stream=None):
        return qwm_attention_ext(self.c, Q, K_seg, V_seg, O, lse, scale, stream)

    def reconstruct(self, t0=0, n=None, stream=None):
        n = self.len - t0 if n is None else n
        return qwm_reconstruct(self.c, t0, n, self.device, stream)

    def top1_shift(self, Q, K_exact, stream=None):
        return qwm_top1_shift(self.c, Q, K_exact, stream)

    # typed views of the packed buffers (for inspection and tests); the centroid
    # tables are those of `cent_version` (default: the version in force)
    def view(self, name: str, cent_version: int | None = None) -> torch.Tensor:
        H, d, C, G, r = (self.cfg.heads, self.cfg.head_dim, self.cfg.n_centroids,
                         self.cfg.group, self.cfg.rank)
        if name in ("cent_k", "cent_v"):
            cv = self.cent_version if cent_version is None else int(cent_version)
            if not 0 <= cv < self.cfg.max_cent_versions:
                raise IndexError(f"centroid-table version {cv} out of range")
            n = H * C * d
            return self.buffers[name][2 * n * cv:2 * n * (cv + 1)].view(torch.int16).view(H, C, d)
        T, ng = self.tcap, d // G
        b = self.buffers[name]
        idt = torch.uint8 if C <= 256 else torch.int16
        shapes = {
            "k_codes": (torch.uint8, (H, T, d // 4)), "v_codes": (torch.uint8, (H, T, d // 4)),
            "k_params": (torch.int16, (H, T, ng, 2)), "v_params": (torch.int16, (H, T, ng, 2)),
            "k_idx": (idt, (H, T)), "v_idx": (idt, (H, T)),
            "k_coef": (torch.int8, (H, T, r)), "k_cscale": (torch.int16, (H, T)),
            "qstats": (torch.float64, (H, d, d)), "sens": (torch.float32, (H, d)),
            "wgroup": (torch.float32, (H, ng)), "tokver": (torch.int16, (T,)),
            "centver": (torch.int16, (T,)),
            "basis": (torch.float32, (self.cfg.max_versions, H, d, max(r, 1))),
            "eigvec": (torch.float64, (H * d * d + H,)),
        }
        dt, shp = shapes[name]
        n = math.prod(shp) * torch.empty((), dtype=dt).element_size()
        return b[:n].view(dt).view(shp)
