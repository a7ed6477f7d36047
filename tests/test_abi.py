"""Host-side checks of the C ABI (no GPU needed): the library loads and exports
every symbol include/qwm.h declares, buffer sizing follows the packed layout,
and invalid calls return the documented status before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

import bit_kv_cache_23_b200 as q
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
MAGIC = 0x51574D31


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "qwm.h")).read()
    return sorted(set(re.findall(r"QWM_API[^;(]*?\b(qwm_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = q.lib()
    names = _declared_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert q.qwm_abi_version() == 2
    assert q.qwm_status_string(3) == "capacity exceeded"


def _cfg(**kw):
    base = dict(heads=40, head_dim=128, n_centroids=256, group=32, n_cand=4, rank=8,
                max_versions=64, flags=0, max_cent_versions=1, max_queries=0, max_tokens=37440)
    base.update(kw)
    return q.qwm_config(**base)


def test_full_quadratic_flag_accepted():
    out = q.qwm_sizes()
    assert q.lib().qwm_cache_sizes(ctypes.byref(_cfg(flags=q.QWM_FLAG_QSAC_FULL)),
                                   ctypes.byref(out)) == 0
    # the fp32 snapshot of M / n fits after 32 Ritz columns in each head's fp64 block
    for d in (64, 128):
        assert 32 * d * 8 + d * d * 4 <= d * d * 8


def test_sizes_follow_layout():
    s = q.qwm_cache_sizes(_cfg())
    assert s.tcap == 37504  # rounded up to a multiple of 128
    H, T = 40, s.tcap
    assert s.bytes[0] == H * T * 32 and s.bytes[1] == H * T * 16 and s.bytes[2] == H * T
    assert s.bytes[3] == H * T * 8 and s.bytes[4] == H * T * 2
    assert s.bytes_per_token_head == 108 == oracle.bytes_per_token_head(128, 256, 32, 8)
    s2 = q.qwm_cache_sizes(_cfg(n_centroids=512))
    assert s2.bytes_per_token_head == 110 and s2.bytes[2] == H * T * 2
    t = q.qwm_cache_sizes(_cfg(heads=1, head_dim=64, n_centroids=16, group=16, rank=4,
                               max_tokens=512))
    assert t.bytes_per_token_head == oracle.bytes_per_token_head(64, 16, 16, 4) == 72


@pytest.mark.parametrize("bad", [dict(head_dim=96), dict(group=8), dict(n_centroids=0),
                                 dict(n_centroids=513), dict(n_cand=9), dict(n_cand=300),
                                 dict(rank=17), dict(max_versions=0), dict(flags=2), dict(flags=-1),
                                 dict(max_tokens=0), dict(heads=0), dict(max_cent_versions=0),
                                 dict(max_cent_versions=65536), dict(max_queries=-1),
                                 dict(max_queries=(1 << 24) + 1)])
def test_invalid_configs_rejected(bad):
    out = q.qwm_sizes()
    st = q.lib().qwm_cache_sizes(ctypes.byref(_cfg(**bad)), ctypes.byref(out))
    assert st == 1


def test_init_validates_pointers_before_device_work():
    cfg = _cfg()
    bufs = q.qwm_buffers()
    c = q.qwm_cache()
    L = q.lib()
    assert L.qwm_cache_init(ctypes.byref(c), ctypes.byref(cfg), ctypes.byref(bufs), None) == 1
    for i in range(q.NBUF):
        bufs.ptr[i] = 0x100000 + 256 * i * 4096
    bufs.ptr[5] += 8
    assert L.qwm_cache_init(ctypes.byref(c), ctypes.byref(cfg), ctypes.byref(bufs), None) == 2
    assert c.magic == 0  # unchanged on error


def _fake_cache(**state):
    c = q.qwm_cache()
    c.cfg = _cfg(max_tokens=1000)
    c.tcap = 1024
    for i in range(q.NBUF):
        c.buf.ptr[i] = 0x100000 + 256 * i * 4096
    c.magic = MAGIC
    c.n_versions = 1
    for k, v in state.items():
        setattr(c, k, v)
    return c


def test_call_order_and_capacity_errors():
    L = q.lib()
    p = ctypes.c_void_p(0x200000)
    c = _fake_cache()
    assert L.qwm_append_kv(ctypes.byref(c), p, p, 10, None) == 4      # no centroids yet
    c = _fake_cache(has_centroids=1, len=1000)
    assert L.qwm_append_kv(ctypes.byref(c), p, p, 25, None) == 3      # 1000 + 25 > 1024
    assert c.len == 1000
    c = _fake_cache(has_centroids=1, len=0)
    assert L.qwm_attention(ctypes.byref(c), p, 4, 0.0, p, None) == 4  # empty cache
    assert L.qwm_append_kv(ctypes.byref(c), ctypes.c_void_p(0x200004), p, 4, None) == 2
    c = _fake_cache(n_versions=64)
    assert L.qwm_update_query_stats(ctypes.byref(c), p, 8, 1, None) == 3  # no basis slot
    c = _fake_cache()
    c.magic = 0
    assert L.qwm_append_kv(ctypes.byref(c), p, p, 4, None) == 1       # not initialised
    c = _fake_cache(has_centroids=1, len=100)
    assert L.qwm_reconstruct(ctypes.byref(c), 90, 20, p, p, None) == 1  # past len
    assert L.qwm_build_centroids(ctypes.byref(c), p, p, 100, 10, None) == 1  # n < C


def test_attention_ext_argument_checks():
    L = q.lib()
    p = ctypes.c_void_p(0x200000)
    c = _fake_cache(has_centroids=1, len=0)
    # no keys at all: empty cache and empty segment
    assert L.qwm_attention_ext(ctypes.byref(c), p, 4, None, None, 0, 0.0, p, None, None) == 4
    # a segment needs both K and V
    assert L.qwm_attention_ext(ctypes.byref(c), p, 4, p, None, 8, 0.0, p, None, None) == 1
    assert L.qwm_attention_ext(ctypes.byref(c), p, 4, p, p, -1, 0.0, p, None, None) == 1
    # 16-byte alignment of the segment, 4-byte alignment of lse
    assert L.qwm_attention_ext(ctypes.byref(c), p, 4, ctypes.c_void_p(0x200008), p, 8, 0.0, p,
                               None, None) == 2
    assert L.qwm_attention_ext(ctypes.byref(c), p, 4, p, p, 8, 0.0, p,
                               ctypes.c_void_p(0x200002), None) == 2
    # a non-empty cache without centroids
    c = _fake_cache(has_centroids=0, len=10)
    assert L.qwm_attention_ext(ctypes.byref(c), p, 4, p, p, 8, 0.0, p, None, None) == 4
    # nothing to do for zero query rows (no device work)
    c = _fake_cache(has_centroids=1, len=0)
    assert L.qwm_attention_ext(ctypes.byref(c), p, 0, p, p, 8, 0.0, p, None, None) == 0


def _probe():
    """Compile tests/c/abi_probe.c against include/qwm.h with gcc, link it to
    libqwm.so and return its "key value" lines as a dict."""
    import tempfile
    lib = q.lib()  # noqa: F841 - the library is built
    libdir = os.path.dirname(q.LIB_PATH)
    with tempfile.TemporaryDirectory() as td:
        exe = os.path.join(td, "abi_probe")
        subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Werror", "-I",
                               os.path.join(ROOT, "include"),
                               os.path.join(ROOT, "tests", "c", "abi_probe.c"), "-L", libdir,
                               "-l:libqwm.so", "-Wl,-rpath," + libdir, "-o", exe])
        out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    d = {}
    for line in out.splitlines():
        k, v = line.rsplit(" ", 1) if not line.startswith("status_") else line.split(" ", 1)
        d[k] = v
    return d


def test_struct_layout_matches_header():
    """The binding's ctypes structures, buffer order and status strings agree
    with what a C compiler makes of include/qwm.h, and qwm_cache_sizes returns
    the same sizes through the header as through the binding."""
    d = _probe()
    assert int(d["abi_macro"]) == int(d["abi_lib"]) == q.qwm_abi_version() == 2
    assert int(d["nbuf"]) == q.NBUF == len(q.BUFFER_NAMES) == 18
    assert int(d["noalloc_bytes"]) == q.QWM_NOALLOC_SCRATCH_BYTES
    assert int(d["flag_qsac_full"]) == q.QWM_FLAG_QSAC_FULL
    assert int(d["attn_max_split"]) == q.QWM_ATTN_MAX_SPLIT
    for name, st in (("qwm_config", q.qwm_config), ("qwm_sizes", q.qwm_sizes),
                     ("qwm_buffers", q.qwm_buffers), ("qwm_cache", q.qwm_cache)):
        assert int(d[f"size {name}"]) == ctypes.sizeof(st), name
    for key, v in d.items():
        if key.startswith("off "):
            sname, field = key[4:].split(".")
            st = getattr(q, sname)
            assert getattr(st, field).offset == int(v), key
    for e in ("K_CODES", "CENT_K", "TOKVER", "CENTVER", "WORKSPACE"):
        assert q.BUFFER_NAMES[int(d[f"enum QWM_BUF_{e}"])] == e.lower(), e
    s = q.qwm_cache_sizes(_cfg(max_cent_versions=2, max_queries=1560))
    assert int(d["sizes_status"]) == 0 and int(d["sizes_bad_status"]) == 1
    assert int(d["sizes_tcap"]) == s.tcap and int(d["sizes_bpth"]) == s.bytes_per_token_head
    for i in range(q.NBUF):
        assert int(d[f"sizes_bytes_{i}"]) == s.bytes[i], q.BUFFER_NAMES[i]
    assert d["status_capacity"] == q.qwm_status_string(3) == "capacity exceeded"


def test_workspace_holds_split_attention_partials():
    """The WORKSPACE buffer covers QWM_ATTN_MAX_SPLIT fp32 partial outputs and
    log-sum-exps of max_queries rows and every head (and is never smaller than
    the centroid build's scratch)."""
    ws = q.BUFFER_NAMES.index("workspace")
    base = q.qwm_cache_sizes(_cfg()).bytes[ws]
    s = q.qwm_cache_sizes(_cfg(max_queries=1560))
    need = q.QWM_ATTN_MAX_SPLIT * 1560 * 40 * (128 + 1) * 4
    assert s.bytes[ws] == max(need, base)
    assert q.qwm_cache_sizes(_cfg(max_queries=1)).bytes[ws] == base


def test_centroid_versions_sizes_and_capacity():
    """Centroid tables take one [H][C][d] bf16 slot per version and CENTVER one
    uint16 per token; a rebuild on a cache that holds tokens needs a free slot
    (QWM_ERR_CAPACITY otherwise, with the cache unchanged)."""
    s1 = q.qwm_cache_sizes(_cfg())
    s3 = q.qwm_cache_sizes(_cfg(max_cent_versions=3))
    ck = q.BUFFER_NAMES.index("cent_k")
    assert s1.bytes[ck] == 40 * 256 * 128 * 2 and s3.bytes[ck] == 3 * s1.bytes[ck]
    assert s1.bytes[q.BUFFER_NAMES.index("centver")] == s1.tcap * 2
    L = q.lib()
    p = ctypes.c_void_p(0x200000)
    c = _fake_cache(has_centroids=1, len=100, n_cent_versions=1)
    assert L.qwm_build_centroids(ctypes.byref(c), p, p, 300, 10, None) == 3
    assert L.qwm_build_centroids_noalloc(ctypes.byref(c), p, p, 300, 10, None) == 3
    assert c.n_cent_versions == 1 and c.cur_cent_version == 0
    # misaligned inputs and bad sizes are refused by both entry points alike
    for fn in (L.qwm_build_centroids, L.qwm_build_centroids_noalloc):
        assert fn(ctypes.byref(c), ctypes.c_void_p(0x200008), p, 300, 10, None) == 2
        assert fn(ctypes.byref(c), p, p, 300, 0, None) == 1
        assert fn(ctypes.byref(c), p, p, 2000, 10, None) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    cfg = _cfg()
    c = _fake_cache(has_centroids=1)
    with pytest.raises(ValueError):
        q.qwm_append_kv(c, torch.zeros((4, 40, 128), dtype=torch.bfloat16),
                        torch.zeros((4, 40, 128), dtype=torch.bfloat16))
