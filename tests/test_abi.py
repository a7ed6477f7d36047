"""Host-side checks of the C ABI (no GPU needed): the library loads and exports
every symbol include/qwm.h declares, buffer sizing follows the packed layout,
and invalid calls return the documented status before touching the device."""
import ctypes
import os
import re

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
    assert q.qwm_abi_version() == 1
    assert q.qwm_status_string(3) == "capacity exceeded"


def _cfg(**kw):
    base = dict(heads=40, head_dim=128, n_centroids=256, group=32, n_cand=4, rank=8,
                max_versions=64, flags=0, max_tokens=37440)
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
                                 dict(max_tokens=0), dict(heads=0)])
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


def test_struct_layout_matches_header():
    assert ctypes.sizeof(q.qwm_config) == 40
    assert ctypes.sizeof(q.qwm_buffers) == 8 * q.NBUF
    assert ctypes.sizeof(q.qwm_cache) == 40 + 8 * q.NBUF + 24 + 24
    assert len(q.BUFFER_NAMES) == q.NBUF == 17


def test_binding_refuses_cpu_tensors():
    import torch
    cfg = _cfg()
    c = _fake_cache(has_centroids=1)
    with pytest.raises(ValueError):
        q.qwm_append_kv(c, torch.zeros((4, 40, 128), dtype=torch.bfloat16),
                        torch.zeros((4, 40, 128), dtype=torch.bfloat16))
