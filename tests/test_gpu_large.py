"""Parity at the full sizes of the large layer configurations.

Every frame runs through the CUDA library for all heads, in the launch
configuration the benchmark times; for sampled heads every token is re-encoded
by the CPU oracle, running on its own state, and compared bit for bit (centroid
tables, indices, INT2 codes, fp16 group parameters, INT8 coefficients and
scales); at every refresh the statistics matrix, s and w are compared bit for
bit and the basis within tolerance with the oracle's refresh, and attention
is compared on sampled query rows against the oracle's fp64 attention over its
own reconstruction of the whole cache.
"""
import pytest

from large_util import run_full
from parity_util import ATOL_MAX, ATOL_MEAN

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _check(out):
    assert out["cent_equal"], "k-means centroids differ"
    assert out["packed_mismatch"] == {}, out["packed_mismatch"]
    assert out["refreshes"] > 0
    assert out["stats_mismatch"] == 0, out["stats_mismatch"]
    assert out["sw_mismatch"] == 0, out["sw_mismatch"]
    assert out["orth_err"] < 1e-5, out["orth_err"]
    assert out["proj_err"] < 1e-3, out["proj_err"]
    assert out["attn"], "no attention check ran"
    for f, h, mx, mean in out["attn"]:
        assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (f, h, mx, mean)


def test_480p_full_size():
    """40 heads x 128, 24 frames x 1560 tokens, C=256: heads 0, 23, 39; at the last
    frame all 1560 query rows of head 23 (the last CTA holds rows 1536-1559)."""
    out = run_full("480p", heads=[0, 23, 39], attn_frames={0, 11, 23}, attn_rows=16,
                   full_rows_head=23)
    _check(out)
    assert out["full_rows"] == 1560


def test_720p_full_size():
    """40 heads x 128, 21 frames x 3600 tokens, C=512 (two-byte indices): heads 5, 38."""
    _check(run_full("720p", heads=[5, 38], attn_frames={0, 20}, attn_rows=16))


def test_1min_full_size():
    """40 heads x 128, 241 frames x 1560 tokens (375960 cached), C=512, basis
    refreshed every 8 frames with a drifting Key mean: head 11."""
    _check(run_full("1min", heads=[11], attn_frames={0, 120, 240}, attn_rows=12))
