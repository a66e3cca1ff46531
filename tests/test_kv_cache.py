"""The library's KV-cache accounting reproduces Table 5 and agrees with the
oracle's reading for other context lengths and schedules."""

import os

import pytest

import oracle.accounting as OA
from token_skipping_sparse_b200 import kv_cache as K

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows():
    with open(os.path.join(GOLDEN, "table5_kv_cache.txt")) as fh:
        return [ln.split() for ln in fh if ln.strip() and not ln.startswith("#")]


def _half_up(x, q):
    from decimal import ROUND_HALF_UP, Decimal
    return str(Decimal(repr(x)).quantize(Decimal(q), rounding=ROUND_HALF_UP))


def test_table5_values():
    rows = _rows()
    assert len(rows) == 4
    for n, full, pap, saving in rows:
        f_ = K.kv_cache_gib(int(n), skipping=False)
        p_ = K.kv_cache_gib(int(n))
        # the table rounds half up (4.125 -> 4.13, 6.625 -> 6.63)
        assert _half_up(f_, "0.01") == full
        assert _half_up(p_, "0.01") == pap
        assert _half_up(100 * (1 - p_ / f_), "0.1") == saving


@pytest.mark.parametrize("n", [1, 1000, 3000, 9216, 50000, 131072])
def test_matches_oracle_reading(n):
    assert K.kv_cache_gib(n) == pytest.approx(OA.kv_cache_gib(n), rel=1e-15)
    assert K.kv_cache_gib(n, skipping=False) == pytest.approx(OA.kv_cache_gib(n, with_pap=False), rel=1e-15)


def test_per_layer_structure():
    per = K.cached_tokens_per_layer(32768)
    assert len(per) == 32
    assert per[:10] == [32768] * 10
    assert per[10:14] == [9216] * 4 and per[14:19] == [7168] * 5
    assert per[19:24] == [4096] * 5 and per[24:29] == [2048] * 5 and per[29:] == [1024] * 3
    assert all(a >= b for a, b in zip(per[9:], per[10:]))       # nested candidate sets never grow
    short = K.cached_tokens_per_layer(500)
    assert short == [500] * 29 + [500] * 3


def test_custom_schedule():
    s = K.SkipSchedule(layers=8, first_skip=2, stage_ends=(3, 5), budgets=(100, 50), after_last=10,
                       kv_heads=8, head_dim=64, bytes_per_value=2)
    assert K.cached_tokens_per_layer(1000, s) == [1000, 1000, 100, 100, 50, 50, 10, 10]
    assert K.kv_cache_bytes([1] * 8, s) == 8 * 2 * 8 * 64 * 2
