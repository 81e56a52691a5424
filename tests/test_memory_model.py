"""Batch-scaling memory model against the numbers the paper prints for it
(Sec. 4.3, Fig. 7; App. C.1).  The per-request cache bytes are closed form and
pinned; the per-request non-cache memory is fitted to the printed slopes, so the
batch limits and headroom are checked within a stated tolerance."""
import json
import os

import pytest

from mla_latent_kv_write_b200 import memory_model as M

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "cache_accounting.json")))


def test_cache_terms_match_the_printed_cache_sizes():
    dense = GOLD["dense_window"]
    assert M.dense_cache_gb() == pytest.approx(dense["gigabytes_bf16"], rel=0.01)          # App. C.1: ~6.0 GB
    assert M.dense_cache_gb() / M.latent_cache_gb(192) == pytest.approx(GOLD["per_token"]["reduction_factor"],
                                                                        rel=0.005)       # 13.7x
    # every printed slope exceeds its cache term (the rest is per-request non-cache memory)
    bs = GOLD["batch_scaling"]
    assert bs["dense_slope_gb_per_request"] > M.dense_cache_gb()
    lo, hi = bs["latent_slope_gb_per_request_range"]
    assert lo > M.latent_cache_gb(64) and hi > M.latent_cache_gb(512)


def test_batch_scaling_reproduces_the_printed_headroom():
    bs = GOLD["batch_scaling"]
    r = M.batch_scaling()
    assert r["dense"]["max_batch"] == bs["dense_oom_batch"] - 1                            # OOM at 28
    rows = r["latent"]
    assert rows[192]["headroom"] == pytest.approx(bs["headroom_default_d_c_192"], rel=0.05)  # 8.0x
    assert rows[64]["headroom"] == pytest.approx(bs["headroom_range"][1], rel=0.05)          # 11.4x
    assert rows[512]["headroom"] == pytest.approx(bs["headroom_range"][0], rel=0.05)         # 4.6x
    lo, hi = bs["slope_reduction_percent_range"]
    assert 100 * rows[512]["slope_reduction"] == pytest.approx(lo, abs=1.0)                 # 77 %
    assert 100 * rows[64]["slope_reduction"] == pytest.approx(hi, abs=1.0)                  # 91 %
    # monotone: a smaller latent always allows a larger batch
    b = [rows[dc]["max_batch"] for dc in (64, 128, 192, 256, 512)]
    assert b == sorted(b, reverse=True)


def test_known_deviation_at_d_c_64():
    """The pages keep d_c = 64 within budget at batch 320; the fitted linear
    model puts its limit ~4 % lower.  Recorded, not hidden."""
    r = M.batch_scaling()
    assert 0.9 * GOLD["batch_scaling"]["d_c_64_within_budget_at_batch"] <= r["latent"][64]["max_batch"] < 320
