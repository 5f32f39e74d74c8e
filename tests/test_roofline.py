"""Algorithmic work counts used by the benchmark's roofline (CPU)."""
import pytest

from block_sparse_attention_pisa_b200 import roofline as R


def test_video_attention_flops():
    # N=32768, H=24, d=128, b=64, k=64 of 512, order 1: 1.649 exact + 0.180 order-0 +
    # 11.545 order-1 TFLOP
    exact = 24 * 32768 * 4 * 64 * 128 * 64
    zero = 24 * 32768 * 4 * 128 * 448
    first = 24 * 32768 * 2 * 128 * 128 * 448
    assert R.attention_flops(1, 24, 32768, 128, 64, 64, 1) == pytest.approx(exact + zero + first)
    assert R.attention_flops(1, 24, 32768, 128, 64, 64, 1) / 1e12 == pytest.approx(13.37, abs=0.01)
    assert R.attention_flops(1, 24, 32768, 128, 64, 64, 0) == pytest.approx(exact + zero)


def test_all_selected_equals_dense():
    assert R.attention_flops(1, 16, 16384, 64, 128, 128, 1) == pytest.approx(R.dense_flops(1, 16, 16384, 64))


def test_stats_and_select_bytes():
    # K, V read (2 x 201 MB) + kbar, S0 (2 x 6.3 MB) + S1 (403 MB) = 818 MB
    assert R.stats_bytes(1, 24, 32768, 128, 64, 1) / 1e6 == pytest.approx(818.0, abs=1.0)
    assert R.select_bytes(1, 24, 32768, 128, 64, 64) / 1e6 == pytest.approx(211.0, abs=1.0)


def test_ragged_counts_real_tokens():
    # long workload: 75600 tokens in 591 blocks of <= 128
    f = R.attention_flops(1, 40, 75600, 128, 128, 60, 1)
    assert f / 1e12 == pytest.approx(65.33, abs=0.05)


def test_hybrid_and_drop_flops():
    # hybrid: exact + order-0 + one d x d product per query; keep-or-drop: exact only
    exact = 24 * 32768 * 4 * 64 * 128 * 64
    zero = 24 * 32768 * 4 * 128 * 448
    hbar = 24 * 32768 * 2 * 128 * 128
    assert R.attention_flops(1, 24, 32768, 128, 64, 64, 2) == pytest.approx(exact + zero + hbar)
    assert R.attention_flops(1, 24, 32768, 128, 64, 64, -1) == pytest.approx(exact)
    # nothing left to approximate: the hybrid term vanishes
    assert R.attention_flops(1, 16, 16384, 64, 128, 128, 2) == pytest.approx(R.dense_flops(1, 16, 16384, 64))


def test_routing_and_hybrid_bytes():
    # per-block S1 read twice (2 x 403 MB) + Hbar + M
    assert R.routing_bytes(1, 24, 32768, 128, 64) / 1e6 == pytest.approx(808.5, abs=1.0)
    # order 2 writes Hbar (64 KB per head) instead of per-block S1
    assert R.stats_bytes(1, 24, 32768, 128, 64, 2) / 1e6 == pytest.approx(416.8, abs=1.0)


def test_grouped_select_flops():
    # video: 512 query blocks, groups of 4 -> 128 proxies scored against 512 key blocks,
    # then 512 members against 128 candidates each: half the plain 512 x 512 scores
    plain = R.select_flops(1, 24, 32768, 128, 64)
    assert plain == pytest.approx(24 * 2 * 512 * 512 * 128)
    grouped = R.select_flops(1, 24, 32768, 128, 64, group=4, cand=128)
    assert grouped == pytest.approx(24 * 2 * 128 * (128 * 512 + 512 * 128))
    assert grouped == pytest.approx(plain / 2)
    # group 1 with every key block a candidate is plain selection
    assert R.select_flops(1, 24, 32768, 128, 64, group=1, cand=512) == pytest.approx(plain)
    # a ragged group count rounds up
    assert R.select_flops(1, 1, 64 * 10, 64, 64, group=4, cand=3) == pytest.approx(2 * 64 * (3 * 10 + 10 * 3))
