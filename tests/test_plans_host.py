"""Host-side launch planning (no GPU): the attention plan's rules as the
library states them, read back through dflash_plan_attention_info."""

from __future__ import annotations

import itertools

import pytest

from block_diffusion_speculative_propose_b200.dflash import DFlashError, attention_plan, gemm_plan


def test_benchmark_workloads_plans():
    # batch 1, context 2048 (130 pages): 17 128-key splits, two CTAs per SM,
    # 64-key tiles on a two-deep ring
    p = attention_plan(1, 8, 130, 16, 4)
    assert (p["tcgen05"], p["keys_per_tile"], p["ring_depth"], p["ctas_per_sm"]) == (1, 64, 2, 2)
    assert (p["chunk_keys"], p["max_splits"], p["transposed_pv"]) == (128, 17, 1)
    # batch 32, contexts up to 8192 (514 pages): 1792-key splits, sized for 8 CTAs per SM
    p = attention_plan(32, 8, 514, 16, 4)
    assert (p["ring_depth"], p["ctas_per_sm"], p["chunk_keys"], p["max_splits"]) == (2, 2, 1792, 5)
    assert p["transposed_pv"] == 1
    # 32-key tiles on a four-deep ring when asked for
    p = attention_plan(32, 8, 514, 16, 4, tile32=True)
    assert (p["keys_per_tile"], p["ring_depth"], p["ctas_per_sm"], p["chunk_keys"]) == (32, 4, 2, 1792)
    # the one-CTA-per-SM kernel when its six-deep ring is asked for
    p = attention_plan(32, 8, 514, 16, 4, forced_ring=6)
    assert (p["ring_depth"], p["ctas_per_sm"], p["chunk_keys"], p["transposed_pv"]) == (6, 1, 3584, 0)
    # eight query heads per kv head: 128 rows per kv group, the mma.sync kernel
    assert attention_plan(2, 4, 258, 16, 8)["tcgen05"] == 0
    # head_dim 64 keeps the M = 64 P V kernel
    assert attention_plan(2, 2, 258, 4, 2, head_dim=64)["transposed_pv"] == 0


def _chunk(B, W, parts):
    c = -(-(B * 8 * W * 16) // (parts * 148))
    c = -(-c // 64) * 64
    return max(128, min(8192, c))


@pytest.mark.parametrize("B,W", list(itertools.product([1, 2, 4, 8, 32, 128], [5, 33, 130, 514, 2050])))
def test_attention_plan_rules(B, W):
    keys = W * 16
    p = attention_plan(B, 8, W, 16, 4)
    assert p["tcgen05"] == 1 and p["keys_per_tile"] == 64 and p["cluster"] == 0
    # head_dim 128 by default: two CTAs per SM, 64-key tiles on a two-deep ring,
    # P V transposed, splits sized for eight CTAs per SM
    assert (p["transposed_pv"], p["ring_depth"], p["ctas_per_sm"]) == (1, 2, 2)
    c = p["chunk_keys"]
    assert c == _chunk(B, W, 8) and c % 64 == 0 and 128 <= c <= 8192
    assert p["max_splits"] == -(-keys // c)
    # a forced ring depth takes the one-kernel-per-tile variant with its own
    # split rule: a split of at least 12 tiles keeps the six-deep ring busy
    for forced in (2, 6):
        f = attention_plan(B, 8, W, 16, 4, forced_ring=forced)
        assert f["ring_depth"] == forced and f["transposed_pv"] == 0
        assert f["chunk_keys"] == _chunk(B, W, 4)
    # the persistent kernel (opt-in) only ever replaces the six-deep ring
    q = attention_plan(B, 8, W, 16, 4, persistent=True)
    assert q["transposed_pv"] == 0
    assert q["persistent"] == (1 if _chunk(B, W, 4) // 64 >= 12 else 0)
    # the cluster combine (opt-in) only with few (request, kv head) pairs
    r = attention_plan(B, 8, W, 16, 4, cluster=True)
    assert r["transposed_pv"] == 0
    if r["cluster"]:
        assert 2 * B * 8 <= 148 and r["keys_per_tile"] == 128 and 2 <= r["max_splits"] <= 8


def test_attention_plan_rejects_bad_sizes():
    with pytest.raises(DFlashError):
        attention_plan(0, 8, 130, 16, 4)
    with pytest.raises(DFlashError):
        attention_plan(1, 8, 0, 16, 4)


# ----------------------------------------------------------------------------
# GEMM plans (dflash_plan_gemm_info)
# ----------------------------------------------------------------------------
def test_gemm_plans_of_the_draft_step():
    # batch 128 (2048 block rows, 1920 LM-head rows): 256 x 256 CTA-pair tiles
    for M, N, K, g in ((2048, 6144, 4096, 128), (2048, 4096, 4096, 32), (2048, 24576, 4096, 32),
                       (2048, 4096, 12288, 32), (1920, 151936, 4096, 32)):
        p = gemm_plan(M, N, K, g)
        assert (p["pair"], p["tile_m"], p["tile_n"], p["k_splits"]) == (1, 256, 256, 1), (M, N, K)
    # batch 32 (512 rows): QKV wide pairs (48 tiles), O narrow pairs (64 tiles
    # of 256 x 128), down and fc with K split over two pairs (32 tiles -> 64 pairs)
    assert gemm_plan(512, 6144, 4096, 128)["tile_n"] == 256
    p = gemm_plan(512, 4096, 4096)
    assert (p["pair"], p["tile_n"], p["k_splits"], p["tiles"]) == (1, 128, 1, 64)
    for M, K in ((512, 12288), (282, 20480)):
        p = gemm_plan(M, 4096, K)
        assert (p["pair"], p["tile_n"], p["k_splits"], p["tiles"], p["grid"]) == (1, 256, 2, 32, 128)
    # no split when the split clusters cannot all run at once, or K is short
    assert gemm_plan(512, 4096, 12288, pair_split_cap=20)["k_splits"] == 1
    assert gemm_plan(512, 4096, 4096, pair_split_cap=37)["k_splits"] == 1
    # batch 1 (16 rows): the staged one-SM kernel; few tiles -> cluster split-K,
    # the LM head's 594 tiles -> stream-K
    p = gemm_plan(16, 4096, 12288)
    assert (p["pair"], p["staged"], p["k_splits"], p["grid"]) == (0, 1, 8, 128)
    p = gemm_plan(15, 151936, 4096)
    assert (p["pair"], p["staged"], p["stream_k"], p["grid"]) == (0, 1, 1, 148)


@pytest.mark.parametrize("M", [1, 16, 32, 33, 128, 129, 256, 300, 512, 768, 2048])
@pytest.mark.parametrize("N,K", [(1024, 1024), (4096, 4096), (6144, 4096), (4096, 12288),
                                 (24576, 4096), (151936, 4096)])
def test_gemm_plan_rules(M, N, K):
    for g in (32, 128):
        p = gemm_plan(M, N, K, g)
        assert p["tiles"] == -(-M // p["tile_m"]) * -(-N // p["tile_n"])
        if p["pair"]:
            # pairs only for several 128-row M tiles, never the staged epilogue
            assert M > 128 and not p["staged"] and not p["stream_k"]
            assert p["tile_m"] == 256 and p["tile_n"] in (128, 256) and p["tile_n"] % g == 0
            if p["k_splits"] == 2:
                assert p["tile_n"] == 256 and K // 64 >= 96 and p["tiles"] <= 37
                assert p["grid"] == 4 * p["tiles"]
            else:
                assert p["k_splits"] == 1 and p["grid"] <= 148 and p["grid"] % 2 == 0
        else:
            assert p["tile_m"] == 128 and p["grid"] <= 148
            assert p["staged"] == (1 if M <= 32 else 0)


def test_gemm_plan_rejects_bad_sizes():
    for args in ((0, 1024, 1024), (16, 0, 1024), (16, 1024, 100), (16, 1024, 1024, 48)):
        with pytest.raises(DFlashError):
            gemm_plan(*args)
