"""Host-side launch planning (no GPU): the attention plan's rules as the
library states them, read back through dflash_plan_attention_info."""

from __future__ import annotations

import itertools

import pytest

from block_diffusion_speculative_propose_b200.dflash import DFlashError, attention_plan


def test_benchmark_workloads_plans():
    # batch 1, context 2048 (130 pages): 17 two-tile splits, two-deep ring, two CTAs per SM
    p = attention_plan(1, 8, 130, 16, 4)
    assert (p["tcgen05"], p["keys_per_tile"], p["ring_depth"], p["ctas_per_sm"]) == (1, 64, 2, 2)
    assert (p["chunk_keys"], p["max_splits"]) == (128, 17)
    # batch 32, contexts up to 8192 (514 pages): 56-tile splits on the six-deep ring
    p = attention_plan(32, 8, 514, 16, 4)
    assert (p["ring_depth"], p["ctas_per_sm"], p["chunk_keys"], p["max_splits"]) == (6, 1, 3584, 3)
    # eight query heads per kv head: 128 rows per kv group, the mma.sync kernel
    assert attention_plan(2, 4, 258, 16, 8)["tcgen05"] == 0


@pytest.mark.parametrize("B,W", list(itertools.product([1, 2, 4, 8, 32, 128], [5, 33, 130, 514, 2050])))
def test_attention_plan_rules(B, W):
    P, keys = 16, W * 16
    p = attention_plan(B, 8, W, 16, 4)
    assert p["tcgen05"] == 1 and p["keys_per_tile"] == 64 and p["cluster"] == 0
    c = p["chunk_keys"]
    assert c % 64 == 0 and 128 <= c <= 8192
    assert p["max_splits"] == -(-keys // c)
    # a split of at least 12 tiles keeps the six-deep ring busy; shorter ones
    # keep two CTAs per SM on the two-deep ring
    assert p["ring_depth"] == (6 if c // 64 >= 12 else 2)
    assert p["ctas_per_sm"] == (1 if p["ring_depth"] == 6 else 2)
    for forced in (2, 6):
        assert attention_plan(B, 8, W, 16, 4, forced_ring=forced)["ring_depth"] == forced
    # the persistent kernel only ever replaces the six-deep ring
    q = attention_plan(B, 8, W, 16, 4, persistent=True)
    assert q["persistent"] == (1 if p["ring_depth"] == 6 else 0)
    # the cluster combine (opt-in) only with few (request, kv head) pairs
    r = attention_plan(B, 8, W, 16, 4, cluster=True)
    if r["cluster"]:
        assert 2 * B * 8 <= 148 and r["keys_per_tile"] == 128 and 2 <= r["max_splits"] <= 8


def test_attention_plan_rejects_bad_sizes():
    with pytest.raises(DFlashError):
        attention_plan(0, 8, 130, 16, 4)
    with pytest.raises(DFlashError):
        attention_plan(1, 8, 0, 16, 4)
