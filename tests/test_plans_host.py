"""Host-side launch planning (no GPU): the attention plan's rules as the
library states them, read back through dflash_plan_attention_info."""

from __future__ import annotations

import itertools

import pytest

from block_diffusion_speculative_propose_b200.dflash import DFlashError, attention_plan


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
