"""Pins of the oracle's tensor-parallel proposal (kv heads, their query heads
and the MLP features split over ranks, row-parallel O and down projections
summed across ranks, vocabulary-split LM head): it must equal the
single-rank oracle — the same drafts, logits and context caches up to float64
summation order — which is itself pinned in test_oracle_pins.py.  CPU only."""

from __future__ import annotations

import numpy as np
import pytest

import oracle as O
from block_diffusion_speculative_propose_b200 import synth


def _weights(cfg, seed):
    return {k: ([x.float().numpy().astype(np.float64) for x in v] if isinstance(v, list)
                else v.float().numpy().astype(np.float64))
            for k, v in synth.make_weights(cfg, seed=seed).items()}


def _case(cfg, ctx_lens, seed):
    rng = np.random.default_rng(seed)
    P, bs = cfg["page_size"], cfg["block_size"]
    need = [-(-(c + bs) // P) for c in ctx_lens]
    num_pages = sum(need) + 1
    table = np.zeros((len(ctx_lens), max(need)), dtype=np.int64)
    perm = rng.permutation(num_pages)
    cur = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[cur:cur + n]
        cur += n
    pos = np.concatenate([np.arange(c) for c in ctx_lens]).astype(np.int64)
    req = np.concatenate([np.full(c, b) for b, c in enumerate(ctx_lens)]).astype(np.int64)
    slots = O.paged_slots(pos, req, table, P)
    aux = rng.standard_normal((len(pos), cfg["n_target_layers"] * cfg["hidden"]))
    bonus = rng.integers(0, cfg["mask_token_id"], size=len(ctx_lens))
    return table, num_pages, pos, slots, aux, bonus


def _shards(vocab, parts):
    groups = vocab // 32
    out, start = [], 0
    for r in range(parts):
        g = groups // parts + (1 if r < groups % parts else 0)
        out.append((start * 32, g * 32))
        start += g
    return out


CFG_GQA = dict(hidden=256, n_layers=2, n_q_heads=8, n_kv_heads=4, head_dim=32,
               intermediate=384, vocab=512, n_target_layers=2, block_size=4,
               mask_token_id=511, page_size=16, rms_eps=1e-6, rope_theta=1e6)


@pytest.mark.parametrize("cfg,sizes", [
    (synth.model_config("tiny"), [1, 2]),
    (CFG_GQA, [2, 4]),
])
def test_tensor_parallel_proposal_equals_single_rank(cfg, sizes):
    oc = O.OracleConfig.from_mapping(cfg)
    W = _weights(cfg, seed=3)
    ctx = [0, 37, 70]
    table, num_pages, pos, slots, aux, bonus = _case(cfg, ctx, seed=5)
    kc, vc = O.empty_caches(oc, num_pages)
    O.inject_context(oc, W, aux, pos, slots, kc, vc, "exact")
    ref = O.propose(oc, W, bonus, ctx, table, kc, vc, "exact")
    for size in sizes:
        kr, vr = O.empty_caches_tp(oc, num_pages, size)
        O.inject_context_tp(oc, W, aux, pos, slots, kr, vr, size)
        got = O.propose_tp(oc, W, bonus, ctx, table, kr, vr, size,
                           _shards(cfg["vocab"], size + 1))
        np.testing.assert_array_equal(got.draft_tokens, ref.draft_tokens)
        np.testing.assert_array_equal(got.block_tokens, ref.block_tokens)
        assert np.max(np.abs(got.logits - ref.logits)) <= 1e-12 * np.max(np.abs(ref.logits))
        # the ranks' caches hold the single-rank caches' heads, in rank order
        # (context and the block's own K/V)
        for l in range(oc.n_layers):
            np.testing.assert_allclose(np.concatenate([kr[r][l] for r in range(size)], axis=1),
                                       kc[l], rtol=0, atol=1e-12)
            np.testing.assert_allclose(np.concatenate([vr[r][l] for r in range(size)], axis=1),
                                       vc[l], rtol=0, atol=1e-12)


def test_tp_slices_partition_heads_and_features():
    oc = O.OracleConfig.from_mapping(CFG_GQA)
    for size in (1, 2, 4):
        sl = [O.tp_slices(oc, r, size) for r in range(size)]
        assert [s.kv_heads.start for s in sl] == [r * 4 // size for r in range(size)]
        assert sl[-1].kv_heads.stop == 4 and sl[-1].q_heads.stop == 8
        assert sl[-1].features.stop == 384
        for s in sl:      # each kv head keeps its own query group (G = 2)
            assert s.q_heads.start == 2 * s.kv_heads.start
            assert s.q_heads.stop == 2 * s.kv_heads.stop
    with pytest.raises(ValueError):
        O.tp_slices(oc, 0, 3)          # 4 kv heads over 3 ranks
    with pytest.raises(ValueError):
        O.tp_slices(oc, 2, 2)
