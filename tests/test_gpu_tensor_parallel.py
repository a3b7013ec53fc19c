"""GPU parity of the vocabulary-parallel LM head: handles that each hold one
shard of the LM head (dflash_create_vocab_shard) propose keys
(dflash_propose_keys); their element-wise maximum — on one GPU the stand-in
for the ranks' all-reduce MAX — decoded by dflash_finalize_draft_keys gives
the drafts of the whole-vocabulary handle and of the oracle (outside
near-ties), and each shard's logits are the matching columns of the whole
LM head's."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from block_diffusion_speculative_propose_b200 import (DFlash, DFlashError, finalize_draft_keys,
                                                      synth)
from block_diffusion_speculative_propose_b200.tensor_parallel import vocab_shards
from tests._util import rel_l2, to_np, weights_to
from tests.test_gpu_propose import Chain, compare_drafts, max_excluded

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def shard_weights(Wg, start, count):
    return dict(Wg, lm_head=Wg["lm_head"][start:start + count].contiguous())


def run_shards(cfg, Wt, ctx_lens, parts_list, seed):
    Wg = weights_to(Wt, DEV)
    h = DFlash(cfg, Wg, max_position=8192)
    try:
        ch = Chain(cfg, Wt, h, ctx_lens, seed=seed)
        d_full, lo_full, blk_full = ch.gpu()
        prop_io = ch.oracle("device")
        K = cfg["block_size"] - 1
        bonus = ch.bonus.to(DEV)
        seq = torch.tensor(ch.ctx_lens, device=DEV)
        table = torch.tensor(ch.table, device=DEV)
        for parts in parts_list:
            keys, logits = [], []
            for start, count in vocab_shards(cfg["vocab"], parts):
                hs = DFlash(cfg, shard_weights(Wg, start, count), max_position=8192,
                            vocab_shard=(start, count))
                try:
                    lo = torch.empty(ch.B * K, count, dtype=torch.float32, device=DEV)
                    keys.append(hs.propose_keys(bonus, seq, table, ch.kc, ch.vc, logits_out=lo))
                    logits.append(lo)
                    torch.cuda.synchronize()
                    assert hs.check_device_errors() == 0
                finally:
                    hs.close()
            kmax = torch.stack(keys).amax(dim=0)
            d, blk = finalize_draft_keys(kmax, bonus, cfg["block_size"], cfg["vocab"])
            torch.cuda.synchronize()
            lo_cat = to_np(torch.cat(logits, dim=1)).astype(np.float64)
            lo_ref = lo_full.astype(np.float64)
            assert rel_l2(lo_cat, lo_ref) < 1e-6
            # the same picks as the whole-vocabulary handle wherever the
            # shards' logits equal its own bit for bit, and as the oracle
            # outside near-ties
            same = np.all(to_np(torch.cat(logits, dim=1)) == lo_full, axis=1)
            gd, fd = to_np(d).reshape(-1), d_full.reshape(-1)
            assert np.array_equal(gd[same], fd[same])
            excluded = compare_drafts(to_np(d), to_np(torch.cat(logits, dim=1)), prop_io,
                                      ch.oracle("exact"), K, name=f"vocab-parallel chain x{parts}")
            assert excluded <= max_excluded(ch.B * K)
            assert np.array_equal(to_np(blk)[:, 0], to_np(ch.bonus))
            assert np.array_equal(to_np(blk)[:, 1:], to_np(d))
    finally:
        h.close()


def test_tiny_vocab_shards():
    cfg = synth.model_config("tiny")
    run_shards(cfg, synth.make_weights(cfg, seed=0), [40, 0, 131], [1, 2, 3, 4], seed=21)


def test_qwen3_heads_vocab_shards():
    cfg = dict(synth.model_config("qwen3_8b"), n_layers=1, vocab=8192, mask_token_id=8191)
    run_shards(cfg, synth.make_weights(cfg, seed=0), [300, 1000], [2, 8], seed=22)


def test_vocab_shard_host_errors():
    cfg = synth.model_config("tiny")
    Wg = weights_to(synth.make_weights(cfg, seed=0), DEV)
    with pytest.raises(DFlashError) as e:
        DFlash(cfg, shard_weights(Wg, 16, 32), vocab_shard=(16, 32))
    assert e.value.status == -4                      # not a multiple of 32
    for bad in ((0, 0), (-32, 64), (992, 64)):
        with pytest.raises(DFlashError) as e:
            DFlash(cfg, shard_weights(Wg, 0, 64), vocab_shard=bad)
        assert e.value.status == -1
    hs = DFlash(cfg, shard_weights(Wg, 32, 64), vocab_shard=(32, 64))
    try:
        ch = Chain(cfg, synth.make_weights(cfg, seed=0), hs, [20], seed=3)
        shape = (ch.num_pages, cfg["n_kv_heads"], cfg["page_size"], cfg["head_dim"])
        kc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV)
              for _ in range(cfg["n_layers"])]
        vc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV)
              for _ in range(cfg["n_layers"])]
        with pytest.raises(DFlashError) as e:      # a shard's argmax is not a draft
            hs.propose(ch.bonus.to(DEV), torch.tensor(ch.ctx_lens, device=DEV),
                       torch.tensor(ch.table, device=DEV), kc, vc)
        assert e.value.status == -1
        # a key that names no vocabulary entry decodes to -1 with the input bit
        err = torch.zeros(1, dtype=torch.int32, device=DEV)
        keys = torch.full((1, cfg["block_size"] - 1), -(2 ** 63), dtype=torch.int64, device=DEV)
        d, _ = finalize_draft_keys(keys, torch.tensor([5], dtype=torch.int32, device=DEV),
                                   cfg["block_size"], cfg["vocab"], device_error=err)
        torch.cuda.synchronize()
        assert (to_np(d) == -1).all() and int(err.item()) & 0x20
    finally:
        hs.close()
