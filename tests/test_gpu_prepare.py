"""GPU parity of dflash_prepare_proposal_inputs (proposal inputs with the
async rejection correction) against the oracle: bit-exact, integer work.
Also the composed device step verify -> prepare with no host round trip."""

from __future__ import annotations

import json
import os

import numpy as np
import pytest
import torch

import oracle as O
from block_diffusion_speculative_propose_b200 import (prepare_proposal_inputs, synth,
                                                      verify_greedy)
from tests._util import to_np
from tests.test_oracle_async import _random_case

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
HERE = os.path.dirname(__file__)


def _dev(a, dtype):
    return torch.tensor(np.asarray(a), dtype=dtype, device=DEV)


def _run(c, err=None):
    prev = c.get("prev_sampled")
    return prepare_proposal_inputs(
        _dev(c["target_positions"], torch.int64), _dev(c["last_token_indices"], torch.int32),
        _dev(c["cur_sampled"], torch.int32), _dev(c["cur_num_draft"], torch.int32),
        _dev(c["block_table"], torch.int32), c["page_size"], c["vocab"],
        None if prev is None else _dev(prev, torch.int32),
        None if prev is None else _dev(c["prev_num_draft"], torch.int32), device_error=err)


def _check(c):
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pos, slots, seq, bonus = _run(c, err)
    torch.cuda.synchronize()
    ref = O.prepare_proposal_inputs(**c)
    np.testing.assert_array_equal(to_np(pos), ref.positions)
    np.testing.assert_array_equal(to_np(slots), ref.slot_mapping)
    np.testing.assert_array_equal(to_np(seq), ref.seq_lens)
    np.testing.assert_array_equal(to_np(bonus), ref.bonus)
    return int(err.item())


def test_hand_worked_example():
    ex = json.load(open(os.path.join(HERE, "golden", "async_prep_example.json")))
    c = {k: ex[k] for k in ("target_positions", "last_token_indices", "cur_sampled",
                            "cur_num_draft", "block_table", "page_size", "vocab",
                            "prev_sampled", "prev_num_draft")}
    assert _check(c) == 0


@pytest.mark.parametrize("B,K,V,with_prev", [(1, 15, 151936, True), (7, 3, 50, True),
                                             (33, 9, 1000, False), (128, 15, 151936, True),
                                             (300, 5, 77, True)])
def test_random_cases(B, K, V, with_prev):
    rng = np.random.default_rng(B * 31 + K)
    for _ in range(3):
        c = _random_case(rng, B=B, K=K, V=V, with_prev=with_prev)
        assert _check(c) == 0


def test_padding_only_and_empty():
    rng = np.random.default_rng(5)
    c = _random_case(rng, B=3, K=4, V=30)
    # no requests: every row is padding
    c0 = dict(c, last_token_indices=np.zeros(0, dtype=np.int64),
              cur_sampled=np.zeros((0, 5), dtype=np.int64), cur_num_draft=np.zeros(0),
              prev_sampled=np.zeros((0, 5), dtype=np.int64), prev_num_draft=np.zeros(0))
    assert _check(c0) == 0


def test_malformed_inputs_set_the_error_bit():
    rng = np.random.default_rng(6)
    c = _random_case(rng, B=4, K=4, V=30)
    bad = dict(c, cur_sampled=np.full((4, 5), -1))        # no valid sampler output
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    _, _, _, bonus = _run(bad, err)
    torch.cuda.synchronize()
    assert int(err.item()) & 0x20 and (to_np(bonus) == -1).all()
    last = np.asarray(c["last_token_indices"]).copy()
    last[2] = last[1]                                      # not strictly increasing
    err.zero_()
    _run(dict(c, last_token_indices=last), err)
    torch.cuda.synchronize()
    assert int(err.item()) & 0x20


def test_verify_then_prepare_on_device():
    """The speculative step's bookkeeping without leaving the device: greedy
    verification of the C5-shaped batch feeds the preparation directly."""
    cfg = synth.model_config("qwen3_8b")
    wl = synth.WORKLOADS["qwen3_b128_ctx8192_32768"]
    B, K, V = wl["batch"], cfg["block_size"] - 1, cfg["vocab"]
    sb = synth.make_step_batch(cfg, B, wl["ctx_lo"], wl["ctx_hi"], accept=wl["accept"], seed=3)
    drafts = sb.prev_drafts.to(DEV)
    logits = sb.target_logits.to(DEV)
    out, n_acc, bonus_v = verify_greedy(drafts, logits)
    starts = to_np(sb.seq_lens).astype(np.int64)
    pos = np.concatenate([s + np.arange(K + 1) for s in starts])   # the step's K+1 target rows
    last = (np.arange(B) + 1) * (K + 1) - 1
    table = to_np(sb.block_table)
    cur_nd = torch.full((B,), K, dtype=torch.int32, device=DEV)
    p, slots, seq, bonus = prepare_proposal_inputs(
        _dev(pos, torch.int64), _dev(last, torch.int32), out, cur_nd,
        _dev(table, torch.int32), 16, V)
    torch.cuda.synchronize()
    ver = O.verify_greedy(to_np(sb.prev_drafts), to_np(sb.target_logits))
    ref = O.prepare_proposal_inputs(pos, last, ver.out_tokens, np.full(B, K), table, 16, V)
    np.testing.assert_array_equal(to_np(seq), ref.seq_lens)
    np.testing.assert_array_equal(to_np(seq), starts + ver.num_accepted + 1)
    np.testing.assert_array_equal(to_np(bonus), ver.bonus)
    np.testing.assert_array_equal(to_np(slots), ref.slot_mapping)
