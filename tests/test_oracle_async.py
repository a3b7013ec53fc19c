"""Pins of the oracle's proposal-input preparation with the async correction
(DFlash Speculative Decoding in the vLLM Neuron Framework, "Async Rejection
and Position Correction", "Paged KV Integration", "Draft Block
Construction").  CPU only."""

from __future__ import annotations

import json
import os

import numpy as np
import pytest

import oracle as O

HERE = os.path.dirname(__file__)


def _example():
    return json.load(open(os.path.join(HERE, "golden", "async_prep_example.json")))


def test_hand_worked_example():
    ex = _example()
    got = O.prepare_proposal_inputs(ex["target_positions"], ex["last_token_indices"],
                                    ex["cur_sampled"], ex["cur_num_draft"], ex["block_table"],
                                    ex["page_size"], ex["vocab"], ex["prev_sampled"],
                                    ex["prev_num_draft"])
    want = ex["expected"]
    for k in ("positions", "req_ids", "slot_mapping", "seq_lens", "bonus"):
        np.testing.assert_array_equal(getattr(got, k), want[k], err_msg=k)


def _random_case(rng, B, K, V, P=16, pad=2, with_prev=True):
    rows = rng.integers(1, K + 2, size=B)                 # target rows per request
    last = np.cumsum(rows) - 1
    n = int(rows.sum()) + pad
    base = rng.integers(0, 200, size=B)
    pos = np.zeros(n, dtype=np.int64)
    for b in range(B):
        s = last[b] - rows[b] + 1
        pos[s:last[b] + 1] = base[b] + 40 + np.arange(rows[b])
    W = (base.max() + 80) // P + 2
    table = rng.permutation(B * W).reshape(B, W)

    def sampled():
        s = rng.integers(0, V, size=(B, K + 1))
        acc = rng.integers(0, K + 1, size=B)
        for b in range(B):
            s[b, acc[b] + 1:] = -1
        return s
    prev = sampled() if with_prev else None
    return dict(target_positions=pos, last_token_indices=last, cur_sampled=sampled(),
                cur_num_draft=np.full(B, K), block_table=table, page_size=P, vocab=V,
                prev_sampled=prev, prev_num_draft=np.full(B, K) if with_prev else None)


def test_request_ids_follow_last_token_indices():
    rng = np.random.default_rng(0)
    for _ in range(20):
        c = _random_case(rng, B=int(rng.integers(1, 6)), K=int(rng.integers(1, 6)), V=40)
        got = O.prepare_proposal_inputs(**c)
        last = c["last_token_indices"]
        n = len(c["target_positions"])
        want = np.array([np.searchsorted(last, r, side="left") if r <= last[-1] else -1
                         for r in range(n)])
        np.testing.assert_array_equal(got.req_ids, want)
        assert (got.slot_mapping[got.req_ids < 0] == -1).all()


def test_no_previous_step_and_identity_tensors_are_no_ops():
    rng = np.random.default_rng(1)
    c = _random_case(rng, B=4, K=5, V=40, with_prev=False)
    a = O.prepare_proposal_inputs(**c)
    live = a.req_ids >= 0
    np.testing.assert_array_equal(a.positions[live], np.asarray(c["target_positions"])[live])
    # "no-op identity tensors": every previous output valid -> nothing rejected
    c2 = dict(c, prev_sampled=np.zeros((4, 6), dtype=np.int64), prev_num_draft=np.full(4, 5))
    b = O.prepare_proposal_inputs(**c2)
    for k in ("positions", "slot_mapping", "seq_lens", "bonus"):
        np.testing.assert_array_equal(getattr(a, k), getattr(b, k))


def test_correction_shifts_each_request_by_its_rejections():
    rng = np.random.default_rng(2)
    for _ in range(10):
        c = _random_case(rng, B=5, K=7, V=30)
        with_prev = O.prepare_proposal_inputs(**c)
        without = O.prepare_proposal_inputs(**dict(c, prev_sampled=None, prev_num_draft=None))
        prev = np.asarray(c["prev_sampled"])
        rejected = (1 + 7) - ((prev != -1) & (prev < 30)).sum(axis=1)
        live = with_prev.req_ids >= 0
        shift = without.positions[live] - with_prev.positions[live]
        np.testing.assert_array_equal(shift, rejected[with_prev.req_ids[live]])
        np.testing.assert_array_equal(without.seq_lens - with_prev.seq_lens, rejected)


def test_composes_with_greedy_verification():
    """Feeding the verifier's output back as the current step's sampler
    output: the post-verify length is the block start + tau (accepted drafts
    + bonus) and the bonus is the verifier's bonus."""
    rng = np.random.default_rng(3)
    B, K, V = 6, 5, 23
    drafts = rng.integers(0, V, size=(B, K))
    logits = rng.standard_normal((B, K + 1, V)).astype(np.float32)
    for b in range(B):
        n = int(rng.integers(0, K + 1))
        for j in range(n):
            logits[b, j, drafts[b, j]] = logits[b, j].max() + 1
    ver = O.verify_greedy(drafts, logits)
    starts = rng.integers(0, 100, size=B)
    rows = np.full(B, K + 1)
    last = np.cumsum(rows) - 1
    pos = np.concatenate([s + np.arange(K + 1) for s in starts])
    table = rng.permutation(B * 16).reshape(B, 16)
    got = O.prepare_proposal_inputs(pos, last, ver.out_tokens, np.full(B, K), table, 16, V)
    np.testing.assert_array_equal(got.seq_lens, starts + ver.num_accepted + 1)
    np.testing.assert_array_equal(got.bonus, ver.bonus)


def test_injecting_rejected_rows_changes_no_proposal():
    """The whole step injects all K+1 verified rows of a request, the rejected
    ones included; they sit at positions >= the post-verify length, which the
    next block covers, so the proposal equals the one made after injecting
    the accepted rows only (the plain reading: n + 1 rows at [seq_len,
    seq_len + n + 1))."""
    from block_diffusion_speculative_propose_b200 import synth
    cfg = synth.model_config("tiny")
    oc = O.OracleConfig.from_mapping(cfg)
    W = {k: ([x.float().numpy() for x in v] if isinstance(v, list) else v.float().numpy())
         for k, v in synth.make_weights(cfg, seed=4).items()}
    rng = np.random.default_rng(8)
    K, bs, P, V = cfg["block_size"] - 1, cfg["block_size"], cfg["page_size"], cfg["vocab"]
    ctx = [21, 50, 3]
    B = len(ctx)
    need = [-(-(c + 2 * bs + 1) // P) for c in ctx]
    table = np.zeros((B, max(need)), dtype=np.int64)
    perm = rng.permutation(sum(need))
    cur = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[cur:cur + n]
        cur += n
    pre_pos = np.concatenate([np.arange(c) for c in ctx]).astype(np.int64)
    pre_req = np.concatenate([np.full(c, b) for b, c in enumerate(ctx)]).astype(np.int64)
    pre_aux = rng.standard_normal((len(pre_pos), cfg["n_target_layers"] * cfg["hidden"]))
    drafts = rng.integers(0, V, size=(B, K))
    logits = rng.standard_normal((B, K + 1, V)).astype(np.float32)
    accept = [0, 2, K]
    for b in range(B):
        for j in range(K):
            if j < accept[b]:
                logits[b, j, drafts[b, j]] = logits[b, j].max() + 1
            else:
                logits[b, j, drafts[b, j]] = logits[b, j].min() - 1
    ver = O.verify_greedy(drafts, logits)
    aux = rng.standard_normal((B * (K + 1), cfg["n_target_layers"] * cfg["hidden"]))
    tpos = np.concatenate([c + np.arange(K + 1) for c in ctx]).astype(np.int64)
    last = (np.arange(1, B + 1) * (K + 1) - 1)
    nd = np.full(B, K)
    pi = O.prepare_proposal_inputs(tpos, last, ver.out_tokens, nd, table, P, V)

    def proposal(rows):
        kc, vc = O.empty_caches(oc, sum(need))
        O.inject_context(oc, W, pre_aux, pre_pos, O.paged_slots(pre_pos, pre_req, table, P),
                         kc, vc, "exact")
        O.inject_context(oc, W, aux[rows], pi.positions[rows], pi.slot_mapping[rows], kc, vc,
                         "exact")
        return O.propose(oc, W, pi.bonus, pi.seq_lens, table, kc, vc, "exact")

    every = proposal(np.arange(B * (K + 1)))
    kept = np.concatenate([b * (K + 1) + np.arange(int(ver.num_accepted[b]) + 1)
                           for b in range(B)])
    accepted_only = proposal(kept)
    np.testing.assert_array_equal(pi.seq_lens, np.asarray(ctx) + ver.num_accepted + 1)
    np.testing.assert_array_equal(every.draft_tokens, accepted_only.draft_tokens)
    np.testing.assert_array_equal(every.logits, accepted_only.logits)
