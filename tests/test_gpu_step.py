"""GPU parity of the whole speculative step (dflash_spec_step and its
library-owned CUDA graph) against the oracle's chain of the same four stages:
verify -> prepare proposal inputs (with the async correction) -> inject the
target rows -> propose.  Integer results (accepted tokens, corrected
positions, slots, lengths, bonus tokens) are bit-exact; drafts are bit-exact
outside near-ties (the band of test_gpu_propose).  The graph replays must give
the same bits as the eager call."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from block_diffusion_speculative_propose_b200 import DFlash, DFlashError, synth
from tests._util import to_np, weights_np, weights_to
from tests.test_gpu_propose import compare_drafts, max_excluded

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


class StepCase:
    """B requests with ctx_lens tokens already injected; this step verifies
    K drafts per request (the first accept[b] of them agree with the target's
    greedy picks) and injects the K+1 verified rows of each request."""

    def __init__(self, cfg, Wt, ctx_lens, accept, seed, prev_rejected=None):
        self.cfg = cfg
        self.oc = O.OracleConfig.from_mapping(cfg)
        self.Wn = weights_np(Wt)
        rng = np.random.default_rng(seed)
        P, bs, V = cfg["page_size"], cfg["block_size"], cfg["vocab"]
        K = bs - 1
        self.B = B = len(ctx_lens)
        self.K = K
        pre = np.zeros(B, dtype=np.int64) if prev_rejected is None else np.asarray(prev_rejected)
        # pages: the context, the verified rows at their optimistic positions
        # and the next block
        need = [-(-(c + int(pre[b]) + 2 * bs + 1) // P) for b, c in enumerate(ctx_lens)]
        self.W = max(need) + 1
        self.num_pages = sum(need) + 2
        perm = rng.permutation(self.num_pages)
        self.table = np.zeros((B, self.W), dtype=np.int32)
        cur = 0
        for b, n in enumerate(need):
            self.table[b, :n] = perm[cur:cur + n]
            cur += n
        # context already in the cache
        self.pre_pos = np.concatenate([np.arange(c) for c in ctx_lens] + [[]]).astype(np.int64)
        self.pre_req = np.concatenate([np.full(c, b) for b, c in enumerate(ctx_lens)]
                                      + [[]]).astype(np.int64)
        self.pre_slots = O.paged_slots(self.pre_pos, self.pre_req, self.table, P)
        self.pre_aux = synth.make_aux(len(self.pre_pos), cfg, seed + 1)
        # drafts under verification and the target's logits for them
        drafts = rng.integers(0, V, size=(B, K)).astype(np.int32)
        g = torch.Generator().manual_seed(seed + 2)
        logits = torch.randn(B, K + 1, V, generator=g).numpy().astype(np.float32)
        for b in range(B):
            for j in range(K + 1):
                if j < accept[b]:
                    logits[b, j, drafts[b, j]] = logits[b, j].max() + 1.0
                elif j < K:
                    logits[b, j, drafts[b, j]] = logits[b, j].min() - 1.0
        self.drafts, self.logits = drafts, logits
        # the K+1 verified rows of each request at their optimistic positions
        self.n = n = B * (K + 1)
        self.tpos = np.concatenate([c + pre[b] + np.arange(K + 1)
                                    for b, c in enumerate(ctx_lens)]).astype(np.int64)
        self.last = (np.arange(1, B + 1) * (K + 1) - 1).astype(np.int32)
        self.num_draft = np.full(B, K, dtype=np.int32)
        self.aux = synth.make_aux(n, cfg, seed + 3)
        if prev_rejected is None:
            self.prev_sampled = self.prev_num_draft = None
        else:
            ps = rng.integers(0, V, size=(B, K + 1)).astype(np.int32)
            for b in range(B):
                ps[b, K + 1 - int(pre[b]):] = -1
            self.prev_sampled, self.prev_num_draft = ps, np.full(B, K, dtype=np.int32)

    def gpu_inputs(self):
        t = lambda a: None if a is None else torch.tensor(a, device=DEV)  # noqa: E731
        return dict(prev_drafts=t(self.drafts), target_logits=t(self.logits),
                    target_positions=t(self.tpos), last_token_indices=t(self.last),
                    num_draft=t(self.num_draft), aux=self.aux.to(DEV),
                    block_table=t(self.table), prev_sampled=t(self.prev_sampled),
                    prev_num_draft=t(self.prev_num_draft))

    def gpu_caches(self, h):
        cfg = self.cfg
        shape = (self.num_pages, cfg["n_kv_heads"], cfg["page_size"], cfg["head_dim"])
        kc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV)
              for _ in range(cfg["n_layers"])]
        vc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV)
              for _ in range(cfg["n_layers"])]
        if len(self.pre_pos):
            h.inject_context(self.pre_aux.to(DEV), torch.tensor(self.pre_pos, device=DEV),
                             torch.tensor(self.pre_slots, device=DEV), kc, vc)
        return kc, vc

    def oracle(self, mode="device"):
        cfg, oc = self.cfg, self.oc
        kc, vc = O.empty_caches(oc, self.num_pages)
        if len(self.pre_pos):
            O.inject_context(oc, self.Wn, to_np(self.pre_aux).astype(np.float64), self.pre_pos,
                             self.pre_slots, kc, vc, mode)
        ver = O.verify_greedy(self.drafts, self.logits)
        pi = O.prepare_proposal_inputs(self.tpos, self.last, ver.out_tokens, self.num_draft,
                                       self.table, cfg["page_size"], cfg["vocab"],
                                       self.prev_sampled, self.prev_num_draft)
        O.inject_context(oc, self.Wn, to_np(self.aux).astype(np.float64), pi.positions,
                         pi.slot_mapping, kc, vc, mode)
        prop = O.propose(oc, self.Wn, pi.bonus, pi.seq_lens, self.table, kc, vc, mode)
        return ver, pi, prop


def check_step(case, out, ver, pi, prop):
    np.testing.assert_array_equal(to_np(out["out_tokens"]), ver.out_tokens)
    np.testing.assert_array_equal(to_np(out["num_accepted"]), ver.num_accepted)
    np.testing.assert_array_equal(to_np(out["positions"]), pi.positions)
    np.testing.assert_array_equal(to_np(out["slot_mapping"]), pi.slot_mapping)
    np.testing.assert_array_equal(to_np(out["seq_lens"]), pi.seq_lens)
    np.testing.assert_array_equal(to_np(out["bonus"]), pi.bonus)
    excluded = compare_drafts(to_np(out["draft_tokens"]), None, prop, None, case.K,
                              name=f"spec step chain B={case.B}")
    assert excluded <= max_excluded(case.B * case.K)
    blk = to_np(out["block_tokens"])
    np.testing.assert_array_equal(blk[:, 0], pi.bonus)
    np.testing.assert_array_equal(blk[:, 1:], to_np(out["draft_tokens"]))


@pytest.fixture(scope="module")
def tiny():
    cfg = synth.model_config("tiny")
    Wt = synth.make_weights(cfg, seed=0)
    h = DFlash(cfg, weights_to(Wt, DEV), max_position=4096)
    yield cfg, Wt, h
    h.close()


@pytest.mark.parametrize("ctx_lens,accept,prev_rejected", [
    ([37], [2], None),
    ([0, 5, 64, 130], [0, 3, 1, 2], None),
    ([16, 200, 9], [3, 0, 2], [0, 2, 3]),           # async correction of the positions
])
def test_tiny_spec_step_eager_and_graph(tiny, ctx_lens, accept, prev_rejected):
    cfg, Wt, h = tiny
    case = StepCase(cfg, Wt, ctx_lens, accept, seed=len(ctx_lens) * 7 + sum(accept),
                    prev_rejected=prev_rejected)
    ver, pi, prop = case.oracle()
    inp = case.gpu_inputs()
    kc, vc = case.gpu_caches(h)
    out = h.spec_step(k_cache=kc, v_cache=vc, **inp)
    torch.cuda.synchronize()
    assert h.check_device_errors() == 0
    check_step(case, out, ver, pi, prop)
    # the same step through the library's CUDA graph, replayed twice on fresh
    # caches: the same bits as the eager call
    kc2, vc2 = case.gpu_caches(h)
    g = h.step_graph(k_cache=kc2, v_cache=vc2, **inp)
    try:
        for _ in range(2):
            for t in g.out.values():
                t.fill_(-7)
            g.launch()
            torch.cuda.synchronize()
            for k in out:
                assert torch.equal(g.out[k], out[k]), k
        for a, b in zip(kc + vc, kc2 + vc2):
            assert torch.equal(a, b)
    finally:
        g.close()
    assert h.check_device_errors() == 0


def test_qwen3_heads_spec_step():
    """Qwen3-8B head layout and hidden size (one layer, 8192-token vocabulary
    so that the oracle stays quick), three requests."""
    cfg = dict(synth.model_config("qwen3_8b"), n_layers=1, vocab=8192, mask_token_id=8191)
    Wt = synth.make_weights(cfg, seed=0)
    h = DFlash(cfg, weights_to(Wt, DEV), max_position=8192)
    try:
        case = StepCase(cfg, Wt, [300, 41, 1200], [15, 4, 0], seed=5, prev_rejected=[1, 0, 9])
        ver, pi, prop = case.oracle()
        kc, vc = case.gpu_caches(h)
        g = h.step_graph(k_cache=kc, v_cache=vc, **case.gpu_inputs())
        try:
            g.launch()
            torch.cuda.synchronize()
            assert h.check_device_errors() == 0
            check_step(case, g.out, ver, pi, prop)
        finally:
            g.close()
    finally:
        h.close()


def test_spec_step_empty_batch_is_a_noop(tiny):
    """B == 0: nothing runs, eager or as a graph (whose launches do nothing)."""
    cfg, Wt, h = tiny
    z32 = torch.zeros(0, dtype=torch.int32, device=DEV)
    inp = dict(prev_drafts=torch.zeros(0, cfg["block_size"] - 1, dtype=torch.int32, device=DEV),
               target_logits=torch.zeros(0, cfg["block_size"], cfg["vocab"], device=DEV),
               target_positions=torch.zeros(0, dtype=torch.int64, device=DEV),
               last_token_indices=z32, num_draft=z32,
               aux=torch.zeros(0, cfg["n_target_layers"] * cfg["hidden"], dtype=torch.bfloat16,
                               device=DEV),
               block_table=torch.zeros(0, 4, dtype=torch.int32, device=DEV))
    shape = (4, cfg["n_kv_heads"], cfg["page_size"], cfg["head_dim"])
    kc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV) for _ in range(cfg["n_layers"])]
    vc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV) for _ in range(cfg["n_layers"])]
    before = h.launch_count()
    out = h.spec_step(k_cache=kc, v_cache=vc, workspace=torch.empty(256, dtype=torch.uint8,
                                                                     device=DEV), **inp)
    g = h.step_graph(k_cache=kc, v_cache=vc, **inp)
    try:
        g.launch()
        torch.cuda.synchronize()
    finally:
        g.close()
    assert h.launch_count() == before
    assert all(t.numel() == 0 for t in out.values())
    assert h.check_device_errors() == 0


def test_spec_step_host_errors(tiny):
    cfg, Wt, h = tiny
    case = StepCase(cfg, Wt, [20, 30], [1, 2], seed=3)
    inp = case.gpu_inputs()
    kc, vc = case.gpu_caches(h)
    # fewer target rows than requests
    bad = dict(inp, target_positions=inp["target_positions"][:1])
    with pytest.raises(DFlashError):
        h.spec_step(k_cache=kc, v_cache=vc, **bad)
    # previous sampler output without its draft counts
    bad = dict(inp, prev_sampled=torch.zeros(2, 4, dtype=torch.int32, device=DEV))
    with pytest.raises(DFlashError):
        h.spec_step(k_cache=kc, v_cache=vc, **bad)
    # too small a workspace
    with pytest.raises(DFlashError):
        h.spec_step(k_cache=kc, v_cache=vc,
                    workspace=torch.empty(256, dtype=torch.uint8, device=DEV), **inp)
    # no graph while launch profiling is on
    h.profile_enable(64)
    try:
        with pytest.raises(DFlashError):
            h.step_graph(k_cache=kc, v_cache=vc, **inp)
    finally:
        h.profile_disable()
    torch.cuda.synchronize()
    assert h.check_device_errors() == 0
