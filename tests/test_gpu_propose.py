"""GPU parity of the whole proposal (inject -> propose) against the oracle.

Why drafts are compared only outside near-ties: every storage rounding point
(fp16 / bf16 activations) turns a relative perturbation delta of its input
into flipped roundings on about delta / ulp of its outputs, i.e. a relative
change of about sqrt(delta * ulp).  After a few such points any two
implementations whose fp32 arithmetic differs at all (summation order, fused
multiply-adds) sit about one ulp apart — the oracle itself moves its logits by
~5e-4 relative L2 when its K/V input is perturbed by 1e-7.  So greedy picks are
bit-exact against the oracle's ``device`` storage-precision mode in every row
whose top-2 logit gap exceeds the noise of that row: 4 * sqrt(2) times the
row's measured rms logit difference (GPU vs that oracle; capped at 1e-2 of the
row's rms), and never less than 1e-3.  Rows inside the noise are counted and
reported, not compared; the LM-head logits must be within relative L2 1e-2 of
the oracle's exact (float64) mode.  The GPU chain and the oracle chain each
inject the same context with their own code; nothing flows from one to the
other.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from block_diffusion_speculative_propose_b200 import DFlash, DFlashError, synth
from tests._util import rel_l2, to_np, weights_np, weights_to

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
GAP_FLOOR = 1e-3
GAP_SIGMAS = 4.0 * np.sqrt(2.0)


def near_tie_gap(gpu_logits, oracle_logits):
    """Per-row top-2 gap below which a greedy pick is inside the logit noise."""
    if gpu_logits is None:
        rms = np.sqrt(np.mean(np.square(oracle_logits), axis=1))
        return np.maximum(GAP_FLOOR, GAP_SIGMAS * 5e-3 * rms)
    d = np.asarray(gpu_logits, dtype=np.float64) - oracle_logits
    sigma = np.sqrt(np.mean(d * d, axis=1))
    rms = np.sqrt(np.mean(np.square(oracle_logits), axis=1))
    return np.maximum(GAP_FLOOR, GAP_SIGMAS * np.minimum(sigma, 1e-2 * rms))


def max_excluded(rows):
    """Bound on rows inside the noise band.  With random-init weights the gap
    between the two largest of V Gaussian logits averages about
    rms / sqrt(2 ln V) (~0.2 rms for V = 152k), while the band reaches up to
    4 * sqrt(2) * 5e-3 rms (~0.03 rms), so ~15% of rows fall inside it; a third
    of the rows (at least 2) is the bound, so that a kernel with large errors
    cannot hide most rows behind a wide band."""
    return max(2, rows // 3)


def compare_drafts(gpu_drafts, gpu_logits, prop_io, prop_ex, K):
    """Bit-exact drafts outside near-ties; logits within 1e-2 rel-L2 of exact."""
    gd = np.asarray(gpu_drafts).reshape(-1)
    od = prop_io.draft_tokens.reshape(-1)
    gap = O.top2_gap_f32(prop_io.logits)
    ok = gap >= near_tie_gap(gpu_logits, prop_io.logits)
    mism = np.nonzero((gd != od) & ok)[0]
    assert mism.size == 0, f"draft mismatch at rows {mism[:10]} gaps {gap[mism[:10]]}"
    if gpu_logits is not None:
        gl = np.asarray(gpu_logits, dtype=np.float64)
        ex = [rel_l2(gl[r], prop_ex.logits[r]) for r in range(gl.shape[0])]
        dv = [rel_l2(gl[r], prop_io.logits[r]) for r in range(gl.shape[0])]
        print(f"logits rel-L2 vs exact: max {max(ex):.3e} mean {np.mean(ex):.3e}; "
              f"vs device-precision oracle: max {max(dv):.3e}; near-ties excluded "
              f"{int((~ok).sum())} of {ok.size}")
        for r in range(gl.shape[0]):
            assert ex[r] < 1e-2, r
    return int((~ok).sum())


class Chain:
    """Context for B requests injected on both sides, then one proposal."""

    def __init__(self, cfg, Wt, h, ctx_lens, seed, table_extra=1):
        self.cfg, self.h = cfg, h
        self.oc = O.OracleConfig.from_mapping(cfg)
        P, bs = cfg["page_size"], cfg["block_size"]
        rng = np.random.default_rng(seed)
        self.B = B = len(ctx_lens)
        need = [-(-(c + bs) // P) for c in ctx_lens]
        self.W = max(need) + table_extra
        self.num_pages = sum(need) + 3
        perm = rng.permutation(self.num_pages)
        self.table = np.zeros((B, self.W), dtype=np.int32)
        cur = 0
        for b, n in enumerate(need):
            self.table[b, :n] = perm[cur:cur + n]
            cur += n
        self.pos = np.concatenate([np.arange(c) for c in ctx_lens]).astype(np.int64)
        self.req = np.concatenate([np.full(c, b) for b, c in enumerate(ctx_lens)]).astype(np.int64)
        self.slots = O.paged_slots(self.pos, self.req, self.table, P)
        self.aux = synth.make_aux(len(self.pos), cfg, seed)
        self.ctx_lens = np.asarray(ctx_lens, dtype=np.int32)
        g = torch.Generator().manual_seed(seed)
        t = torch.randint(0, cfg["vocab"] - 1, (B,), generator=g)
        self.bonus = torch.where(t >= cfg["mask_token_id"], t + 1, t).to(torch.int32)
        self.Wn = weights_np(Wt)

    def gpu(self, logits=True):
        cfg, h = self.cfg, self.h
        shape = (self.num_pages, cfg["n_kv_heads"], cfg["page_size"], cfg["head_dim"])
        self.kc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV) for _ in range(cfg["n_layers"])]
        self.vc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV) for _ in range(cfg["n_layers"])]
        if len(self.pos):
            h.inject_context(self.aux.to(DEV), torch.tensor(self.pos, device=DEV),
                             torch.tensor(self.slots, device=DEV), self.kc, self.vc)
        K = cfg["block_size"] - 1
        lo = torch.empty(self.B * K, cfg["vocab"], dtype=torch.float32, device=DEV) if logits else None
        blk = torch.empty(self.B, cfg["block_size"], dtype=torch.int32, device=DEV)
        d = h.propose(self.bonus.to(DEV), torch.tensor(self.ctx_lens, device=DEV),
                      torch.tensor(self.table, device=DEV), self.kc, self.vc,
                      block_tokens=blk, logits_out=lo)
        torch.cuda.synchronize()
        assert h.check_device_errors() == 0
        return to_np(d), (to_np(lo) if logits else None), to_np(blk)

    def oracle(self, mode):
        kc, vc = O.empty_caches(self.oc, self.num_pages)
        if len(self.pos):
            O.inject_context(self.oc, self.Wn, to_np(self.aux).astype(np.float64), self.pos,
                             self.slots, kc, vc, mode)
        return O.propose(self.oc, self.Wn, to_np(self.bonus), self.ctx_lens, self.table, kc, vc,
                         mode)


@pytest.fixture(scope="module")
def tiny():
    cfg = synth.model_config("tiny")
    Wt = synth.make_weights(cfg, seed=0)
    h = DFlash(cfg, weights_to(Wt, DEV), max_position=4096)
    yield cfg, Wt, h
    h.close()


@pytest.mark.parametrize("ctx_lens", [[64], [0, 1, 15, 16, 17, 100], [333] * 3])
def test_tiny_chain(tiny, ctx_lens):
    cfg, Wt, h = tiny
    ch = Chain(cfg, Wt, h, ctx_lens, seed=sum(ctx_lens) + len(ctx_lens))
    d, lo, blk = ch.gpu()
    p_io, p_ex = ch.oracle("device"), ch.oracle("exact")
    K = cfg["block_size"] - 1
    excluded = compare_drafts(d, lo, p_io, p_ex, K)
    assert excluded <= max_excluded(len(ctx_lens) * K)
    np.testing.assert_array_equal(blk[:, 0], to_np(ch.bonus))
    np.testing.assert_array_equal(blk[:, 1:], d)


def test_propose_is_deterministic(tiny):
    cfg, Wt, h = tiny
    ch = Chain(cfg, Wt, h, [50, 70], seed=3)
    a = ch.gpu()
    b = ch.gpu()
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_empty_calls_are_noops(tiny):
    cfg, Wt, h = tiny
    shape = (4, cfg["n_kv_heads"], 16, cfg["head_dim"])
    kc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV) for _ in range(cfg["n_layers"])]
    h.inject_context(torch.zeros(0, 768, dtype=torch.bfloat16, device=DEV),
                     torch.zeros(0, dtype=torch.int64, device=DEV),
                     torch.zeros(0, dtype=torch.int64, device=DEV), kc, kc)
    d = h.propose(torch.zeros(0, dtype=torch.int32, device=DEV),
                  torch.zeros(0, dtype=torch.int32, device=DEV),
                  torch.zeros(0, 4, dtype=torch.int32, device=DEV), kc, kc)
    torch.cuda.synchronize()
    assert d.shape == (0, cfg["block_size"] - 1)
    assert all(int(t.abs().sum()) == 0 for t in kc)


def test_device_bounds_are_flagged_not_faulted(tiny):
    """Out-of-range inputs that only the device can see set error bits and
    skip the access; the context stays usable."""
    cfg, Wt, h = tiny
    shape = (4, cfg["n_kv_heads"], 16, cfg["head_dim"])
    kc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV) for _ in range(cfg["n_layers"])]
    vc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV) for _ in range(cfg["n_layers"])]
    table = torch.tensor([[0, 1]], dtype=torch.int32, device=DEV)
    # seq_len 40 + bs 4 needs 3 pages, the table has 2
    h.propose(torch.tensor([5], dtype=torch.int32, device=DEV),
              torch.tensor([40], dtype=torch.int32, device=DEV), table, kc, vc)
    bits = h.check_device_errors()
    assert bits & 4                      # DFLASH_DEVERR_TABLE
    # page id outside the pool
    h.propose(torch.tensor([5], dtype=torch.int32, device=DEV),
              torch.tensor([3], dtype=torch.int32, device=DEV),
              torch.tensor([[9, 1]], dtype=torch.int32, device=DEV), kc, vc)
    assert h.check_device_errors() & 2   # DFLASH_DEVERR_SLOT
    # bonus token outside the vocabulary
    h.propose(torch.tensor([cfg["vocab"] + 5], dtype=torch.int32, device=DEV),
              torch.tensor([3], dtype=torch.int32, device=DEV), table, kc, vc)
    assert h.check_device_errors() & 8   # DFLASH_DEVERR_TOKEN
    # inject slot outside the pool
    h.inject_context(synth.make_aux(2, cfg, 0).to(DEV),
                     torch.tensor([0, 1], device=DEV), torch.tensor([3, 4 * 16], device=DEV),
                     kc, vc)
    assert h.check_device_errors() & 2
    # and a clean call afterwards is clean
    h.propose(torch.tensor([5], dtype=torch.int32, device=DEV),
              torch.tensor([3], dtype=torch.int32, device=DEV), table, kc, vc)
    assert h.check_device_errors() == 0


def test_host_argument_errors(tiny):
    cfg, Wt, h = tiny
    shape = (4, cfg["n_kv_heads"], 16, cfg["head_dim"])
    kc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV) for _ in range(cfg["n_layers"])]
    small_ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    with pytest.raises(DFlashError) as e:
        h.propose(torch.tensor([5], dtype=torch.int32, device=DEV),
                  torch.tensor([3], dtype=torch.int32, device=DEV),
                  torch.tensor([[0, 1]], dtype=torch.int32, device=DEV), kc, kc,
                  workspace=small_ws)
    assert e.value.status == -3
    with pytest.raises(DFlashError) as e:
        h.linear(torch.zeros(4, 100, dtype=torch.bfloat16, device=DEV),
                 torch.zeros(32, 100, dtype=torch.bfloat16, device=DEV))
    assert e.value.status == -4


# ----------------------------------------------------------------------------
# Qwen3-8B-shaped draft, batch 1, context 2048 (one full step)
# ----------------------------------------------------------------------------
def test_qwen3_b1_step():
    cfg = synth.model_config("qwen3_8b")
    Wt = synth.make_weights(cfg, seed=0)
    h = DFlash(cfg, weights_to(Wt, DEV), max_position=40960)
    try:
        oc = O.OracleConfig.from_mapping(cfg)
        sb = synth.make_step_batch(cfg, 1, 2048, 2048, accept="uniform", seed=7,
                                   with_logits=False)
        P = 16
        shape = (sb.num_pages, cfg["n_kv_heads"], P, cfg["head_dim"])
        # context already in the cache: seeded N(0,1) values on both sides
        kc = [torch.empty(shape, dtype=torch.bfloat16) for _ in range(cfg["n_layers"])]
        vc = [torch.empty(shape, dtype=torch.bfloat16) for _ in range(cfg["n_layers"])]
        synth.fill_cache_random(kc + vc, seed=11)
        slots = O.paged_slots(to_np(sb.inject_positions), to_np(sb.inject_req_ids),
                              to_np(sb.block_table), P)
        kg = [t.to(DEV) for t in kc]
        vg = [t.to(DEV) for t in vc]
        h.inject_context(sb.aux.to(DEV), sb.inject_positions.to(DEV),
                         torch.tensor(slots, device=DEV), kg, vg)
        K = cfg["block_size"] - 1
        lo = torch.empty(K, cfg["vocab"], dtype=torch.float32, device=DEV)
        d = h.propose(sb.bonus.to(DEV), sb.seq_lens.to(DEV), sb.block_table.to(DEV), kg, vg,
                      logits_out=lo)
        torch.cuda.synchronize()
        assert h.check_device_errors() == 0
        Wn = weights_np(Wt)
        res = {}
        for mode in ("device", "exact"):
            ko = [to_np(t).astype(np.float64) for t in kc]
            vo = [to_np(t).astype(np.float64) for t in vc]
            O.inject_context(oc, Wn, to_np(sb.aux).astype(np.float64),
                             to_np(sb.inject_positions), slots, ko, vo, mode)
            res[mode] = O.propose(oc, Wn, to_np(sb.bonus), to_np(sb.seq_lens),
                                  to_np(sb.block_table), ko, vo, mode)
        excluded = compare_drafts(to_np(d), to_np(lo), res["device"], res["exact"], K)
        assert excluded <= max_excluded(K)
    finally:
        h.close()


def test_chain_launch_matches_oracle(monkeypatch):
    """The opt-in schedules — one-launch gate/up + down (few rows) and
    cluster-combined attention splits — give the same drafts as the oracle
    outside near-ties, like the default schedule."""
    monkeypatch.setenv("DFLASH_CHAIN", "1")
    monkeypatch.setenv("DFLASH_ATTN_CLUSTER", "1")
    cfg = dict(synth.model_config("qwen3_8b"), n_layers=1, vocab=8192, mask_token_id=8191)
    Wt = synth.make_weights(cfg, seed=0)
    h = DFlash(cfg, weights_to(Wt, DEV), max_position=4096)
    try:
        for ctx in ([700], [300, 1300]):
            ch = Chain(cfg, Wt, h, ctx, seed=11 + len(ctx))
            h.profile_enable(1024)
            d, lo, blk = ch.gpu()
            prof = h.profile_read()
            h.profile_disable()
            assert prof.get("gemm_mlp", (0, 0.0))[0] == cfg["n_layers"]   # the chain ran
            assert prof.get("gemm_gate_up", (0, 0.0))[0] == 0
            K = cfg["block_size"] - 1
            excluded = compare_drafts(d, lo, ch.oracle("device"), ch.oracle("exact"), K)
            assert excluded <= max_excluded(len(ctx) * K)
    finally:
        h.close()
