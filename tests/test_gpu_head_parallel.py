"""GPU parity of the head-parallel (tensor-parallel) draft layers on one GPU.

Each of S shard handles (dflash_create_tp_shard) holds one rank's kv heads with
their query groups, its MLP features, the matching columns of Wo and W_down
and its vocabulary rows of the LM head ("DFlash Speculative Decoding in the
vLLM Neuron Framework", §Context KV Injection: "this rank's KV heads only";
§DFlashQwen3ForCausalLM: a column-parallel LM head).  The ranks run as host
threads of this process, each on its own stream, calling dflash_propose_tp;
their exchange hook is the all-reduce SUM of the row-parallel O / down partial
sums: every rank synchronizes its stream, waits on a host barrier until all
ranks have reached the same exchange point, and sums the partials (kernels of
different ranks never wait on one another; only the host threads do).  The
vocabulary keys are then combined by their element-wise maximum, the stand-in
for the all-reduce MAX.  Drafts must match the single-rank oracle (the
tensor-parallel oracle is pinned equal to it) under the whole-chain rules of
test_gpu_propose; each rank's injected K/V must be its heads' slice of the
whole-model handle's.
"""

from __future__ import annotations

import threading

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


class LockstepExchange:
    """All-reduce SUM among `size` rank threads sharing one GPU."""

    def __init__(self, size, workspaces, streams):
        self.size, self.ws, self.streams = size, workspaces, streams
        self.bar = threading.Barrier(size, timeout=120)
        self.views = [None] * size
        self.calls = [0] * size

    def hook(self, r):
        def f(data, count, _stream=None):
            s = self.streams[r]
            s.synchronize()                          # this rank's partials are complete
            off = data - self.ws[r].data_ptr()
            self.views[r] = self.ws[r][off:off + 4 * count].view(torch.float32)
            self.calls[r] += 1
            self.bar.wait()                          # every rank's partials are complete
            with torch.cuda.stream(s):
                total = self.views[0].clone()
                for j in range(1, self.size):
                    total += self.views[j]
            s.synchronize()
            self.bar.wait()                          # every rank has read every partial
            with torch.cuda.stream(s):
                self.views[r].copy_(total)
            s.synchronize()
            return 0
        return f


def bf16_ulp_distance(a: torch.Tensor, b: torch.Tensor) -> torch.Tensor:
    """Number of bf16 values between a and b (element-wise, same-signed
    ordering of the bit patterns; -0 == +0)."""
    def ordered(x):
        u = x.contiguous().view(torch.int16).to(torch.int32) & 0xFFFF
        neg = (u & 0x8000) != 0
        return torch.where(neg, 0x8000 - (u & 0x7FFF), 0x8000 + u)
    return (ordered(a) - ordered(b)).abs()


def _small_qwen3(n_layers=2):
    return dict(synth.model_config("qwen3_8b"), n_layers=n_layers, vocab=8192,
                mask_token_id=8191)


@pytest.mark.parametrize("size,ctx", [(2, [300, 1000]), (4, [700]), (8, [64, 200, 900])])
def test_head_parallel_matches_oracle(size, ctx):
    cfg = _small_qwen3()
    Wt = synth.make_weights(cfg, seed=0)
    Wg = weights_to(Wt, DEV)
    h = DFlash(cfg, Wg, max_position=8192)
    shards = []
    try:
        ch = Chain(cfg, Wt, h, ctx, seed=size + len(ctx))
        d_full, lo_full, _ = ch.gpu()
        K, V, P, d = cfg["block_size"] - 1, cfg["vocab"], 16, cfg["head_dim"]
        hk = cfg["n_kv_heads"] // size
        vs = vocab_shards(V, size)
        shards = [DFlash(cfg, Wg, max_position=8192, tp=(r, size), vocab_shard=vs[r])
                  for r in range(size)]
        shape = (ch.num_pages, hk, P, d)
        kcs = [[torch.zeros(shape, dtype=torch.bfloat16, device=DEV)
                for _ in range(cfg["n_layers"])] for _ in range(size)]
        vcs = [[torch.zeros(shape, dtype=torch.bfloat16, device=DEV)
                for _ in range(cfg["n_layers"])] for _ in range(size)]
        pos = torch.tensor(ch.pos, device=DEV)
        slots = torch.tensor(ch.slots, device=DEV)
        for r in range(size):
            shards[r].inject_context(ch.aux.to(DEV), pos, slots, kcs[r], vcs[r])
        torch.cuda.synchronize()
        # each rank's caches: its kv heads of the whole model's (block slots
        # included, written by the whole-model proposal; compare context only)
        ctx_pages = set()
        for b, n in enumerate(ch.ctx_lens):
            ctx_pages.update(int(x) for x in ch.table[b, :int(n) // P])
        sel = torch.tensor(sorted(ctx_pages), dtype=torch.long, device=DEV)
        if len(sel):
            for r in range(size):
                for l in range(cfg["n_layers"]):
                    for got, full in ((kcs[r][l], ch.kc[l]), (vcs[r][l], ch.vc[l])):
                        a = got.index_select(0, sel)
                        b_ = full[:, r * hk:(r + 1) * hk].index_select(0, sel)
                        # the shard's K/V GEMM has other tiles, so its fp32 sums
                        # differ in the last bits: a value may round the other
                        # way (one bf16 ulp of the larger), and values near zero
                        # (cancellation) carry the sums' absolute error, about
                        # 2^-12 of the entries' rms
                        af, bf = a.float(), b_.float()
                        rms = float(bf.square().mean().sqrt())
                        tol = 2.0 ** -7 * torch.maximum(af.abs(), bf.abs()) + 2.0 ** -12 * rms
                        worst = float(((af - bf).abs() / tol).max())
                        assert worst <= 1.0, (worst, r, l)
                        # (measured: 0.1-0.3% of the values round the other way)
                        assert int((bf16_ulp_distance(a, b_) > 0).sum()) <= a.numel() // 100

        bonus = ch.bonus.to(DEV)
        seq = torch.tensor(ch.ctx_lens, device=DEV)
        table = torch.tensor(ch.table, device=DEV)
        streams = [torch.cuda.Stream(device=DEV) for _ in range(size)]
        wss = [torch.empty(shards[r].propose_workspace_bytes(ch.B, ch.W), dtype=torch.uint8,
                           device=DEV) for r in range(size)]
        ex = LockstepExchange(size, wss, streams)
        keys = [None] * size
        logits = [torch.empty(ch.B * K, vs[r][1], dtype=torch.float32, device=DEV)
                  for r in range(size)]
        errors = []

        def rank(r):
            try:
                keys[r] = shards[r].propose_tp(bonus, seq, table, kcs[r], vcs[r], ex.hook(r),
                                               logits_out=logits[r], workspace=wss[r],
                                               stream=streams[r])
                streams[r].synchronize()
            except Exception as e:      # surfaced below
                errors.append((r, e))
                ex.bar.abort()

        threads = [threading.Thread(target=rank, args=(r,)) for r in range(size)]
        for th in threads:
            th.start()
        for th in threads:
            th.join(timeout=300)
        assert not errors, errors
        assert ex.calls == [2 * cfg["n_layers"]] * size     # O and down, every layer
        for r in range(size):
            assert shards[r].check_device_errors() == 0
        kmax = torch.stack(keys).amax(dim=0)
        drafts, blk = finalize_draft_keys(kmax, bonus, cfg["block_size"], V)
        torch.cuda.synchronize()
        lo = to_np(torch.cat(logits, dim=1)).astype(np.float64)
        # the same model up to summation order (partial sums added across
        # ranks, other attention splits): within the logit budget of each other
        assert all(k is not None for k in keys)
        assert rel_l2(lo, lo_full.astype(np.float64)) < 1e-2
        excluded = compare_drafts(to_np(drafts), lo, ch.oracle("device"), ch.oracle("exact"), K,
                                  name=f"head-parallel chain x{size}")
        assert excluded <= max_excluded(ch.B * K)
        np.testing.assert_array_equal(to_np(blk)[:, 0], to_np(ch.bonus))
    finally:
        for s in shards:
            s.close()
        h.close()


def test_head_parallel_rejections():
    cfg = _small_qwen3(n_layers=1)
    Wg = weights_to(synth.make_weights(cfg, seed=0), DEV)
    # kv heads (8) not divisible by 3
    with pytest.raises(DFlashError) as e:
        DFlash(cfg, Wg, max_position=1024, tp=(0, 3))
    assert e.value.status == -4
    sh = DFlash(cfg, Wg, max_position=1024, tp=(1, 2), vocab_shard=(4096, 4096))
    try:
        kc = [torch.zeros(4, 4, 16, 128, dtype=torch.bfloat16, device=DEV)]
        args = (torch.tensor([5], dtype=torch.int32, device=DEV),
                torch.tensor([3], dtype=torch.int32, device=DEV),
                torch.tensor([[0, 1]], dtype=torch.int32, device=DEV), kc, kc)
        # a shard proposes only through dflash_propose_tp
        with pytest.raises(DFlashError):
            sh.propose_keys(*args)
        # a failing exchange is reported, not ignored
        with pytest.raises(DFlashError) as e:
            sh.propose_tp(*args, lambda data, count, st: 7)
        assert e.value.status == -9
    finally:
        sh.close()
