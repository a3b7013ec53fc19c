"""Host side of the vocabulary-parallel LM head on CPU: the shard partition and
the one exchange step (an all-reduce MAX of ordered 64-bit keys) between two
gloo ranks.  The keys are built here from the encoding that include/dflash.h
states for dflash_propose_keys, so the test pins that the signed maximum over
ranks is the whole vocabulary's greedy pick (largest logit, ties -> lowest
id, -0 == +0, NaN counts as -inf)."""

from __future__ import annotations

import os
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from block_diffusion_speculative_propose_b200.tensor_parallel import vocab_shards  # noqa: E402


def ordered_bits(v: np.float32) -> int:
    """32-bit pattern that sorts like the float (as the header defines it)."""
    if np.isnan(v):
        v = np.float32(-np.inf)
    if v == 0:
        v = np.float32(0.0)
    u = int(np.array([v], dtype=np.float32).view(np.uint32)[0])
    return (~u) & 0xFFFFFFFF if u & 0x80000000 else u | 0x80000000


def encode(v: np.float32, token: int) -> int:
    """dflash_propose_keys' key of (value, token) as a signed int64."""
    key = (ordered_bits(v) << 32) | (0xFFFFFFFF - token)
    key ^= 1 << 63
    return key - (1 << 64) if key >= (1 << 63) else key


def decode(key) -> int:
    u = ((int(key) + (1 << 64)) % (1 << 64)) ^ (1 << 63)
    return 0xFFFFFFFF - (u & 0xFFFFFFFF)


def shard_keys(logits: np.ndarray, start: int, count: int) -> np.ndarray:
    """Per row: the key of this shard's greedy pick (ties -> lowest id)."""
    out = np.empty(logits.shape[0], dtype=np.int64)
    for r in range(logits.shape[0]):
        best = None
        for j in range(start, start + count):
            k = encode(logits[r, j], j)
            best = k if best is None or k > best else best
        out[r] = best
    return out


def reference_pick(row: np.ndarray) -> int:
    """Largest logit, NaN as -inf, ties -> lowest index (plain definition)."""
    vals = np.where(np.isnan(row), -np.inf, row)
    return int(np.flatnonzero(vals == vals.max())[0])


def make_logits(rows: int, vocab: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    lg = rng.standard_normal((rows, vocab)).astype(np.float32)
    lg[0, 5] = lg[0, vocab - 3] = lg[0].max() + 1.0          # a tie across shards
    lg[1, :] = -1.0                                          # every value equal
    lg[2, 7] = np.nan                                        # NaN never wins
    lg[3, :] = -0.0
    lg[3, vocab - 1] = 0.0                                   # -0 ties +0: lowest id wins
    lg[4, :] = -np.inf                                       # all -inf: id 0
    lg[5, vocab // 2 + 1] = np.inf
    return lg


def test_vocab_shards_partition():
    for vocab in (1024, 128256, 151936):
        for parts in range(1, 9):
            sh = vocab_shards(vocab, parts)
            assert len(sh) == parts and sh[0][0] == 0
            assert sum(c for _, c in sh) == vocab
            for (s0, c0), (s1, _) in zip(sh, sh[1:]):
                assert s0 + c0 == s1
            assert all(s % 32 == 0 and c % 32 == 0 and c > 0 for s, c in sh)
            assert max(c for _, c in sh) - min(c for _, c in sh) <= 32
    with pytest.raises(ValueError):
        vocab_shards(1000, 2)
    with pytest.raises(ValueError):
        vocab_shards(64, 3)


def test_key_order_matches_the_plain_argmax():
    lg = make_logits(8, 96, seed=1)
    for r in range(lg.shape[0]):
        assert decode(shard_keys(lg[r:r + 1], 0, 96)[0]) == reference_pick(lg[r])


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from block_diffusion_speculative_propose_b200.tensor_parallel import (exchange_draft_keys,
                                                                          vocab_shards)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lg = make_logits(8, 96, seed=2)
        start, count = vocab_shards(96, world)[rank]
        keys = torch.tensor(shard_keys(lg, start, count))
        exchange_draft_keys(keys)
        q.put((rank, [decode(int(k)) for k in keys]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_exchange_keys(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29530 + world
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    lg = make_logits(8, 96, seed=2)
    want = [reference_pick(lg[r]) for r in range(lg.shape[0])]
    for r in range(world):
        assert res[r] == want


# ----------------------------------------------------------------------------
# head-parallel layers: the exchange hook of dflash_propose_tp between gloo ranks
# ----------------------------------------------------------------------------
def _hook_rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from block_diffusion_speculative_propose_b200.tensor_parallel import allreduce_hook
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # a host "workspace" whose middle holds this rank's partial sums; the
        # hook receives only the pointer and the count, as from the library
        ws = torch.zeros(4096, dtype=torch.uint8)
        off, count = 1024, 100
        part = ws[off:off + 4 * count].view(torch.float32)
        g = torch.Generator().manual_seed(rank)
        part.copy_(torch.randn(count, generator=g))
        hook = allreduce_hook(ws)
        rc = hook(ws.data_ptr() + off, count)
        bad = hook(ws.data_ptr() + 4000, 100)    # past the workspace: refused, nothing sent
        q.put((rank, rc, bad, part.tolist(), ws[:off].abs().sum().item(),
               ws[off + 4 * count:].abs().sum().item()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_sum_partials_in_place(world):
    """The hook sums every rank's row-parallel partials in place, touching
    nothing else of the workspace, and refuses a range outside it."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29560 + world
    procs = [ctx.Process(target=_hook_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, rc, bad, vals, before, after = q.get(timeout=120)
        res[rank] = vals
        assert rc == 0 and bad == 1 and before == 0 and after == 0
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import torch
    want = sum(torch.randn(100, generator=torch.Generator().manual_seed(r)) for r in range(world))
    for r in range(world):
        np.testing.assert_allclose(res[r], want.numpy(), rtol=1e-6, atol=1e-6)
