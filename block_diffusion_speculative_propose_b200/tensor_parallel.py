"""Tensor parallelism across ranks (one process per GPU).

Vocabulary-parallel LM head: the draft's LM head is the target's, aliased;
split over the vocabulary like a column-parallel linear layer ("DFlash
Speculative Decoding in the vLLM Neuron Framework", §DFlashQwen3ForCausalLM),
each rank holds a handle whose LM head is its shard (``DFlash(...,
vocab_shard=...)``) and runs the rest of the draft in full.  A rank's greedy
pick per draft row is one ordered 64-bit key (dflash_propose_keys); the only
exchange is an all-reduce MAX of those keys, 8 bytes per row, through
torch.distributed (NCCL over NVLink on GPUs), after which every rank decodes
the same drafts (dflash_finalize_draft_keys).

Head-parallel layers: each rank also holds only its kv heads (with their query
groups) and its MLP features (``DFlash(..., tp=(rank, size))``; §Context KV
Injection: "this rank's KV heads only"), and the row-parallel O and down
projections' partial sums are all-reduced (SUM) before each residual add,
through the exchange hook that dflash_propose_tp calls between its kernels.
"""

from __future__ import annotations

from typing import List, Tuple

import torch
import torch.distributed as dist

from .dflash import DFlash, finalize_draft_keys


def vocab_shards(vocab: int, parts: int) -> List[Tuple[int, int]]:
    """(start, count) of each of `parts` shards of [0, vocab): contiguous,
    multiples of 32 (the LM head's column groups), sizes within 32 of each
    other.  vocab must be a multiple of 32 and parts <= vocab / 32."""
    if vocab % 32 or parts < 1 or parts > vocab // 32:
        raise ValueError(f"cannot split a vocabulary of {vocab} into {parts} shards")
    groups = vocab // 32
    out, start = [], 0
    for r in range(parts):
        g = groups // parts + (1 if r < groups % parts else 0)
        out.append((start * 32, g * 32))
        start += g
    return out


def exchange_draft_keys(draft_keys: torch.Tensor, group=None) -> torch.Tensor:
    """In place: the maximum over the group's ranks of each row's key — the
    whole vocabulary's greedy pick (ties -> lowest id)."""
    dist.all_reduce(draft_keys, op=dist.ReduceOp.MAX, group=group)
    return draft_keys


def propose_vocab_parallel(h: DFlash, bonus_tokens, seq_lens, block_table, k_cache, v_cache,
                           group=None, workspace=None, stream=None):
    """One proposal on a vocabulary-shard handle: local keys, exchange, decode.
    Returns (draft_tokens [B, K], block_tokens [B, bs]) on every rank."""
    keys = h.propose_keys(bonus_tokens, seq_lens, block_table, k_cache, v_cache,
                          workspace=workspace, stream=stream)
    exchange_draft_keys(keys, group)
    return finalize_draft_keys(keys, bonus_tokens, h.cfg["block_size"], h.cfg["vocab"],
                               stream=stream)


def allreduce_hook(workspace: torch.Tensor, group=None, stream=None):
    """The exchange of dflash_propose_tp for this rank: the `count` fp32 values
    at `data` (inside `workspace`) summed over the group in place, through
    torch.distributed.  On GPUs (NCCL) the all-reduce is ordered on `stream`
    (the stream the proposal runs on); with tensors on the host (gloo) it runs
    synchronously."""
    base = workspace.data_ptr()

    def hook(data: int, count: int, _stream_ptr=None) -> int:
        off = data - base
        if off < 0 or off + 4 * count > workspace.numel():
            return 1
        t = workspace[off:off + 4 * count].view(torch.float32)
        if t.is_cuda:
            with torch.cuda.stream(stream if stream is not None else torch.cuda.current_stream()):
                dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
        else:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
        return 0
    return hook


def propose_head_parallel(h: DFlash, bonus_tokens, seq_lens, block_table, k_cache, v_cache,
                          group=None, workspace=None, stream=None):
    """One proposal on a head-parallel shard (every rank of the group calls
    it with the same batch and its own KV pools): layers with the O / down
    partial sums all-reduced, then the vocabulary keys exchanged and decoded.
    Returns (draft_tokens [B, K], block_tokens [B, bs]) on every rank."""
    B, W = int(bonus_tokens.shape[0]), int(block_table.shape[1])
    ws = workspace if workspace is not None else torch.empty(
        max(h.propose_workspace_bytes(B, W), 256), dtype=torch.uint8, device=h.device)
    keys = h.propose_tp(bonus_tokens, seq_lens, block_table, k_cache, v_cache,
                        allreduce_hook(ws, group, stream), workspace=ws, stream=stream)
    exchange_draft_keys(keys, group)
    return finalize_draft_keys(keys, bonus_tokens, h.cfg["block_size"], h.cfg["vocab"],
                               stream=stream)

