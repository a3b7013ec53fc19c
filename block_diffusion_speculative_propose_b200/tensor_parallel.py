"""Vocabulary-parallel LM head across ranks (one process per GPU).

The draft's LM head is the target's, aliased; split over the vocabulary like
a column-parallel linear layer ("DFlash Speculative Decoding in the vLLM
Neuron Framework", §DFlashQwen3ForCausalLM), each rank holds a handle whose
LM head is its shard (``DFlash(..., vocab_shard=...)``) and runs the rest of
the draft in full.  A rank's greedy pick per draft row is one ordered 64-bit
key (dflash_propose_keys); the only exchange is an all-reduce MAX of those
keys, 8 bytes per row, through torch.distributed (NCCL over NVLink on GPUs),
after which every rank decodes the same drafts (dflash_finalize_draft_keys).
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
