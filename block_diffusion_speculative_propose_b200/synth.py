"""Seeded synthetic inputs for the DFlash draft-proposal step.

This module only draws numbers and lays out pages; it holds none of the
method's arithmetic, so the CUDA path and the CPU oracle can both be fed from
it.  All draws go through ``torch.Generator`` objects seeded explicitly, on
the CPU by default (bit-identical everywhere) or on a CUDA device when the
caller only needs a workload of the right shape and distribution (the bench).

Model shapes follow the pages' reference checkpoints: a Qwen3-8B-paired draft
(block 16) and a Llama-3.1-8B-paired draft (block 10, mask id 128002), both
with five Qwen3-style layers and five tapped target layers; plus a tiny model.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import torch

# ----------------------------------------------------------------------------
# model geometries
# ----------------------------------------------------------------------------
MODELS: Dict[str, dict] = {
    "tiny": dict(hidden=256, n_layers=2, n_q_heads=4, n_kv_heads=2, head_dim=64,
                 intermediate=512, vocab=1024, n_target_layers=3, block_size=4,
                 mask_token_id=1023, page_size=16, rms_eps=1e-6, rope_theta=1e6,
                 target_layer_ids=(0, 1, 2)),
    "qwen3_8b": dict(hidden=4096, n_layers=5, n_q_heads=32, n_kv_heads=8,
                     head_dim=128, intermediate=12288, vocab=151936,
                     n_target_layers=5, block_size=16, mask_token_id=151935,
                     page_size=16, rms_eps=1e-6, rope_theta=1e6,
                     target_layer_ids=(1, 9, 17, 25, 33)),
    "llama31_8b": dict(hidden=4096, n_layers=5, n_q_heads=32, n_kv_heads=8,
                       head_dim=128, intermediate=14336, vocab=128256,
                       n_target_layers=5, block_size=10, mask_token_id=128002,
                       page_size=16, rms_eps=1e-6, rope_theta=1e6,
                       target_layer_ids=(1, 8, 15, 22, 29)),
}

# ----------------------------------------------------------------------------
# workloads (batch, context-length mix, acceptance mix)
# ----------------------------------------------------------------------------
WORKLOADS: Dict[str, dict] = {
    # tiny draft, batch 1, 64 context tokens
    "tiny_b1_ctx64": dict(model="tiny", batch=1, ctx_lo=64, ctx_hi=64,
                          accept="uniform"),
    # Qwen3-8B-shaped draft, batch 1, context 2048
    "qwen3_b1_ctx2048": dict(model="qwen3_8b", batch=1, ctx_lo=2048,
                             ctx_hi=2048, accept="uniform"),
    # batch 32, contexts U[512, 8192]
    "qwen3_b32_ctx512_8192": dict(model="qwen3_8b", batch=32, ctx_lo=512,
                                  ctx_hi=8192, accept="uniform"),
    # Llama-3.1-8B-paired draft, batch 128, block 10, contexts U[1024, 16384]
    "llama_b128_ctx1024_16384": dict(model="llama31_8b", batch=128, ctx_lo=1024,
                                     ctx_hi=16384, accept="uniform"),
    # long-context full step, batch 128, contexts U[8192, 32768], E[tau] ~ 6
    "qwen3_b128_ctx8192_32768": dict(model="qwen3_8b", batch=128, ctx_lo=8192,
                                     ctx_hi=32768, accept="geometric"),
}

# per-draft acceptance probability giving E[1 + n] = 6.00 with n capped at 15
GEOMETRIC_P = 0.8445


def model_config(name: str) -> dict:
    return dict(MODELS[name])


# ----------------------------------------------------------------------------
# weights
# ----------------------------------------------------------------------------
def _normal(g: torch.Generator, shape, std: float, device) -> torch.Tensor:
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    return (t * std).to(torch.bfloat16)


def _norm_weight(g: torch.Generator, n: int, device) -> torch.Tensor:
    t = torch.randn(n, generator=g, device=device, dtype=torch.float32)
    return (1.0 + 0.02 * t).to(torch.bfloat16)


def make_weights(cfg: dict, seed: int = 0, device="cpu",
                 std: float = 0.02) -> Dict[str, object]:
    """Random-init draft weights, bf16, row-major [out, in].

    Dense weights ~ N(0, std^2); norm weights 1 + N(0, 0.02^2).  Per-layer
    entries are lists of length n_layers.  ``embed`` and ``lm_head`` stand for
    the target's aliased tables."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    H, L = cfg["hidden"], cfg["n_layers"]
    Hq, Hkv, d = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    I, V, T = cfg["intermediate"], cfg["vocab"], cfg["n_target_layers"]
    W: Dict[str, object] = {
        "fc_w": _normal(g, (H, T * H), std, device),
        "hidden_norm_w": _norm_weight(g, H, device),
        "embed": _normal(g, (V, H), std, device),
        "lm_head": _normal(g, (V, H), std, device),
        "final_norm_w": _norm_weight(g, H, device),
    }
    per = {k: [] for k in ("in_norm_w", "post_norm_w", "wq", "wk", "wv", "wo",
                           "q_norm_w", "k_norm_w", "w_gate", "w_up", "w_down")}
    for _ in range(L):
        per["in_norm_w"].append(_norm_weight(g, H, device))
        per["wq"].append(_normal(g, (Hq * d, H), std, device))
        per["wk"].append(_normal(g, (Hkv * d, H), std, device))
        per["wv"].append(_normal(g, (Hkv * d, H), std, device))
        per["q_norm_w"].append(_norm_weight(g, d, device))
        per["k_norm_w"].append(_norm_weight(g, d, device))
        per["wo"].append(_normal(g, (H, Hq * d), std, device))
        per["post_norm_w"].append(_norm_weight(g, H, device))
        per["w_gate"].append(_normal(g, (I, H), std, device))
        per["w_up"].append(_normal(g, (I, H), std, device))
        per["w_down"].append(_normal(g, (H, I), std, device))
    W.update(per)
    return W


def target_config(draft_cfg: dict, n_layers: int) -> dict:
    """A small causal target for a draft: the draft's layer shape and
    vocabulary with its own depth."""
    keys = ("hidden", "n_q_heads", "n_kv_heads", "head_dim", "intermediate", "vocab",
            "rms_eps", "rope_theta")
    return dict({k: draft_cfg[k] for k in keys}, n_layers=n_layers)


def make_target_weights(tcfg: dict, seed: int = 0, device="cpu",
                        std: float = 0.05) -> Dict[str, object]:
    """Random-init target weights as float32 tensors holding bf16 values (so
    that a draft's bf16 aliases of the embedding and LM head carry the same
    numbers).  Same names and layouts as make_weights, without fc / hidden_norm."""
    W = make_weights(dict(tcfg, n_target_layers=1, block_size=2, mask_token_id=0), seed,
                     device, std)
    del W["fc_w"], W["hidden_norm_w"]
    return {k: ([x.float() for x in v] if isinstance(v, list) else v.float())
            for k, v in W.items()}


# ----------------------------------------------------------------------------
# one step's batch
# ----------------------------------------------------------------------------
@dataclass
class StepBatch:
    """Inputs of one speculative step for B requests.

    Request b has ``ctx_lens[b]`` tokens injected before the step.  The step
    verifies the previous drafts (``prev_drafts`` against ``target_logits``,
    built so that exactly ``n_accept[b]`` drafts are accepted), injects the
    ``n_accept[b] + 1`` accepted rows at positions ctx .. ctx + n_accept, and
    proposes the next block at ``seq_lens = ctx_lens + n_accept + 1``."""

    B: int
    block_size: int
    ctx_lens: torch.Tensor          # [B] int32
    n_accept: torch.Tensor          # [B] int32
    seq_lens: torch.Tensor          # [B] int32
    block_table: torch.Tensor       # [B, max_pages_per_seq] int32
    num_pages: int
    inject_positions: torch.Tensor  # [R] int64 (absolute positions)
    inject_req_ids: torch.Tensor    # [R] int64
    aux: Optional[torch.Tensor]     # [R, T*H] bf16
    bonus: torch.Tensor             # [B] int32
    prev_drafts: torch.Tensor       # [B, K] int32
    target_logits: Optional[torch.Tensor]  # [B, K+1, V] fp32
    pages_of: List[torch.Tensor] = field(default_factory=list)  # per request


def _tokens_except(g, n, vocab, mask_id, device) -> torch.Tensor:
    """n uniform token ids from [0, vocab) without the mask id."""
    t = torch.randint(0, vocab - 1, (n,), generator=g, device=device,
                      dtype=torch.int64)
    return torch.where(t >= mask_id, t + 1, t)


def make_step_batch(cfg: dict, batch: int, ctx_lo: int, ctx_hi: int,
                    accept: str = "uniform", seed: int = 1,
                    with_aux: bool = True, with_logits: bool = True,
                    page_slack: int = 8, table_pages: Optional[int] = None
                    ) -> StepBatch:
    """Draw one step's batch on the CPU (seeded)."""
    g = torch.Generator()
    g.manual_seed(seed)
    B, bs, P = batch, cfg["block_size"], cfg["page_size"]
    K, V, mask = bs - 1, cfg["vocab"], cfg["mask_token_id"]
    ctx = torch.randint(ctx_lo, ctx_hi + 1, (B,), generator=g, dtype=torch.int64)
    if accept == "uniform":
        n_acc = torch.randint(0, K + 1, (B,), generator=g, dtype=torch.int64)
    elif accept == "geometric":
        u = torch.rand(B, K, generator=g, dtype=torch.float64)
        ok = (u < GEOMETRIC_P).to(torch.int64)
        n_acc = torch.cumprod(ok, dim=1).sum(dim=1)       # leading successes
    elif accept == "full":
        n_acc = torch.full((B,), K, dtype=torch.int64)
    elif accept == "none":
        n_acc = torch.zeros(B, dtype=torch.int64)
    else:
        raise ValueError(accept)
    seq = ctx + n_acc + 1
    # pages: every request owns enough pages for seq_len + block_size tokens
    need = [int(math.ceil((int(s) + bs) / P)) for s in seq]
    width = table_pages or int(math.ceil((ctx_hi + K + 1 + bs) / P))
    assert max(need) <= width
    num_pages = sum(need) + page_slack
    perm = torch.randperm(num_pages, generator=g, dtype=torch.int64)
    table = torch.zeros(B, width, dtype=torch.int32)
    pages_of, cur = [], 0
    for b in range(B):
        pg = perm[cur:cur + need[b]]
        cur += need[b]
        table[b, :need[b]] = pg.to(torch.int32)
        pages_of.append(pg)
    # rows injected this step: accepted prefix (previous bonus + n drafts)
    pos = torch.cat([torch.arange(int(c), int(c) + int(n) + 1, dtype=torch.int64)
                     for c, n in zip(ctx, n_acc)]) if B else torch.zeros(0, dtype=torch.int64)
    req = torch.cat([torch.full((int(n) + 1,), b, dtype=torch.int64)
                     for b, n in enumerate(n_acc)]) if B else torch.zeros(0, dtype=torch.int64)
    R = int(pos.numel())
    aux = None
    if with_aux:
        aux = torch.randn(R, cfg["n_target_layers"] * cfg["hidden"], generator=g,
                          dtype=torch.float32).to(torch.bfloat16)
    bonus = _tokens_except(g, B, V, mask, "cpu").to(torch.int32)
    drafts = _tokens_except(g, B * K, V, mask, "cpu").reshape(B, K).to(torch.int32)
    logits = None
    if with_logits:
        logits = make_target_logits(g, drafts, n_acc, V)
    return StepBatch(B=B, block_size=bs, ctx_lens=ctx.to(torch.int32),
                     n_accept=n_acc.to(torch.int32), seq_lens=seq.to(torch.int32),
                     block_table=table, num_pages=num_pages,
                     inject_positions=pos, inject_req_ids=req, aux=aux,
                     bonus=bonus, prev_drafts=drafts, target_logits=logits,
                     pages_of=pages_of)


def make_target_logits(g: torch.Generator, drafts: torch.Tensor,
                       n_acc: torch.Tensor, vocab: int,
                       device="cpu") -> torch.Tensor:
    """fp32 logits [B, K+1, V] ~ N(0, 1) shaped so that the first ``n_acc[b]``
    drafts of request b are the target's top choice and draft ``n_acc[b]`` (if
    any) is not: entries at the accepted draft ids are raised one above the
    row maximum; at the first rejected row the draft's entry is pushed one
    below the row minimum."""
    B, K = drafts.shape
    T = torch.randn(B, K + 1, vocab, generator=g, device=device,
                    dtype=torch.float32)
    d = drafts.to(device=device, dtype=torch.int64)
    n = n_acc.to(device=device, dtype=torch.int64)
    rowmax = T.amax(dim=2)
    rowmin = T.amin(dim=2)
    j = torch.arange(K, device=device)[None, :].expand(B, K)
    acc = j < n[:, None]
    rej = j == n[:, None]
    cur = torch.gather(T[:, :K, :], 2, d[:, :, None])[:, :, 0]
    new = torch.where(acc, rowmax[:, :K] + 1.0,
                      torch.where(rej, rowmin[:, :K] - 1.0, cur))
    T[:, :K, :].scatter_(2, d[:, :, None], new[:, :, None])
    return T


def make_aux(rows: int, cfg: dict, seed: int, device="cpu") -> torch.Tensor:
    """Concatenated tapped hidden states, [rows, T*H] bf16 ~ N(0, 1)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(rows, cfg["n_target_layers"] * cfg["hidden"], generator=g,
                       device=device, dtype=torch.float32).to(torch.bfloat16)


def fill_cache_random(caches: List[torch.Tensor], seed: int) -> None:
    """Fill KV pools in place with N(0, 1) bf16 values (stand-in for context
    that an earlier injection would have written)."""
    g = torch.Generator(device=caches[0].device)
    g.manual_seed(seed)
    for c in caches:
        c.copy_(torch.randn(c.shape, generator=g, device=c.device,
                            dtype=torch.float32).to(torch.bfloat16))
