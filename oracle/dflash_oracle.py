"""CPU oracle for the DFlash draft-proposal step (propose + inject + greedy verify).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or runs
this module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may call it.  It shares no code with the CUDA library; both
sides only receive the same seeded inputs.

What it is: a plain, slow, obviously correct restatement of what the DFlash
pages say the proposal step computes, in float64 arithmetic (numpy), with a
library matmul as the only non-elementary step.  Every function names the
passage it follows.  The three pages are cited by title:

  [NEURON]  "DFlash Speculative Decoding in the vLLM Neuron Framework"
            (AWS Neuron design doc), sections as named there.
  [VLLM]    "[Feat][Spec Decode] DFlash" (vLLM pull request #36847),
            unit test ``test_set_inputs_first_pass_dflash`` and the
            acceptance-metric helpers.
  [QEFF]    "Dflash: Block Diffusion Speculative Decoding" (QEfficient pull
            request #995), PR description and commit notes.

Precision modes
---------------
``exact``   every intermediate stays float64.  Used for the logits check
            (relative L2 against the GPU path).
``device``  rounds (round-to-nearest-even, via float32) at the storage points
            of ``STORAGE_POINTS`` to the format the device path stores there,
            and uses the fp16 copies of the weights that the device path
            multiplies in fp16; everything else stays float64.  Used for
            bit-exact draft / acceptance comparison.
``bf16``    rounds every storage point to bfloat16 (an all-bf16 pipeline; for
            error analysis).
Argmax decisions are taken on float32-rounded logits in every mode (the
kernel's decision precision).

Readings where the pages are silent (each is also listed in the design notes):
  * every norm is RMSNorm ``x * rsqrt(mean(x^2) + eps) * w`` (weight multiplies
    directly), q/k norms are per head over head_dim;
  * context vectors feed Wk/Wv directly (no input_layernorm on the context),
    per [NEURON] "Context KV Injection" step 2;
  * no biases anywhere; one final RMSNorm before the LM head;
  * RoPE is the rotate-half form, pairs (i, i + d/2), inv_freq_i =
    theta^(-2i/d), angles from integer positions in float64, attention scaling 1;
  * softmax scale 1/sqrt(head_dim), no soft-cap, no window;
  * argmax ties go to the lowest index, NaN compares equal to -inf;
  * K = block_size - 1 drafts per request.

Parity pins: see tests/test_oracle_pins.py.  The whole draft stack beyond the
single-layer library comparison and the invariants there is "parity unpinned"
in the sense that no page prints model outputs.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Mapping, Sequence

import numpy as np

# Storage points of the proposal path and the format the device path keeps
# there.  Operands that are bounded by construction (RMSNorm outputs: |y_i| <=
# sqrt(H) max|w|; attention outputs: convex combinations of V rows) are held in
# fp16; the KV cache, q (attended against that cache) and the MLP hidden stay
# bf16.  ``device`` mode rounds to these formats; ``bf16`` mode to bf16 everywhere.
STORAGE_POINTS = {
    "context": "fp16",     # c = hidden_norm(fc(x)), fed to the K/V projection
    "kv": "bf16",          # K (after k_norm + RoPE) and V entries of the paged cache
    "norm": "fp16",        # input / post-attention RMSNorm outputs fed to projections
    "q": "bf16",           # block q after q_norm + RoPE
    "attn_out": "fp16",    # attention output o, fed to Wo
    "mlp_hidden": "bf16",  # silu(gate) * up, fed to Wd
    "final": "fp16",       # final-normed kept rows, fed to the LM head
}
# Weights multiplied in fp16 by the device path (held there as fp16 copies).
FP16_WEIGHTS = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "lm_head")


# ----------------------------------------------------------------------------
# configuration
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class OracleConfig:
    """Draft-model geometry.  Field names follow the [NEURON] DFlashConfig
    (block size, mask token id, target layer ids) plus the Qwen3 layer shape
    ([NEURON] "DFlash Draft Model Architecture")."""

    hidden: int
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    intermediate: int
    vocab: int
    n_target_layers: int
    block_size: int
    mask_token_id: int
    page_size: int = 16
    rms_eps: float = 1e-6
    rope_theta: float = 1e6

    @staticmethod
    def from_mapping(m: Mapping) -> "OracleConfig":
        names = OracleConfig.__dataclass_fields__.keys()
        return OracleConfig(**{k: m[k] for k in names if k in m})

    @property
    def num_drafts(self) -> int:
        # [NEURON] "Configuration Parameters": one block slot is the bonus
        # token, so the draft width is block_size - 1.
        return self.block_size - 1


# ----------------------------------------------------------------------------
# rounding
# ----------------------------------------------------------------------------
def round_bf16(a) -> np.ndarray:
    """Round to bfloat16 (nearest, ties to even) and return float64 values.

    Goes through float32 first (float64 -> float32 is IEEE nearest-even), then
    drops the low 16 bits of the float32 pattern with nearest-even rounding.
    Inputs are finite in every workload this oracle sees."""
    f = np.asarray(a, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def round_fp16(a) -> np.ndarray:
    """Round to IEEE binary16 (nearest, ties to even; via float32, subnormals
    kept, overflow to inf) and return float64 values."""
    f = np.asarray(a, dtype=np.float64).astype(np.float32)
    with np.errstate(over="ignore"):
        return f.astype(np.float16).astype(np.float64)


def _identity(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


_ROUND = {"bf16": round_bf16, "fp16": round_fp16}
MODES = ("exact", "device", "bf16")


class Rounding:
    """Callable ``rnd(point, value)`` for one precision mode."""

    def __init__(self, mode: str):
        if mode not in MODES:
            raise ValueError(f"unknown precision mode {mode!r}")
        self.mode = mode

    def __call__(self, point: str, a) -> np.ndarray:
        if self.mode == "exact":
            return _identity(a)
        if self.mode == "bf16":
            return round_bf16(a)
        return _ROUND[STORAGE_POINTS[point]](a)

    def weight(self, name: str, w) -> np.ndarray:
        """A weight as the mode's GEMM sees it (fp16 copies in device mode)."""
        if self.mode == "device" and name in FP16_WEIGHTS:
            return round_fp16(w)
        return w


def rounding(mode: str) -> Rounding:
    return Rounding(mode)


# ----------------------------------------------------------------------------
# elementary operations
# ----------------------------------------------------------------------------
def rms_norm(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * w.

    [NEURON] names "hidden_norm" and "pre-norms" of a standard Qwen3 decoder
    layer without defining them; the Qwen3 norm is RMSNorm."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(w, dtype=np.float64)


def silu(x: np.ndarray) -> np.ndarray:
    """SiLU(x) = x * sigmoid(x), the SwiGLU gate of a Qwen3 MLP."""
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def linear(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """y = x @ w^T with w stored [out, in] (no bias).  float64 matmul."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T


def rope_inv_freq(head_dim: int, theta: float) -> np.ndarray:
    """inv_freq_i = theta^(-2i/d), i < d/2 (default RoPE, attention scaling 1;
    [QEFF] commit notes fold attention_scaling into the sin/cos table)."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return theta ** (-(2.0 * i) / head_dim)


def apply_rope(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE on the last axis of ``x`` (shape [..., n, heads, d] or
    [n, d]) at integer ``positions`` (shape [n]).

    out[i]       = x[i] cos(a_i) - x[i + d/2] sin(a_i)
    out[i + d/2] = x[i + d/2] cos(a_i) + x[i] sin(a_i),  a_i = pos * inv_freq_i
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    pos = np.asarray(positions, dtype=np.float64)
    ang = pos[:, None] * rope_inv_freq(d, theta)[None, :]  # [n, d/2]
    cos, sin = np.cos(ang), np.sin(ang)
    # broadcast [n, d/2] against x's [n, (heads,) d/2]
    extra = x.ndim - 2
    shape = (ang.shape[0],) + (1,) * extra + (half,)
    cos = cos.reshape(shape)
    sin = sin.reshape(shape)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def argmax_f32(logits: np.ndarray) -> np.ndarray:
    """Greedy pick over the last axis, decided on float32 values.

    Ties go to the lowest index (np.argmax returns the first maximum); NaN is
    treated as -inf so it never wins over a number."""
    f = np.asarray(logits).astype(np.float32)
    f = np.where(np.isnan(f), np.float32(-np.inf), f)
    return np.argmax(f, axis=-1).astype(np.int64)


# ----------------------------------------------------------------------------
# paged KV addressing and block construction
# ----------------------------------------------------------------------------
def paged_slots(positions, req_ids, block_table, page_size: int) -> np.ndarray:
    """Map absolute positions to cache slots, [NEURON] "Paged KV Integration":
    page number = pos // page clamped to the table width - 1, page id looked
    up in the request's block-table row, slot = page_id * page + pos % page."""
    positions = np.asarray(positions, dtype=np.int64)
    req_ids = np.asarray(req_ids, dtype=np.int64)
    bt = np.asarray(block_table, dtype=np.int64)
    max_blocks = bt.shape[1]
    flat = bt.reshape(-1)
    block_numbers = np.minimum(positions // page_size, max_blocks - 1)
    block_ids = flat[req_ids * max_blocks + block_numbers]
    return block_ids * page_size + positions % page_size


@dataclass
class ProposalInputs:
    positions: np.ndarray      # [n] corrected context positions (int64)
    slot_mapping: np.ndarray   # [n] context slots, -1 for trailing padding rows (int64)
    req_ids: np.ndarray        # [n] request of each row, -1 for padding (int64)
    seq_lens: np.ndarray       # [B] post-verify sequence lengths (int64)
    bonus: np.ndarray          # [B] bonus tokens (int64)


def _valid_count(sampled, vocab: int) -> np.ndarray:
    """Per request, the sampler outputs that are real tokens: != -1 and
    < vocab ([NEURON] "Async Rejection and Position Correction")."""
    s = np.asarray(sampled, dtype=np.int64)
    return np.sum((s != -1) & (s < vocab), axis=1)


def prepare_proposal_inputs(target_positions, last_token_indices, cur_sampled, cur_num_draft,
                            block_table, page_size: int, vocab: int, prev_sampled=None,
                            prev_num_draft=None) -> ProposalInputs:
    """Device-side proposal-input preparation with the async correction,
    [NEURON] "Async Rejection and Position Correction", "Paged KV
    Integration" and "Draft Block Construction", in the pages' order:

    1. the request of each target row follows from last_token_indices (rows
       of request b end at last_token_indices[b]; rows past the last
       request's end are trailing padding);
    2. _correct_target_positions_for_async: prev_num_rejected =
       (1 + prev_num_draft_tokens) - prev_valid_count, subtracted from each
       row's optimistic position (no previous step: no correction);
    3. _current_seq_lens: the post-verify length removes this step's
       rejected positions from the optimistic length (the request's last
       corrected position + 1), using cur_num_draft_tokens;
    4. the bonus token is the last valid rejection-sampler output;
    5. context slots from the paged-slot formula, -1 for padding rows."""
    pos_in = np.asarray(target_positions, dtype=np.int64)
    last = np.asarray(last_token_indices, dtype=np.int64)
    n, B = pos_in.shape[0], last.shape[0]
    req = np.full(n, -1, dtype=np.int64)
    start = 0
    for b in range(B):
        for r in range(start, last[b] + 1):
            req[r] = b
        start = last[b] + 1
    if prev_sampled is None:
        prev_rej = np.zeros(B, dtype=np.int64)
    else:
        prev_rej = (1 + np.asarray(prev_num_draft, dtype=np.int64)) - _valid_count(prev_sampled,
                                                                                    vocab)
    pos = pos_in.copy()
    for r in range(n):
        if req[r] >= 0:
            pos[r] = pos_in[r] - prev_rej[req[r]]
    cur = np.asarray(cur_sampled, dtype=np.int64)
    cur_rej = (1 + np.asarray(cur_num_draft, dtype=np.int64)) - _valid_count(cur, vocab)
    seq_lens = np.array([pos[last[b]] + 1 - cur_rej[b] for b in range(B)], dtype=np.int64)
    bonus = np.full(B, -1, dtype=np.int64)
    for b in range(B):
        for j in range(cur.shape[1]):
            if cur[b, j] != -1 and cur[b, j] < vocab:
                bonus[b] = cur[b, j]
    slots = np.full(n, -1, dtype=np.int64)
    live = req >= 0
    if live.any():
        slots[live] = paged_slots(pos[live], req[live], block_table, page_size)
    return ProposalInputs(pos, slots, req, seq_lens, bonus)


@dataclass
class QueryBlock:
    input_ids: np.ndarray         # [B * bs]
    positions: np.ndarray         # [B * bs]
    req_ids: np.ndarray           # [B * bs]
    keep_idx: np.ndarray          # [B * (bs - 1)]
    query_start_loc: np.ndarray   # [B + 1]


def build_query_block(bonus_tokens, seq_lens, block_size: int,
                      mask_token_id: int) -> QueryBlock:
    """[NEURON] "Draft Block Construction": each request contributes
    [bonus, mask, ..., mask] (block_size slots) at positions
    seq_len + [0 .. block_size-1]; keep_idx selects slots 1 .. block_size-1.
    [VLLM] test_set_inputs_first_pass_dflash prints a worked example of the
    same layout, with query_start_loc = [0, bs, 2 bs, ...]."""
    bonus = np.asarray(bonus_tokens, dtype=np.int64)
    lens = np.asarray(seq_lens, dtype=np.int64)
    B = bonus.shape[0]
    ids = np.full((B, block_size), mask_token_id, dtype=np.int64)
    ids[:, 0] = bonus
    pos = lens[:, None] + np.arange(block_size, dtype=np.int64)[None, :]
    req = np.repeat(np.arange(B, dtype=np.int64), block_size)
    keep = (np.arange(B, dtype=np.int64)[:, None] * block_size
            + np.arange(1, block_size, dtype=np.int64)[None, :]).reshape(-1)
    qsl = np.arange(B + 1, dtype=np.int64) * block_size
    return QueryBlock(ids.reshape(-1), pos.reshape(-1), req, keep, qsl)


# ----------------------------------------------------------------------------
# (a1) context fusion, (a2) context K/V injection
# ----------------------------------------------------------------------------
def context_fusion(cfg: OracleConfig, W: Mapping, aux: np.ndarray,
                   mode: str = "exact") -> np.ndarray:
    """[NEURON] "Context KV Injection" step 1 and [QEFF] (concat -> fc ->
    hidden_norm): ctx = hidden_norm(fc(aux)).  ``aux`` is the concatenation of
    the tapped target states, [n, n_target * hidden]."""
    rnd = rounding(mode)
    aux = np.asarray(aux, dtype=np.float64)
    assert aux.shape[-1] == cfg.n_target_layers * cfg.hidden
    f = linear(aux, W["fc_w"])
    return rnd("context", rms_norm(f, W["hidden_norm_w"], cfg.rms_eps))


def context_kv(cfg: OracleConfig, W: Mapping, ctx: np.ndarray,
               positions: np.ndarray, mode: str = "exact"):
    """[NEURON] "Context KV Injection" step 2: one matmul of ctx against all
    layers' stacked K/V weights, then each layer's keys are k-normed and
    RoPE-encoded at the context's own positions.  Returns per-layer lists of
    K and V, each [n, n_kv_heads, head_dim]."""
    rnd = rounding(mode)
    L, Hkv, d = cfg.n_layers, cfg.n_kv_heads, cfg.head_dim
    fused = np.concatenate(
        [np.concatenate([rnd.weight("wk", W["wk"][l]), rnd.weight("wv", W["wv"][l])], axis=0)
         for l in range(L)], axis=0)              # [L * 2 * Hkv * d, hidden]
    kv = linear(ctx, fused).reshape(ctx.shape[0], L, 2, Hkv, d)
    ks, vs = [], []
    for l in range(L):
        k = rms_norm(kv[:, l, 0], W["k_norm_w"][l], cfg.rms_eps)
        k = apply_rope(k, positions, cfg.rope_theta)
        ks.append(rnd("kv", k))
        vs.append(rnd("kv", kv[:, l, 1]))
    return ks, vs


def write_slots(cache: np.ndarray, slots: np.ndarray, values: np.ndarray,
                page_size: int) -> None:
    """index_put of per-token [Hkv, d] rows into a [pages, Hkv, page, d]
    cache ([NEURON] "Context KV Injection" step 3).  Negative slots are padding
    rows and are skipped (vLLM slot-mapping convention)."""
    slots = np.asarray(slots, dtype=np.int64)
    for r, s in enumerate(slots):
        if s < 0:
            continue
        cache[s // page_size, :, s % page_size, :] = values[r]


def inject_context(cfg: OracleConfig, W: Mapping, aux, positions, slot_mapping,
                   k_caches: Sequence[np.ndarray], v_caches: Sequence[np.ndarray],
                   mode: str = "exact") -> None:
    """precompute_and_store_context_kv ([NEURON] "Context KV Injection"
    steps 1-3): fuse, project, norm + rotate keys, scatter into each layer's
    paged cache at ``slot_mapping``."""
    aux = np.asarray(aux, dtype=np.float64)
    if aux.shape[0] == 0:
        return
    ctx = context_fusion(cfg, W, aux, mode)
    ks, vs = context_kv(cfg, W, ctx, positions, mode)
    for l in range(cfg.n_layers):
        write_slots(k_caches[l], slot_mapping, ks[l], cfg.page_size)
        write_slots(v_caches[l], slot_mapping, vs[l], cfg.page_size)


# ----------------------------------------------------------------------------
# (a5) non-causal block attention over the paged cache
# ----------------------------------------------------------------------------
def gather_kv(cache: np.ndarray, block_table_row, n_keys: int,
              page_size: int) -> np.ndarray:
    """Logical keys 0 .. n_keys-1 of one request, [n_keys, Hkv, d], gathered
    through the request's block-table row with the paged-slot formula."""
    pos = np.arange(n_keys, dtype=np.int64)
    slots = paged_slots(pos, np.zeros(n_keys, dtype=np.int64),
                        np.asarray(block_table_row)[None, :], page_size)
    return cache[slots // page_size, :, slots % page_size, :]


def attention_one_request(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                          n_q_heads: int, n_kv_heads: int) -> np.ndarray:
    """Non-causal attention of every query row over every key
    ([NEURON] "What is DFlash": each query position attends to the injected
    context and the rest of the block; vLLM runs it with causal=False).

    q [nq, Hq, d], k/v [nk, Hkv, d]  ->  o [nq, Hq, d].  Query head h reads
    kv head h // (Hq / Hkv).  Scores scaled by 1/sqrt(d); plain softmax."""
    G = n_q_heads // n_kv_heads
    d = q.shape[-1]
    out = np.empty(q.shape, dtype=np.float64)
    for h in range(n_q_heads):
        kh = k[:, h // G, :]
        vh = v[:, h // G, :]
        s = (q[:, h, :] @ kh.T) / np.sqrt(d)           # [nq, nk]
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ vh
    return out


def block_attention(cfg: OracleConfig, q: np.ndarray, k_cache: np.ndarray,
                    v_cache: np.ndarray, block_table, seq_lens) -> np.ndarray:
    """q [B * bs, Hq, d] for the query blocks -> o [B * bs, Hq, d].  Request b
    sees logical keys [0, seq_len_b + bs): its context plus its whole block."""
    bs = cfg.block_size
    bt = np.asarray(block_table)
    o = np.empty(q.shape, dtype=np.float64)
    for b, n_ctx in enumerate(np.asarray(seq_lens, dtype=np.int64)):
        n_keys = int(n_ctx) + bs
        k = gather_kv(k_cache, bt[b], n_keys, cfg.page_size)
        v = gather_kv(v_cache, bt[b], n_keys, cfg.page_size)
        rows = slice(b * bs, (b + 1) * bs)
        o[rows] = attention_one_request(q[rows], k.astype(np.float64),
                                        v.astype(np.float64),
                                        cfg.n_q_heads, cfg.n_kv_heads)
    return o


# ----------------------------------------------------------------------------
# (a3)-(a7) the proposal forward
# ----------------------------------------------------------------------------
@dataclass
class Proposal:
    draft_tokens: np.ndarray      # [B, K]
    block_tokens: np.ndarray      # [B, bs]  (bonus + drafts)
    logits: np.ndarray            # [B * K, V] float64 (before the float32 pick)
    hidden: np.ndarray            # [B * bs, H] final residual stream (pre final norm)


def draft_layer(cfg: OracleConfig, W: Mapping, l: int, x: np.ndarray,
                qb: QueryBlock, block_table, seq_lens,
                k_cache: np.ndarray, v_cache: np.ndarray,
                rnd: Rounding) -> np.ndarray:
    """One DFlashQwen3DecoderLayer ([NEURON] "DFlash Draft Model
    Architecture": a standard Qwen3 decoder layer, attention + MLP with
    pre-norms, attention run non-causally):

      n  = RMSNorm(x; input_norm)
      q, k, v = Wq n, Wk n, Wv n;  q, k per-head RMSNorm; RoPE at block positions
      block k, v written to the block's paged slots ([NEURON] "Paged KV
      Integration": the same slot helper serves the query block)
      o  = non-causal attention over [0, seq_len + bs)
      x += Wo o
      n2 = RMSNorm(x; post_attention_norm)
      x += Wd (silu(Wg n2) * Wu n2)
    """
    Hq, Hkv, d, eps = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.rms_eps
    M = x.shape[0]
    w = rnd.weight
    n = rnd("norm", rms_norm(x, W["in_norm_w"][l], eps))
    q = linear(n, w("wq", W["wq"][l])).reshape(M, Hq, d)
    k = linear(n, w("wk", W["wk"][l])).reshape(M, Hkv, d)
    v = linear(n, w("wv", W["wv"][l])).reshape(M, Hkv, d)
    q = rnd("q", apply_rope(rms_norm(q, W["q_norm_w"][l], eps), qb.positions,
                            cfg.rope_theta))
    k = rnd("kv", apply_rope(rms_norm(k, W["k_norm_w"][l], eps), qb.positions,
                             cfg.rope_theta))
    v = rnd("kv", v)
    slots = paged_slots(qb.positions, qb.req_ids, block_table, cfg.page_size)
    write_slots(k_cache, slots, k, cfg.page_size)
    write_slots(v_cache, slots, v, cfg.page_size)
    o = rnd("attn_out", block_attention(cfg, q, k_cache, v_cache, block_table, seq_lens))
    x = x + linear(o.reshape(M, Hq * d), w("wo", W["wo"][l]))
    n2 = rnd("norm", rms_norm(x, W["post_norm_w"][l], eps))
    h = rnd("mlp_hidden", silu(linear(n2, w("w_gate", W["w_gate"][l])))
            * linear(n2, w("w_up", W["w_up"][l])))
    return x + linear(h, W["w_down"][l])


def lm_head_logits(W: Mapping, rows: np.ndarray, chunk: int = 16384,
                   weight: Callable = lambda name, w: w) -> np.ndarray:
    """rows @ lm_head^T in float64, a vocabulary chunk at a time."""
    V = W["lm_head"].shape[0]
    out = np.empty((rows.shape[0], V), dtype=np.float64)
    for v0 in range(0, V, chunk):
        out[:, v0:v0 + chunk] = linear(rows, weight("lm_head", W["lm_head"][v0:v0 + chunk]))
    return out


def propose(cfg: OracleConfig, W: Mapping, bonus_tokens, seq_lens, block_table,
            k_caches: Sequence[np.ndarray], v_caches: Sequence[np.ndarray],
            mode: str = "exact") -> Proposal:
    """DFlashQwen3ForCausalLM.forward after injection ([NEURON] code block):
    build [bonus, mask..] blocks, embed with the (aliased) target embedding,
    run the decoder stack non-causally over the injected context, keep slots
    1..bs-1, final RMSNorm, (aliased) target LM head, greedy pick; the block
    output is cat(bonus, drafts).  Writes the block's K/V into the caches."""
    rnd = rounding(mode)
    bonus = np.asarray(bonus_tokens, dtype=np.int64)
    B, bs, K = bonus.shape[0], cfg.block_size, cfg.num_drafts
    qb = build_query_block(bonus, seq_lens, bs, cfg.mask_token_id)
    x = np.asarray(W["embed"])[qb.input_ids].astype(np.float64)
    for l in range(cfg.n_layers):
        x = draft_layer(cfg, W, l, x, qb, block_table, seq_lens,
                        k_caches[l], v_caches[l], rnd)
    kept = x[qb.keep_idx]
    f = rnd("final", rms_norm(kept, W["final_norm_w"], cfg.rms_eps))
    logits = lm_head_logits(W, f, weight=rnd.weight)
    drafts = argmax_f32(logits).reshape(B, K)
    block = np.concatenate([bonus[:, None], drafts], axis=1)
    return Proposal(drafts, block, logits, x)


# ----------------------------------------------------------------------------
# (a8) greedy verification
# ----------------------------------------------------------------------------
@dataclass
class Verification:
    out_tokens: np.ndarray     # [B, K+1], -1 after the bonus
    num_accepted: np.ndarray   # [B]
    bonus: np.ndarray          # [B]


def verify_greedy(drafts, target_logits) -> Verification:
    """Greedy acceptance against the target's predictions.

    Target row j (j = 0..K) predicts the token after block slot j, slot 0
    being the previous bonus token and slot j the draft d_{j-1} (0-based
    d_0..d_{K-1} = drafts[:, 0..K-1]).  Drafts are accepted while
    d_j == argmax T_j; n = number accepted; the bonus token is argmax T_n; the
    emitted row is [d_0 .. d_{n-1}, bonus, -1, ...] of length K+1 — the
    sampler output with rejected slots marked -1 ([NEURON] "Async Rejection
    and Position Correction" counts valid entries as != -1).  The output is
    what plain greedy decoding of the target emits ([QEFF]: verification by
    the frozen target guarantees output identical to standard decoding)."""
    d = np.asarray(drafts, dtype=np.int64)
    B, K = d.shape
    t = argmax_f32(target_logits)                     # [B, K+1]
    assert t.shape == (B, K + 1)
    out = np.full((B, K + 1), -1, dtype=np.int64)
    n_acc = np.zeros(B, dtype=np.int64)
    bonus = np.zeros(B, dtype=np.int64)
    for b in range(B):
        n = 0
        while n < K and d[b, n] == t[b, n]:
            n += 1
        out[b, :n] = d[b, :n]
        out[b, n] = t[b, n]
        n_acc[b] = n
        bonus[b] = t[b, n]
    return Verification(out, n_acc, bonus)


def acceptance_length(num_accepted_tokens: int, num_drafts: int) -> float:
    """[VLLM] compute_acceptance_len: 1 + accepted / drafts (1 if none)."""
    return 1.0 if num_drafts == 0 else 1.0 + num_accepted_tokens / num_drafts


def acceptance_rate(num_accepted_tokens: int, num_draft_tokens: int) -> float:
    """[VLLM] compute_acceptance_rate: accepted / draft tokens (nan if none)."""
    return float("nan") if num_draft_tokens == 0 else \
        num_accepted_tokens / num_draft_tokens


# ----------------------------------------------------------------------------
# helpers for callers
# ----------------------------------------------------------------------------
def empty_caches(cfg: OracleConfig, num_pages: int, dtype=np.float64):
    """Per-layer zeroed K and V pools, [num_pages, Hkv, page, d] each."""
    shape = (num_pages, cfg.n_kv_heads, cfg.page_size, cfg.head_dim)
    return ([np.zeros(shape, dtype=dtype) for _ in range(cfg.n_layers)],
            [np.zeros(shape, dtype=dtype) for _ in range(cfg.n_layers)])


def top2_gap_f32(logits: np.ndarray) -> np.ndarray:
    """Gap between the largest and second-largest float32 logit per row; used
    to flag near-ties whose greedy pick legitimately depends on rounding."""
    f = np.asarray(logits).astype(np.float32).astype(np.float64)
    part = np.partition(f, -2, axis=-1)
    return part[..., -1] - part[..., -2]


# ----------------------------------------------------------------------------
# tensor parallelism across ranks (the next step of the path; exact mode only)
#
# [NEURON] "Context KV Injection": each rank projects and stores "this rank's
# KV heads only"; [NEURON] "DFlashQwen3ForCausalLM": the aliased LM head is a
# column-parallel linear over the vocabulary.  Reading of what the pages leave
# open (the usual column-/row-parallel split of a decoder layer): rank r of S
# holds the contiguous kv heads [r Hkv/S, (r+1) Hkv/S) with their query heads
# (each kv head keeps its own query group) and the MLP features
# [r I/S, (r+1) I/S); the O and down projections are row-parallel, so each
# rank forms a partial sum of the layer's output and the partials are added
# across ranks (an all-reduce) before the residual add.  Every norm, the
# embedding, fc + hidden_norm and the residual stream are replicated.
# ----------------------------------------------------------------------------
@dataclass
class TPSlices:
    q_heads: slice      # query heads of this rank
    kv_heads: slice     # kv heads of this rank
    features: slice     # MLP features of this rank


def tp_slices(cfg: OracleConfig, rank: int, size: int) -> TPSlices:
    """Rank `rank` of `size`: its kv heads, their query heads, its MLP
    features (contiguous blocks); `size` must divide n_kv_heads and intermediate."""
    Hq, Hkv, I = cfg.n_q_heads, cfg.n_kv_heads, cfg.intermediate
    if size < 1 or Hkv % size or I % size or not 0 <= rank < size:
        raise ValueError(f"cannot split {Hkv} kv heads / {I} features over {size} ranks")
    hk, hq, fi = Hkv // size, Hq // size, I // size
    return TPSlices(slice(rank * hq, (rank + 1) * hq), slice(rank * hk, (rank + 1) * hk),
                    slice(rank * fi, (rank + 1) * fi))


def _rows(w: np.ndarray, heads: slice, d: int) -> np.ndarray:
    """The output rows of a [heads * d, in] projection that belong to `heads`."""
    return np.asarray(w)[heads.start * d:heads.stop * d]


def empty_caches_tp(cfg: OracleConfig, num_pages: int, size: int):
    """Per rank, per layer zeroed K and V pools of the rank's kv heads,
    [num_pages, Hkv / size, page, d]."""
    shape = (num_pages, cfg.n_kv_heads // size, cfg.page_size, cfg.head_dim)
    return ([[np.zeros(shape) for _ in range(cfg.n_layers)] for _ in range(size)],
            [[np.zeros(shape) for _ in range(cfg.n_layers)] for _ in range(size)])


def inject_context_tp(cfg: OracleConfig, W: Mapping, aux, positions, slot_mapping,
                      k_caches, v_caches, size: int) -> None:
    """inject_context with each rank projecting and storing its kv heads only
    ([NEURON] "Context KV Injection"); k_caches[r][l] is rank r's layer-l pool."""
    aux = np.asarray(aux, dtype=np.float64)
    if aux.shape[0] == 0:
        return
    d = cfg.head_dim
    ctx = context_fusion(cfg, W, aux, "exact")             # replicated on every rank
    for r in range(size):
        sl = tp_slices(cfg, r, size)
        for l in range(cfg.n_layers):
            k = linear(ctx, _rows(W["wk"][l], sl.kv_heads, d)).reshape(ctx.shape[0], -1, d)
            v = linear(ctx, _rows(W["wv"][l], sl.kv_heads, d)).reshape(ctx.shape[0], -1, d)
            k = apply_rope(rms_norm(k, W["k_norm_w"][l], cfg.rms_eps), positions,
                           cfg.rope_theta)
            write_slots(k_caches[r][l], slot_mapping, k, cfg.page_size)
            write_slots(v_caches[r][l], slot_mapping, v, cfg.page_size)


def draft_layer_tp(cfg: OracleConfig, W: Mapping, l: int, x: np.ndarray, qb: QueryBlock,
                   block_table, seq_lens, k_caches, v_caches, size: int) -> np.ndarray:
    """draft_layer split over `size` ranks: each rank's heads attend over its
    own cache shard, its O and down projections give partial sums, and the
    partials are added across ranks (in rank order) before each residual add."""
    eps, d, M = cfg.rms_eps, cfg.head_dim, x.shape[0]
    n = rms_norm(x, W["in_norm_w"][l], eps)
    attn_parts = []
    for r in range(size):
        sl = tp_slices(cfg, r, size)
        hq, hk = sl.q_heads.stop - sl.q_heads.start, sl.kv_heads.stop - sl.kv_heads.start
        q = linear(n, _rows(W["wq"][l], sl.q_heads, d)).reshape(M, hq, d)
        k = linear(n, _rows(W["wk"][l], sl.kv_heads, d)).reshape(M, hk, d)
        v = linear(n, _rows(W["wv"][l], sl.kv_heads, d)).reshape(M, hk, d)
        q = apply_rope(rms_norm(q, W["q_norm_w"][l], eps), qb.positions, cfg.rope_theta)
        k = apply_rope(rms_norm(k, W["k_norm_w"][l], eps), qb.positions, cfg.rope_theta)
        slots = paged_slots(qb.positions, qb.req_ids, block_table, cfg.page_size)
        write_slots(k_caches[r][l], slots, k, cfg.page_size)
        write_slots(v_caches[r][l], slots, v, cfg.page_size)
        rank_cfg = OracleConfig(**{**cfg.__dict__, "n_q_heads": hq, "n_kv_heads": hk})
        o = block_attention(rank_cfg, q, k_caches[r][l], v_caches[r][l], block_table, seq_lens)
        wo_cols = np.asarray(W["wo"][l])[:, sl.q_heads.start * d:sl.q_heads.stop * d]
        attn_parts.append(linear(o.reshape(M, hq * d), wo_cols))
    x = x + sum(attn_parts)                                  # all-reduce of the O partials
    n2 = rms_norm(x, W["post_norm_w"][l], eps)
    mlp_parts = []
    for r in range(size):
        f = tp_slices(cfg, r, size).features
        h = silu(linear(n2, np.asarray(W["w_gate"][l])[f])) * linear(n2, np.asarray(W["w_up"][l])[f])
        mlp_parts.append(linear(h, np.asarray(W["w_down"][l])[:, f]))
    return x + sum(mlp_parts)                                # all-reduce of the down partials


def propose_tp(cfg: OracleConfig, W: Mapping, bonus_tokens, seq_lens, block_table,
               k_caches, v_caches, size: int, vocab_shards) -> Proposal:
    """propose over `size` ranks: draft_layer_tp for the stack, then the LM
    head over the vocabulary shards [(start, count), ...] (a column-parallel
    linear, [NEURON] "DFlashQwen3ForCausalLM"): each shard's greedy pick (its
    largest float32 logit, lowest id on ties) and the best of those across
    shards (largest value, lowest id on ties)."""
    bonus = np.asarray(bonus_tokens, dtype=np.int64)
    B, bs, K = bonus.shape[0], cfg.block_size, cfg.num_drafts
    qb = build_query_block(bonus, seq_lens, bs, cfg.mask_token_id)
    x = np.asarray(W["embed"])[qb.input_ids].astype(np.float64)
    for l in range(cfg.n_layers):
        x = draft_layer_tp(cfg, W, l, x, qb, block_table, seq_lens, k_caches, v_caches, size)
    f = rms_norm(x[qb.keep_idx], W["final_norm_w"], cfg.rms_eps)
    lm = np.asarray(W["lm_head"])
    parts, picks = [], []
    for start, count in vocab_shards:
        lg = linear(f, lm[start:start + count])
        parts.append(lg)
        loc = argmax_f32(lg)
        picks.append((lg.astype(np.float32)[np.arange(lg.shape[0]), loc], loc + start))
    vals = np.stack([p[0] for p in picks])                   # [shards, rows] float32
    ids = np.stack([p[1] for p in picks])
    vals = np.where(np.isnan(vals), -np.inf, vals)
    best = np.empty(f.shape[0], dtype=np.int64)
    for row in range(f.shape[0]):
        top = vals[:, row].max()
        best[row] = ids[vals[:, row] == top, row].min()
    drafts = best.reshape(B, K)
    block = np.concatenate([bonus[:, None], drafts], axis=1)
    return Proposal(drafts, block, np.concatenate(parts, axis=1), x)
