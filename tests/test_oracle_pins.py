"""Pins of the CPU oracle to things outside itself (no GPU needed).

Each test checks the oracle against a value the pages print (the vLLM worked
example), a library routine (torch, transformers' Qwen3), a closed form, an
invariant of the method, or brute force on tiny inputs — chosen so that a
dropped term, a wrong sign or index, or a transposed operand in the oracle
fails at least one of them.
"""

from __future__ import annotations

import itertools
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O
from block_diffusion_speculative_propose_b200 import synth
from tests._util import weights_np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TINY = synth.model_config("tiny")


def tiny_cfg(**kw):
    c = dict(TINY)
    c.update(kw)
    return c


# ----------------------------------------------------------------------------
# block construction: the worked example printed in the vLLM pull request
# ----------------------------------------------------------------------------
def test_block_construction_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "vllm_block_example.json")))
    M = 777
    qb = O.build_query_block(g["next_token_ids"], g["seq_lens"], g["block_size"], M)
    ids = [M if v == g["mask_placeholder"] else v for v in g["expected_input_ids"]]
    assert qb.input_ids.tolist() == ids
    assert qb.positions.tolist() == g["expected_query_positions"]
    assert qb.keep_idx.tolist() == g["expected_token_indices_to_sample"]
    assert qb.query_start_loc.tolist() == g["expected_query_start_loc"]
    assert int(np.diff(qb.query_start_loc).max()) == g["expected_max_query_len"]


# ----------------------------------------------------------------------------
# paged slots
# ----------------------------------------------------------------------------
def test_paged_gather_equals_page_copy():
    """Writing a logical sequence into a shuffled pool page by page (block
    copies through the table) and gathering it back through the slot formula
    returns the logical sequence."""
    rng = np.random.default_rng(0)
    P, W, num_pages, Hkv, d = 16, 7, 20, 2, 4
    table = rng.permutation(num_pages)[:W].reshape(1, W)
    logical = rng.standard_normal((W * P, Hkv, d))
    pool = np.zeros((num_pages, Hkv, P, d))
    for j in range(W):
        pool[table[0, j]] = logical[j * P:(j + 1) * P].transpose(1, 0, 2)
    for n in (1, 15, 16, 17, W * P):
        got = O.gather_kv(pool, table[0], n, P)
        np.testing.assert_array_equal(got, logical[:n])


def test_paged_slots_clamp_and_requests():
    """Two requests with their own rows; positions past the table clamp onto
    the row's last page, as the slot helper's formula states."""
    P = 16
    table = np.array([[5, 2, 9], [7, 1, 3]])
    pos = np.array([0, 15, 16, 33, 47, 48, 100, 0, 20, 47])
    req = np.array([0, 0, 0, 0, 0, 0, 0, 1, 1, 1])
    got = O.paged_slots(pos, req, table, P)
    want = [80, 95, 32, 145, 159, 144, 148, 112, 20, 63]
    assert got.tolist() == want


# ----------------------------------------------------------------------------
# elementary operations against torch
# ----------------------------------------------------------------------------
def test_rms_norm_matches_torch_and_closed_form():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 64))
    w = 1 + 0.1 * rng.standard_normal(64)
    ref = F.rms_norm(torch.tensor(x), (64,), torch.tensor(w), eps=1e-6).numpy()
    np.testing.assert_allclose(O.rms_norm(x, w, 1e-6), ref, rtol=1e-13, atol=1e-13)
    # constant vector c: y = c / sqrt(c^2 + eps) * w
    c = 3.0
    y = O.rms_norm(np.full(8, c), np.arange(1, 9, dtype=float), 1e-6)
    np.testing.assert_allclose(y, c / np.sqrt(c * c + 1e-6) * np.arange(1, 9), rtol=1e-15)


def test_silu_matches_torch():
    x = np.linspace(-30, 30, 601)
    np.testing.assert_allclose(O.silu(x), F.silu(torch.tensor(x)).numpy(), rtol=1e-14,
                               atol=1e-300)
    assert O.silu(np.zeros(1))[0] == 0.0


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.standard_normal(10000) * 10.0 ** rng.integers(-8, 8, 10000),
                        # exact ties between two bf16 neighbours
                        (np.arange(1, 200, dtype=np.float64) * 2 + 1) * 2.0 ** -8])
    ref = torch.tensor(x, dtype=torch.float64).float().to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(O.round_bf16(x), ref)


def test_round_fp16_matches_torch():
    rng = np.random.default_rng(14)
    x = np.concatenate([rng.standard_normal(10000) * 10.0 ** rng.integers(-9, 6, 10000),
                        [70000.0, -1e6, 6.1e-5, 3e-8, 65504.0, 65520.0]])
    ref = torch.tensor(x, dtype=torch.float64).float().to(torch.float16).double().numpy()
    np.testing.assert_array_equal(O.round_fp16(x), ref)


def test_storage_modes():
    """device mode rounds each storage point to its declared format; weights
    multiplied in fp16 are fp16-rounded; exact mode leaves values alone."""
    x = np.array([1.0 + 2.0 ** -9, 1.0 + 2.0 ** -12, 3.0e-6])
    dev, ex, b16 = O.rounding("device"), O.rounding("exact"), O.rounding("bf16")
    for point, fmt in O.STORAGE_POINTS.items():
        want = O.round_fp16(x) if fmt == "fp16" else O.round_bf16(x)
        np.testing.assert_array_equal(dev(point, x), want)
        np.testing.assert_array_equal(b16(point, x), O.round_bf16(x))
        np.testing.assert_array_equal(ex(point, x), x)
    np.testing.assert_array_equal(dev.weight("lm_head", x), O.round_fp16(x))
    np.testing.assert_array_equal(dev.weight("fc_w", x), x)
    np.testing.assert_array_equal(dev.weight("w_down", x), x)


def test_argmax_ties_and_nan():
    rng = np.random.default_rng(3)
    a = rng.integers(0, 4, (200, 9)).astype(np.float32)  # many ties
    np.testing.assert_array_equal(O.argmax_f32(a), torch.argmax(torch.tensor(a), -1).numpy())
    row = np.array([np.nan, 1.0, 5.0, np.nan, 5.0], dtype=np.float32)
    assert O.argmax_f32(row) == 2
    assert O.argmax_f32(np.array([np.nan, -np.inf, np.nan], dtype=np.float32)) == 0


# ----------------------------------------------------------------------------
# RoPE
# ----------------------------------------------------------------------------
def test_rope_two_dim_rotation():
    """d = 2: a single pair rotated by pos * theta^0 = pos radians."""
    x = np.array([[0.3, -1.7]])
    for pos in (0, 1, 5, 1234):
        got = O.apply_rope(x, np.array([pos]), 1e6)
        c, s = np.cos(pos), np.sin(pos)
        np.testing.assert_allclose(got, [[0.3 * c + 1.7 * s, -1.7 * c + 0.3 * s]], rtol=1e-13)


def test_rope_matches_transformers_and_relative_invariance():
    from transformers.models.qwen3.modeling_qwen3 import (Qwen3RotaryEmbedding,
                                                          apply_rotary_pos_emb)
    from tests._hf import qwen3_config
    for d in (64, 128):
        cfg = tiny_cfg(head_dim=d)
        rot = Qwen3RotaryEmbedding(qwen3_config(cfg))
        # the library evaluates inverse frequencies and angles in float32
        np.testing.assert_allclose(O.rope_inv_freq(d, 1e6), rot.inv_freq.double().numpy(),
                                   rtol=2e-7)
        rng = np.random.default_rng(d)
        for pos, tol in ((np.array([0, 1, 2, 7]), 2e-6),
                         (np.array([300, 4095, 32767]), 1e-2)):
            q = rng.standard_normal((len(pos), 3, d))
            cos, sin = rot(torch.zeros(1, dtype=torch.float32), torch.tensor(pos)[None])
            qt = torch.tensor(q).permute(1, 0, 2)[None]             # [1, heads, n, d]
            ref, _ = apply_rotary_pos_emb(qt, qt, cos.double(), sin.double())
            ref = ref[0].permute(1, 0, 2).numpy()
            np.testing.assert_allclose(O.apply_rope(q, pos, 1e6), ref, rtol=tol, atol=tol)
    # q_m . k_n depends only on m - n; pair norms are preserved
    rng = np.random.default_rng(9)
    q, k = rng.standard_normal((1, 64)), rng.standard_normal((1, 64))
    dots = [(O.apply_rope(q, np.array([m]), 1e6) @ O.apply_rope(k, np.array([m - 5]), 1e6).T).item()
            for m in (5, 6, 100, 9000)]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-9)
    r = O.apply_rope(q, np.array([77]), 1e6)
    np.testing.assert_allclose(r[:, :32] ** 2 + r[:, 32:] ** 2, q[:, :32] ** 2 + q[:, 32:] ** 2,
                               rtol=1e-12)


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------
def _sdpa(q, k, v, G):
    """torch scaled_dot_product_attention, non-causal, kv heads repeated."""
    qt = torch.tensor(q).permute(1, 0, 2)[None]
    kt = torch.tensor(k).permute(1, 0, 2).repeat_interleave(G, 0)[None]
    vt = torch.tensor(v).permute(1, 0, 2).repeat_interleave(G, 0)[None]
    o = F.scaled_dot_product_attention(qt, kt, vt, is_causal=False)
    return o[0].permute(1, 0, 2).numpy()


def test_attention_matches_sdpa():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((16 * 1, 8, 64))
    k = rng.standard_normal((300, 2, 64)) * 2
    v = rng.standard_normal((300, 2, 64))
    np.testing.assert_allclose(O.attention_one_request(q, k, v, 8, 2), _sdpa(q, k, v, 4),
                               rtol=1e-10, atol=1e-12)


def _random_pool(rng, cfg, seq_lens, extra_pages=3):
    P, bs = cfg["page_size"], cfg["block_size"]
    need = [-(-(s + bs) // P) for s in seq_lens]
    W = max(need) + 1
    num_pages = sum(need) + extra_pages
    perm = rng.permutation(num_pages)
    table = np.zeros((len(seq_lens), W), dtype=np.int64)
    cur = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[cur:cur + n]
        cur += n
    shape = (num_pages, cfg["n_kv_heads"], P, cfg["head_dim"])
    return table, rng.standard_normal(shape), rng.standard_normal(shape)


def test_block_attention_bs1_is_decode_attention():
    """block_size 1: each request has one query over its seq_len + 1 keys —
    ordinary single-query decode attention."""
    cfg = O.OracleConfig.from_mapping(tiny_cfg(block_size=1))
    rng = np.random.default_rng(5)
    seq_lens = [0, 5, 16, 40]
    table, kc, vc = _random_pool(rng, tiny_cfg(block_size=1), seq_lens)
    q = rng.standard_normal((len(seq_lens), cfg.n_q_heads, cfg.head_dim))
    o = O.block_attention(cfg, q, kc, vc, table, seq_lens)
    G = cfg.n_q_heads // cfg.n_kv_heads
    for b, s in enumerate(seq_lens):
        k = O.gather_kv(kc, table[b], s + 1, 16)
        v = O.gather_kv(vc, table[b], s + 1, 16)
        np.testing.assert_allclose(o[b:b + 1], _sdpa(q[b:b + 1], k, v, G), rtol=1e-10,
                                   atol=1e-12)


def test_block_attention_invariances():
    cfg_d = tiny_cfg()
    cfg = O.OracleConfig.from_mapping(cfg_d)
    rng = np.random.default_rng(6)
    seq_lens = [3, 33, 64]
    table, kc, vc = _random_pool(rng, cfg_d, seq_lens)
    q = rng.standard_normal((len(seq_lens) * cfg.block_size, cfg.n_q_heads, cfg.head_dim))
    o = O.block_attention(cfg, q, kc, vc, table, seq_lens)
    # (1) physical page shuffle + table update: bitwise identical
    perm = rng.permutation(kc.shape[0])
    inv = np.argsort(perm)
    o2 = O.block_attention(cfg, q, kc[perm], vc[perm], inv[table], seq_lens)
    np.testing.assert_array_equal(o, o2)
    # (2) non-causal: permuting the logical order of (k, v) pairs changes nothing
    b, s = 1, seq_lens[1]
    n = s + cfg.block_size
    k = O.gather_kv(kc, table[b], n, 16)
    v = O.gather_kv(vc, table[b], n, 16)
    p = rng.permutation(n)
    rows = slice(b * cfg.block_size, (b + 1) * cfg.block_size)
    a1 = O.attention_one_request(q[rows], k, v, cfg.n_q_heads, cfg.n_kv_heads)
    a2 = O.attention_one_request(q[rows], k[p], v[p], cfg.n_q_heads, cfg.n_kv_heads)
    np.testing.assert_allclose(a1, a2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(o[rows], a1, rtol=1e-13, atol=1e-14)
    # (3) identical keys: softmax is uniform, output is the mean of V
    k_same = np.repeat(k[:1], n, axis=0)
    a3 = O.attention_one_request(q[rows], k_same, v, cfg.n_q_heads, cfg.n_kv_heads)
    G = cfg.n_q_heads // cfg.n_kv_heads
    for h in range(cfg.n_q_heads):
        np.testing.assert_allclose(a3[:, h], np.broadcast_to(v[:, h // G].mean(0), a3[:, h].shape),
                                   rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------
# injection against library routines
# ----------------------------------------------------------------------------
def _tiny_weights(seed=0, **over):
    cfg = tiny_cfg(**over)
    W = weights_np(synth.make_weights(cfg, seed=seed))
    return cfg, W


def test_context_fusion_matches_torch():
    cfg, W = _tiny_weights()
    oc = O.OracleConfig.from_mapping(cfg)
    aux = np.random.default_rng(7).standard_normal((9, 3 * 256))
    ref = F.rms_norm(F.linear(torch.tensor(aux), torch.tensor(W["fc_w"], dtype=torch.float64)),
                     (256,), torch.tensor(W["hidden_norm_w"], dtype=torch.float64), eps=1e-6)
    np.testing.assert_allclose(O.context_fusion(oc, W, aux), ref.numpy(), rtol=1e-12,
                               atol=1e-13)


def test_context_kv_matches_qwen3_attention_modules():
    """Injected K/V of every layer equal transformers' Qwen3Attention k/v path
    (k_proj -> per-head k_norm -> RoPE at the context position; v_proj)
    applied to the context vector, layer by layer."""
    from transformers.models.qwen3.modeling_qwen3 import (Qwen3RotaryEmbedding,
                                                          apply_rotary_pos_emb)
    from tests._hf import qwen3_config, qwen3_from_draft_weights
    cfg, W = _tiny_weights(seed=3)
    oc = O.OracleConfig.from_mapping(cfg)
    rng = np.random.default_rng(8)
    ctx = rng.standard_normal((11, cfg["hidden"]))
    # small positions: the library's float32 angles are exact to ~1e-6 there
    pos = rng.integers(0, 8, 11)
    ks, vs = O.context_kv(oc, W, ctx, pos)
    m = qwen3_from_draft_weights(cfg, W)
    rot = Qwen3RotaryEmbedding(qwen3_config(cfg))
    cos, sin = rot(torch.zeros(1, dtype=torch.float32), torch.tensor(pos)[None])
    cos, sin = cos.double(), sin.double()
    c = torch.tensor(ctx)
    with torch.no_grad():
        for l, layer in enumerate(m.model.layers):
            a = layer.self_attn
            k = a.k_norm(a.k_proj(c).view(11, cfg["n_kv_heads"], cfg["head_dim"]))
            kt = k.permute(1, 0, 2)[None]
            _, kr = apply_rotary_pos_emb(kt, kt, cos, sin)
            np.testing.assert_allclose(ks[l], kr[0].permute(1, 0, 2).numpy(), rtol=5e-6,
                                       atol=5e-6)
            v = a.v_proj(c).view(11, cfg["n_kv_heads"], cfg["head_dim"]).numpy()
            np.testing.assert_allclose(vs[l], v, rtol=1e-12, atol=1e-13)


def test_inject_scatter_and_padding_rows():
    cfg, W = _tiny_weights(seed=4)
    oc = O.OracleConfig.from_mapping(cfg)
    rng = np.random.default_rng(10)
    n = 21
    aux = rng.standard_normal((n, 768))
    pos = np.arange(n) + 40
    table = rng.permutation(12)[:6].reshape(1, 6)
    slots = O.paged_slots(pos, np.zeros(n, dtype=np.int64), table, 16)
    slots[[3, 9]] = -1                                  # padding rows
    kc, vc = O.empty_caches(oc, 12)
    O.inject_context(oc, W, aux, pos, slots, kc, vc)
    ctx = O.context_fusion(oc, W, aux)
    ks, vs = O.context_kv(oc, W, ctx, pos)
    for l in range(oc.n_layers):
        got_k = O.gather_kv(kc[l], table[0], 40 + n, 16)[40:]
        got_v = O.gather_kv(vc[l], table[0], 40 + n, 16)[40:]
        keep = np.ones(n, bool)
        keep[[3, 9]] = False
        np.testing.assert_array_equal(got_k[keep], ks[l][keep])
        np.testing.assert_array_equal(got_v[keep], vs[l][keep])
        assert not got_k[~keep].any() and not got_v[~keep].any()


# ----------------------------------------------------------------------------
# the draft stack against transformers' Qwen3
# ----------------------------------------------------------------------------
def test_propose_without_context_is_noncausal_qwen3():
    """seq_len = 0: the block attends only to itself, so the DFlash forward is
    a Qwen3 decoder stack + final norm + LM head run non-causally over the
    block at positions 0..bs-1."""
    from tests._hf import full_mask, qwen3_from_draft_weights
    cfg, W = _tiny_weights(seed=5, block_size=6)
    oc = O.OracleConfig.from_mapping(cfg)
    bonus = np.array([17, 900])
    table = np.array([[0], [1]])
    kc, vc = O.empty_caches(oc, 2)
    prop = O.propose(oc, W, bonus, [0, 0], table, kc, vc)
    m = qwen3_from_draft_weights(cfg, W)
    for b in range(2):
        ids = torch.tensor([[int(bonus[b])] + [cfg["mask_token_id"]] * 5])
        with torch.no_grad():
            out = m(input_ids=ids, attention_mask=full_mask(6, 6),
                    position_ids=torch.arange(6)[None]).logits[0].numpy()
        # the library's RoPE angles are float32 (~1e-7 here)
        np.testing.assert_allclose(prop.logits[b * 5:(b + 1) * 5], out[1:], rtol=1e-5,
                                   atol=1e-6)
        # and the HF model with its default causal mask differs (non-causality matters)
        with torch.no_grad():
            causal = m(input_ids=ids, position_ids=torch.arange(6)[None]).logits[0].numpy()
        assert np.abs(causal[1:] - out[1:]).max() > 1e-3


def test_propose_one_layer_with_context_matches_qwen3():
    """One draft layer with unit input-norm and hidden-norm weights: the
    context vector c has unit RMS, so the layer's own input RMSNorm leaves it
    unchanged (up to eps) and the injected K/V equal those a Qwen3 layer
    computes from hidden state c.  The block rows of a Qwen3 model run on
    [c_0..c_{n-1}, embed(block)] with nothing masked then equal the proposal."""
    from tests._hf import full_mask, qwen3_from_draft_weights
    cfg, W = _tiny_weights(seed=6, n_layers=1, block_size=5)
    W["in_norm_w"] = [np.ones(cfg["hidden"], dtype=np.float32)]
    W["hidden_norm_w"] = np.ones(cfg["hidden"], dtype=np.float32)
    oc = O.OracleConfig.from_mapping(cfg)
    rng = np.random.default_rng(11)
    n = 37
    aux = rng.standard_normal((n, 768))
    table = np.array([[4, 0, 3, 1]])
    kc, vc = O.empty_caches(oc, 6)
    pos = np.arange(n)
    O.inject_context(oc, W, aux, pos, O.paged_slots(pos, np.zeros(n, np.int64), table, 16),
                     kc, vc)
    prop = O.propose(oc, W, [321], [n], table, kc, vc)
    ctx = O.context_fusion(oc, W, aux)
    m = qwen3_from_draft_weights(cfg, W)
    emb = W["embed"][[321] + [cfg["mask_token_id"]] * 4].astype(np.float64)
    inp = torch.tensor(np.concatenate([ctx, emb]))[None]
    with torch.no_grad():
        out = m(inputs_embeds=inp, attention_mask=full_mask(n + 5, n + 5),
                position_ids=torch.arange(n + 5)[None]).logits[0].numpy()
    ref = out[n + 1:]
    assert np.linalg.norm(prop.logits - ref) / np.linalg.norm(ref) < 2e-5


# ----------------------------------------------------------------------------
# greedy verification
# ----------------------------------------------------------------------------
def _greedy_emit(drafts, targets):
    """Sequential greedy decoding with the drafts as guesses: the target emits
    its greedy token at each step; decoding past a step is only trusted while
    the guess for that step was right."""
    out = []
    for j, t in enumerate(targets):
        out.append(t)
        if j == len(drafts) or drafts[j] != t:
            break
    return out


def test_verify_brute_force_tiny():
    V, K = 3, 2
    for d in itertools.product(range(V), repeat=K):
        for t in itertools.product(range(V), repeat=K + 1):
            logits = np.full((1, K + 1, V), -1.0, dtype=np.float32)
            for j, tj in enumerate(t):
                logits[0, j, tj] = 2.0
            r = O.verify_greedy(np.array([d]), logits)
            emit = _greedy_emit(d, t)
            n = len(emit) - 1
            assert r.num_accepted[0] == n
            assert r.bonus[0] == emit[-1]
            assert r.out_tokens[0].tolist() == emit + [-1] * (K + 1 - len(emit))


def test_verify_special_cases_and_metrics():
    rng = np.random.default_rng(12)
    B, K, V = 4, 5, 50
    logits = rng.standard_normal((B, K + 1, V)).astype(np.float32)
    t = logits.argmax(-1)
    full = O.verify_greedy(t[:, :K], logits)             # drafts = target argmaxes
    assert (full.num_accepted == K).all() and (full.bonus == t[:, K]).all()
    none = O.verify_greedy((t[:, :K] + 1) % V, logits)    # first draft wrong
    assert (none.num_accepted == 0).all() and (none.bonus == t[:, 0]).all()
    assert (none.out_tokens[:, 1:] == -1).all()
    tie = np.zeros((1, 2, 4), dtype=np.float32)
    tie[0, :, 1] = tie[0, :, 3] = 1.0                     # tie -> lowest index
    assert O.verify_greedy(np.array([[1]]), tie).num_accepted[0] == 1
    assert O.verify_greedy(np.array([[3]]), tie).num_accepted[0] == 0
    # acceptance metrics as the vLLM helpers define them
    acc = int(full.num_accepted.sum())
    assert O.acceptance_length(acc, B) == 1 + K
    assert O.acceptance_rate(acc, B * K) == 1.0
    assert O.acceptance_length(0, 0) == 1.0


# ----------------------------------------------------------------------------
# end to end: speculative decoding with the oracle drafter is lossless
# ----------------------------------------------------------------------------
def _target_forward(model, tokens):
    with torch.no_grad():
        out = model(input_ids=torch.tensor([tokens]), output_hidden_states=True)
    hs = out.hidden_states
    aux = torch.cat([hs[0][0], hs[1][0], hs[2][0]], dim=-1).numpy()
    return out.logits[0].numpy(), aux


@pytest.mark.parametrize("drafter", ["dflash", "true_continuation"])
def test_speculative_loop_is_lossless(drafter):
    """A tiny random Qwen3 target (2 layers, 3 tapped states) decodes greedily;
    the DFlash loop (inject accepted rows -> propose -> target verifies the
    block -> greedy acceptance) must emit exactly the same tokens.  With the
    target's true continuation as drafts every block is fully accepted."""
    from tests._hf import random_target
    cfg = tiny_cfg(block_size=5)
    oc = O.OracleConfig.from_mapping(cfg)
    target = random_target(cfg, n_layers=2, seed=1)
    W = weights_np(synth.make_weights(cfg, seed=2))
    W["embed"] = target.model.embed_tokens.weight.detach().numpy().astype(np.float32)
    W["lm_head"] = target.lm_head.weight.detach().numpy().astype(np.float32)
    rng = np.random.default_rng(13)
    prompt = rng.integers(0, cfg["mask_token_id"], 12).tolist()
    N = 30
    ref = list(prompt)
    for _ in range(N + oc.block_size):
        logits, _ = _target_forward(target, ref)
        ref.append(int(O.argmax_f32(logits[-1])))
    ref_new = ref[len(prompt):]

    table = rng.permutation(8)[:5].reshape(1, 5)
    kc, vc = O.empty_caches(oc, 8)

    def inject(aux_rows, start):
        pos = np.arange(start, start + len(aux_rows))
        O.inject_context(oc, W, aux_rows, pos,
                         O.paged_slots(pos, np.zeros(len(pos), np.int64), table, 16), kc, vc)

    tokens = list(prompt)
    logits, aux = _target_forward(target, tokens)
    inject(aux, 0)
    seq_len = len(tokens)
    bonus = int(O.argmax_f32(logits[-1]))
    emitted = [bonus]
    accepted_total = blocks = 0
    while len(emitted) < N:
        if drafter == "dflash":
            drafts = O.propose(oc, W, [bonus], [seq_len], table, kc, vc).draft_tokens[0]
        else:
            drafts = np.array(ref_new[len(emitted):len(emitted) + oc.num_drafts])
        logits, aux = _target_forward(target, tokens + [bonus] + drafts.tolist())
        T = logits[len(tokens):len(tokens) + oc.block_size][None]
        r = O.verify_greedy(drafts[None], T)
        n = int(r.num_accepted[0])
        inject(aux[len(tokens):len(tokens) + n + 1], seq_len)
        tokens += [bonus] + drafts[:n].tolist()
        seq_len += n + 1
        assert seq_len == len(tokens)
        bonus = int(r.bonus[0])
        emitted += drafts[:n].tolist() + [bonus]
        accepted_total += n
        blocks += 1
    assert emitted[:N] == ref_new[:N]
    if drafter == "true_continuation":
        assert accepted_total >= oc.num_drafts * (blocks - 1)
