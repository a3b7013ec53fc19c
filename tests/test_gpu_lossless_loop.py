"""The whole speculative loop on the device is lossless (QEfficient PR
"Dflash: Block Diffusion Speculative Decoding": output identical to standard
decoding; "DFlash Speculative Decoding in the vLLM Neuron Framework",
§Target Auxiliary Hidden State Extraction for the capture convention).

A small causal target model runs on the GPU (the library's dflash_target_*):
it returns its logits and the pre-layer residual states of the capture layers
(the draft checkpoint's target_layer_ids plus one), concatenated, as the
injection input.  The loop — target forward over [bonus, drafts] -> greedy
verification -> injection of the accepted rows -> proposal of the next block —
must emit exactly the target's own greedy continuation, computed by decoding
one token at a time.  The target's rows are reduced in a fixed order, so the
two agree bit for bit by construction; and the target itself is pinned to
transformers' Qwen3 model in float64 on the same weights (logits, captured
states, greedy continuation), the library model that also pins the oracle's
own lossless loop.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from block_diffusion_speculative_propose_b200 import (DFlash, TargetModel, aux_capture_layers,
                                                      paged_slots, synth, verify_greedy)
from tests._util import rel_l2, to_np, weights_to

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TARGET_LAYERS = 4
TARGET_LAYER_IDS = [0, 1, 2]        # draft checkpoint ids: the state after layers 0, 1, 2
MAX_LEN = 160


def _setup():
    dcfg = dict(synth.model_config("tiny"), target_layer_ids=TARGET_LAYER_IDS)
    tcfg = synth.target_config(dcfg, TARGET_LAYERS)
    Wt = synth.make_target_weights(tcfg, seed=3)
    Wd = synth.make_weights(dcfg, seed=4)
    Wd["embed"] = Wt["embed"].to(torch.bfloat16)     # aliased from the target (exact)
    Wd["lm_head"] = Wt["lm_head"].to(torch.bfloat16)
    cap = aux_capture_layers(TARGET_LAYER_IDS, TARGET_LAYERS)
    return dcfg, tcfg, Wt, Wd, cap


def _hf_target(tcfg, Wt):
    from tests._hf import qwen3_from_draft_weights
    Wn = {k: ([to_np(x) for x in v] if isinstance(v, list) else to_np(v)) for k, v in Wt.items()}
    return qwen3_from_draft_weights(dict(tcfg, n_layers=TARGET_LAYERS), Wn)


def _hf_forward(model, tokens, capture):
    """Logits and the pre-layer residual states at the capture layers
    (layer j < L: the input of decoder layer j; L: the input of the final norm)."""
    states = {}
    hooks = [layer.register_forward_pre_hook(
        lambda mod, args, j=j: states.__setitem__(j, args[0][0].detach().clone()))
        for j, layer in enumerate(model.model.layers)]
    hooks.append(model.model.norm.register_forward_pre_hook(
        lambda mod, args: states.__setitem__(TARGET_LAYERS, args[0][0].detach().clone())))
    try:
        with torch.no_grad():
            out = model(input_ids=torch.tensor([tokens]))
    finally:
        for h in hooks:
            h.remove()
    aux = torch.cat([states[j] for j in capture], dim=-1).numpy()
    return out.logits[0].numpy(), aux


def _argmax(logits_row) -> int:
    return int(torch.argmax(logits_row).item())


def test_target_matches_library_model():
    """The device target equals transformers' Qwen3 (float64) on its weights:
    logits and captured states to fp32 accuracy, over a prompt and then one
    more token at a time (the cache path)."""
    dcfg, tcfg, Wt, Wd, cap = _setup()
    assert cap == [1, 2, 3]
    tm = TargetModel(tcfg, weights_to(Wt, DEV), cap, MAX_LEN)
    try:
        model = _hf_target(tcfg, Wt)
        rng = np.random.default_rng(5)
        toks = rng.integers(0, dcfg["vocab"] - 1, 20).tolist()
        lo, ax = tm.forward(torch.tensor(toks[:17], dtype=torch.int32, device=DEV), 0)
        lo2, ax2 = tm.forward(torch.tensor(toks[17:], dtype=torch.int32, device=DEV), 17)
        torch.cuda.synchronize()
        assert tm.check_device_errors() == 0
        ref_lo, ref_ax = _hf_forward(model, toks, cap)
        g_lo = np.concatenate([to_np(lo), to_np(lo2)])
        g_ax = np.concatenate([to_np(ax), to_np(ax2)]).astype(np.float64)
        for r in range(len(toks)):
            assert rel_l2(g_lo[r], ref_lo[r]) < 1e-5, r
        # captured states are stored in bf16: within half a bf16 ulp of the reference
        assert np.all(np.abs(g_ax - ref_ax) <= 2.0 ** -8 * np.abs(ref_ax) + 1e-6)
    finally:
        tm.close()


def _gpu_greedy(tcfg, Wt, cap, prompt, N):
    tm = TargetModel(tcfg, weights_to(Wt, DEV), cap, MAX_LEN)
    try:
        lo, _ = tm.forward(torch.tensor(prompt, dtype=torch.int32, device=DEV), 0)
        out = [_argmax(lo[-1])]
        pos = len(prompt)
        while len(out) < N:
            lo, _ = tm.forward(torch.tensor([out[-1]], dtype=torch.int32, device=DEV), pos)
            pos += 1
            out.append(_argmax(lo[-1]))
        assert tm.check_device_errors() == 0
        return out
    finally:
        tm.close()


def _pool(dcfg, n_pages, seed):
    rng = np.random.default_rng(seed)
    table = torch.tensor(rng.permutation(n_pages + 2)[:n_pages].reshape(1, n_pages),
                         dtype=torch.int32, device=DEV)
    shape = (n_pages + 2, dcfg["n_kv_heads"], dcfg["page_size"], dcfg["head_dim"])
    kc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV) for _ in range(dcfg["n_layers"])]
    vc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV) for _ in range(dcfg["n_layers"])]
    return table, kc, vc


def _inject(h, aux_rows, start, table, kc, vc, P):
    n = aux_rows.shape[0]
    pos = torch.arange(start, start + n, dtype=torch.int64, device=DEV)
    req = torch.zeros(n, dtype=torch.int64, device=DEV)
    h.inject_context(aux_rows.contiguous(), pos, paged_slots(pos, req, table, P), kc, vc)


def test_speculative_loop_on_device_is_lossless():
    dcfg, tcfg, Wt, Wd, cap = _setup()
    K, P, V = dcfg["block_size"] - 1, dcfg["page_size"], dcfg["vocab"]
    rng = np.random.default_rng(13)
    prompt = rng.integers(0, dcfg["mask_token_id"], 12).tolist()
    N = 48
    ref = _gpu_greedy(tcfg, Wt, cap, prompt, N + K + 1)

    # the same continuation from transformers' Qwen3 in float64 (one full
    # forward per token), compared up to its first near-tie
    model = _hf_target(tcfg, Wt)
    toks = list(prompt)
    lib_ref, gaps = [], []
    for _ in range(N):
        lg, _ = _hf_forward(model, toks, cap)
        gaps.append(float(O.top2_gap_f32(lg[-1][None])[0]))
        lib_ref.append(int(O.argmax_f32(lg[-1])))
        toks.append(lib_ref[-1])
    first_tie = next((i for i, g in enumerate(gaps) if g < 1e-4), N)
    assert first_tie >= 24
    upto = min(first_tie + 1, N)
    assert ref[:upto] == lib_ref[:upto]

    h = DFlash(dcfg, weights_to(Wd, DEV), max_position=MAX_LEN + 64)
    tm = TargetModel(tcfg, weights_to(Wt, DEV), cap, MAX_LEN)
    try:
        table, kc, vc = _pool(dcfg, MAX_LEN // P + 2, seed=7)
        lo, aux = tm.forward(torch.tensor(prompt, dtype=torch.int32, device=DEV), 0)
        _inject(h, aux, 0, table, kc, vc, P)
        seq_len = len(prompt)
        bonus = _argmax(lo[-1])
        emitted = [bonus]
        blocks = accepted = 0
        while len(emitted) < N:
            drafts = h.propose(torch.tensor([bonus], dtype=torch.int32, device=DEV),
                               torch.tensor([seq_len], dtype=torch.int32, device=DEV), table,
                               kc, vc)
            blk = torch.cat([torch.tensor([bonus], dtype=torch.int32, device=DEV),
                             drafts.reshape(-1)])
            lo, aux = tm.forward(blk, seq_len)
            out_tok, n_acc, new_bonus = verify_greedy(drafts, lo.view(1, K + 1, V))
            n = int(n_acc[0])
            _inject(h, aux[:n + 1], seq_len, table, kc, vc, P)
            seq_len += n + 1
            emitted += to_np(drafts)[0, :n].tolist() + [int(new_bonus[0])]
            assert to_np(out_tok)[0, :n + 1].tolist() == emitted[-(n + 1):]
            bonus = int(new_bonus[0])
            blocks += 1
            accepted += n
        torch.cuda.synchronize()
        assert h.check_device_errors() == 0 and tm.check_device_errors() == 0
        assert emitted[:N] == ref[:N]
        # the drafter is untrained, but greedy acceptance still takes some drafts
        print(f"lossless loop: {blocks} blocks, {accepted} drafts accepted")
    finally:
        tm.close()
        h.close()


def test_step_graph_loop_on_device_is_lossless():
    """The same loop with the library's whole-step CUDA graph (verify ->
    prepare -> inject all verified rows -> propose) replayed on the target's
    outputs, which the target writes straight into the graph's input buffers."""
    dcfg, tcfg, Wt, Wd, cap = _setup()
    K, P, V, T, H = (dcfg["block_size"] - 1, dcfg["page_size"], dcfg["vocab"],
                     dcfg["n_target_layers"], dcfg["hidden"])
    rng = np.random.default_rng(17)
    prompt = rng.integers(0, dcfg["mask_token_id"], 9).tolist()
    N = 40
    ref = _gpu_greedy(tcfg, Wt, cap, prompt, N + K + 1)
    h = DFlash(dcfg, weights_to(Wd, DEV), max_position=MAX_LEN + 64)
    tm = TargetModel(tcfg, weights_to(Wt, DEV), cap, MAX_LEN)
    try:
        table, kc, vc = _pool(dcfg, MAX_LEN // P + 2, seed=9)
        lo, aux = tm.forward(torch.tensor(prompt, dtype=torch.int32, device=DEV), 0)
        _inject(h, aux, 0, table, kc, vc, P)
        seq_len = len(prompt)
        bonus = _argmax(lo[-1])
        drafts0 = h.propose(torch.tensor([bonus], dtype=torch.int32, device=DEV),
                            torch.tensor([seq_len], dtype=torch.int32, device=DEV), table,
                            kc, vc)
        # the graph's input buffers, rewritten in place every iteration
        prev_drafts = drafts0.clone()
        logits_in = torch.empty(1, K + 1, V, dtype=torch.float32, device=DEV)
        aux_in = torch.empty(K + 1, T * H, dtype=torch.bfloat16, device=DEV)
        tpos = torch.empty(K + 1, dtype=torch.int64, device=DEV)
        last = torch.tensor([K], dtype=torch.int32, device=DEV)
        nd = torch.tensor([K], dtype=torch.int32, device=DEV)
        g = h.step_graph(prev_drafts, logits_in, tpos, last, nd, aux_in, table, kc, vc)
        emitted = [bonus]
        try:
            while len(emitted) < N:
                blk = torch.cat([torch.tensor([bonus], dtype=torch.int32, device=DEV),
                                 prev_drafts.reshape(-1)])
                tm.forward(blk, seq_len, logits=logits_in.view(K + 1, V), aux=aux_in)
                tpos.copy_(torch.arange(seq_len, seq_len + K + 1, device=DEV))
                g.launch()
                n = int(g.out["num_accepted"][0])
                emitted += to_np(prev_drafts)[0, :n].tolist() + [int(g.out["bonus"][0])]
                assert int(g.out["seq_lens"][0]) == seq_len + n + 1
                seq_len += n + 1
                bonus = int(g.out["bonus"][0])
                prev_drafts.copy_(g.out["draft_tokens"])
            torch.cuda.synchronize()
            assert h.check_device_errors() == 0 and tm.check_device_errors() == 0
        finally:
            g.close()
        assert emitted[:N] == ref[:N]
    finally:
        tm.close()
        h.close()
