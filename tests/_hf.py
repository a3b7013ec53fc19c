"""Library reference models for pinning the oracle: transformers' Qwen3 classes
loaded with the same weights, run in float64 on the CPU."""

from __future__ import annotations

import numpy as np
import torch


def qwen3_config(cfg: dict, n_layers: int | None = None):
    from transformers import Qwen3Config
    return Qwen3Config(
        vocab_size=cfg["vocab"], hidden_size=cfg["hidden"],
        intermediate_size=cfg["intermediate"],
        num_hidden_layers=n_layers if n_layers is not None else cfg["n_layers"],
        num_attention_heads=cfg["n_q_heads"], num_key_value_heads=cfg["n_kv_heads"],
        head_dim=cfg["head_dim"], rms_norm_eps=cfg["rms_eps"], rope_theta=cfg["rope_theta"],
        max_position_embeddings=1 << 16, tie_word_embeddings=False, attention_bias=False,
        attn_implementation="eager")


def _t(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, dtype=np.float64))


def qwen3_from_draft_weights(cfg: dict, W: dict):
    """Qwen3ForCausalLM whose decoder layers, final norm, embedding and LM head
    carry the draft weights (oracle format: numpy, [out, in])."""
    from transformers.models.qwen3.modeling_qwen3 import Qwen3ForCausalLM
    m = Qwen3ForCausalLM(qwen3_config(cfg)).double().eval()
    with torch.no_grad():
        m.model.embed_tokens.weight.copy_(_t(W["embed"]))
        m.lm_head.weight.copy_(_t(W["lm_head"]))
        m.model.norm.weight.copy_(_t(W["final_norm_w"]))
        for l, layer in enumerate(m.model.layers):
            layer.input_layernorm.weight.copy_(_t(W["in_norm_w"][l]))
            layer.post_attention_layernorm.weight.copy_(_t(W["post_norm_w"][l]))
            a = layer.self_attn
            a.q_proj.weight.copy_(_t(W["wq"][l]))
            a.k_proj.weight.copy_(_t(W["wk"][l]))
            a.v_proj.weight.copy_(_t(W["wv"][l]))
            a.o_proj.weight.copy_(_t(W["wo"][l]))
            a.q_norm.weight.copy_(_t(W["q_norm_w"][l]))
            a.k_norm.weight.copy_(_t(W["k_norm_w"][l]))
            layer.mlp.gate_proj.weight.copy_(_t(W["w_gate"][l]))
            layer.mlp.up_proj.weight.copy_(_t(W["w_up"][l]))
            layer.mlp.down_proj.weight.copy_(_t(W["w_down"][l]))
    return m


def full_mask(n_q: int, n_kv: int) -> torch.Tensor:
    """Additive 4-D mask with nothing masked (non-causal attention)."""
    return torch.zeros(1, 1, n_q, n_kv, dtype=torch.float64)


def random_target(cfg: dict, n_layers: int, seed: int):
    """A tiny random-weight Qwen3 causal LM (the target model of the lossless
    test), float64."""
    from transformers.models.qwen3.modeling_qwen3 import Qwen3ForCausalLM
    torch.manual_seed(seed)
    m = Qwen3ForCausalLM(qwen3_config(cfg, n_layers)).double().eval()
    with torch.no_grad():
        for p in m.parameters():
            if p.dim() >= 2:
                p.normal_(0.0, 0.05)
            else:
                p.copy_(1.0 + 0.02 * torch.randn_like(p))
    return m
