"""The C-ABI library loads, exports every function include/dflash.h declares,
and rejects bad arguments on the host (no GPU needed for any of this)."""

from __future__ import annotations

import ctypes
import os
import re

import pytest
import torch

from block_diffusion_speculative_propose_b200 import build as build_mod
from block_diffusion_speculative_propose_b200 import dflash as D

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dflash.h")


@pytest.fixture(scope="module")
def L():
    build_mod.build()
    return D.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dflash_[a-z_]+)\s*\(", text)))


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("dflash_inject_context", "dflash_propose", "dflash_verify_greedy"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code, name in D.STATUS.items():
        assert D.status_string(code) == name
    assert "sm_100a" in D.version()


def test_host_validation_without_gpu(L):
    out = ctypes.c_void_p(1)
    assert L.dflash_create(None, None, 0, ctypes.byref(out)) == -1
    assert out.value is None
    assert L.dflash_create(None, None, 0, None) == -1
    # negative sizes and no-op sizes return before touching the device
    assert L.dflash_verify_greedy(None, None, -1, 3, 10, None, None, None, None, 0, None) == -1
    assert L.dflash_verify_greedy(None, None, 0, 3, 10, None, None, None, None, 0, None) == 0
    assert L.dflash_verify_greedy(None, None, 2, 200, 10, None, None, None, None, 0, None) == -1
    assert L.dflash_paged_slots(None, None, 0, None, 4, 16, None, None) == 0
    assert L.dflash_paged_slots(None, None, -1, None, 4, 16, None, None) == -1
    assert L.dflash_inject_context(None, None, None, None, 0, None, None, 1, None, 0, None) == -1
    assert L.dflash_propose(None, None, None, None, 1, 1, None, None, 1, None, None, None,
                            None, 0, None) == -1
    assert L.dflash_check_device_errors(None, None) == -1
    assert L.dflash_verify_workspace_bytes(128, 15, 151936) > 0
    assert L.dflash_verify_workspace_bytes(0, 15, 151936) == 0
    assert L.dflash_inject_workspace_bytes(None, 16) == 0
    assert L.dflash_propose_workspace_bytes(None, 1, 10) == 0
    # proposal preparation: (n, B) = (0, 0) is a no-op; bad sizes / pointer
    # combinations are rejected before any launch
    prep = L.dflash_prepare_proposal_inputs
    args = dict(tp=None, n=0, last=None, B=0, cur=None, cw=4, cnd=None, prev=None, pw=0,
                pnd=None, bt=None, W=4, P=16, V=10, po=None, so=None, sl=None, bo=None,
                err=None, st=None)

    def call(**kw):
        a = dict(args, **kw)
        return prep(a["tp"], a["n"], a["last"], a["B"], a["cur"], a["cw"], a["cnd"], a["prev"],
                    a["pw"], a["pnd"], a["bt"], a["W"], a["P"], a["V"], a["po"], a["so"],
                    a["sl"], a["bo"], a["err"], a["st"])
    assert call() == 0
    assert call(n=-1) == -1
    assert call(B=-1) == -1
    assert call(cw=0) == -1
    assert call(P=0) == -1
    assert call(V=0) == -1
    assert call(prev=16) == -1          # prev_sampled without prev_num_draft
    assert call(pnd=16) == -1
    assert call(n=4) == -1              # rows without their pointers
    assert call(B=2) == -1


def test_spec_step_host_validation_without_gpu(L):
    """The whole-step entry points reject a missing handle or buffers before
    anything reaches the device, and the graph calls accept NULL as documented."""
    io = D._StepIO()
    io.B, io.n = 1, 16
    assert L.dflash_spec_step(None, ctypes.byref(io), None, 0, None) == -1
    assert L.dflash_spec_step(None, None, None, 0, None) == -1
    out = ctypes.c_void_p(1)
    assert L.dflash_step_graph_create(None, ctypes.byref(io), None, 0, ctypes.byref(out)) == -1
    assert out.value is None                          # *out cleared on failure
    assert L.dflash_step_graph_create(None, ctypes.byref(io), None, 0, None) == -1
    assert L.dflash_step_graph_launch(None, None) == -1
    L.dflash_step_graph_destroy(None)                 # no-op
    assert L.dflash_spec_step_workspace_bytes(None, 1, 16, 8) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_create_without_device_fails_cleanly(L):
    from block_diffusion_speculative_propose_b200 import synth
    cfg = synth.model_config("tiny")
    c = D._Config(cfg["hidden"], cfg["n_layers"], cfg["n_q_heads"], cfg["n_kv_heads"],
                  cfg["head_dim"], cfg["intermediate"], cfg["vocab"], cfg["n_target_layers"],
                  None, cfg["block_size"], cfg["mask_token_id"], 16, 1e-6, 1e6, 1024)
    w = D._Weights()
    dummy = (ctypes.c_void_p * cfg["n_layers"])(*([16] * cfg["n_layers"]))
    for k in ("fc_w", "hidden_norm_w", "embed", "lm_head", "final_norm_w"):
        setattr(w, k, 16)
    for k in ("in_norm_w", "post_norm_w", "wq", "wk", "wv", "wo", "q_norm_w", "k_norm_w",
              "w_gate", "w_up", "w_down"):
        setattr(w, k, ctypes.cast(dummy, D._PP))
    out = ctypes.c_void_p()
    assert L.dflash_create(ctypes.byref(c), ctypes.byref(w), 0, ctypes.byref(out)) == -2
    assert out.value is None
