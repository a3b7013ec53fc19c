"""The workspace-free greedy verification, dflash_verify_greedy_noalloc.

It exists for callers that cannot allocate device memory (an embedding runtime
that pre-reserved the GPU for its own pool, a plugin that only receives its
buffers, a decode loop where cudaMalloc's synchronization is not acceptable):
its scratch is a fixed array inside the library.  Called through the C ABI, it
must give exactly what dflash_verify_greedy gives (verification is bit-exact),
on consecutive calls that reuse the shared scratch, and must refuse batches
larger than that scratch before launching anything.
"""

from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from block_diffusion_speculative_propose_b200 import dflash as D
from block_diffusion_speculative_propose_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _case(B, K, V, seed):
    g = torch.Generator().manual_seed(seed)
    n_acc = torch.randint(0, K + 1, (B,), generator=g)
    drafts = torch.randint(0, V, (B, K), generator=g, dtype=torch.int32)
    logits = synth.make_target_logits(g, drafts, n_acc, V)
    return drafts.to(DEV), logits.to(DEV)


def _noalloc(drafts, logits):
    B, K1, V = logits.shape
    out = torch.full((B, K1), -7, dtype=torch.int32, device=DEV)
    n = torch.full((B,), -7, dtype=torch.int32, device=DEV)
    bonus = torch.full((B,), -7, dtype=torch.int32, device=DEV)
    st = D.lib().dflash_verify_greedy_noalloc(
        ctypes.c_void_p(drafts.data_ptr()), ctypes.c_void_p(logits.data_ptr()), B, K1 - 1, V,
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(n.data_ptr()),
        ctypes.c_void_p(bonus.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out, n, bonus


def test_noalloc_verify_matches_workspace_verify_on_consecutive_calls():
    # two calls in a row with different shapes: the second reuses (and must not
    # be disturbed by) whatever the first left in the shared scratch
    for B, K, V, seed in ((128, 15, 151936, 1), (3, 9, 128256, 2), (37, 4, 1027, 3)):
        drafts, logits = _case(B, K, V, seed)
        ref = D.verify_greedy(drafts, logits)
        st, out, n, bonus = _noalloc(drafts, logits)
        torch.cuda.synchronize()
        assert st == 0, D.STATUS.get(st, st)
        np.testing.assert_array_equal(out.cpu().numpy(), ref[0].cpu().numpy())
        np.testing.assert_array_equal(n.cpu().numpy(), ref[1].cpu().numpy())
        np.testing.assert_array_equal(bonus.cpu().numpy(), ref[2].cpu().numpy())


def test_noalloc_verify_rejects_batches_beyond_its_scratch():
    B, K, V = 1024, 15, 2048      # 16384 partial keys > 8192
    drafts, logits = _case(B, K, V, 4)
    st, out, n, bonus = _noalloc(drafts, logits)
    torch.cuda.synchronize()
    assert st == -3                # DFLASH_ERR_WORKSPACE, nothing launched
    assert int((out != -7).sum()) == 0
