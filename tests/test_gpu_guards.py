"""Guards of the device path that need a GPU but fault nothing.

- The fp16 storage range: dflash_create refuses weights that fp16 cannot hold
  (a weight beyond 65504, weights so small that most are fp16 subnormals, a
  norm weight whose RMSNorm output bound sqrt(hidden) * max|w| exceeds 65504)
  with DFLASH_ERR_RANGE.
- Bounded waits: a kernel whose one wait can never complete (an mbarrier that
  nothing arrives on) gives up after the device's wait limit, the handle
  reports DFLASH_ERR_DEVICE_TIMEOUT, and the context stays usable: the next
  proposal is clean and identical to one taken before.
- Request count: more requests than an attention launch can index are refused
  on the host before any launch.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from block_diffusion_speculative_propose_b200 import DFlash, DFlashError, set_wait_limit, synth
from tests._util import to_np, weights_to

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
DEVERR_TIMEOUT = 1
ERR_RANGE = -8
ERR_DEVICE_TIMEOUT = -7
ERR_UNSUPPORTED_SHAPE = -4


def _tiny():
    cfg = synth.model_config("tiny")
    return cfg, weights_to(synth.make_weights(cfg, seed=0), DEV)


def _create_status(cfg, W):
    try:
        DFlash(cfg, W, max_position=1024).close()
        return 0
    except DFlashError as e:
        return e.status


def test_fp16_range_guard():
    cfg, W = _tiny()
    assert _create_status(cfg, W) == 0
    big = dict(W, wq=[w.clone() for w in W["wq"]])
    big["wq"][1][3, 5] = 7.0e4                     # beyond fp16's largest finite value
    assert _create_status(cfg, big) == ERR_RANGE
    big = dict(W, lm_head=W["lm_head"].clone())
    big["lm_head"][7, 0] = -7.0e4
    assert _create_status(cfg, big) == ERR_RANGE
    tiny_w = dict(W, w_up=[w * 1e-4 for w in W["w_up"]])   # ~2e-6: mostly fp16 subnormals
    assert _create_status(cfg, tiny_w) == ERR_RANGE
    # sqrt(256) * 5000 = 80000 > 65504: the post-attention RMSNorm output may overflow
    nrm = dict(W, post_norm_w=[w.clone() for w in W["post_norm_w"]])
    nrm["post_norm_w"][0][11] = 5000.0
    assert _create_status(cfg, nrm) == ERR_RANGE
    # within range: sqrt(256) * 4000 = 64000
    nrm["post_norm_w"][0][11] = 4000.0
    assert _create_status(cfg, nrm) == 0


def _propose(h, cfg):
    P, bs = cfg["page_size"], cfg["block_size"]
    shape = (8, cfg["n_kv_heads"], P, cfg["head_dim"])
    g = torch.Generator(device=DEV)
    g.manual_seed(5)
    kc = [torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
          for _ in range(cfg["n_layers"])]
    vc = [torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
          for _ in range(cfg["n_layers"])]
    table = torch.tensor([[3, 1, 6, 0], [2, 7, 5, 4]], dtype=torch.int32, device=DEV)
    d = h.propose(torch.tensor([11, 400], dtype=torch.int32, device=DEV),
                  torch.tensor([37, 50], dtype=torch.int32, device=DEV), table, kc, vc)
    torch.cuda.synchronize()
    return to_np(d)


def test_bounded_wait_runs_out_and_context_survives():
    cfg, W = _tiny()
    h = DFlash(cfg, W, max_position=1024)
    try:
        before = _propose(h, cfg)
        assert h.check_device_errors() == 0
        set_wait_limit(0, 2_000_000)              # ~1 ms at 1.9 GHz
        try:
            h.selftest_wait_timeout()
            status, bits = h.check_device_status()
            assert status == ERR_DEVICE_TIMEOUT and bits & DEVERR_TIMEOUT
            # read and cleared: the handle is clean again
            assert h.check_device_status() == (0, 0)
        finally:
            set_wait_limit(0, 4_000_000_000)
        after = _propose(h, cfg)
        assert h.check_device_errors() == 0
        np.testing.assert_array_equal(before, after)
    finally:
        h.close()


def test_request_count_limit_refused_before_any_launch():
    """The attention grid carries the request index in one of its dimensions
    (at most 65535): a proposal or an attention call for 65536 requests is
    DFLASH_ERR_UNSUPPORTED_SHAPE on the host, before any launch or buffer
    access (the buffers passed here are deliberately too small to be read)."""
    cfg, W = _tiny()
    h = DFlash(cfg, W, max_position=1024)
    try:
        B = 65536
        bonus = torch.zeros(B, dtype=torch.int32, device=DEV)
        seq = torch.zeros(B, dtype=torch.int32, device=DEV)
        table = torch.zeros(B, 1, dtype=torch.int32, device=DEV)
        shape = (1, cfg["n_kv_heads"], cfg["page_size"], cfg["head_dim"])
        kc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV) for _ in range(cfg["n_layers"])]
        vc = [torch.zeros(shape, dtype=torch.bfloat16, device=DEV) for _ in range(cfg["n_layers"])]
        ws = torch.zeros(1024, dtype=torch.uint8, device=DEV)
        with pytest.raises(DFlashError) as e:
            h.propose(bonus, seq, table, kc, vc, workspace=ws)
        assert e.value.status == ERR_UNSUPPORTED_SHAPE
        q = torch.zeros(cfg["block_size"], cfg["n_q_heads"], cfg["head_dim"], dtype=torch.bfloat16,
                        device=DEV)
        with pytest.raises(DFlashError) as e:
            h.block_attention(q, seq, table, kc[0], vc[0], workspace=ws)
        assert e.value.status == ERR_UNSUPPORTED_SHAPE
        torch.cuda.synchronize()
        assert h.check_device_errors() == 0
        # the handle still proposes
        _propose(h, cfg)
        assert h.check_device_errors() == 0
    finally:
        h.close()
