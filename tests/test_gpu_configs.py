"""GPU parity at the benchmark workloads' full sizes, in the launch
configuration bench.py times (verify -> paged slots -> inject -> propose on
the whole batch).  Greedy verification is compared bit-exactly on the whole
batch; injection + proposal are recomputed by the oracle for sampled requests
(requests are independent), from copies of those requests' pages taken before
the step.
"""

from __future__ import annotations

import gc

import numpy as np
import pytest
import torch

import oracle as O
from block_diffusion_speculative_propose_b200 import (DFlash, paged_slots, synth,
                                                      verify_greedy)
from tests._util import rel_l2, to_np, weights_np, weights_to
from tests.test_gpu_propose import check_lm_head_stage, compare_drafts, max_excluded

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _fill_pool(shape, n_layers, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    out = []
    for _ in range(2 * n_layers):
        t = torch.empty(shape, dtype=torch.bfloat16, device=DEV)
        for i in range(0, shape[0], 4096):
            blk = t[i:i + 4096]
            blk.copy_(torch.randn(blk.shape, generator=g, device=DEV).to(torch.bfloat16))
        out.append(t)
    return out[:n_layers], out[n_layers:]


@pytest.mark.parametrize("workload,samples", [
    ("qwen3_b32_ctx512_8192", 2),
    ("llama_b128_ctx1024_16384", 2),
    ("qwen3_b128_ctx8192_32768", 2),
])
def test_full_step_at_bench_size(workload, samples):
    wl = synth.WORKLOADS[workload]
    cfg = synth.model_config(wl["model"])
    B, bs, K, P, V = wl["batch"], cfg["block_size"], cfg["block_size"] - 1, 16, cfg["vocab"]
    Wt = synth.make_weights(cfg, seed=0)
    h = DFlash(cfg, weights_to(Wt, DEV), max_position=wl["ctx_hi"] + 4 * bs + 64)
    try:
        sb = synth.make_step_batch(cfg, B, wl["ctx_lo"], wl["ctx_hi"], accept=wl["accept"],
                                   seed=1)
        shape = (sb.num_pages, cfg["n_kv_heads"], P, cfg["head_dim"])
        kc, vc = _fill_pool(shape, cfg["n_layers"], seed=8)
        rng = np.random.default_rng(0)
        seq = to_np(sb.seq_lens)
        pick = sorted({int(np.argmax(seq)), *rng.choice(B, samples - 1, replace=False).tolist()})
        # pages of the sampled requests, before the step writes anything
        pages = [to_np(sb.block_table[b, :-(-(int(seq[b]) + bs) // P)]).astype(np.int64)
                 for b in pick]
        all_pages = np.concatenate(pages)
        idx = torch.tensor(all_pages, device=DEV)
        k_pre = [to_np(t.index_select(0, idx)).astype(np.float32) for t in kc]
        v_pre = [to_np(t.index_select(0, idx)).astype(np.float32) for t in vc]

        # ---- the GPU step, as bench.py runs it
        dv = {k: getattr(sb, k).to(DEV) for k in ("prev_drafts", "target_logits",
                                                  "inject_positions", "inject_req_ids", "aux",
                                                  "bonus", "seq_lens", "block_table")}
        out_tok, n_acc, new_bonus = verify_greedy(dv["prev_drafts"], dv["target_logits"])
        slots = paged_slots(dv["inject_positions"], dv["inject_req_ids"], dv["block_table"], P)
        h.inject_context(dv["aux"], dv["inject_positions"], slots, kc, vc)
        Wpages = int(sb.block_table.shape[1])
        ws = torch.empty(h.propose_workspace_bytes(B, Wpages), dtype=torch.uint8, device=DEV)
        drafts = h.propose(dv["bonus"], dv["seq_lens"], dv["block_table"], kc, vc,
                           workspace=ws)
        torch.cuda.synchronize()
        assert h.check_device_errors() == 0
        # the LM head's greedy pick on the rows it saw, stage-isolated: every
        # sampled request's rows plus random rows of the whole batch
        Wn = weights_np(Wt)
        lm_rows = sorted({*np.concatenate([np.arange(b * K, (b + 1) * K) for b in pick]).tolist(),
                          *rng.choice(B * K, min(B * K, 64), replace=False).tolist()})
        check_lm_head_stage(h, ws, B, Wpages, to_np(drafts), Wn, lm_rows,
                            f"{workload} lm-head")
        # the same step with the debug logits gives the same drafts
        logits = torch.empty(B * K, V, dtype=torch.float32, device=DEV)
        drafts2 = h.propose(dv["bonus"], dv["seq_lens"], dv["block_table"], kc, vc,
                            logits_out=logits)
        torch.cuda.synchronize()
        assert torch.equal(drafts, drafts2)

        # ---- verification: whole batch, bit-exact
        ver = O.verify_greedy(to_np(sb.prev_drafts), to_np(sb.target_logits))
        np.testing.assert_array_equal(to_np(out_tok), ver.out_tokens)
        np.testing.assert_array_equal(to_np(n_acc), ver.num_accepted)
        np.testing.assert_array_equal(to_np(new_bonus), ver.bonus)
        np.testing.assert_array_equal(ver.num_accepted, to_np(sb.n_accept))
        ref_slots = O.paged_slots(to_np(sb.inject_positions), to_np(sb.inject_req_ids),
                                  to_np(sb.block_table), P)
        np.testing.assert_array_equal(to_np(slots), ref_slots)
        gpu_drafts = to_np(drafts)[pick]
        rows = np.concatenate([np.arange(b * K, (b + 1) * K) for b in pick])
        gpu_logits = to_np(logits[torch.tensor(rows, device=DEV)])
        del logits, kc, vc, dv
        gc.collect()
        torch.cuda.empty_cache()

        # ---- oracle: inject + propose for the sampled requests on a compact pool
        oc = O.OracleConfig.from_mapping(cfg)
        remap = {int(p): i for i, p in enumerate(all_pages)}
        width = max(len(p) for p in pages)
        table = np.zeros((len(pick), width), dtype=np.int64)
        for j, p in enumerate(pages):
            table[j, :len(p)] = [remap[int(x)] for x in p]
        req = to_np(sb.inject_req_ids)
        sel = np.isin(req, pick)
        pos = to_np(sb.inject_positions)[sel]
        local_req = np.searchsorted(np.array(pick), req[sel])
        local_slots = O.paged_slots(pos, local_req, table, P)
        aux = to_np(sb.aux)[sel].astype(np.float64)
        del Wt
        res = {}
        for mode in ("device", "exact"):
            ko = [k.astype(np.float64) for k in k_pre]
            vo = [v.astype(np.float64) for v in v_pre]
            O.inject_context(oc, Wn, aux, pos, local_slots, ko, vo, mode)
            res[mode] = O.propose(oc, Wn, to_np(sb.bonus)[pick], seq[pick], table, ko, vo, mode)
        excluded = compare_drafts(gpu_drafts, gpu_logits, res["device"], res["exact"], K,
                                  name=f"{workload} chain")
        assert excluded <= max_excluded(len(pick) * K)
    finally:
        h.close()
        gc.collect()
        torch.cuda.empty_cache()
