#!/usr/bin/env python3
"""Benchmark of the DFlash draft-proposal step on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
  greedy verification of the previous drafts against target logits
  -> paged-slot mapping of the accepted rows -> context K/V injection of those
  rows -> one block proposal (all draft layers + LM head + greedy pick).
Inputs are resident in HBM when the timed region starts (value); the e2e
figure repeats the step through the public API with pinned host buffers and
the host<->device copies inside the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

With N > 1 (torchrun, one rank per GPU) every rank runs its own batch
(requests are independent: weak scaling, no collective on the data path);
the step time is the max over ranks.  ``--impl reference`` times the CPU
oracle on the host cores instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "draft blocks/sec and draft tokens/sec at batch B; % HBM / tensor-core roofline"
DEFAULT_WORKLOAD = "qwen3_b128_ctx8192_32768"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch measured with ncu (dram__bytes_read.sum +
# dram__bytes_write.sum) for the kernel family that dominates a workload,
# keyed by the digest of the kernel sources it was measured on.
TRAFFIC = {
    # attention of the batch-128, 8k-32k-context step, scaled from one launch of
    # `bench.py --ncu-case attention` (16 requests of the same context
    # distribution: 1.3782 GB read + 27.4 MB written for 1.3738 GB of
    # algorithmic bytes, ratio 1.0232) to the launch's algorithmic bytes
    ("qwen3_b128_ctx8192_32768", "attention"): {"ratio_to_algorithmic": 1.0232,
                                                "digest": "2f2ef01b70758d65"},
    # the same for the batch-32, 512-8192-context workload (16 requests: 300.6 MB
    # read + 16.4 MB written for 298.7 MB) and the Llama-paired batch-128 one
    # (592.1 MB + 16.7 MB for 590.2 MB)
    ("qwen3_b32_ctx512_8192", "attention"): {"ratio_to_algorithmic": 1.0614,
                                             "digest": "2f2ef01b70758d65"},
    ("llama_b128_ctx1024_16384", "attention"): {"ratio_to_algorithmic": 1.0316,
                                                "digest": "2f2ef01b70758d65"},
    # gate/up GEMM of the batch-1 step, one launch of `bench.py --workload
    # qwen3_b1_ctx2048 --ncu-case gemms` (the step's shapes): 201.5 MB read +
    # 3.5 MB written
    ("qwen3_b1_ctx2048", "gemm_gate_up"): {"bytes_per_launch": 205062144,
                                           "digest": "6384f9db5e3108f3"},
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-graph", action="store_true", help="eager launches for the value loop")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the sub-measurements")
    ap.add_argument("--ncu-case", choices=["attention", "gemms", "verify"], default=None,
                    help="run one kernel family twice on a reduced case of the workload "
                         "(for a profiler capture of the second run) and exit")
    ap.add_argument("--seed", type=int, default=1)
    a = ap.parse_args()
    a.warmup = max(a.warmup, 3)
    a.steps = max(a.steps, 1)
    return a


# Sources a kernel family is compiled from (its traffic figure is void once
# any of them changes).
FAMILY_SOURCES = {"gemm": ("gemm_tcgen05.cuh", "gemm_pair.cuh", "dflash_device.cuh"),
                  "attention": ("attention_tc2.cuh", "attention_tc.cuh", "attention.cuh",
                                "dflash_device.cuh")}


def source_digest(family: str = "gemm") -> str:
    h = hashlib.sha256()
    for name in FAMILY_SOURCES["attention" if family == "attention" else "gemm"]:
        h.update(open(os.path.join(ROOT, "block_diffusion_speculative_propose_b200", "csrc",
                                   name), "rb").read())
    return h.hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------
def dist_init(gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return rank, world, local


def dist_max(x: float) -> float:
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def shard_seed(seed: int, rank: int) -> int:
    """Each rank draws its own batch: requests are independent units."""
    return seed + 1000 * rank


# ----------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_index: int, out_path: str):
        self.path = out_path
        self.proc = None
        try:
            self.f = open(out_path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(gpu_index), "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(parts)
            except Exception:
                pass
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------
# the step on the GPU
# ----------------------------------------------------------------------------
class GpuStep:
    def __init__(self, wl_name: str, device: int, seed: int):
        from block_diffusion_speculative_propose_b200 import (DFlash, Workspace, synth,
                                                              verify_workspace_bytes)
        self.synth = synth
        wl = synth.WORKLOADS[wl_name]
        self.wl_name, self.wl = wl_name, wl
        cfg = synth.model_config(wl["model"])
        self.cfg = cfg
        self.dev = torch.device("cuda", device)
        torch.cuda.set_device(self.dev)
        B, bs = wl["batch"], cfg["block_size"]
        self.B, self.bs, self.K = B, bs, bs - 1
        W = synth.make_weights(cfg, seed=0, device=self.dev)
        self.h = DFlash(cfg, W, device=device, max_position=wl["ctx_hi"] + 4 * bs + 64)
        self.W = W
        sb = synth.make_step_batch(cfg, B, wl["ctx_lo"], wl["ctx_hi"], accept=wl["accept"],
                                   seed=seed)
        self.sb = sb
        d = self.dev
        # step inputs (pinned host copies kept for the e2e loop)
        self.host = {
            "prev_drafts": sb.prev_drafts.pin_memory(),
            "target_logits": sb.target_logits.pin_memory(),
            "inject_pos": sb.inject_positions.pin_memory(),
            "inject_req": sb.inject_req_ids.pin_memory(),
            "aux": sb.aux.pin_memory(),
            "bonus": sb.bonus.pin_memory(),
            "seq_lens": sb.seq_lens.pin_memory(),
            "block_table": sb.block_table.pin_memory(),
        }
        self.inp = {k: v.to(d) for k, v in self.host.items()}
        shape = (sb.num_pages, cfg["n_kv_heads"], cfg["page_size"], cfg["head_dim"])
        self.kc = [torch.empty(shape, dtype=torch.bfloat16, device=d) for _ in range(cfg["n_layers"])]
        self.vc = [torch.empty(shape, dtype=torch.bfloat16, device=d) for _ in range(cfg["n_layers"])]
        fill = torch.Generator(device=d)
        fill.manual_seed(seed + 7)
        for c in self.kc + self.vc:
            for i in range(0, c.shape[0], 4096):
                blk = c[i:i + 4096]
                blk.copy_(torch.randn(blk.shape, generator=fill, device=d,
                                      dtype=torch.float32).to(torch.bfloat16))
        R = int(sb.inject_positions.numel())
        self.R = R
        Wd = int(sb.block_table.shape[1])
        self.ws_prop = torch.empty(self.h.propose_workspace_bytes(B, Wd), dtype=torch.uint8, device=d)
        self.ws_inj = torch.empty(max(self.h.inject_workspace_bytes(R), 256), dtype=torch.uint8, device=d)
        self.ws_ver = torch.empty(max(verify_workspace_bytes(B, self.K, cfg["vocab"]), 256),
                                  dtype=torch.uint8, device=d)
        self.out = {
            "slots": torch.empty(R, dtype=torch.int64, device=d),
            "drafts": torch.empty(B, self.K, dtype=torch.int32, device=d),
            "block": torch.empty(B, bs, dtype=torch.int32, device=d),
            "ver_tokens": torch.empty(B, self.K + 1, dtype=torch.int32, device=d),
            "n_acc": torch.empty(B, dtype=torch.int32, device=d),
            "new_bonus": torch.empty(B, dtype=torch.int32, device=d),
        }
        self.graph = None

    def run(self, stream=None):
        from block_diffusion_speculative_propose_b200 import paged_slots, verify_greedy
        i, o = self.inp, self.out
        verify_greedy(i["prev_drafts"], i["target_logits"], out_tokens=o["ver_tokens"],
                      num_accepted=o["n_acc"], bonus=o["new_bonus"], workspace=self.ws_ver,
                      stream=stream)
        paged_slots(i["inject_pos"], i["inject_req"], i["block_table"],
                    self.cfg["page_size"], slots=o["slots"], stream=stream)
        self.h.inject_context(i["aux"], i["inject_pos"], o["slots"], self.kc, self.vc,
                              workspace=self.ws_inj, stream=stream)
        self.h.propose(i["bonus"], i["seq_lens"], i["block_table"], self.kc, self.vc,
                       draft_tokens=o["drafts"], block_tokens=o["block"],
                       workspace=self.ws_prop, stream=stream)

    def capture(self):
        s = torch.cuda.Stream(device=self.dev)
        s.wait_stream(torch.cuda.current_stream(self.dev))
        with torch.cuda.stream(s):
            self.run()
        torch.cuda.current_stream(self.dev).wait_stream(s)
        torch.cuda.synchronize(self.dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run()
        torch.cuda.synchronize(self.dev)
        self.graph = g

    def step(self):
        if self.graph is not None:
            self.graph.replay()
        else:
            self.run()

    def launches_per_step(self) -> int:
        before = self.h.launch_count()
        self.run()
        torch.cuda.synchronize(self.dev)
        return int(self.h.launch_count() - before) + 3   # + verify (2) + paged_slots (1)

    def e2e_setup(self):
        """Two sets of device inputs / outputs and a captured graph of the step
        for each, for the pipelined end-to-end loop."""
        self.inp_sets = [self.inp, {k: torch.empty_like(v) for k, v in self.inp.items()}]
        self.out_sets = [self.out, {k: torch.empty_like(v) for k, v in self.out.items()}]
        self.host_out_sets = [{k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
                               for k, v in self.out.items()} for _ in range(2)]
        self.e2e_graphs = []
        keep_inp, keep_out = self.inp, self.out
        for j in range(2):
            self.inp, self.out = self.inp_sets[j], self.out_sets[j]
            for k in self.inp:
                self.inp[k].copy_(self.host[k])
            self.capture()
            self.e2e_graphs.append(self.graph)
        self.inp, self.out = keep_inp, keep_out
        self.graph = self.e2e_graphs[0]

    def e2e_pipelined(self, steps: int, warmup: int) -> float:
        """Seconds per step through the public API from pinned host buffers,
        every step copying its inputs host -> device and reading its results
        back, with step i+1's input copies (its own buffer set) overlapping
        step i's compute, as a serving loop would.  Timed on the device from
        the first copy to the last read-back."""
        dev = self.dev
        comp = torch.cuda.current_stream(dev)
        h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        done = [torch.cuda.Event(), torch.cuda.Event()]
        copied = [torch.cuda.Event(), torch.cuda.Event()]
        read = [torch.cuda.Event(), torch.cuda.Event()]
        for e in done + read:
            e.record(comp)
        keys_in = ("prev_drafts", "target_logits", "inject_pos", "inject_req", "aux", "bonus",
                   "seq_lens", "block_table")
        keys_out = ("drafts", "block", "ver_tokens", "n_acc", "new_bonus")

        def one(i):
            j = i & 1
            with torch.cuda.stream(h2d):
                h2d.wait_event(done[j])            # step i-2 has finished with set j
                for k in keys_in:
                    self.inp_sets[j][k].copy_(self.host[k], non_blocking=True)
                copied[j].record(h2d)
            comp.wait_event(copied[j])
            comp.wait_event(read[j])               # step i-2's results have been read back
            self.e2e_graphs[j].replay()
            done[j].record(comp)
            with torch.cuda.stream(d2h):
                d2h.wait_event(done[j])
                for k in keys_out:
                    self.host_out_sets[j][k].copy_(self.out_sets[j][k], non_blocking=True)
                read[j].record(d2h)
        for i in range(warmup):
            one(i)
        torch.cuda.synchronize(dev)
        dist_barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        h2d.wait_stream(comp)
        for i in range(steps):
            one(i)
        comp.wait_stream(d2h)
        e1.record(comp)
        torch.cuda.synchronize(dev)
        dist_barrier()
        return e0.elapsed_time(e1) / 1e3 / steps

    def e2e_step(self):
        """The step through the public API from pinned host buffers: H2D of the
        step's inputs, the four calls, D2H of the step's results."""
        for k in ("prev_drafts", "target_logits", "inject_pos", "inject_req", "aux", "bonus",
                  "seq_lens", "block_table"):
            self.inp[k].copy_(self.host[k], non_blocking=True)
        self.run()
        for k in ("drafts", "block", "ver_tokens", "n_acc", "new_bonus"):
            self.host_out[k].copy_(self.out[k], non_blocking=True)

    def e2e_bytes(self):
        h2d = sum(self.host[k].numel() * self.host[k].element_size() for k in
                  ("prev_drafts", "target_logits", "inject_pos", "inject_req", "aux", "bonus",
                   "seq_lens", "block_table"))
        d2h = sum(self.out[k].numel() * self.out[k].element_size() for k in
                  ("drafts", "block", "ver_tokens", "n_acc", "new_bonus"))
        return h2d, d2h

    # ------------------------------------------------------------ accounting
    def algorithmic(self, family: str):
        """Algorithmic (bytes, flops) of ONE launch of a kernel family."""
        c, B, bs, K = self.cfg, self.B, self.bs, self.K
        H, L, Hq, Hkv, d, I, V = (c["hidden"], c["n_layers"], c["n_q_heads"], c["n_kv_heads"],
                                  c["head_dim"], c["intermediate"], c["vocab"])
        M, MK, R = B * bs, B * K, self.R
        seq = self.sb.seq_lens.double()
        keys = float((seq + bs).sum())

        def gemm(m, n, k, extra):
            return n * k * 2 + m * k * 2 + extra, 2.0 * m * n * k
        if family == "gemm_qkv":
            return gemm(M, (Hq + 2 * Hkv) * d, H, M * (Hq + 2 * Hkv) * d * 2)
        if family == "gemm_o":
            return gemm(M, H, Hq * d, M * H * 8)
        if family == "gemm_gate_up":
            return gemm(M, 2 * I, H, M * I * 2)
        if family == "gemm_down":
            return gemm(M, H, I, M * H * 8)
        if family == "gemm_mlp":     # gate/up + down in one launch (few rows)
            b1, f1 = gemm(M, 2 * I, H, M * I * 2)
            b2, f2 = gemm(M, H, I, M * H * 8)
            return b1 + b2, f1 + f2
        if family == "gemm_lm_head":
            return gemm(MK, V, H, MK * 8)
        if family == "gemm_fc":
            return gemm(R, H, c["n_target_layers"] * H, R * H * 4)
        if family == "gemm_kv_inject":
            return gemm(R, L * 2 * Hkv * d, H, R * L * 2 * Hkv * d * 2)
        if family == "attention":
            return keys * Hkv * d * 2 * 2 + 2 * M * Hq * d * 2, 4.0 * keys * bs * Hq * d
        if family == "verify":
            return B * (K + 1) * V * 4.0, 0.0
        return None


def graph_seconds(fn, dev, reps: int = 10, iters: int = 5) -> float:
    """Device seconds per call of `fn`, replayed from a CUDA graph of `reps`
    calls (so host launch cost is excluded), median-free mean over `iters`."""
    fn()
    torch.cuda.synchronize(dev)
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        fn()
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fn()
    g.replay()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        g.replay()
    e1.record()
    torch.cuda.synchronize(dev)
    del g
    return e0.elapsed_time(e1) / 1e3 / (iters * reps)


def roof_of(byts: float, flops: float, seconds: float, peaks: dict) -> dict:
    """Roofline fraction of work (bytes, flops) done in `seconds`: against the
    slower of the HBM time and the tensor time (measured peaks)."""
    t_hbm = byts / (peaks["hbm_gbs"] * 1e9)
    tc = peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"]
    t_tc = flops / (tc * 1e12)
    bound = "tensor" if t_tc > t_hbm else "hbm"
    return {"bound": bound, "roofline_us": max(t_hbm, t_tc) * 1e6, "us": seconds * 1e6,
            "frac": max(t_hbm, t_tc) / seconds if seconds > 0 else None,
            "algorithmic_bytes": byts, "algorithmic_flops": flops}


def extra_measurements(st, peaks) -> dict:
    """Sub-measurements of the same workload: the prefill injection of the
    first request's whole context (batch-1 workloads) and the device-side
    proposal-input preparation at the workload's batch."""
    from block_diffusion_speculative_propose_b200 import paged_slots, prepare_proposal_inputs
    c, dev, out = st.cfg, st.dev, {}
    H, L, Hkv, d, T = (c["hidden"], c["n_layers"], c["n_kv_heads"], c["head_dim"],
                       c["n_target_layers"])
    if st.B == 1:
        n = int(st.sb.ctx_lens[0])
        g = torch.Generator(device=dev)
        g.manual_seed(11)
        aux = torch.randn(n, T * H, generator=g, device=dev).to(torch.bfloat16)
        pos = torch.arange(n, dtype=torch.int64, device=dev)
        req = torch.zeros(n, dtype=torch.int64, device=dev)
        slots = paged_slots(pos, req, st.inp["block_table"], c["page_size"])
        ws = torch.empty(st.h.inject_workspace_bytes(n), dtype=torch.uint8, device=dev)
        t = graph_seconds(lambda: st.h.inject_context(aux, pos, slots, st.kc, st.vc,
                                                       workspace=ws), dev, reps=4)
        byts = 2.0 * (H * T * H + L * 2 * Hkv * d * H) + n * (T * H * 2 + L * 2 * Hkv * d * 2)
        flops = 2.0 * n * (T * H * H + H * L * 2 * Hkv * d)
        out["prefill_inject"] = dict(rows=n, **roof_of(byts, flops, t, peaks))
        del aux, ws
    K, B = st.K, st.B
    starts = st.sb.seq_lens.to(torch.int64).to(dev)
    tp = (starts[:, None] + torch.arange(K + 1, device=dev)[None, :]).reshape(-1)
    last = ((torch.arange(B, device=dev) + 1) * (K + 1) - 1).to(torch.int32)
    nd = torch.full((B,), K, dtype=torch.int32, device=dev)
    ver = st.out["ver_tokens"]
    t = graph_seconds(lambda: prepare_proposal_inputs(tp, last, ver, nd, st.inp["block_table"],
                                                      c["page_size"], c["vocab"], ver, nd),
                      dev, reps=20)
    out["prepare_proposal_inputs"] = {"rows": int(tp.numel()), "us": t * 1e6}
    out["spec_step_graph"] = spec_step_graph(st)
    out["vocab_parallel_propose"] = vocab_parallel_propose(st)
    out["head_parallel_propose"] = head_parallel_propose(st)
    return out


def vocab_parallel_propose(st, parts_list=(1, 2, 4, 8)) -> dict:
    """One rank's share of a vocabulary-parallel proposal: the proposal with a
    1/parts shard of the LM head (dflash_propose_keys on a shard handle), as
    each rank of a parts-GPU group would run it before the all-reduce of its
    8-byte keys per draft row.  The exchange itself is not timed (one GPU)."""
    from block_diffusion_speculative_propose_b200 import DFlash
    from block_diffusion_speculative_propose_b200.tensor_parallel import vocab_shards
    c, dev, B, K = st.cfg, st.dev, st.B, st.K
    keys = torch.empty(B, K, dtype=torch.int64, device=dev)
    args = (st.inp["bonus"], st.inp["seq_lens"], st.inp["block_table"], st.kc, st.vc)
    out = {}
    for parts in parts_list:
        start, count = vocab_shards(c["vocab"], parts)[0]
        if parts == 1:
            hs = st.h
        else:
            hs = DFlash(c, dict(st.W, lm_head=st.W["lm_head"][start:start + count]),
                        device=dev.index, max_position=st.h.max_position,
                        vocab_shard=(start, count))
        try:
            t = graph_seconds(lambda: hs.propose_keys(*args, draft_keys=keys,
                                                      workspace=st.ws_prop), dev, reps=4)
        finally:
            if hs is not st.h:
                hs.close()
        out[str(parts)] = {"vocab_rows": count, "us": t * 1e6}
    return out


def head_parallel_propose(st, sizes=(2, 4, 8)) -> dict:
    """One rank's share of a head-parallel proposal (dflash_propose_tp on the
    rank-0 shard of `size`: its kv heads with their query groups, its MLP
    features and its vocabulary shard), on that rank's own K/V pool of the same
    pages.  The exchange hook is a no-op here (one GPU: the two all-reduces per
    layer are not timed), so the figure is the rank's compute alone."""
    from block_diffusion_speculative_propose_b200 import DFlash
    from block_diffusion_speculative_propose_b200.tensor_parallel import vocab_shards
    c, dev, B, K = st.cfg, st.dev, st.B, st.K
    out = {}
    args = (st.inp["bonus"], st.inp["seq_lens"], st.inp["block_table"])
    for size in sizes:
        if c["n_kv_heads"] % size:
            continue
        shard = DFlash(c, st.W, device=dev.index, max_position=st.h.max_position,
                       tp=(0, size), vocab_shard=vocab_shards(c["vocab"], size)[0])
        kc = vc = None
        try:
            shape = (st.kc[0].shape[0], c["n_kv_heads"] // size) + tuple(st.kc[0].shape[2:])
            kc = [torch.empty(shape, dtype=torch.bfloat16, device=dev) for _ in st.kc]
            vc = [torch.empty(shape, dtype=torch.bfloat16, device=dev) for _ in st.vc]
            for x in kc + vc:
                x.normal_()
            keys = torch.empty(B, K, dtype=torch.int64, device=dev)
            t = graph_seconds(lambda: shard.propose_tp(*args, kc, vc, lambda d, n, s: 0,
                                                       draft_keys=keys), dev, reps=4)
            out[str(size)] = {"kv_heads": c["n_kv_heads"] // size,
                              "intermediate": c["intermediate"] // size, "us": t * 1e6}
        finally:
            shard.close()
            del kc, vc
            torch.cuda.empty_cache()
    return out


def spec_step_graph(st, reps: int = 20) -> dict:
    """The closed-loop speculative step through the library's own CUDA graph
    (dflash_step_graph_create / _launch): verify the workload's drafts against
    its target logits, prepare the proposal inputs on the device, inject all
    K+1 verified rows of every request and propose the next block — nothing
    from the host between the stages.  The verified rows end where the
    workload's context ends, so every block lies inside the block table."""
    c, dev, K, B = st.cfg, st.dev, st.K, st.B
    T, H = c["n_target_layers"], c["hidden"]
    starts = (st.sb.seq_lens.to(torch.int64) - (K + 1)).clamp(min=0).to(dev)
    tp = (starts[:, None] + torch.arange(K + 1, device=dev)[None, :]).reshape(-1)
    last = ((torch.arange(B, device=dev) + 1) * (K + 1) - 1).to(torch.int32)
    nd = torch.full((B,), K, dtype=torch.int32, device=dev)
    g0 = torch.Generator(device=dev)
    g0.manual_seed(13)
    aux = torch.randn(B * (K + 1), T * H, generator=g0, device=dev).to(torch.bfloat16)
    g = st.h.step_graph(st.inp["prev_drafts"], st.inp["target_logits"], tp, last, nd, aux,
                        st.inp["block_table"], st.kc, st.vc)
    try:
        for _ in range(3):
            g.launch()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.launch()
        e1.record()
        torch.cuda.synchronize(dev)
        t = e0.elapsed_time(e1) / 1e3 / reps
        if st.h.check_device_errors():
            raise RuntimeError("device error in the closed-loop step")
        acc = float(g.out["num_accepted"].float().mean())
    finally:
        g.close()
    return {"rows": int(tp.numel()), "us": t * 1e6, "blocks_per_s": B / t,
            "mean_accepted": acc, "launches": reps}


def run_ours(a, rank, world, local):
    peaks, peaks_src = load_peaks()
    st = GpuStep(a.workload, local, shard_seed(a.seed, rank))
    dev = st.dev
    launches = st.launches_per_step()
    if not a.no_graph:
        st.capture()

    # ---------------------------------------------------------- timed value loop
    # the raw nvidia-smi samples go to BENCH_CLOCKS_DIR (default: the system
    # temporary directory); their summary is in the JSON line
    clocks_dir = os.environ.get("BENCH_CLOCKS_DIR") or tempfile.gettempdir()
    os.makedirs(clocks_dir, exist_ok=True)
    sampler = ClockSampler(local, os.path.join(clocks_dir, f"clocks_rank{rank}.csv"))
    for _ in range(a.warmup):
        st.step()
    torch.cuda.synchronize(dev)
    dist_barrier()
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream(dev)
    ev0.record(stream)
    for _ in range(a.steps):
        st.step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    dist_barrier()
    clocks = sampler.stop()
    t_step = dist_max(ev0.elapsed_time(ev1) / a.steps) / 1e3     # seconds, max over ranks
    B, K = st.B, st.K
    value = world * B / t_step

    # ---------------------------------------------------------- e2e (host buffers)
    e2e = None
    if not a.no_e2e:
        if a.no_graph:
            st.host_out = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
                           for k, v in st.out.items()}
            for _ in range(a.warmup):
                st.e2e_step()
            torch.cuda.synchronize(dev)
            dist_barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(a.steps):
                st.e2e_step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            dist_barrier()
            te = dist_max(e0.elapsed_time(e1) / a.steps) / 1e3
        else:
            st.e2e_setup()
            te = dist_max(st.e2e_pipelined(a.steps, a.warmup))
        h2d, d2h = st.e2e_bytes()
        e2e = {"value": world * B / te, "unit": "blocks/s", "ms_per_step": te * 1e3,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipelined": not a.no_graph}

    # ---------------------------------------------------------- per-kernel profile
    n_prof = min(a.steps, 50)
    st.h.profile_enable(launches * n_prof + 64)
    torch.cuda.synchronize(dev)
    v0, v1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    vt = 0.0
    for _ in range(n_prof):
        st.run()
    prof = st.h.profile_read()
    # verify is a handle-free call: bracket it with events on the same stream
    for _ in range(n_prof):
        v0.record(stream)
        from block_diffusion_speculative_propose_b200 import verify_greedy
        verify_greedy(st.inp["prev_drafts"], st.inp["target_logits"],
                      out_tokens=st.out["ver_tokens"], num_accepted=st.out["n_acc"],
                      bonus=st.out["new_bonus"], workspace=st.ws_ver)
        v1.record(stream)
        torch.cuda.synchronize(dev)
        vt += v0.elapsed_time(v1)
    prof["verify"] = (n_prof, vt)
    st.h.profile_disable()
    total = sum(t for _, t in prof.values())
    shares = {k: {"launches_per_step": c / n_prof, "ms_per_step": t / n_prof,
                  "share": t / total} for k, (c, t) in prof.items()}
    dom = max(prof.items(), key=lambda kv: kv[1][1])[0]
    c_dom, t_dom = prof[dom]
    per_launch_s = t_dom / c_dom / 1e3
    alg = st.algorithmic(dom)
    if alg is None:   # a light kernel dominates: report the largest GEMM family instead
        dom = max((k for k in prof if st.algorithmic(k) is not None),
                  key=lambda k: prof[k][1])
        c_dom, t_dom = prof[dom]
        per_launch_s = t_dom / c_dom / 1e3
        alg = st.algorithmic(dom)
    byts, flops = alg
    ridge = peaks.get("bf16_tflops_sustained", 1400.0) * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if flops > 0 and flops / byts > ridge:
        ach = flops / per_launch_s / 1e12
        peak = peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": ach / peak}
    else:
        ach = byts / per_launch_s / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                "frac": ach / peak}
    tr = TRAFFIC.get((a.workload, dom))
    traffic = None
    if tr and tr["digest"] == source_digest(dom):
        traffic = (tr["bytes_per_launch"] if "bytes_per_launch" in tr
                   else tr["ratio_to_algorithmic"] * byts)
    roof.update({"traffic": traffic, "kernel": dom, "algorithmic_bytes_per_launch": byts,
                 "algorithmic_flops_per_launch": flops, "launch_ms": per_launch_s * 1e3,
                 "peak_source": f"{peaks_src} ({'sustained bf16' if roof['bound'] == 'tensor' else 'HBM copy'})"})

    # per-kernel and whole-step rooflines (event-bracketed launch times)
    step_b, step_f = 0.0, 0.0
    for k, v in shares.items():
        alg_k = st.algorithmic(k)
        if alg_k is None or v["launches_per_step"] <= 0:
            continue
        per = v["ms_per_step"] / 1e3 / v["launches_per_step"]
        r = roof_of(alg_k[0], alg_k[1], per, peaks)
        v.update({"bound": r["bound"], "frac": r["frac"],
                  "algorithmic_bytes_per_launch": alg_k[0]})
        step_b += alg_k[0] * v["launches_per_step"]
        step_f += alg_k[1] * v["launches_per_step"]
    step_roof = roof_of(step_b, step_f, t_step, peaks)
    extras = extra_measurements(st, peaks) if rank == 0 and not a.no_extras else {}

    assert st.h.check_device_errors() == 0, "device error flags raised"

    line = {
        "metric": METRIC, "value": value, "unit": "blocks/s",
        "draft_tokens_per_s": value * K, "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": a.workload, "batch_per_gpu": B, "block_size": st.bs,
                   "drafts_per_block": K, "context": [st.wl["ctx_lo"], st.wl["ctx_hi"]],
                   "accept": st.wl["accept"], "injected_rows_per_step": st.R,
                   "parallelism": f"replicas x{world} (requests sharded by rank)",
                   "cuda_graph": not a.no_graph,
                   "l2": "inputs larger than L2: every step streams the draft weights "
                         f"({weight_bytes(st.cfg) / 1e9:.2f} GB) and the KV context"},
        "roofline": roof,
        "step_roofline": step_roof,
        "kernels": shares,
        "extras": extras,
        "gpu_launches": launches * a.steps,
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
        "clock_samples": clocks["samples"],
        "e2e": e2e,
    }
    # ---------------------------------------------------------- CPU baseline
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(a.workload, a.seed, target_s=10.0)
    if rank == 0:
        print(json.dumps(line), flush=True)
    st.h.close()


def weight_bytes(cfg) -> float:
    H, L, Hq, Hkv, d, I, V, T = (cfg["hidden"], cfg["n_layers"], cfg["n_q_heads"],
                                 cfg["n_kv_heads"], cfg["head_dim"], cfg["intermediate"],
                                 cfg["vocab"], cfg["n_target_layers"])
    layer = (Hq + 2 * Hkv) * d * H + H * Hq * d + 3 * I * H
    return 2.0 * (L * layer + V * H + T * H * H + L * 2 * Hkv * d * H)


# ----------------------------------------------------------------------------
# the oracle on the host cores
# ----------------------------------------------------------------------------
class OracleStep:
    """One step of the same workload run by the CPU oracle on a bounded sample
    of requests (all of them when B <= 2): verify of the sampled rows, their
    injection, and one proposal."""

    def __init__(self, wl_name: str, seed: int, max_requests: int = 2):
        import oracle as O
        from block_diffusion_speculative_propose_b200 import synth
        self.O = O
        wl = synth.WORKLOADS[wl_name]
        cfg = synth.model_config(wl["model"])
        self.cfg = cfg
        self.oc = O.OracleConfig.from_mapping(cfg)
        Wt = synth.make_weights(cfg, seed=0)
        W = {}
        for k, v in Wt.items():
            if isinstance(v, list):
                W[k] = [x.float().numpy() for x in v]
            else:
                W[k] = v.float().numpy()
        del Wt
        self.W = W
        sb = synth.make_step_batch(cfg, wl["batch"], wl["ctx_lo"], wl["ctx_hi"],
                                   accept=wl["accept"], seed=seed)
        self.B = wl["batch"]
        self.n = min(max_requests, self.B)
        P, bs = cfg["page_size"], cfg["block_size"]
        sel = list(range(self.n))
        # compact pool with just the sampled requests' pages (contents random)
        tables, pages = [], 0
        for b in sel:
            need = int(math.ceil((int(sb.seq_lens[b]) + bs) / P))
            tables.append(np.arange(pages, pages + need))
            pages += need
        width = max(len(t) for t in tables)
        self.table = np.zeros((self.n, width), dtype=np.int64)
        for i, t in enumerate(tables):
            self.table[i, :len(t)] = t
        rng = np.random.default_rng(seed)
        shape = (pages, cfg["n_kv_heads"], P, cfg["head_dim"])
        self.kc = [rng.standard_normal(shape).astype(np.float32) for _ in range(cfg["n_layers"])]
        self.vc = [rng.standard_normal(shape).astype(np.float32) for _ in range(cfg["n_layers"])]
        rows = np.isin(sb.inject_req_ids.numpy(), sel)
        self.aux = sb.aux.float().numpy()[rows].astype(np.float64)
        self.pos = sb.inject_positions.numpy()[rows]
        self.req = sb.inject_req_ids.numpy()[rows]
        self.bonus = sb.bonus.numpy()[sel]
        self.seq = sb.seq_lens.numpy()[sel]
        self.drafts = sb.prev_drafts.numpy()[sel]
        self.logits = sb.target_logits.numpy()[sel]

    def step(self):
        O = self.O
        O.verify_greedy(self.drafts, self.logits)
        slots = O.paged_slots(self.pos, self.req, self.table, self.cfg["page_size"])
        O.inject_context(self.oc, self.W, self.aux, self.pos, slots, self.kc, self.vc, "device")
        O.propose(self.oc, self.W, self.bonus, self.seq, self.table, self.kc, self.vc, "device")


def one_thread():
    """The oracle runs single-threaded: numpy's BLAS pool limited to one thread
    for the duration of the CPU legs."""
    from threadpoolctl import threadpool_limits
    return threadpool_limits(limits=1, user_api="blas")


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def cpu_baseline(wl_name: str, seed: int, target_s: float = 10.0) -> dict:
    os_ = OracleStep(wl_name, seed)
    with one_thread():
        threads = blas_threads()
        t0 = time.perf_counter()
        n = 0
        while True:
            os_.step()
            n += 1
            if time.perf_counter() - t0 >= target_s:
                break
        dt = (time.perf_counter() - t0) / n
    extrap = os_.n < os_.B
    return {"value": os_.n / dt, "unit": "blocks/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} oracle step(s) of {os_.n} of {os_.B} request(s) (verify + inject + "
                      f"propose, device storage precision, whole contexts), {dt:.2f} s per step; "
                      f"numpy float64 on one thread"
                      + (f"; requests are independent, so the per-request rate of the sample "
                         f"stands for the batch of {os_.B} (extrapolated)" if extrap else ""),
            "extrapolated": extrap, "host_cores": os.cpu_count(), "cpu_model": cpu_model()}


# Wall-clock bound of the reference arm's timed steps: one oracle step of a
# batch-1 workload takes about ten seconds on the host cores, so the K timed
# steps run whole oracle steps on an evenly spaced subset of them (all K when
# they fit the bound) and the value is requests processed / elapsed time.
REF_BUDGET_S = 120.0


def run_reference(a, rank, world):
    if rank != 0:
        return
    os_ = OracleStep(a.workload, a.seed)
    lim = one_thread()
    threads = blas_threads()
    # warm-up: one whole oracle step, which also times it (taken even when W = 0)
    t0 = time.perf_counter()
    os_.step()
    t_one = time.perf_counter() - t0
    n_run = max(1, min(a.steps, int(REF_BUDGET_S // max(t_one, 1e-9))))
    done = 0
    t0 = time.perf_counter()
    for i in range(a.steps):
        if (i + 1) * n_run // a.steps > done:     # n_run evenly spaced steps
            os_.step()
            done += 1
    elapsed = time.perf_counter() - t0
    lim.restore_original_limits()
    dt = elapsed / a.steps
    value = done * os_.n / elapsed
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "blocks/s",
        "draft_tokens_per_s": value * (os_.cfg["block_size"] - 1), "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": a.workload, "batch_per_gpu": os_.B,
                   "block_size": os_.cfg["block_size"]},
        "cpu_baseline": {"value": value, "unit": "blocks/s", "cores": threads,
                         "kind": "oracle",
                         "sample": f"{done} whole oracle step(s) of {os_.n} of {os_.B} "
                                   f"request(s) (verify + inject + propose at the device "
                                   f"storage precision, whole contexts, {t_one:.1f} s each, one "
                                   f"thread) spread evenly over the {a.steps} timed steps to "
                                   f"bound the run at {REF_BUDGET_S:.0f} s; value = requests "
                                   f"processed / elapsed time"
                                   + ("; the per-request rate of the sample stands for the "
                                      "whole batch (extrapolated)" if os_.n < os_.B else ""),
                         "extrapolated": os_.n < os_.B, "cpu_model": cpu_model()},
        "oracle_steps_timed": done,
        "e2e": {"value": value, "unit": "blocks/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def ncu_case(a):
    """Reduced cases of the workload's hot kernel families, each run twice, so
    that a profiler can capture the second launch on a few GB of device memory:
      attention  one layer of block attention for 16 requests drawn from the
                 workload's context-length distribution (paged, shuffled pages)
      gemms      injection + proposal at the workload's batch with 64-token
                 contexts: the GEMM shapes of the full step (block rows, LM-head
                 rows, injected rows) with a small KV pool
      verify     greedy verification of the workload's [B, K+1, V] fp32 logits"""
    from block_diffusion_speculative_propose_b200 import DFlash, paged_slots, synth, verify_greedy
    wl = synth.WORKLOADS[a.workload]
    cfg = synth.model_config(wl["model"])
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(a.seed)
    B, bs, P = wl["batch"], cfg["block_size"], cfg["page_size"]
    Hkv, d = cfg["n_kv_heads"], cfg["head_dim"]
    if a.ncu_case == "verify":
        V, K = cfg["vocab"], bs - 1
        lo = torch.randn(B, K + 1, V, generator=g, device=dev)
        dr = torch.randint(0, V, (B, K), generator=g, device=dev).to(torch.int32)
        for _ in range(2):
            verify_greedy(dr, lo)
        torch.cuda.synchronize()
        print(json.dumps({"ncu_case": "verify", "algorithmic_bytes": lo.numel() * 4.0}))
        return
    if a.ncu_case == "attention":
        c1 = dict(cfg, n_layers=1, vocab=2048, mask_token_id=2047)
        h = DFlash(c1, synth.make_weights(c1, seed=0, device=dev),
                   max_position=wl["ctx_hi"] + 2 * bs)
        rng = np.random.default_rng(a.seed)
        n = 16
        seq = rng.integers(wl["ctx_lo"], wl["ctx_hi"] + 1, size=n).astype(np.int32)
        need = [-(-(int(s) + bs) // P) for s in seq]
        perm = rng.permutation(sum(need))
        table = np.zeros((n, max(need)), dtype=np.int32)
        cur = 0
        for b, m in enumerate(need):
            table[b, :m] = perm[cur:cur + m]
            cur += m
        shape = (sum(need), Hkv, P, d)
        kc = torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)
        vc = torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)
        q = torch.randn(n * bs, cfg["n_q_heads"], d, generator=g, device=dev).to(torch.bfloat16)
        seq_t, table_t = torch.tensor(seq, device=dev), torch.tensor(table, device=dev)
        for _ in range(2):
            h.block_attention(q, seq_t, table_t, kc, vc)
        torch.cuda.synchronize()
        keys = float((seq.astype(np.float64) + bs).sum())
        byts = keys * Hkv * d * 2 * 2 + 2 * n * bs * cfg["n_q_heads"] * d * 2
        print(json.dumps({"ncu_case": "attention", "requests": n, "algorithmic_bytes": byts,
                          "device_errors": h.check_device_errors()}))
        h.close()
        return
    # gemms
    h = DFlash(cfg, synth.make_weights(cfg, seed=0, device=dev), max_position=4096)
    ctx = 64
    per = -(-(ctx + 2 * bs) // P)
    table = torch.arange(B * per, dtype=torch.int32, device=dev).view(B, per)
    shape = (B * per, Hkv, P, d)
    kc = [torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)
          for _ in range(cfg["n_layers"])]
    vc = [torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)
          for _ in range(cfg["n_layers"])]
    rows_per = 6 if wl["accept"] == "geometric" else (bs + 1) // 2
    rows = B * rows_per
    req = (torch.arange(rows, device=dev) % B).to(torch.int64)
    pos = (ctx - rows_per + torch.arange(rows, device=dev) // B).to(torch.int64)
    slots = paged_slots(pos, req, table, P)
    aux = torch.randn(rows, cfg["n_target_layers"] * cfg["hidden"], generator=g,
                      device=dev).to(torch.bfloat16)
    bonus = torch.randint(0, cfg["vocab"] - 1, (B,), generator=g, device=dev).to(torch.int32)
    seq = torch.full((B,), ctx, dtype=torch.int32, device=dev)
    for _ in range(2):
        h.inject_context(aux, pos, slots, kc, vc)
        h.propose(bonus, seq, table, kc, vc)
    torch.cuda.synchronize()
    print(json.dumps({"ncu_case": "gemms", "block_rows": B * bs, "injected_rows": rows,
                      "device_errors": h.check_device_errors()}))
    h.close()


def main():
    a = parse_args()
    if a.ncu_case:
        ncu_case(a)
        return
    rank, world, local = dist_init(a.gpus)
    try:
        if a.impl == "reference":
            run_reference(a, rank, world)
        else:
            run_ours(a, rank, world, local)
    finally:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
