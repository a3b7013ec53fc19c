"""Host-side logic of bench.py on CPU: the N > 1 path with two gloo ranks
(sharded batches, max-over-ranks timing) and the oracle reference arm."""

from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    from block_diffusion_speculative_propose_b200 import synth
    r, w, local = bench.dist_init(world)
    try:
        t = bench.dist_max(1.0 + rank)            # per-rank "step time"
        cfg = synth.model_config("tiny")
        sb = synth.make_step_batch(cfg, 4, 10, 500, seed=bench.shard_seed(1, rank),
                                   with_aux=False, with_logits=False)
        bench.dist_barrier()
        q.put((rank, w, t, sb.seq_lens.tolist()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_take_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29511
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, t0, s0), (r1, w1, t1, s1) = res
    assert (w0, w1) == (2, 2)
    assert t0 == t1 == 2.0                 # both ranks see the slowest rank's time
    assert s0 != s1                        # each rank draws its own requests


def test_reference_arm_prints_one_json_line():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--workload", "tiny_b1_ctx64", "--steps", "2", "--warmup", "3"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "blocks/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["steps"] == 2 and d["warmup"] == 3


def test_reference_arm_bounds_its_run(monkeypatch, capsys):
    """With many timed steps, the reference arm runs only as many whole oracle
    steps as fit its wall-clock bound, spread over the K steps, and says so."""
    sys.path.insert(0, ROOT)
    import time
    import types

    import bench

    class FakeOracle:
        calls = 0

        def __init__(self, wl_name, seed):
            self.n, self.B, self.cfg = 1, 1, {"block_size": 4}

        def step(self):
            FakeOracle.calls += 1
            time.sleep(0.02)

    monkeypatch.setattr(bench, "OracleStep", FakeOracle)
    monkeypatch.setattr(bench, "REF_BUDGET_S", 0.1)
    a = types.SimpleNamespace(workload="tiny_b1_ctx64", seed=1, steps=200, warmup=3)
    bench.run_reference(a, 0, 1)
    d = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    timed = d["oracle_steps_timed"]
    assert 1 <= timed <= 6 and FakeOracle.calls == timed + 1     # + the calibration step
    assert d["steps"] == 200 and d["value"] > 0
    assert f"{timed} whole oracle step" in d["cpu_baseline"]["sample"]
    # few steps: all of them run
    FakeOracle.calls = 0
    a.steps = 2
    bench.run_reference(a, 0, 1)
    d = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert d["oracle_steps_timed"] == 2 and FakeOracle.calls == 3


def test_traffic_records_match_the_kernel_sources():
    """Every ncu traffic record in bench.py was taken on the kernel sources as
    they stand: a kernel change without a new capture would make the bench
    line's roofline.traffic read null."""
    import bench
    for (workload, family), rec in bench.TRAFFIC.items():
        fam = "attention" if family == "attention" else "gemm"
        assert rec["digest"] == bench.source_digest(fam), (workload, family)
        assert ("ratio_to_algorithmic" in rec) != ("bytes_per_launch" in rec)
        if "ratio_to_algorithmic" in rec:
            assert 1.0 <= rec["ratio_to_algorithmic"] < 1.2
    # the default workload's dominant kernel has a record
    assert (bench.DEFAULT_WORKLOAD, "attention") in bench.TRAFFIC
