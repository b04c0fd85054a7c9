"""The multi-process (N > 1) host logic of bench.py, on CPU.

The path shards into independent replicas (one per GPU, its own seeded
inputs, no collective in the data path); the only cross-rank step is the max
of the timings, so that the slowest rank sets the job's time. Here two
``gloo`` ranks run that step, and a two-rank torchrun launch runs the
reference arm, which must print one line from rank 0 and none elsewhere.
The bench's CPU-baseline leg, which runs on the host alone, is checked here
too.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from trainable_gated_block_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


# per-rank timings (ms): the max is taken element by element
TIMES = {0: [5.0, 10.0, 0.25], 1: [7.0, 3.0, 0.5]}


def _gloo_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, _ = bench.rank_env()
        got = bench.max_over_ranks(TIMES[rank], dist, torch.device("cpu"))
        res = dict(world=w, rank=r, max=got, tflops=bench.weak_tflops(w, 1e12, got[0]))
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.spawn(_gloo_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    want = [max(a, b) for a, b in zip(TIMES[0], TIMES[1])]
    for rank in (0, 1):
        with open(tmp_path / f"rank{rank}.json") as f:
            res = json.load(f)
        assert res["world"] == 2 and res["rank"] == rank
        assert res["max"] == want                       # every rank sees the slowest rank's times
        # whole-job throughput: both replicas' work over the slowest rank's time
        assert res["tflops"] == pytest.approx(2 * 1e12 / (want[0] * 1e-3) / 1e12)


def test_single_process_is_identity():
    vals = [1.5, 2.0]
    assert bench.max_over_ranks(vals, dist, torch.device("cpu")) == vals
    assert bench.max_over_ranks(vals, None, None) == vals


def test_rank_env(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.rank_env() == (1, 0, 0)
    monkeypatch.setenv("WORLD_SIZE", "4")
    monkeypatch.setenv("RANK", "3")
    monkeypatch.setenv("LOCAL_RANK", "3")
    assert bench.rank_env() == (4, 3, 3)


def test_replicas_get_different_inputs():
    cfg = inputs.PrefillConfig("small", "bf16", 1, 256, 4, 2, 128, 2, "normal", 1.0, seed=7)
    seeds = [bench.replica_seed(cfg.seed, r) for r in range(4)]
    assert len(set(seeds)) == 4
    x0 = inputs.make_prefill(cfg, seed=seeds[0])
    x1 = inputs.make_prefill(cfg, seed=seeds[1])
    assert not torch.equal(x0["q"], x1["q"]) and not torch.equal(x0["s"], x1["s"])
    assert torch.equal(x0["q"], inputs.make_prefill(cfg, seed=seeds[0])["q"])   # and are reproducible


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "1", "--prefill", "qwen3-4b-8k"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout                   # rank 0 alone prints
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_cpu_baseline_line_on_cpu():
    """The bench's CPU-baseline leg (the fp64 oracle on a bounded sample) runs on the host alone."""
    cfg = inputs.workload("qwen3-4b-8k")
    x = inputs.make_prefill(cfg)
    cb = bench.cpu_baseline(cfg, x, 0.5)
    assert cb["kind"] == "oracle" and cb["unit"] == "TFLOPS" and cb["value"] > 0
    assert cb["cores"] >= 1 and cb["affinity_cores"] >= 1
    assert set(cb["parts_s"]) == {"select", "fwd", "bwd"} and all(v >= 0 for v in cb["parts_s"].values())
    assert cb["fwd_tflops"] > 0 and cb["bwd_tflops"] > 0
