"""Host logic of the multi-rank benchmark on CPU: two gloo ranks.

The chunked forward shards by batch: every rank runs an independent batch of
the same workload and no collective touches the data path.  What the ranks do
share is the timing protocol (barrier, max over ranks) and the whole-job
throughput; these tests run that logic as two gloo processes on 127.0.0.1.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    import bench
    import workloads
    w_, r_, l_ = bench.dist_setup(world, backend="gloo")
    assert (w_, r_, l_) == (world, rank, rank)
    dev = torch.device("cpu")
    bench.barrier(world, dev)
    # Per-rank step times: the job time is the slowest rank's.
    ms_local = 2.0 + 3.0 * rank
    ms = bench.max_over_ranks(ms_local, world, dev)
    w = workloads.workload("tiny_fp32")
    inp = workloads.chunk_inputs(w, seed=bench.rank_seed(w, rank))
    res = {"ms": ms, "value": bench.whole_job_value(w.token_heads, world, ms),
           "q0": float(inp["q"].flatten()[0]), "token_heads": w.token_heads}
    with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
        json.dump(res, f)
    bench.barrier(world, dev)
    dist.destroy_process_group()


def test_two_gloo_ranks_timing_protocol(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r = [json.load(open(tmp_path / ("rank%d.json" % i))) for i in range(world)]
    # Max over ranks: both ranks see the slower rank's 5 ms.
    assert r[0]["ms"] == r[1]["ms"] == 5.0
    # Weak scaling: both ranks' units over the slowest time.
    assert r[0]["value"] == pytest.approx(world * r[0]["token_heads"] / 5e-3)
    # Independent batches per rank.
    assert r[0]["q0"] != r[1]["q0"]


def test_whole_job_value_single_rank():
    import bench
    assert bench.whole_job_value(1000, 1, 2.0) == pytest.approx(5e5)
    assert bench.whole_job_value(1000, 4, 2.0) == pytest.approx(2e6)


def test_reference_arm_only_rank0_works():
    """Under torchrun the reference arm runs on rank 0 alone; rank 1 exits 0 silently."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert p.returncode == 0
    assert p.stdout.strip() == ""


def test_reference_arm_rank0_json_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["unit"] == "tokens·heads/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
