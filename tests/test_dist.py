"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): the
max-over-ranks timing reduction and the per-rank independent batches.  The
layer itself does not shard, so N GPUs run N independent replicas."""
import json
import os
import socket
import subprocess
import sys
from datetime import timedelta

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    from sparse_mixture_experts_04_b200.synth import CONFIGS
    step_ms = [2.5, 3.25][rank]
    v = bench.max_over_ranks(step_ms, world, device="cpu")
    seed = bench.rank_config(CONFIGS["mixtral"], rank).seed
    q.put((rank, v, seed))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_independent_batches_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    assert [o[1] for o in out] == [3.25, 3.25]          # every rank sees the slowest rank's time
    assert out[0][2] != out[1][2]                        # each rank draws its own batch


def test_reference_arm_prints_one_json_line_on_cpu():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_fp32",
                        "--steps", "3", "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_non_zero_ranks_exit_quietly():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_fp32",
                        "--steps", "3", "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]
