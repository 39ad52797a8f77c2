"""Multi-process host logic of the benchmark on CPU (gloo, world size 2).

The attention path shards with no exchange: every rank runs its own batch
(weak scaling) and only the timing takes the max over ranks. These tests run
that logic on two CPU processes, and the reference arm under torchrun, where
rank 0 alone does the work and prints."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    from causal_sliding_window_rope_b200 import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + rank, 3.0 * (1 - rank)]
        got = bench.reduce_max(local, dist, "cpu")
        x = synth.layer_inputs(1, 4, 2, 1, 4, False, torch.float32,
                               config=bench.rank_config_id(rank))["q"]
        gathered = [torch.zeros_like(x) for _ in range(world)]
        dist.all_gather(gathered, x)
        out.put((rank, got, bool(torch.equal(gathered[0], gathered[1]))))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_distinct_shards():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = [out.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, same in results:
        assert got == [11.0, 3.0]       # max over ranks, identical everywhere
        assert not same                 # each rank draws its own batch


def test_reference_arm_under_torchrun_prints_once_on_rank0():
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="4")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["n_gpus"] == 2
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
