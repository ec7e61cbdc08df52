"""Multi-process paths of bench.py on CPU (gloo, world size 2).

The decode has no exchange step: ranks decode their own tensors and meet
only to time the step (barrier, maximum over ranks) and to add up the work.
These tests run those reductions in two real processes, and the reference
arm under the launcher the benchmark driver uses.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.setup_dist()
    try:
        bench.barrier(w)
        q.put((r, bench.max_over_ranks(1.5 + r, w), bench.sum_over_ranks(10.0 * (r + 1), w)))
    finally:
        dist.destroy_process_group()


def test_rank_reductions_with_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == [(0, 2.5, 30.0), (1, 2.5, 30.0)]


def test_reference_arm_under_the_launcher_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", "bench.py", "--impl",
           "reference", "--config", "single", "--steps", "3", "--warmup", "3",
           "--cpu-budget-s", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["unit"] == "GB/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] == 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0


@pytest.mark.parametrize("config", ["block", "stack"])
def test_decode_groups(config):
    sys.path.insert(0, ROOT)
    import bench
    names = [u[0] for u in bench.workload_units(config, 0)]
    groups = bench.block_groups(config, names)
    assert sorted(i for g in groups for i in g) == list(range(len(names)))
    if config == "stack":
        assert len(groups) == 38 and all(len(g) == 7 for g in groups[1:-1])
    else:
        assert groups == [list(range(7))]
