"""Multi-process path of bench.py on the host: world size 2 over gloo (no GPU).

bench.py --gpus N runs one process per GPU; every rank replicates the workload (weak
scaling: the heads of the path are independent, no data-path collective), the timing is
bracketed by barriers and reduced with a max over ranks, and the work is summed over
ranks.  These tests run that rank logic with two CPU processes.
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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    w, r, _ = bench.init_dist(backend="gloo")
    bench.barrier(w)
    cpu = torch.device("cpu")
    out.put((r, w, bench.max_over_ranks(float(r + 1) * 1.5, w, cpu), bench.sum_over_ranks(float(r + 1), w, cpu)))
    bench.barrier(w)
    dist.destroy_process_group()


def test_rank_helpers_gloo_world2():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, *_ in res] == [0, 1]
    for _, w, mx, sm in res:
        assert w == 2
        assert mx == 3.0          # max over ranks of (rank + 1) * 1.5
        assert sm == 3.0          # sum over ranks of (rank + 1)


def test_reference_arm_torchrun_world2():
    """Under torchrun with 2 ranks the reference arm runs on rank 0 only, which prints one
    JSON line carrying the launched world size; the other rank exits 0 without output."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT,
                       env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
