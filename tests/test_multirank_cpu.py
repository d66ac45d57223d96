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


# ---- head-sharded attention for sequence-sharded callers (two gloo ranks) -------------------

def _oracle_heads(q, k, v, shape, thr, window, scale):
    """The hot path on a rank's heads, computed by the oracle (fp64, natural order in/out)."""
    import numpy as np
    import oracle
    T, Hg, W, P = shape.T, shape.Hg, shape.W, shape.P
    out = torch.empty(q.shape, dtype=torch.float64)
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            qf, kf, vf = (oracle.reorder(x[b, h].double().numpy()[None, None], T, Hg, W, P)
                          for x in (q, k, v))
            mk, _, _ = oracle.nabla_mask(qf, kf, T, Hg, W, P, thr, window, scale=scale)
            o, _ = oracle.block_sparse_attention(qf, kf, vf, mk, P * P, scale)
            out[b, h] = torch.from_numpy(oracle.inverse_reorder(o, T, Hg, W, P)[0, 0])
    return out


def _sharded_worker(rank, world, port, wl_args, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from adaptive_block_sparse_b200 import sharding
    from synth import Workload, make_qkv
    dist.init_process_group("gloo", rank=rank, world_size=world)
    wl = Workload(**wl_args)
    q, k, v = make_qkv(wl)
    s = wl.S // world
    mine = slice(rank * s, (rank + 1) * s)       # this rank's contiguous token range
    x = [t[:, :, mine].contiguous() for t in (q, k, v)]
    # the two exchanges alone: a round trip returns the input, and the head shard holds
    # every token of the rank's heads
    heads = sharding.seq_to_heads(x[0])
    hpr = wl.H // world
    assert torch.equal(heads, q[:, rank * hpr:(rank + 1) * hpr])
    assert torch.equal(sharding.heads_to_seq(heads), x[0])
    o = sharding.sharded_nabla_attention(*x, wl.T, wl.Hg, wl.W, wl.thrs[0], wl.window,
                                         compute=_oracle_heads, balance="contiguous")
    out.put((rank, o))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("wl_args", [
    dict(name="sh_a", B=1, H=2, T=2, Hg=16, W=16, D=64, thrs=(0.8,), seed=1101),
    dict(name="sh_b", B=2, H=4, T=2, Hg=16, W=8, D=64, thrs=(0.6,), window=(1, 1, 1), seed=1102),
])
def test_sharded_attention_gloo_world2(wl_args):
    """Sequence-sharded inputs -> all-to-all to head shards -> per-head path -> all-to-all
    back: equals the unsharded computation exactly."""
    import math
    from adaptive_block_sparse_b200 import Shape
    from synth import Workload, make_qkv
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_worker, args=(r, 2, port, wl_args, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(out.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = Workload(**wl_args)
    q, k, v = make_qkv(wl)
    shape = Shape(wl.B, wl.H, wl.T, wl.Hg, wl.W, wl.D)
    ref = _oracle_heads(q, k, v, shape, wl.thrs[0], wl.window, 1 / math.sqrt(wl.D))
    got = torch.cat([res[0], res[1]], dim=2)
    assert torch.equal(got, ref)


# ---- head balance: units assigned to ranks by load (longest processing time first) ----------

def test_lpt_assign_plan_and_bound():
    from adaptive_block_sparse_b200.sharding import lpt_assign
    # one heavy head and many light ones: the contiguous split would give 102 against 52
    loads = [100, 1, 1, 1, 1, 50]
    plan = lpt_assign(loads, 2)
    assert plan == [[0], [1, 2, 3, 4, 5]]
    rng = __import__("numpy").random.default_rng(3)
    for n in (2, 3, 4, 8):
        for _ in range(20):
            loads = [int(x) for x in rng.integers(1, 1000, size=int(rng.integers(n, 50)))]
            plan = lpt_assign(loads, n)
            assert sorted(u for p in plan for u in p) == list(range(len(loads)))
            span = max(sum(loads[u] for u in p) for p in plan)
            lower = max(max(loads), sum(loads) / n)       # no split can do better than this
            assert span <= 4.0 / 3.0 * lower + 1e-9


def _lpt_worker(rank, world, port, wl_args, loads, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from adaptive_block_sparse_b200 import sharding
    from synth import Workload, make_qkv
    dist.init_process_group("gloo", rank=rank, world_size=world)
    wl = Workload(**wl_args)
    q, k, v = make_qkv(wl)
    s = wl.S // world
    mine = slice(rank * s, (rank + 1) * s)
    x = [t[:, :, mine].contiguous() for t in (q, k, v)]
    plan = sharding.lpt_assign(loads, world)
    # the uneven exchanges alone: every token of this rank's units, and back
    u = sharding.seq_to_units(x[0], plan)
    assert torch.equal(u[0], q.reshape(wl.B * wl.H, wl.S, wl.D)[plan[rank]])
    assert torch.equal(sharding.units_to_seq(u, plan, wl.B, wl.H), x[0])
    o = sharding.sharded_nabla_attention(*x, wl.T, wl.Hg, wl.W, wl.thrs[0], wl.window,
                                         compute=_oracle_heads, balance="lpt", loads=loads)
    out.put((rank, o, len(plan[rank])))
    dist.barrier()
    dist.destroy_process_group()


def test_sharded_attention_lpt_gloo_world2():
    """Deliberately skewed head loads: the heavy head gets a rank of its own, the light
    ones share the other; the result equals the unsharded computation exactly."""
    import math
    from adaptive_block_sparse_b200 import Shape
    from synth import Workload, make_qkv
    wl_args = dict(name="sh_lpt", B=2, H=3, T=2, Hg=16, W=16, D=64, thrs=(0.7,), seed=1103)
    loads = [900, 5, 7, 3, 400, 2]        # per (b, h): units 0 and 4 dominate
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_lpt_worker, args=(r, 2, port, wl_args, loads, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = {r: (o, nu) for r, o, nu in (out.get(timeout=300) for _ in procs)}
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][1] == 1 and res[1][1] == 5          # plan [[0], [1, 2, 3, 4, 5]]
    wl = Workload(**wl_args)
    q, k, v = make_qkv(wl)
    shape = Shape(wl.B, wl.H, wl.T, wl.Hg, wl.W, wl.D)
    ref = _oracle_heads(q, k, v, shape, wl.thrs[0], wl.window, 1 / math.sqrt(wl.D))
    got = torch.cat([res[0][0], res[1][0]], dim=2)
    assert torch.equal(got, ref)
