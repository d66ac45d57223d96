"""Benchmark of the NABLA hot path on B200 (one JSON line on stdout, rank 0).

A step is one pass of the whole hot path over one batch of synthetic video-latent input
already resident in HBM:
  reorder Q, K, V (fused block pooling of Q and K)  ->  adaptive mask build (pooled
  scores, softmax, CDF threshold, optional STA union)  ->  block-sparse attention forward
  [-> backward for the training workload].
The headline value is the kept-block throughput of the whole step: kept (query block,
key block) tiles x 4*64*64*D FLOPs (x 3.5 with the backward: 2 + 5 GEMMs) / step time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config wan720p] [--impl ours]
  python bench.py --impl reference ...     # the CPU oracle arm (host cores)

Multi-GPU: heads are independent, so every rank runs its own copy of the workload
(weak scaling, no data-path collective); the step time is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import WORKLOADS, make_dout, make_qkv  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
PROFILE_FWD = os.path.join(ROOT, "profiles", "attn_fwd_wan720p_h8_full.md")
KERNEL_SOURCES = [os.path.join(ROOT, "adaptive_block_sparse_b200", "csrc", f)
                  for f in ("attn_fwd.cu", "common.cuh")]


def measured_traffic(workload: str):
    """DRAM bytes per forward launch from the committed ncu summary, or None.

    The summary carries the figure for the 40-head 720p-like launch (measured on heads
    0-7, scaled by heads) and a hash of the kernel sources it was taken from; the value is
    only reported while the sources are unchanged and for that workload.
    """
    import hashlib
    if workload != "wan720p" or not os.path.exists(PROFILE_FWD):
        return None
    fields = {}
    for line in open(PROFILE_FWD):
        if ":" in line and line.split(":")[0].strip() in ("traffic_bytes_per_launch", "source_sha256"):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(f, "rb") as fh:
            h.update(fh.read())
    if fields.get("source_sha256") != h.hexdigest() or "traffic_bytes_per_launch" not in fields:
        return None
    return float(fields["traffic_bytes_per_launch"])

FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "NABLA attn fwd ms & TFLOP/s (kept blocks), % bf16 TC peak, vs dense; mask GB/s"


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK}, "measured"
    except (OSError, ValueError, KeyError, TypeError):
        return dict(FALLBACK), "fallback"


# --------------------------------------------------------------------------------------
# clocks sampler (nvidia-smi during the timed region)
# --------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        time.sleep(0.05)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------------------
# distributed plumbing
# --------------------------------------------------------------------------------------
def init_dist(backend=None):
    """One process per GPU (torchrun environment).  NCCL on GPUs; gloo when there is no
    GPU (the rank logic is exercised on the host).  Returns (world, rank, local rank)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        timeout = datetime.timedelta(seconds=300)
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timeout)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, dev):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, world, dev):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# --------------------------------------------------------------------------------------
# the CUDA path
# --------------------------------------------------------------------------------------
class Path:
    """Buffers and the step of the hot path for one workload on one GPU."""

    def __init__(self, wl, dev, units=None):
        """``units``: optional list of flat (b*H + h) heads of ``wl`` to keep (the rank's
        share of a strong-scaling run); they form a problem of B = 1, H = len(units)."""
        import dataclasses
        import adaptive_block_sparse_b200 as m
        self.m = m
        full_wl = wl
        self.q, self.k, self.v = make_qkv(wl, device=dev)          # natural order
        if units is not None:
            pick = torch.tensor(units, dtype=torch.long, device=dev)
            self.q, self.k, self.v = (t.reshape(wl.B * wl.H, wl.S, wl.D)[pick][None].contiguous()
                                      for t in (self.q, self.k, self.v))
            wl = dataclasses.replace(wl, B=1, H=len(units))
        self.wl = wl
        self.dev = dev
        self.shape = m.Shape(wl.B, wl.H, wl.T, wl.Hg, wl.W, wl.D, wl.P)
        sh = self.shape
        self.thr = wl.thrs[0] if len(wl.thrs) == 1 else 0.8
        # Both steps read Q, K, V in their natural order (no reordered copy): only the
        # pooled means are computed beforehand.  Training also converts V to fp16 in place
        # order (the P V products and the backward take fp16 P and V), and the forward
        # writes f32 O for the backward.
        self.natural = True
        if wl.backward:
            self.vh = torch.empty(self.q.shape, dtype=torch.float16, device=dev)
        self.qp = torch.empty(wl.B, wl.H, sh.nb, wl.D, dtype=torch.float64, device=dev)
        self.kp = torch.empty_like(self.qp)
        # the forward reads the bitmask only; the lists serve the backward
        self.bits, self.ridx, self.rcnt, self.cidx, self.ccnt = m.alloc_mask(
            sh, dev, lists=wl.backward, cols=wl.backward)
        self.mask_ws = torch.zeros(m.nabla_mask_workspace_bytes(sh), dtype=torch.uint8, device=dev)
        self.fwd_ws = torch.zeros(m.nabla_fwd_workspace_bytes(sh), dtype=torch.uint8, device=dev)
        self.o_dtype = m.NABLA_F32 if wl.backward else m.NABLA_BF16
        self.o = torch.empty(self.q.shape, device=dev,
                             dtype=torch.float32 if wl.backward else torch.bfloat16)
        self.lse = torch.empty(wl.B, wl.H, wl.S, dtype=torch.float32, device=dev)
        if wl.backward:
            self.do = make_dout(full_wl, device=dev)
            if units is not None:
                self.do = self.do.reshape(full_wl.B * full_wl.H, wl.S, wl.D)[pick][None].contiguous()
            self.dq, self.dk, self.dv = (torch.empty(self.q.shape, dtype=torch.float32, device=dev)
                                         for _ in range(3))
            self.bwd_ws = torch.zeros(m.nabla_bwd_workspace_bytes(sh), dtype=torch.uint8, device=dev)
        self.ev = {}

    def launches_per_step(self):
        """Kernels of this library launched by one step (memsets not counted).

        Inference: the mask (pooling + fp16 split of Q, of K, logits, select, fp64
        rescue); forward (schedule: per-head sort + head placement; attention).  Training:
        V to fp16; the mask as above + column lists; forward; backward (2 schedules of 2
        launches, preprocess, dK/dV, dQ).
        """
        if not self.wl.backward:
            return 5 + 3
        return 1 + 5 + 1 + 3 + 7

    def fill_pools(self):
        """The fp64 pooled means of Q and K (for the measurements made from pools)."""
        self.m.nabla_reorder(self.q, None, self.shape, pool_out=self.qp)
        self.m.nabla_reorder(self.k, None, self.shape, pool_out=self.kp)

    def _mark(self, name, timing):
        if timing:
            e = torch.cuda.Event(enable_timing=True)
            e.record()
            self.ev.setdefault(name, []).append(e)

    def step(self, timing=False):
        m, sh, wl = self.m, self.shape, self.wl
        self._mark("t0", timing)
        if wl.backward:
            m.nabla_reorder(self.v, self.vh, sh, inverse=m.REORDER_KEEP)
        self._mark("t_reorder", timing)
        # the mask pools Q and K itself (natural order), one pass over each
        m.nabla_build_mask(self.q, self.k, sh, self.thr, wl.window, mask_bits=self.bits,
                           row_idx=self.ridx, row_cnt=self.rcnt, col_idx=self.cidx,
                           col_cnt=self.ccnt, workspace=self.mask_ws,
                           layout=m.NABLA_LAYOUT_NATURAL)
        self._mark("t_mask", timing)
        v = self.vh if wl.backward else self.v
        m.nabla_attn_fwd(self.q, self.k, v, self.bits, sh, o=self.o, o_dtype=self.o_dtype,
                         lse=self.lse, workspace=self.fwd_ws, layout=m.NABLA_LAYOUT_NATURAL)
        self._mark("t_fwd", timing)
        if wl.backward:
            m.nabla_attn_bwd(self.q, self.k, self.vh, self.o, self.do, self.lse, self.ridx,
                             self.rcnt, self.cidx, self.ccnt, sh, dq=self.dq, dk=self.dk,
                             dv=self.dv, workspace=self.bwd_ws, layout=m.NABLA_LAYOUT_NATURAL)
            self._mark("t_bwd", timing)

    def segment_ms(self, a, b):
        return [x.elapsed_time(y) for x, y in zip(self.ev[a], self.ev[b])]

    def kept_pairs(self):
        return int(self.rcnt.to(torch.int64).sum().item())

    def check_status(self):
        for ws in [self.fwd_ws] + ([self.bwd_ws] if self.wl.backward else []):
            code = self.m.nabla_read_device_status(ws)
            if code:
                raise RuntimeError(f"device status 0x{code:x}")


def head_loads(wl, dev):
    """Kept tiles of every (b, h) of a workload (pools + mask on the GPU), for the
    strong-scaling split; every rank computes the same numbers."""
    import adaptive_block_sparse_b200 as m
    sh = m.Shape(wl.B, wl.H, wl.T, wl.Hg, wl.W, wl.D, wl.P)
    q, k, _ = make_qkv(wl, device=dev)
    qp = torch.empty(wl.B, wl.H, sh.nb, wl.D, dtype=torch.float64, device=dev)
    kp = torch.empty_like(qp)
    m.nabla_reorder(q, None, sh, pool_out=qp)
    m.nabla_reorder(k, None, sh, pool_out=kp)
    cnt = torch.empty(wl.B, wl.H, sh.nb, dtype=torch.int32, device=dev)
    thr = wl.thrs[0] if len(wl.thrs) == 1 else 0.8
    m.nabla_build_mask(None, None, sh, thr, wl.window, row_cnt=cnt, q_pool=qp, k_pool=kp)
    loads = cnt.to(torch.int64).sum(dim=-1).reshape(-1).tolist()
    del q, k, qp, kp, cnt
    torch.cuda.empty_cache()
    return loads


def time_call(fn, iters, warm=2):
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(iters):
        fn()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / iters


# --------------------------------------------------------------------------------------
# CPU oracle timing (bounded sample)
# --------------------------------------------------------------------------------------
def oracle_sample(wl, q_nat, k_nat, v_nat, rcnt, budget_s=20.0):
    """Times the CPU oracle on a bounded sample and extrapolates the whole step.

    Sample: the oracle mask of ``n_mask`` heads (pool -> pooled softmax -> CDF -> STA) and
    the oracle attention forward of query blocks drawn from several heads.  Full-step time
    = mask time per head x B*H + kept FLOPs / (oracle attention FLOP rate).
    """
    import oracle
    cores = len(os.sched_getaffinity(0))
    BH = wl.B * wl.H
    thr = wl.thrs[0] if len(wl.thrs) == 1 else 0.8
    scale = 1 / math.sqrt(wl.D)
    t0 = time.perf_counter()
    n_mask = 0
    masks = {}
    for bh in range(BH):
        b, h = divmod(bh, wl.H)
        qf = oracle.reorder(q_nat[b, h].double().numpy()[None, None], wl.T, wl.Hg, wl.W, wl.P)
        kf = oracle.reorder(k_nat[b, h].double().numpy()[None, None], wl.T, wl.Hg, wl.W, wl.P)
        mk, _, _ = oracle.nabla_mask(qf, kf, wl.T, wl.Hg, wl.W, wl.P, thr, wl.window)
        masks[bh] = (qf, kf, mk[0, 0])
        n_mask += 1
        if time.perf_counter() - t0 > budget_s * 0.3 or n_mask >= 4:
            break
    t_mask = (time.perf_counter() - t0) / n_mask
    t1 = time.perf_counter()
    flops = 0.0
    blocks = 0
    rng = np.random.default_rng(0)
    for bh, (qf, kf, mk) in masks.items():
        b, h = divmod(bh, wl.H)
        vf = oracle.reorder(v_nat[b, h].double().numpy()[None, None], wl.T, wl.Hg, wl.W, wl.P)
        for i in rng.choice(wl.nb, size=min(4, wl.nb), replace=False):
            rows = np.arange(i * wl.N, (i + 1) * wl.N)
            oracle.block_sparse_attention_rows(qf[0, 0], kf[0, 0], vf[0, 0], mk, wl.N, scale, rows)
            flops += 4.0 * wl.N * wl.N * wl.D * mk[i].sum()
            blocks += 1
        if time.perf_counter() - t1 > budget_s * 0.7:
            break
    t_attn = time.perf_counter() - t1
    rate = flops / max(t_attn, 1e-9)
    kept_flops = 4.0 * wl.N * wl.N * wl.D * float(rcnt)
    est = t_mask * BH + kept_flops / rate
    return {
        "value": kept_flops / est / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
        "threads_blas": os.environ.get("OMP_NUM_THREADS", "default"),
        "sample": (f"oracle mask of {n_mask} head(s) ({t_mask:.2f} s/head) + oracle forward of "
                   f"{blocks} query blocks ({flops / 1e9:.2f} GFLOP in {t_attn:.2f} s); full "
                   f"step extrapolated to {BH} heads and {rcnt} kept tiles: {est:.1f} s"),
        "est_step_s": est,
    }


# --------------------------------------------------------------------------------------
def workload_config(wl, thr, world, scaling="weak"):
    """The ``config`` object of a bench line; both arms print the same one."""
    return {"workload": wl.name, "B": wl.B, "H": wl.H, "grid": [wl.T, wl.Hg, wl.W],
            "D": wl.D, "P": wl.P, "thr": thr, "sta": list(wl.window),
            "step": ("mask from natural-order Q/K (pooling fused), attn fwd on natural-order "
                     "Q/K/V" if not wl.backward
                     else "V to fp16, mask + lists from natural-order Q/K (pooling fused), attn "
                          "fwd and bwd on natural-order Q/K/V/dO"),
            "l2": "inputs larger than L2 (no flush)",
            "parallelism": (f"heads-replicated x{world}" if scaling == "weak"
                            else f"heads split over {world} ranks (LPT by kept tiles)")}


def run_reference(args, wl, world, rank):
    """The reference arm: the CPU oracle, as it stands, on the host cores.

    Set-up (untimed): the inputs of the GPU arm (drawn on the GPU when there is one, so
    that both arms see the same tensors; on the host otherwise) and the oracle mask of
    every head, which gives the exact kept-tile count.  Each step is a bounded 1/(B*H)
    slice of the workload, timed as it runs: the oracle mask of one head (heads in turn)
    plus the oracle forward over query blocks drawn in a fixed shuffled order across all
    heads until they hold (kept tiles) / (B*H) tiles; the attention time is scaled by the
    small overshoot of the last block.  value = the slice's kept-tile FLOPs / its time.
    """
    if rank != 0:
        return
    import oracle
    BH = wl.B * wl.H
    thr = wl.thrs[0] if len(wl.thrs) == 1 else 0.8
    scale = 1 / math.sqrt(wl.D)
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    q, k, v = (t.cpu() for t in make_qkv(wl, device=gen_dev))
    cores = len(os.sched_getaffinity(0))
    heads = []
    kept_all = 0
    for bh in range(BH):
        b, h = divmod(bh, wl.H)
        qf, kf, vf = (oracle.reorder(t[b, h].double().numpy()[None, None], wl.T, wl.Hg, wl.W, wl.P)[0, 0]
                      for t in (q, k, v))
        heads.append((qf, kf, vf))
    masks = []
    for bh in range(BH):
        qf, kf, _ = heads[bh]
        mk, _, _ = oracle.nabla_mask(qf[None, None], kf[None, None], wl.T, wl.Hg, wl.W, wl.P, thr, wl.window)
        masks.append(mk[0, 0])
        kept_all += int(mk.sum())
    budget = kept_all / BH
    order = [(bh, i) for bh in range(BH) for i in range(wl.nb) if masks[bh][i].any()]
    np.random.default_rng(0).shuffle(order)
    fl = 4.0 * wl.N * wl.N * wl.D
    cursor = 0
    times, samples = [], []
    for s in range(args.warmup + args.steps):
        bh_m = s % BH
        qf, kf, _ = heads[bh_m]
        t0 = time.perf_counter()
        oracle.nabla_mask(qf[None, None], kf[None, None], wl.T, wl.Hg, wl.W, wl.P, thr, wl.window)
        t_mask = time.perf_counter() - t0
        done = 0
        t1 = time.perf_counter()
        while done < budget:
            bh, i = order[cursor % len(order)]
            cursor += 1
            qh, kh, vh = heads[bh]
            rows = np.arange(i * wl.N, (i + 1) * wl.N)
            oracle.block_sparse_attention_rows(qh, kh, vh, masks[bh], wl.N, scale, rows)
            done += int(masks[bh][i].sum())
        t_attn = (time.perf_counter() - t1) * budget / done
        if s >= args.warmup:
            times.append(t_mask + t_attn)
            samples.append((t_mask, t_attn))
    step_s = statistics.median(times)
    val = budget * fl / step_s / 1e12
    sample = (f"1/{BH} of the workload per step: oracle mask of one head (median "
              f"{statistics.median(t for t, _ in samples):.2f} s) + oracle forward over {budget:.0f} "
              f"kept tiles (median {statistics.median(a for _, a in samples):.2f} s); kept tiles of all "
              f"{BH} heads from the oracle masks: {kept_all}")
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": workload_config(wl, thr, world),
            "kept_tiles": kept_all,
            "cpu_baseline": {"kind": "oracle", "cores": cores, "sample": sample, "value": val,
                             "unit": "TFLOP/s"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="wan720p", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=4)
    ap.add_argument("--no-side", action="store_true",
                    help="skip the side measurements (training step, forward vs sparsity)")
    ap.add_argument("--scaling", default="weak", choices=["weak", "strong"],
                    help="weak: every rank runs the whole workload; strong: the workload's "
                         "heads are split over the ranks (LPT by kept tiles)")
    args = ap.parse_args()
    wl = WORKLOADS[args.config]
    world, rank, local = init_dist() if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    if args.impl == "reference":
        run_reference(args, wl, world, rank)
        return
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pk, pk_kind = peaks()
    full_wl = wl
    units = None
    if args.scaling == "strong":
        from adaptive_block_sparse_b200.sharding import lpt_assign
        plan = lpt_assign(head_loads(wl, dev), world)
        units = plan[rank]
        args.no_side = True
        if not units:
            raise SystemExit(f"rank {rank} has no heads: {world} ranks for {wl.B * wl.H} heads")
    path = Path(wl, dev, units=units)
    wl = path.wl

    for _ in range(max(3, args.warmup)):
        path.step()
    torch.cuda.synchronize()
    path.check_status()
    kept = path.kept_pairs()
    nb = path.shape.nb
    BH = wl.B * wl.H

    # ---- timed region ---------------------------------------------------------------------
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    path.ev = {}
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(args.steps):
        path.step(timing=True)
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    ms_local = start.elapsed_time(end) / args.steps
    ms = max_over_ranks(ms_local, world, dev)
    path.check_status()
    fwd_ms = statistics.mean(path.segment_ms("t_mask", "t_fwd"))
    mask_ms_step = statistics.mean(path.segment_ms("t_reorder", "t_mask"))
    v16_ms = statistics.mean(path.segment_ms("t0", "t_reorder")) if wl.backward else None
    bwd_ms = statistics.mean(path.segment_ms("t_fwd", "t_bwd")) if wl.backward else None

    fl_fwd = 4.0 * 64 * 64 * wl.D
    step_flops = kept * fl_fwd * (3.5 if wl.backward else 1.0)
    total_flops = sum_over_ranks(step_flops, world, dev)
    value = total_flops / (ms * 1e-3) / 1e12
    fwd_tflops = kept * fl_fwd / (fwd_ms * 1e-3) / 1e12
    bwd_tflops = kept * fl_fwd * 2.5 / (bwd_ms * 1e-3) / 1e12 if wl.backward else None

    # ---- side measurements (outside the timed region) ----------------------------------------
    m, sh = path.m, path.shape
    # the mask from bf16 Q and K in the natural order (the step's call: pooling included)
    def mask_from_qk():
        m.nabla_build_mask(path.q, path.k, sh, path.thr, wl.window, mask_bits=path.bits,
                           row_idx=path.ridx, row_cnt=path.rcnt, workspace=path.mask_ws,
                           layout=m.NABLA_LAYOUT_NATURAL)
    mask_ms = time_call(mask_from_qk, 5)
    mask_bytes = 2 * BH * wl.S * wl.D * 2 + BH * nb * sh.nw * 4
    # the same in two passes: the fp64 pools alone (the pooling pass of the reorder entry
    # point), then the mask from the pools
    pool_ms = time_call(path.fill_pools, 5)
    pool_bytes = 2 * BH * wl.S * wl.D * 2 + 2 * BH * nb * wl.D * 8
    mask_pools_ms = time_call(lambda: m.nabla_build_mask(
        None, None, sh, path.thr, wl.window, mask_bits=path.bits, row_idx=path.ridx,
        row_cnt=path.rcnt, q_pool=path.qp, k_pool=path.kp, workspace=path.mask_ws), 5)
    # several thresholds from one pooled map (the pools of the step), against one mask
    # call per threshold; the masks are the same bit for bit
    sweep_thrs = (0.5, 0.7, 0.8, 0.9, 0.95)
    sw_bits = torch.empty(len(sweep_thrs), wl.B, wl.H, nb, sh.nw, dtype=torch.int32, device=dev)
    sw_cnt = torch.empty(len(sweep_thrs), wl.B, wl.H, nb, dtype=torch.int32, device=dev)
    sweep_call = lambda: m.nabla_build_mask_sweep(None, None, sh, sweep_thrs, wl.window,
                                                  mask_bits=sw_bits, row_cnt=sw_cnt, q_pool=path.qp,
                                                  k_pool=path.kp, workspace=path.mask_ws)

    def separate_calls():
        for t, thr in enumerate(sweep_thrs):
            m.nabla_build_mask(None, None, sh, thr, wl.window, mask_bits=sw_bits[t], row_cnt=sw_cnt[t],
                               q_pool=path.qp, k_pool=path.kp, workspace=path.mask_ws)
    sweep_ms = time_call(sweep_call, 3)
    separate_ms = time_call(separate_calls, 3)
    sweep = {"thrs": list(sweep_thrs), "ms": sweep_ms, "ms_separate_calls": separate_ms,
             "sparsity": m.sparsity_curve(sw_cnt, sh)}
    del sw_bits, sw_cnt
    # all-ones mask (padding bits are ignored by the kernels)
    dense_bits = torch.full((wl.B, wl.H, nb, sh.nw), -1, dtype=torch.int32, device=dev)
    dense_iters = 2 if nb > 1000 else 5
    v_fwd = path.vh if wl.backward else path.v
    dense_call = lambda: m.nabla_attn_fwd(path.q, path.k, v_fwd, dense_bits, sh, o=path.o,  # noqa: E731
                                          o_dtype=path.o_dtype, lse=path.lse,
                                          workspace=path.fwd_ws, layout=m.NABLA_LAYOUT_NATURAL)
    dense_ms = time_call(dense_call, dense_iters, warm=1)
    dense_tflops = BH * nb * nb * fl_fwd / (dense_ms * 1e-3) / 1e12
    path.check_status()
    del dense_bits

    # per-head sparsity (from the step's row counts) and the near-threshold blocks: blocks
    # (outside the static window) whose ranked mass E lies within 1e-6 of thr, counted as
    # kept(thr + 1e-6) - kept(thr - 1e-6) from two exact masks of the step's pooled map
    head_kept = path.rcnt.to(torch.int64).reshape(BH, nb).sum(dim=1).cpu().tolist()
    head_sp = sorted(1.0 - x / (nb * nb) for x in head_kept)
    per_head = {"min": head_sp[0], "median": statistics.median(head_sp), "max": head_sp[-1]}
    near = None
    if 0.0 < path.thr < 1.0:
        nt_bits = torch.empty(2, wl.B, wl.H, nb, sh.nw, dtype=torch.int32, device=dev)
        nt_cnt = torch.empty(2, wl.B, wl.H, nb, dtype=torch.int32, device=dev)
        m.nabla_build_mask_sweep(None, None, sh, (path.thr - 1e-6, path.thr + 1e-6), wl.window,
                                 mask_bits=nt_bits, row_cnt=nt_cnt, q_pool=path.qp, k_pool=path.kp,
                                 workspace=path.mask_ws)
        c = nt_cnt.to(torch.int64).reshape(2, -1).sum(dim=1).tolist()
        near = int(c[1] - c[0])
        del nt_bits, nt_cnt

    side = {}
    if not args.no_side:
        # forward throughput against sparsity: the same pooled map cut at several thresholds,
        # up to the pages' operating range (80-92% sparsity) where the data reaches it
        fvs = []
        for thr_s in (0.5, 0.8, 0.9, 0.95, 0.99, 0.999):
            b_s = torch.empty_like(path.bits)
            c_s = torch.empty(wl.B, wl.H, nb, dtype=torch.int32, device=dev)
            m.nabla_build_mask(None, None, sh, thr_s, wl.window, mask_bits=b_s, row_cnt=c_s,
                               q_pool=path.qp, k_pool=path.kp, workspace=path.mask_ws)
            kept_s = int(c_s.to(torch.int64).sum())
            call = lambda: m.nabla_attn_fwd(path.q, path.k, v_fwd, b_s, sh, o=path.o,  # noqa: E731
                                            o_dtype=path.o_dtype, lse=path.lse,
                                            workspace=path.fwd_ws, layout=m.NABLA_LAYOUT_NATURAL)
            ms_s = time_call(call, 3, warm=1)
            tf = kept_s * fl_fwd / (ms_s * 1e-3) / 1e12
            fvs.append({"thr": thr_s, "sparsity": 1.0 - kept_s / (BH * nb * nb), "kept_tiles": kept_s,
                        "ms": ms_s, "tflops_kept": tf, "frac": tf / pk["bf16_tflops"]})
            del b_s, c_s
        path.check_status()
        side["fwd_vs_sparsity"] = fvs
        if not wl.backward:
            # the training step (forward + backward) on the training-like workload, beside
            # the headline inference step
            twl = WORKLOADS["train_mid"]
            tpath = Path(twl, dev)
            for _ in range(3):
                tpath.step()
            torch.cuda.synchronize()
            tpath.check_status()
            tpath.ev = {}
            for _ in range(10):
                tpath.step(timing=True)
            torch.cuda.synchronize()
            tpath.check_status()
            tk = tpath.kept_pairs()
            t_bwd = statistics.mean(tpath.segment_ms("t_fwd", "t_bwd"))
            t_fwd = statistics.mean(tpath.segment_ms("t_mask", "t_fwd"))
            t_step = statistics.mean(tpath.segment_ms("t0", "t_bwd"))
            fl_b = 10.0 * 64 * 64 * twl.D
            btf = tk * fl_b / (t_bwd * 1e-3) / 1e12
            side.update({
                "train_workload": twl.name, "train_step_ms": t_step, "train_fwd_ms": t_fwd,
                "train_kept_tiles": tk, "bwd_ms": t_bwd, "bwd_tflops_kept": btf,
                "bwd_roofline": {"bound": "tensor", "kernel": "attn_bwd_dkdv_kernel + attn_bwd_dq_kernel "
                                 "(+ preprocess)", "achieved": btf, "peak": pk["bf16_tflops"],
                                 "unit": "TFLOP/s", "frac": btf / pk["bf16_tflops"],
                                 "peak_kind": f"{pk_kind} burst bf16 dense",
                                 "algorithmic_per_launch": f"{tk} kept 64x64 tiles x {int(fl_b)} FLOP"}})
            del tpath
            torch.cuda.empty_cache()
        if wl.name == "wan720p":
            # the hybrid mask on the same shape (NABLA at thr 0.7 OR a 3x3x5 STA window):
            # the same step, timed beside the headline
            swl = WORKLOADS["wan720p_sta"]
            spath = Path(swl, dev)
            for _ in range(3):
                spath.step()
            torch.cuda.synchronize()
            spath.check_status()
            spath.ev = {}
            for _ in range(10):
                spath.step(timing=True)
            torch.cuda.synchronize()
            spath.check_status()
            sk = spath.kept_pairs()
            s_fwd = statistics.mean(spath.segment_ms("t_mask", "t_fwd"))
            side["sta_hybrid"] = {
                "workload": swl.name, "thr": spath.thr, "sta": list(swl.window), "kept_tiles": sk,
                "sparsity": 1.0 - sk / (BH * nb * nb), "step_ms": statistics.mean(spath.segment_ms("t0", "t_fwd")),
                "mask_ms": statistics.mean(spath.segment_ms("t_reorder", "t_mask")), "fwd_ms": s_fwd,
                "fwd_tflops_kept": sk * fl_fwd / (s_fwd * 1e-3) / 1e12,
                "fwd_frac": sk * fl_fwd / (s_fwd * 1e-3) / 1e12 / pk["bf16_tflops"]}
            del spath
            torch.cuda.empty_cache()
            # the small configuration's threshold sweep, each forward next to the dense one
            # on the same tensors (natural layout)
            mwl = WORKLOADS["small"]
            msh = m.Shape(mwl.B, mwl.H, mwl.T, mwl.Hg, mwl.W, mwl.D, mwl.P)
            mq, mk, mv = make_qkv(mwl, device=dev)
            mws = torch.zeros(m.nabla_fwd_workspace_bytes(msh), dtype=torch.uint8, device=dev)
            mo = torch.empty_like(mq)
            mnb = msh.nb
            mdense = torch.full((mwl.B, mwl.H, mnb, msh.nw), -1, dtype=torch.int32, device=dev)
            dms = time_call(lambda: m.nabla_attn_fwd(mq, mk, mv, mdense, msh, o=mo, workspace=mws,
                                                     layout=m.NABLA_LAYOUT_NATURAL), 20, warm=3)
            rows = []
            for thr_m in mwl.thrs:
                mc = torch.empty(mwl.B, mwl.H, mnb, dtype=torch.int32, device=dev)
                mb, *_ = m.nabla_build_mask(mq, mk, msh, thr_m, mwl.window, row_cnt=mc,
                                            layout=m.NABLA_LAYOUT_NATURAL)
                kept_m = int(mc.to(torch.int64).sum())
                sms_ = time_call(lambda: m.nabla_attn_fwd(mq, mk, mv, mb, msh, o=mo, workspace=mws,
                                                          layout=m.NABLA_LAYOUT_NATURAL), 20, warm=3)
                rows.append({"thr": thr_m, "kept_tiles": kept_m,
                             "sparsity": 1.0 - kept_m / (mwl.B * mwl.H * mnb * mnb),
                             "ms": sms_, "dense_ms": dms, "speedup_vs_dense": dms / sms_})
            code = m.nabla_read_device_status(mws)
            if code:
                raise RuntimeError(f"device status 0x{code:x}")
            side["small_thr_sweep"] = {"workload": mwl.name, "l2": "inputs fit in L2 (25 MB)",
                                       "rows": rows}
            del mq, mk, mv, mo, mdense, mws

    # ---- end to end through the public API with host buffers --------------------------------
    # Every step copies its own inputs host -> device and its result back inside the timed
    # region.  Two copies of the step's device state alternate on two streams, so the PCIe
    # copies of consecutive steps overlap (inputs of step i+1 in flight while step i
    # computes and returns its result), as a serving loop would run them.
    hq, hk, hv = (t.cpu().pin_memory() for t in (path.q, path.k, path.v))
    hdo = path.do.cpu().pin_memory() if wl.backward else None
    paths = [path, Path(full_wl, dev, units=units)]
    streams = [torch.cuda.Stream(device=dev) for _ in paths]
    houts = [(torch.empty(path.o.shape, dtype=path.o.dtype).pin_memory(),
              [torch.empty(path.q.shape, dtype=torch.float32).pin_memory() for _ in range(3)]
              if wl.backward else []) for _ in paths]
    barrier(world)
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream()
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_s.record(cur)
    for st in streams:
        st.wait_event(e_s)
    for i in range(args.e2e_steps):
        p_i, st, (ho, hgrads) = paths[i % 2], streams[i % 2], houts[i % 2]
        with torch.cuda.stream(st):
            p_i.q.copy_(hq, non_blocking=True)
            p_i.k.copy_(hk, non_blocking=True)
            p_i.v.copy_(hv, non_blocking=True)
            if wl.backward:
                p_i.do.copy_(hdo, non_blocking=True)
            p_i.step()
            ho.copy_(p_i.o, non_blocking=True)
            for hg, g in zip(hgrads, (p_i.dq, p_i.dk, p_i.dv) if wl.backward else ()):
                hg.copy_(g, non_blocking=True)
    for st in streams:
        cur.wait_stream(st)
    e_e.record(cur)
    torch.cuda.synchronize()
    barrier(world)
    for p_i in paths:
        p_i.check_status()
    e2e_ms = max_over_ranks(e_s.elapsed_time(e_e) / args.e2e_steps, world, dev)
    h2d = 3 * path.q.numel() * 2 + (path.do.numel() * 2 if wl.backward else 0)
    d2h = path.o.numel() * path.o.element_size() + (3 * path.q.numel() * 4 if wl.backward else 0)
    del paths[1], streams, houts
    e2e_value = total_flops / (e2e_ms * 1e-3) / 1e12

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = oracle_sample(wl, path.q.cpu(), path.k.cpu(), path.v.cpu(), kept, budget_s=20.0)
        cpu = {k2: cb[k2] for k2 in ("value", "unit", "cores", "kind", "sample")}

    peak_burst = pk["bf16_tflops"]
    roof = {"bound": "tensor", "kernel": "attn_fwd_kernel<128>" if wl.D == 128 else "attn_fwd_kernel<64>",
            "achieved": fwd_tflops, "peak": peak_burst, "unit": "TFLOP/s",
            "frac": fwd_tflops / peak_burst, "peak_kind": f"{pk_kind} burst bf16 dense",
            "frac_of_sustained": fwd_tflops / pk["bf16_tflops_sustained"],
            "traffic": measured_traffic(wl.name),
            "traffic_note": "dram read+write bytes per launch from ncu (heads 0-7, scaled by heads); "
                            "null when the kernel changed since the capture",
            "algorithmic_per_launch": f"{kept} kept 64x64 tiles x {int(fl_fwd)} FLOP"}
    sparsity = 1.0 - kept / (BH * nb * nb)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": args.scaling, "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(full_wl, path.thr, world, args.scaling),
        "fwd_ms": fwd_ms, "fwd_tflops_kept": fwd_tflops,
        "dense_fwd_ms": dense_ms, "dense_tflops": dense_tflops, "speedup_vs_dense": dense_ms / fwd_ms,
        "mask_ms": mask_ms, "mask_gbs": mask_bytes / (mask_ms * 1e-3) / 1e9,
        "mask_frac_hbm": mask_bytes / (mask_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
        "mask_ms_in_step": mask_ms_step, "mask_ms_from_pools": mask_pools_ms,
        "pool_ms": pool_ms, "pool_gbs": pool_bytes / (pool_ms * 1e-3) / 1e9,
        "mask_sweep_from_pools": sweep, "v_to_f16_ms": v16_ms,
        "bwd_ms": bwd_ms, "bwd_tflops_kept": bwd_tflops,
        "kept_tiles": kept, "sparsity": sparsity, "sparsity_per_head": per_head,
        "near_threshold_blocks": near,
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
                "overlap": "two device copies of the step state on two streams: the copies of "
                           "consecutive steps overlap"},
        "gpu_launches": path.launches_per_step() * args.steps,
        "clocks": clocks,
    }
    for key, val in side.items():
        if line.get(key) is None:
            line[key] = val
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
