"""Helpers shared by the GPU parity tests: run the CUDA path, run the oracle, compare."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

BAND = 1e-6          # blocks whose ranked mass lies this close to thr may differ
FWD_MAX_ABS = 2e-2   # O, dQ, dK, dV against the fp64 oracle
FWD_MEAN_ABS = 2e-3


def nbl():
    import adaptive_block_sparse_b200 as m
    m.load_library()
    return m


def shape_of(wl):
    return nbl().Shape(wl.B, wl.H, wl.T, wl.Hg, wl.W, wl.D, wl.P)


def gpu_reorder(x_nat, shape, pool=False, dtype=torch.bfloat16):
    m = nbl()
    dst = torch.empty(x_nat.shape, dtype=dtype, device=x_nat.device)
    pool_out = (torch.empty(shape.B, shape.H, shape.nb, shape.D, dtype=torch.float64,
                            device=x_nat.device) if pool else None)
    m.nabla_reorder(x_nat, dst, shape, pool_out=pool_out)
    return dst, pool_out


def gpu_mask(q, k, shape, thr, window=(0, 0, 0), cols=True, **kw):
    m = nbl()
    bits, ridx, rcnt, cidx, ccnt = m.alloc_mask(shape, q.device if q is not None else kw["q_pool"].device,
                                                cols=cols)
    m.nabla_build_mask(q, k, shape, thr, window, mask_bits=bits, row_idx=ridx, row_cnt=rcnt,
                       col_idx=cidx, col_cnt=ccnt, **kw)
    torch.cuda.synchronize()
    return bits, ridx, rcnt, cidx, ccnt


def bits_to_mask(bits, nb):
    return oracle.unpack_mask_bits(bits.cpu().numpy().view(np.uint32), nb)


def to64(t):
    return t.detach().cpu().double().numpy()


def oracle_mask_per_head(q_nat_cpu, k_nat_cpu, wl, thr, window):
    """Oracle mask head by head (bounded memory).  Inputs: bf16 natural-order CPU tensors."""
    B, H = q_nat_cpu.shape[:2]
    nb = wl.nb
    mask = np.empty((B, H, nb, nb), dtype=bool)
    E = np.empty((B, H, nb, nb))
    for b in range(B):
        for h in range(H):
            qf = oracle.reorder(q_nat_cpu[b, h].double().numpy()[None, None], wl.T, wl.Hg, wl.W, wl.P)
            kf = oracle.reorder(k_nat_cpu[b, h].double().numpy()[None, None], wl.T, wl.Hg, wl.W, wl.P)
            m, e, _ = oracle.nabla_mask(qf, kf, wl.T, wl.Hg, wl.W, wl.P, thr, window)
            mask[b, h], E[b, h] = m[0, 0], e[0, 0]
    return mask, E


def check_mask(gmask, omask, E, thr):
    """Bit-exact except blocks within BAND of thr.  Returns (mismatches, ambiguous)."""
    mism = gmask != omask
    amb = np.abs(E - thr) <= BAND if thr < 1.0 else np.zeros_like(mism)
    bad = mism & ~amb
    assert not bad.any(), f"{int(bad.sum())} mask blocks differ outside the {BAND} band"
    return int(mism.sum()), int(amb.sum())


def check_lists(ridx, rcnt, gmask):
    """Row lists equal the ascending set bits of the GPU mask (bit-exact)."""
    idx, cnt = oracle.row_lists(gmask)
    rc = rcnt.cpu().numpy()
    assert np.array_equal(rc, cnt)
    ri = ridx.cpu().numpy()
    valid = np.arange(gmask.shape[-1])[None, None, None, :] < cnt[..., None]
    assert np.array_equal(np.where(valid, ri, -1), idx)


def bf16_half_ulp(x):
    ax = np.maximum(np.abs(x), 1e-30)
    return 0.5 * np.exp2(np.floor(np.log2(ax)) - 7)


def check_close(got, ref, what, storage_bf16=False):
    """max-abs / mean-abs gates; bf16 storage adds half an ulp of the reference value."""
    err = np.abs(got - ref)
    slack = bf16_half_ulp(ref) if storage_bf16 else 0.0
    max_gate = FWD_MAX_ABS + slack
    assert np.all(err <= max_gate), f"{what}: max abs err {err.max():.3e} (worst excess {(err - max_gate).max():.3e})"
    mean_gate = FWD_MEAN_ABS + (np.mean(slack) if storage_bf16 else 0.0)
    assert err.mean() <= mean_gate, f"{what}: mean abs err {err.mean():.3e} > {mean_gate:.3e}"
    return float(err.max()), float(err.mean())


def check_lse(got, ref):
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref))
    if fin.any():
        err = np.abs(got[fin] - ref[fin])
        assert err.max() <= FWD_MAX_ABS, f"lse max abs err {err.max():.3e}"


def scale_of(D):
    return 1.0 / math.sqrt(D)
