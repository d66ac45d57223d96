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


def bf16_round(x):
    """x (float64) rounded to the nearest bfloat16, ties to even, returned as float64.

    Done on the fp64 value directly (frexp, 8 significant bits, round half to even), so
    there is no double rounding through fp32.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def bf16_ulp(y):
    """Spacing of bfloat16 values at |y| (y itself a bf16 value); 0 maps to the smallest."""
    ay = np.maximum(np.abs(y), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(ay)) - 7)


def check_close(got, ref, what, storage_bf16=False):
    """max-abs / mean-abs gates of the fp64 reference.

    f32 outputs: |got - ref| <= FWD_MAX_ABS everywhere and mean <= FWD_MEAN_ABS.

    bf16 outputs: the reference is rounded to bf16 first (the output format cannot hold
    anything closer) and the same two gates apply to |got - bf16(ref)|, the mean gate
    without any slack.  Where one bf16 step exceeds the max gate (|ref| >= 4, step
    2^-5), a result that rounded to the neighbouring bf16 value (one step away) is a
    storage effect, not an error of the kernel, and is accepted; nothing further is.
    Returns (max, mean) of |got - bf16(ref)| (bf16) or |got - ref| (f32), and prints the
    unrounded error beside it for bf16 outputs.
    """
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if storage_bf16:
        ref_r = bf16_round(ref)
        err = np.abs(got - ref_r)
        max_gate = np.maximum(FWD_MAX_ABS, bf16_ulp(ref_r))
        raw = np.abs(got - ref)
        print(f"{what}: vs bf16(ref) max {err.max():.3e} mean {err.mean():.3e}; "
              f"vs ref max {raw.max():.3e} mean {raw.mean():.3e}; "
              f"one-step bf16 flips above the max gate: {int((err > FWD_MAX_ABS).sum())}")
    else:
        err = np.abs(got - ref)
        max_gate = FWD_MAX_ABS
    assert np.all(err <= max_gate), \
        f"{what}: max abs err {err.max():.3e} (worst excess {(err - max_gate).max():.3e})"
    assert err.mean() <= FWD_MEAN_ABS, f"{what}: mean abs err {err.mean():.3e} > {FWD_MEAN_ABS:.3e}"
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
