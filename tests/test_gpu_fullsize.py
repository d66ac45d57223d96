"""Parity at the benchmark's full sizes, in the launch configuration bench.py times.

Masks: every head against the oracle (bit-exact outside the 1e-6 band).  Forward: every
row of the head with the most kept tiles, plus six query blocks of each of four other
distinct heads, computed by the oracle on the GPU's mask.  Backward (training workload):
two sampled heads in full.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from parity_lib import bits_to_mask, check_close, check_lists, check_lse, check_mask, to64
from synth import WORKLOADS

pytestmark = pytest.mark.gpu


def _run(name):
    import bench
    wl = WORKLOADS[name]
    path = bench.Path(wl, torch.device("cuda", 0))
    path.step()
    torch.cuda.synchronize()
    path.check_status()
    return wl, path


def _head(t, b, h, wl, reorder=False):
    x = t[b, h].detach().cpu().double().numpy()
    return oracle.reorder(x[None, None], wl.T, wl.Hg, wl.W, wl.P)[0, 0] if reorder else x


@pytest.mark.parametrize("name", ["wan720p", "wan720p_sta", "train_mid"])
def test_fullsize_mask_and_forward(name):
    wl, path = _run(name)
    thr = path.thr
    # every output is computed in a fixed order: a second run is bitwise identical
    o1, bits1 = path.o.clone(), path.bits.clone()
    path.step()
    torch.cuda.synchronize()
    path.check_status()
    assert torch.equal(path.bits, bits1), "mask differs between two runs"
    assert torch.equal(path.o.view(torch.int16) if path.o.dtype == torch.bfloat16 else path.o, 
                       o1.view(torch.int16) if o1.dtype == torch.bfloat16 else o1), \
        "forward output differs between two runs"
    gm = bits_to_mask(path.bits, wl.nb)
    # counts from the mask build; row lists rebuilt from the bitmask when the step did not
    # ask for them (the forward reads only the bitmask)
    ridx = path.ridx
    if ridx is None:
        ridx = torch.empty(wl.B, wl.H, wl.nb, wl.nb, dtype=torch.int32, device=path.bits.device)
        rcnt2 = torch.empty_like(path.rcnt)
        path.m.nabla_mask_lists(path.bits, path.shape, ridx, rcnt2)
        assert torch.equal(rcnt2, path.rcnt)
    check_lists(ridx, path.rcnt, gm)
    mism = amb = 0
    qn, kn = path.q.cpu(), path.k.cpu()
    for b in range(wl.B):
        for h in range(wl.H):
            qf = oracle.reorder(qn[b, h].double().numpy()[None, None], wl.T, wl.Hg, wl.W, wl.P)
            kf = oracle.reorder(kn[b, h].double().numpy()[None, None], wl.T, wl.Hg, wl.W, wl.P)
            om, E, _ = oracle.nabla_mask(qf, kf, wl.T, wl.Hg, wl.W, wl.P, thr, wl.window)
            m1, a1 = check_mask(gm[b, h][None, None], om, E, thr)
            mism += m1
            amb += a1
    print(f"{name}: sparsity {1 - gm.mean():.4f}, near-threshold blocks {amb}, differing {mism}")
    # Forward.  (1) Every query row of the head that keeps the most tiles: its tiles are
    # the longest walks of the launch (hundreds of key blocks per tile on the 720p-like
    # workload), which exercise long online-softmax runs and the rescaling of O.  (2) Six
    # query blocks of each of four further distinct heads.
    rng = np.random.default_rng(7)
    bf16_out = path.o.dtype == torch.bfloat16
    scale = 1 / math.sqrt(wl.D)
    perm = oracle.fractal_permutation(wl.T, wl.Hg, wl.W, wl.P)
    kept_per_head = gm.reshape(wl.B * wl.H, -1).sum(axis=1)
    heavy = int(np.argmax(kept_per_head))
    others = [x for x in range(wl.B * wl.H) if x != heavy]
    picks = [(heavy, None)] + [(int(x), rng.choice(wl.nb, size=6, replace=False))
                               for x in rng.choice(others, size=min(4, len(others)), replace=False)]
    for bh, blocks in picks:
        b, h = divmod(bh, wl.H)
        q, k, v = (_head(t, b, h, wl, reorder=True) for t in (path.q, path.k, path.v))
        if blocks is None:
            O, L = oracle.block_sparse_attention(q[None, None], k[None, None], v[None, None],
                                                 gm[b:b + 1, h:h + 1], wl.N, scale)
            O, L = O[0, 0], L[0, 0]
            rows = np.arange(wl.S)
            what = f"O {name} heaviest head {b},{h} ({int(kept_per_head[bh])} tiles), every row"
        else:
            rows = (blocks[:, None] * wl.N + np.arange(wl.N)[None, :]).reshape(-1)
            O, L = oracle.block_sparse_attention_rows(q, k, v, gm[b, h], wl.N, scale, rows)
            what = f"O {name} head {b},{h}"
        # outputs in natural order (the inference path) sit at the tokens' natural indices
        at = torch.from_numpy(perm[rows] if path.natural else rows).cuda()
        got = path.o[b, h, at].detach().cpu().double().numpy()
        mx, mean = check_close(got, O, what, storage_bf16=bf16_out)
        print(f"{what}: max err {mx:.2e} mean {mean:.2e}")
        lse = path.lse[b, h, at].cpu().double().numpy()
        check_lse(lse, L)


def test_fullsize_backward():
    """The training step as bench.py times it: natural-order Q, K, V (fp16 V), dO; the
    gradients land at natural indices.  Two heads in full against the oracle gradients of
    the reordered tensors, inverse-reordered."""
    wl, path = _run("train_mid")
    gm = bits_to_mask(path.bits, wl.nb)
    check_lists(path.cidx, path.ccnt, np.swapaxes(gm, -1, -2))
    scale = 1 / math.sqrt(wl.D)
    for b, h in ((0, 3), (1, 17)):
        q, k, v, do = (_head(t, b, h, wl, reorder=True) for t in (path.q, path.k, path.vh, path.do))
        ref = oracle.block_sparse_attention_bwd(q[None, None], k[None, None], v[None, None],
                                                do[None, None], gm[b:b + 1, h:h + 1], wl.N, scale)
        for got, r, what in zip((path.dq, path.dk, path.dv), ref, ("dQ", "dK", "dV")):
            r_nat = oracle.inverse_reorder(r[0, 0][None, None], wl.T, wl.Hg, wl.W, wl.P)[0, 0]
            mx, mean = check_close(to64(got[b, h]), r_nat, f"{what} train_mid head {b},{h}")
            print(f"train_mid {what} head {b},{h}: max err {mx:.2e} mean {mean:.2e}")
