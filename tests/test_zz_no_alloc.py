"""Allocation-free forward entry point (nabla_attn_fwd_noalloc), through the C ABI.

It exists for callers that cannot allocate device memory where they run attention
(a framework that owns all device memory through its own pool, a latency-critical
loop): its workspace is a fixed 1 MiB array inside the library.  This file is named to
be collected last, so a run that stops at the first failure has already run every
other test; it also passes alone in a fresh process (the first call sets up the array).
"""
import numpy as np
import pytest
import torch

from parity_lib import FWD_MAX_ABS, FWD_MEAN_ABS, gpu_mask, gpu_reorder, nbl, shape_of
from synth import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("name,o_dtype", [("small", torch.float32), ("tiny", torch.bfloat16)])
def test_noalloc_forward_matches_regular_entry_point(name, o_dtype):
    m = nbl()
    wl = WORKLOADS[name]
    shape = shape_of(wl)
    q, k, v = make_qkv(wl, device=DEV)
    qf, _ = gpu_reorder(q, shape)
    kf, _ = gpu_reorder(k, shape)
    vk, _ = gpu_reorder(v, shape, dtype=torch.float16)
    bits, _, _, _, _ = gpu_mask(qf, kf, shape, wl.thrs[-1], (0, 0, 0), cols=False)
    odt = m.NABLA_F32 if o_dtype == torch.float32 else m.NABLA_BF16
    lse_ref = torch.empty(wl.B, wl.H, wl.S, dtype=torch.float32, device=DEV)
    ws = torch.zeros(m.nabla_fwd_workspace_bytes(shape), dtype=torch.uint8, device=DEV)
    o_ref, _ = m.nabla_attn_fwd(qf, kf, vk, bits, shape, o_dtype=odt, lse=lse_ref, workspace=ws)
    torch.cuda.synchronize()
    assert m.nabla_read_device_status(ws) == 0
    ref = o_ref.double().cpu().numpy()
    for call in range(2):                      # two calls in a row share the scratch array
        o = torch.full(q.shape, float("nan"), dtype=o_dtype, device=DEV)
        lse = torch.full((wl.B, wl.H, wl.S), float("nan"), dtype=torch.float32, device=DEV)
        m.nabla_attn_fwd_noalloc(qf, kf, vk, bits, shape, o, lse)
        torch.cuda.synchronize()
        err = np.abs(o.double().cpu().numpy() - ref)
        assert err.max() <= FWD_MAX_ABS and err.mean() <= FWD_MEAN_ABS, (call, err.max())
        lerr = np.abs(lse.cpu().numpy() - lse_ref.cpu().numpy())
        assert np.nanmax(lerr) <= FWD_MAX_ABS and not np.isnan(lerr).any(), call


def test_noalloc_rejects_problems_beyond_its_scratch():
    m = nbl()
    big = m.Shape(1, 2000, 21, 48, 80, 128)    # 1.26 M tiles: schedule > 1 MiB
    assert m.nabla_fwd_workspace_bytes(big) > (1 << 20)
    x = torch.zeros(16, dtype=torch.bfloat16, device=DEV)    # never read: rejected first
    i = torch.zeros(16, dtype=torch.int32, device=DEV)
    with pytest.raises(m.NablaError) as e:
        m.nabla_attn_fwd_noalloc(x, x, x.to(torch.float16), i, big, x)
    assert e.value.status == m.NABLA_ERR_UNSUPPORTED
