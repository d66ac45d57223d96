"""Allocation-free forward entry point (nabla_attn_fwd_noalloc), through the C ABI.

It exists for callers that cannot allocate device memory where they run attention
(a framework that owns all device memory through its own pool, a latency-critical
loop): its workspace is a fixed 1 MiB array inside the library.  The kernels are the
regular forward's and deterministic, so the output must equal nabla_attn_fwd's bit for
bit, on both token layouts and on two calls in a row (the array keeps the previous
call's contents).  After every call the array's status word is read back through
nabla_attn_fwd_noalloc_status.  This file is named to be collected last, so a run that
stops at the first failure has already run every other test; it also passes alone in a
fresh process (the first call sets up the array).
"""
import pytest
import torch

from parity_lib import gpu_mask, gpu_reorder, nbl, shape_of
from synth import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("name,o_dtype,natural", [("small", torch.float32, False),
                                                  ("tiny", torch.bfloat16, False),
                                                  ("small", torch.bfloat16, True)])
def test_noalloc_forward_matches_regular_entry_point(name, o_dtype, natural):
    m = nbl()
    wl = WORKLOADS[name]
    shape = shape_of(wl)
    q, k, v = make_qkv(wl, device=DEV)
    qf, qp = gpu_reorder(q, shape, pool=True)
    kf, kp = gpu_reorder(k, shape, pool=True)
    bits, _, _, _, _ = gpu_mask(None, None, shape, wl.thrs[-1], (0, 0, 0), cols=False,
                                q_pool=qp, k_pool=kp)
    if natural:
        # the inference layout: natural-order Q, K, V (bf16 V) read in place
        layout, qa, ka, va = m.NABLA_LAYOUT_NATURAL, q, k, v
    else:
        vk, _ = gpu_reorder(v, shape, dtype=torch.float16)
        layout, qa, ka, va = m.NABLA_LAYOUT_REORDERED, qf, kf, vk
    odt = m.NABLA_F32 if o_dtype == torch.float32 else m.NABLA_BF16
    lse_ref = torch.empty(wl.B, wl.H, wl.S, dtype=torch.float32, device=DEV)
    ws = torch.zeros(m.nabla_fwd_workspace_bytes(shape), dtype=torch.uint8, device=DEV)
    o_ref, _ = m.nabla_attn_fwd(qa, ka, va, bits, shape, o_dtype=odt, lse=lse_ref, workspace=ws,
                                layout=layout)
    torch.cuda.synchronize()
    assert m.nabla_read_device_status(ws) == 0
    for call in range(2):                      # two calls in a row share the scratch array
        o = torch.full(q.shape, float("nan"), dtype=o_dtype, device=DEV)
        lse = torch.full((wl.B, wl.H, wl.S), float("nan"), dtype=torch.float32, device=DEV)
        m.nabla_attn_fwd_noalloc(qa, ka, va, bits, shape, o, lse, layout=layout)
        assert m.nabla_attn_fwd_noalloc_status() == 0, call
        assert torch.equal(o.view(torch.int16) if o_dtype == torch.bfloat16 else o.view(torch.int32),
                           o_ref.view(torch.int16) if o_dtype == torch.bfloat16 else o_ref.view(torch.int32)), call
        assert torch.equal(lse.view(torch.int32), lse_ref.view(torch.int32)), call


def test_noalloc_rejects_problems_beyond_its_scratch():
    m = nbl()
    big = m.Shape(1, 2000, 21, 48, 80, 128)    # 1.26 M tiles: schedule > 1 MiB
    assert m.nabla_fwd_workspace_bytes(big) > (1 << 20)
    x = torch.zeros(16, dtype=torch.bfloat16, device=DEV)    # never read: rejected first
    i = torch.zeros(16, dtype=torch.int32, device=DEV)
    with pytest.raises(m.NablaError) as e:
        m.nabla_attn_fwd_noalloc(x, x, x.to(torch.float16), i, big, x)
    assert e.value.status == m.NABLA_ERR_UNSUPPORTED
