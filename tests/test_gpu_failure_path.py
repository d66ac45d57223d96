"""Failure detection without a GPU fault: a bounded barrier wait that nothing completes
gives up after its limit, records a status code, and the context stays usable."""
import math
import time

import numpy as np
import pytest
import torch

import oracle
from parity_lib import bits_to_mask, check_close, gpu_mask, gpu_reorder, shape_of, to64
from synth import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_context_stays_usable():
    import adaptive_block_sparse_b200 as m
    dev = torch.device("cuda", 0)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    t0 = time.time()
    m.nabla_selftest_bounded_wait(ws)
    code = m.nabla_read_device_status(ws)          # synchronises the stream
    waited = time.time() - t0
    assert code == m.DEVICE_TIMEOUT_SELFTEST, hex(code)
    assert 1.0 < waited < 30.0, waited              # the wait ran out its ~2 s limit
    assert m.nabla_read_device_status(ws) == 0      # reading cleared the word
    # the same stream and context still run the path correctly
    wl = WORKLOADS["tiny"]
    shape = shape_of(wl)
    q, k, v = make_qkv(wl, device=dev)
    qf, _ = gpu_reorder(q, shape)
    kf, _ = gpu_reorder(k, shape)
    vf, _ = gpu_reorder(v, shape)
    bits, *_ = gpu_mask(qf, kf, shape, wl.thrs[0], wl.window, cols=False)
    fws = torch.zeros(m.nabla_fwd_workspace_bytes(shape), dtype=torch.uint8, device=dev)
    o, _ = m.nabla_attn_fwd(qf, kf, vf, bits, shape, o_dtype=m.NABLA_F32, workspace=fws)
    torch.cuda.synchronize()
    assert m.nabla_read_device_status(fws) == 0
    gm = bits_to_mask(bits, wl.nb)
    O, _ = oracle.block_sparse_attention(to64(qf), to64(kf), to64(vf), gm, wl.N, 1 / math.sqrt(wl.D))
    check_close(to64(o), O, "forward after the self-test")
