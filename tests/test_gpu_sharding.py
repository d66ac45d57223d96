"""Head-sharded attention on the GPU with one NCCL rank: the exchanges are identities and
the per-rank path (pools, mask, natural-layout forward) matches the oracle."""
import math
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from parity_lib import check_close
from synth import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu


def test_sharded_attention_one_nccl_rank():
    import torch.distributed as dist
    from adaptive_block_sparse_b200 import Shape, sharding
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        wl = WORKLOADS["small"]
        q, k, v = make_qkv(wl, device="cuda")
        thr = 0.8
        o = sharding.sharded_nabla_attention(q, k, v, wl.T, wl.Hg, wl.W, thr)
        shape = Shape(wl.B, wl.H, wl.T, wl.Hg, wl.W, wl.D)
        direct = sharding.nabla_local_heads(q, k, v, shape, thr, scale=1 / math.sqrt(wl.D))
        torch.cuda.synchronize()
        assert torch.equal(o, direct)
        scale = 1 / math.sqrt(wl.D)
        for h in (0, wl.H - 1):
            qf, kf, vf = (oracle.reorder(x[0, h].double().cpu().numpy()[None, None], wl.T, wl.Hg, wl.W, wl.P)
                          for x in (q, k, v))
            mk, _, _ = oracle.nabla_mask(qf, kf, wl.T, wl.Hg, wl.W, wl.P, thr)
            ref, _ = oracle.block_sparse_attention(qf, kf, vf, mk, wl.N, scale)
            ref = oracle.inverse_reorder(ref, wl.T, wl.Hg, wl.W, wl.P)[0, 0]
            check_close(o[0, h].double().cpu().numpy(), ref, f"sharded head {h}", storage_bf16=True)
    finally:
        dist.destroy_process_group()
