"""Head-sharded NABLA attention for callers whose activations are sharded by sequence.

Every (batch, head) pair goes through the whole path independently: each head pools its
own Q and K, builds its own block mask and attends over its own kept tiles (lsdiaocha.cn
article on NABLA, section 2: the mask is formed per head from that head's pooled map).
So heads, not tokens, are the unit to distribute.  A model that keeps its activations
sharded by sequence (rank r holding a contiguous range of S/N tokens of every head)
exchanges them once before attention and once after:

    [B, H, S/N, D] per rank  --all-to-all-->  [B, H/N, S, D] per rank   (seq_to_heads)
    hot path on the rank's H/N heads (pool, mask, forward in the natural token order)
    [B, H/N, S, D] per rank  --all-to-all-->  [B, H, S/N, D] per rank   (heads_to_seq)

The exchanges are ``torch.distributed.all_to_all_single`` calls (NCCL over NVLink /
NVSwitch on GPUs; any backend with all-to-all, e.g. gloo on the host), each moving
(N-1)/N of the tensor.  Token ranges are contiguous in the latent's natural order
(frames outermost), and the exchange is exact data movement, so the sharded result
equals the unsharded one bit for bit.
"""
import math

import torch
import torch.distributed as dist


def seq_to_heads(x, group=None):
    """[B, H, S/N, D] (this rank's tokens of every head) -> [B, H/N, S, D] (every token of
    this rank's heads: heads [r H/N, (r+1) H/N) on rank r, tokens in rank order)."""
    n = dist.get_world_size(group)
    B, H, s, D = x.shape
    if H % n:
        raise ValueError(f"{H} heads do not split over {n} ranks")
    send = x.reshape(B, n, H // n, s, D).permute(1, 0, 2, 3, 4).contiguous()   # [dst, B, H/N, s, D]
    recv = torch.empty_like(send)                                               # [src, B, H/N, s, D]
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 2, 0, 3, 4).reshape(B, H // n, n * s, D)


def heads_to_seq(y, group=None):
    """Inverse of seq_to_heads: [B, H/N, S, D] -> [B, H, S/N, D]."""
    n = dist.get_world_size(group)
    B, h, S, D = y.shape
    if S % n:
        raise ValueError(f"{S} tokens do not split over {n} ranks")
    s = S // n
    send = y.reshape(B, h, n, s, D).permute(2, 0, 1, 3, 4).contiguous()        # [dst, B, h, s, D]
    recv = torch.empty_like(send)                                               # [src, B, h, s, D]
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 0, 2, 3, 4).reshape(B, n * h, s, D)


def nabla_local_heads(q, k, v, shape, thr, window=(0, 0, 0), scale=None):
    """The hot path on one rank's heads, natural token order in and out: fp64 pools of Q
    and K, the block mask from them, the forward reading Q, K, V in place.  Returns bf16 O
    [B, h, S, D]."""
    import adaptive_block_sparse_b200 as m
    dev = q.device
    qp = torch.empty(shape.B, shape.H, shape.nb, shape.D, dtype=torch.float64, device=dev)
    kp = torch.empty_like(qp)
    m.nabla_reorder(q, None, shape, pool_out=qp)
    m.nabla_reorder(k, None, shape, pool_out=kp)
    bits, _, _, _, _ = m.nabla_build_mask(None, None, shape, thr, window, scale=scale,
                                          q_pool=qp, k_pool=kp)
    o, _ = m.nabla_attn_fwd(q, k, v, bits, shape, scale=scale, layout=m.NABLA_LAYOUT_NATURAL)
    return o


def sharded_nabla_attention(q, k, v, T, Hg, W, thr, window=(0, 0, 0), scale=None, group=None,
                            compute=None):
    """NABLA attention for sequence-sharded inputs.

    q, k, v : [B, H, S/N, D] bf16, this rank's contiguous token range of every head
              (natural order, S = T * Hg * W).
    compute : the per-rank hot path, called as compute(q, k, v, shape, thr, window, scale)
              on [B, H/N, S, D] tensors with ``shape`` the rank's Shape; defaults to
              nabla_local_heads (the CUDA path).
    Returns O [B, H, S/N, D] in the caller's sharding.
    """
    from adaptive_block_sparse_b200 import Shape
    n = dist.get_world_size(group)
    B, H, s, D = q.shape
    if s * n != T * Hg * W:
        raise ValueError("the token shards do not cover the latent")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    qh, kh, vh = (seq_to_heads(x, group) for x in (q, k, v))
    shape = Shape(B, H // n, T, Hg, W, D)
    o = (compute or nabla_local_heads)(qh, kh, vh, shape, thr, window, scale)
    return heads_to_seq(o, group)
