"""Head-sharded NABLA attention for callers whose activations are sharded by sequence.

Every (batch, head) pair goes through the whole path independently: each head pools its
own Q and K, builds its own block mask and attends over its own kept tiles (lsdiaocha.cn
article on NABLA, section 2: the mask is formed per head from that head's pooled map).
So heads, not tokens, are the unit to distribute.  A model that keeps its activations
sharded by sequence (rank r holding a contiguous range of S/N tokens of every head)
exchanges them once before attention and once after:

    [B, H, S/N, D] per rank  --all-to-all-->  every token of this rank's heads
    hot path on the rank's heads (mask with its pooling, forward; natural token order)
    this rank's heads          --all-to-all-->  [B, H, S/N, D] per rank

Two ways to assign heads to ranks:
  * ``balance="contiguous"``: heads [r H/N, (r+1) H/N) on rank r (seq_to_heads /
    heads_to_seq), equal head counts;
  * ``balance="lpt"`` (default): heads by their work.  The kept-tile count of a head is
    known once its mask is built, and it differs by two orders of magnitude between
    heads (a head with flat pooled scores keeps hundreds of key blocks per row, a peaked
    one a handful), so equal head counts can leave one rank with most of the work.
    Each rank pools its own token range (whole rows of 8 x 8 patches), the pooled means
    are all-gathered (B*H*nb*D fp64 values, small beside Q, K, V), every rank builds the
    same masks of all heads from them, and the (b, h) units go to ranks longest
    processing time first (units by kept tiles descending, each to the least loaded
    rank).  The exchanges are then uneven all-to-alls.

The exchanges are ``torch.distributed`` collectives (NCCL over NVLink / NVSwitch on
GPUs; any backend with all-to-all, e.g. gloo on the host), plain data movement, so the
sharded result equals the unsharded one bit for bit.
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


def lpt_assign(loads, n):
    """Longest-processing-time-first assignment of units (with ``loads``) to ``n`` ranks.

    Units are taken by load descending (index ascending on ties); each goes to the rank
    with the smallest total so far (lowest rank on ties).  Deterministic, so every rank
    computes the same plan.  The largest rank total is at most 4/3 of the optimum
    (Graham's bound for this greedy order).  Returns one ascending unit list per rank.
    """
    order = sorted(range(len(loads)), key=lambda u: (-loads[u], u))
    totals = [0] * n
    plan = [[] for _ in range(n)]
    for u in order:
        r = min(range(n), key=lambda x: (totals[x], x))
        plan[r].append(u)
        totals[r] += loads[u]
    return [sorted(p) for p in plan]


def seq_to_units(x, plan, group=None):
    """[B, H, S/N, D] (this rank's tokens of every head) -> [1, U, S, D]: every token of
    this rank's units plan[rank] (flat indices b*H + h, ascending), tokens in rank order.
    One uneven all_to_all_single."""
    n = dist.get_world_size(group)
    me = dist.get_rank(group)
    B, H, s, D = x.shape
    flat = x.reshape(B * H, s, D)
    send = torch.cat([flat[plan[d]] for d in range(n)], dim=0).contiguous()
    u = len(plan[me])
    recv = torch.empty((n * u, s, D), dtype=x.dtype, device=x.device)
    dist.all_to_all_single(recv, send, output_split_sizes=[u] * n,
                           input_split_sizes=[len(plan[d]) for d in range(n)], group=group)
    return recv.reshape(n, u, s, D).permute(1, 0, 2, 3).reshape(1, u, n * s, D)


def units_to_seq(y, plan, B, H, group=None):
    """Inverse of seq_to_units: [1, U, S, D] of this rank's units -> [B, H, S/N, D]."""
    n = dist.get_world_size(group)
    _, u, S, D = y.shape
    s = S // n
    send = y.reshape(u, n, s, D).permute(1, 0, 2, 3).contiguous().reshape(n * u, s, D)
    counts = [len(plan[d]) for d in range(n)]
    recv = torch.empty((sum(counts), s, D), dtype=y.dtype, device=y.device)
    dist.all_to_all_single(recv, send, output_split_sizes=counts, input_split_sizes=[u] * n,
                           group=group)
    out = torch.empty((B * H, s, D), dtype=y.dtype, device=y.device)
    out[[x for d in range(n) for x in plan[d]]] = recv
    return out.reshape(B, H, s, D)


def nabla_local_heads(q, k, v, shape, thr, window=(0, 0, 0), scale=None):
    """The hot path on one rank's heads, natural token order in and out: the block mask
    from Q and K (pooled by the mask build itself), the forward reading Q, K, V in place.
    Returns bf16 O [B, h, S, D]."""
    import adaptive_block_sparse_b200 as m
    bits, _, _, _, _ = m.nabla_build_mask(q, k, shape, thr, window, scale=scale,
                                          layout=m.NABLA_LAYOUT_NATURAL)
    o, _ = m.nabla_attn_fwd(q, k, v, bits, shape, scale=scale, layout=m.NABLA_LAYOUT_NATURAL)
    return o


def unit_loads(q, k, T, Hg, W, thr, window=(0, 0, 0), scale=None, group=None):
    """Kept tiles of every (b, h) unit of a sequence-sharded problem, and the masks.

    q, k: [B, H, S/N, D] bf16, this rank's contiguous token range of every head (natural
    order; S/N must hold whole rows of 8 x 8 patches, a multiple of 8 * W tokens).  Each
    rank pools its range (viewed as one latent frame of S/(N W) rows), the pools are
    all-gathered, and every rank builds the masks of all heads from them (the same bits
    on every rank).  Returns (loads: list of B*H ints, mask_bits [B, H, nb, nw]).
    """
    import adaptive_block_sparse_b200 as m
    n = dist.get_world_size(group)
    B, H, s, D = q.shape
    if s % (8 * W):
        raise ValueError("a token shard must hold whole rows of 8 x 8 patches")
    local = m.Shape(B, H, 1, s // W, W, D)
    qp = torch.empty(B, H, local.nb, D, dtype=torch.float64, device=q.device)
    kp = torch.empty_like(qp)
    m.nabla_reorder(q, None, local, pool_out=qp)
    m.nabla_reorder(k, None, local, pool_out=kp)
    gq = [torch.empty_like(qp) for _ in range(n)]
    gk = [torch.empty_like(kp) for _ in range(n)]
    dist.all_gather(gq, qp, group=group)
    dist.all_gather(gk, kp, group=group)
    full = m.Shape(B, H, T, Hg, W, D)
    cnt = torch.empty(B, H, full.nb, dtype=torch.int32, device=q.device)
    bits, _, _, _, _ = m.nabla_build_mask(None, None, full, thr, window, scale=scale, row_cnt=cnt,
                                          q_pool=torch.cat(gq, dim=2).contiguous(),
                                          k_pool=torch.cat(gk, dim=2).contiguous())
    return cnt.to(torch.int64).sum(dim=-1).reshape(-1).tolist(), bits


def sharded_nabla_attention(q, k, v, T, Hg, W, thr, window=(0, 0, 0), scale=None, group=None,
                            compute=None, balance="lpt", loads=None):
    """NABLA attention for sequence-sharded inputs.

    q, k, v : [B, H, S/N, D] bf16, this rank's contiguous token range of every head
              (natural order, S = T * Hg * W).
    balance : "lpt" (heads to ranks by kept tiles) or "contiguous" (H/N heads per rank).
    loads   : optional per-unit work (B*H numbers, b*H + h) for "lpt"; by default the
              exact kept-tile counts from unit_loads (whose masks are then reused).
    compute : the per-rank hot path, called as compute(q, k, v, shape, thr, window, scale)
              on the rank's heads with ``shape`` their Shape; defaults to the CUDA path.
    Returns O [B, H, S/N, D] in the caller's sharding.
    """
    import adaptive_block_sparse_b200 as m
    n = dist.get_world_size(group)
    B, H, s, D = q.shape
    if s * n != T * Hg * W:
        raise ValueError("the token shards do not cover the latent")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if balance == "contiguous":
        qh, kh, vh = (seq_to_heads(x, group) for x in (q, k, v))
        shape = m.Shape(B, H // n, T, Hg, W, D)
        o = (compute or nabla_local_heads)(qh, kh, vh, shape, thr, window, scale)
        return heads_to_seq(o, group)
    if balance != "lpt":
        raise ValueError(f"unknown balance {balance!r}")
    bits = None
    if loads is None:
        loads, bits = unit_loads(q, k, T, Hg, W, thr, window, scale, group)
    if len(loads) != B * H:
        raise ValueError("loads must give one number per (b, h)")
    plan = lpt_assign(list(loads), n)
    mine = plan[dist.get_rank(group)]
    qu, ku, vu = (seq_to_units(x, plan, group) for x in (q, k, v))
    shape = m.Shape(1, len(mine), T, Hg, W, D)
    if not mine:
        o = torch.empty((1, 0, T * Hg * W, D), dtype=torch.bfloat16, device=q.device)
    elif compute is not None:
        o = compute(qu, ku, vu, shape, thr, window, scale)
    elif bits is not None:
        # the masks of this rank's units were built with everyone's; reuse them
        ub = bits.reshape(B * H, *bits.shape[2:])[mine].reshape(1, len(mine), *bits.shape[2:]).contiguous()
        o, _ = m.nabla_attn_fwd(qu, ku, vu, ub, shape, scale=scale, layout=m.NABLA_LAYOUT_NATURAL)
    else:
        o = nabla_local_heads(qu, ku, vu, shape, thr, window, scale)
    return units_to_seq(o, plan, B, H, group)
