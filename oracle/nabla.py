"""NABLA hot path, restated in plain NumPy fp64 (test infrastructure; see package header).

Citations name the page and its section:
  [ZH-TS]  "NABLA: Neighborhood Adaptive Block-Level Attention", gist.science (Chinese
           edition), technical summary, section "Methodology" (token reordering,
           adaptive mask construction, hybrid integration with STA).
  [LSD-2]  lsdiaocha.cn article on NABLA (arXiv 2507.13546), section 2, "the core
           innovation of the NABLA algorithm" (three steps: pooled scouting, CDF
           filtering, exact mapping back; OR-union with STA).
  [LSD-4]  same article, section 4, "technical principles" (N tokens pooled per
           block; sort each row, accumulate probability; smaller thr => sparser).

Notation follows the pages: Q, K, V; P = patch side (P x P spatial patch), N = P*P tokens
per block; thr = CDF threshold; M = M_nabla OR M_STA.  Tensors are [B, H, S, D] with
S = T * Hg * W tokens; nb = S / N blocks.

Readings taken where the pages are silent (each restated at the function that uses it):
  * row-major patch order and row-major order inside a patch;
  * the pooled map is scaled by 1/sqrt(D) like token attention;
  * block j is kept iff the probability mass ranked strictly before it (ranking by
    probability descending, ties by lower block index first) is < thr, which equals
    "ascending CDF > 1 - thr"; thr >= 1 keeps every block;
  * STA window is centred on the query block and truncated at the grid edges;
  * the mask is a constant for the backward pass.
"""

from __future__ import annotations

import math

import numpy as np


# --------------------------------------------------------------------------------------
# Token reordering ("fractal flatten")                                         [ZH-TS]
# --------------------------------------------------------------------------------------
def fractal_permutation(T: int, Hg: int, W: int, P: int) -> np.ndarray:
    """Return ``perm`` with ``perm[r]`` = natural index of the token at reordered slot r.

    [ZH-TS] "token reordering (fractal flatten)": the tokens of every P x P spatial patch
    are grouped into one contiguous run, and the time dimension stays in order.  The
    natural index of token (t, h, w) is (t*Hg + h)*W + w.  Patches are visited row-major
    (patch row, then patch column) inside each frame, and the P*P tokens of a patch are
    visited row-major (reading taken: the pages describe a single level of P x P grouping).
    """
    if Hg % P or W % P:
        raise ValueError("Hg and W must be multiples of P")
    Hb, Wb = Hg // P, W // P
    perm = np.empty(T * Hg * W, dtype=np.int64)
    r = 0
    for t in range(T):
        for hb in range(Hb):
            for wb in range(Wb):
                for dh in range(P):
                    for dw in range(P):
                        h = hb * P + dh
                        w = wb * P + dw
                        perm[r] = (t * Hg + h) * W + w
                        r += 1
    return perm


def reorder(x: np.ndarray, T: int, Hg: int, W: int, P: int) -> np.ndarray:
    """Natural [..., S, D] -> fractal order [..., S, D] (dst[r] = src[perm[r]])."""
    perm = fractal_permutation(T, Hg, W, P)
    return np.ascontiguousarray(x[..., perm, :])


def inverse_reorder(y: np.ndarray, T: int, Hg: int, W: int, P: int) -> np.ndarray:
    """Fractal order -> natural order; the inverse of :func:`reorder`."""
    perm = fractal_permutation(T, Hg, W, P)
    out = np.empty_like(y)
    out[..., perm, :] = y
    return out


# --------------------------------------------------------------------------------------
# Adaptive mask construction                                             [ZH-TS, LSD-2]
# --------------------------------------------------------------------------------------
def pool_blocks(x: np.ndarray, N: int) -> np.ndarray:
    """Average-pool every run of N consecutive (reordered) tokens: [..., S, D] -> [..., nb, D].

    [ZH-TS] "downsampling": Q and K are reshaped and average-pooled per block; [LSD-4]
    N adjacent tokens form one block.  The N rows are summed one after another in fp64
    (token 0 first), then divided by N.  For bf16 inputs this sum is exact.
    """
    x = np.asarray(x, dtype=np.float64)
    S, D = x.shape[-2], x.shape[-1]
    if S % N:
        raise ValueError("S must be a multiple of N")
    xb = x.reshape(x.shape[:-2] + (S // N, N, D))
    acc = np.zeros(x.shape[:-2] + (S // N, D), dtype=np.float64)
    for j in range(N):
        acc = acc + xb[..., j, :]
    return acc / N


def pooled_logits(q_pool: np.ndarray, k_pool: np.ndarray, scale: float) -> np.ndarray:
    """[ZH-TS] "reduced attention": full attention logits on the pooled map, Qp Kp^T * scale."""
    return np.matmul(q_pool, np.swapaxes(k_pool, -1, -2)) * scale


def pooled_softmax(logits: np.ndarray) -> np.ndarray:
    """Row softmax of the pooled logits ([LSD-2] step 2: softmax normalisation)."""
    m = np.max(logits, axis=-1, keepdims=True)
    e = np.exp(logits - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def cdf_keep_row(p_row: np.ndarray, thr: float):
    """Binarise one row of the pooled probability map.  Returns (keep, E).

    [ZH-TS] "CDF thresholding": per row compute the cumulative distribution and keep
    the blocks whose cumulative probability exceeds 1 - thr.  [LSD-4]: sort the row and
    accumulate; a smaller thr gives a sparser mask.  With an ascending sort the CDF at
    block j is C_j = 1 - E_j, where E_j is the mass of the blocks ranked above j, so the
    kept set is {j : E_j < thr}: the smallest set of top blocks holding >= thr of the
    mass.  Ranking: probability descending, ties by lower block index first.  E is
    accumulated sequentially in rank order.  thr >= 1 keeps every block.
    """
    p_row = np.asarray(p_row, dtype=np.float64)
    order = np.argsort(-p_row, kind="stable")
    ps = p_row[order]
    e_sorted = np.empty_like(ps)
    acc = 0.0
    for r in range(ps.shape[0]):
        e_sorted[r] = acc
        acc = acc + ps[r]
    E = np.empty_like(p_row)
    E[order] = e_sorted
    keep = np.ones(p_row.shape, dtype=bool) if thr >= 1.0 else (E < thr)
    return keep, E


def cdf_mask(p: np.ndarray, thr: float):
    """Row-wise :func:`cdf_keep_row` over the last axis (vectorised; same arithmetic).

    ``np.cumsum`` along the last axis accumulates sequentially, exactly like the loop in
    :func:`cdf_keep_row`.
    """
    p = np.asarray(p, dtype=np.float64)
    order = np.argsort(-p, axis=-1, kind="stable")
    ps = np.take_along_axis(p, order, axis=-1)
    csum = np.cumsum(ps, axis=-1)
    e_sorted = np.concatenate([np.zeros(ps.shape[:-1] + (1,)), csum[..., :-1]], axis=-1)
    E = np.empty_like(p)
    np.put_along_axis(E, order, e_sorted, axis=-1)
    keep = np.ones(p.shape, dtype=bool) if thr >= 1.0 else (E < thr)
    return keep, E


def block_coords(T: int, Hb: int, Wb: int) -> np.ndarray:
    """(t, hb, wb) of every block in reordered order: block i = (t*Hb + hb)*Wb + wb."""
    i = np.arange(T * Hb * Wb)
    return np.stack([i // (Hb * Wb), (i // Wb) % Hb, i % Wb], axis=-1)


def sta_mask(T: int, Hb: int, Wb: int, window) -> np.ndarray:
    """Static sliding-tile window at block granularity, [nb, nb] bool.

    [ZH-TS] "hybrid integration with STA": a static window mask M_STA.  Query block
    (t, hb, wb) keeps key block (t', hb', wb') iff |t-t'| <= wt//2, |hb-hb'| <= wh//2 and
    |wb-wb'| <= ww//2 (window sizes in blocks, odd).  Reading taken: the window is
    centred and truncated at the grid edges.  window == (0, 0, 0) means no STA.
    """
    wt, wh, ww = (int(a) for a in window)
    nb = T * Hb * Wb
    if (wt, wh, ww) == (0, 0, 0):
        return np.zeros((nb, nb), dtype=bool)
    c = block_coords(T, Hb, Wb)
    d = np.abs(c[:, None, :] - c[None, :, :])
    return (d[..., 0] <= wt // 2) & (d[..., 1] <= wh // 2) & (d[..., 2] <= ww // 2)


def nabla_mask(q: np.ndarray, k: np.ndarray, T: int, Hg: int, W: int, P: int,
               thr: float, window=(0, 0, 0), scale: float | None = None):
    """Full mask build on reordered Q, K [B, H, S, D].  Returns (mask, E, p).

    Steps in the pages' order [ZH-TS]: pool Q and K per block of N = P*P tokens, full
    attention on the pooled map, row softmax, CDF threshold, then M = M_nabla OR M_STA.
    ``mask`` is bool [B, H, nb, nb]; ``E`` holds each block's exclusive ranked mass
    (so ``|E - thr|`` measures how close a block is to the threshold); ``p`` is the
    pooled probability map.  Heads are processed one by one ([LSD-2]: each head builds
    its own mask).
    """
    q = np.asarray(q)
    k = np.asarray(k)
    B, H, S, D = q.shape
    N = P * P
    nb = S // N
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    sta = sta_mask(T, Hg // P, W // P, window)
    mask = np.empty((B, H, nb, nb), dtype=bool)
    E = np.empty((B, H, nb, nb), dtype=np.float64)
    p = np.empty((B, H, nb, nb), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            qp = pool_blocks(q[b, h], N)
            kp = pool_blocks(k[b, h], N)
            p[b, h] = pooled_softmax(pooled_logits(qp, kp, scale))
            keep, E[b, h] = cdf_mask(p[b, h], thr)
            mask[b, h] = keep | sta
    return mask, E, p


# --------------------------------------------------------------------------------------
# Mask formats (bitmask words, ascending row / column lists)
# --------------------------------------------------------------------------------------
def pack_mask_bits(mask: np.ndarray) -> np.ndarray:
    """bool [..., nb, nb] -> uint32 [..., nb, ceil(nb/32)]; bit (j % 32) of word j // 32."""
    nb = mask.shape[-1]
    nw = (nb + 31) // 32
    padded = np.zeros(mask.shape[:-1] + (nw * 32,), dtype=np.uint64)
    padded[..., :nb] = mask
    padded = padded.reshape(mask.shape[:-1] + (nw, 32))
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    return (padded * weights).sum(axis=-1).astype(np.uint32)


def unpack_mask_bits(bits: np.ndarray, nb: int) -> np.ndarray:
    bits = np.asarray(bits, dtype=np.uint64)
    j = np.arange(nb)
    return ((bits[..., j // 32] >> (j % 32).astype(np.uint64)) & np.uint64(1)).astype(bool)


def row_lists(mask: np.ndarray):
    """Kept key-block indices of every query-block row, ascending; padded with -1."""
    nb = mask.shape[-1]
    cnt = mask.sum(axis=-1).astype(np.int32)
    idx = np.full(mask.shape, -1, dtype=np.int32)
    flat_m = mask.reshape(-1, nb)
    flat_i = idx.reshape(-1, nb)
    for r in range(flat_m.shape[0]):
        nz = np.nonzero(flat_m[r])[0]
        flat_i[r, : nz.size] = nz
    return idx, cnt


def col_lists(mask: np.ndarray):
    """Query-block indices that keep each key block, ascending; padded with -1."""
    return row_lists(np.swapaxes(mask, -1, -2))


# --------------------------------------------------------------------------------------
# Block-sparse attention                                                 [ZH-TS, LSD-2]
# --------------------------------------------------------------------------------------
def _kept_tokens(mask_row: np.ndarray, N: int) -> np.ndarray:
    """[ZH-TS] "expansion": a kept pooled entry (i, j) keeps the whole N x N tile."""
    blocks = np.nonzero(mask_row)[0]
    return (blocks[:, None] * N + np.arange(N)[None, :]).reshape(-1)


def block_sparse_attention(q, k, v, mask, N: int, scale: float):
    """Exact softmax attention restricted to the kept N x N tiles.  Returns (O, LSE).

    For every query token r of block i: O_r = sum_c softmax_c(scale * Q_r . K_c) V_c over
    the tokens c of the kept key blocks of row i; LSE_r = log sum_c exp(scale * Q_r . K_c)
    (natural log).  A row with no kept block gives O = 0 and LSE = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, H, S, D = q.shape
    nb = S // N
    O = np.zeros((B, H, S, D))
    LSE = np.full((B, H, S), -np.inf)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                cols = _kept_tokens(mask[b, h, i], N)
                if cols.size == 0:
                    continue
                rows = slice(i * N, (i + 1) * N)
                s = (q[b, h, rows] @ k[b, h, cols].T) * scale
                m = s.max(axis=-1, keepdims=True)
                e = np.exp(s - m)
                l = e.sum(axis=-1, keepdims=True)
                O[b, h, rows] = (e @ v[b, h, cols]) / l
                LSE[b, h, rows] = (m + np.log(l))[:, 0]
    return O, LSE


def block_sparse_attention_rows(q_bh, k_bh, v_bh, mask_bh, N: int, scale: float, rows):
    """Same as :func:`block_sparse_attention` for selected token rows of one (b, h).

    ``q_bh`` etc. are [S, D] for one head; returns (O [len(rows), D], LSE [len(rows)]).
    """
    q_bh = np.asarray(q_bh, dtype=np.float64)
    k_bh = np.asarray(k_bh, dtype=np.float64)
    v_bh = np.asarray(v_bh, dtype=np.float64)
    rows = np.asarray(rows)
    O = np.zeros((rows.size, q_bh.shape[-1]))
    LSE = np.full(rows.size, -np.inf)
    for n, r in enumerate(rows):
        cols = _kept_tokens(mask_bh[r // N], N)
        if cols.size == 0:
            continue
        s = (k_bh[cols] @ q_bh[r]) * scale
        m = s.max()
        e = np.exp(s - m)
        l = e.sum()
        O[n] = (e @ v_bh[cols]) / l
        LSE[n] = m + math.log(l)
    return O, LSE


def block_sparse_attention_bwd(q, k, v, dout, mask, N: int, scale: float, heads=None):
    """Gradients of :func:`block_sparse_attention` with the mask held constant.

    Standard softmax-attention backward on the kept tiles ([LSD-2] / [ZH-TS] say NABLA
    accelerates training; the binary mask has no gradient, so it is a constant):
      P = softmax(scale * Q K^T) on kept tiles,  dV = P^T dO,  dP = dO V^T,
      D_r = sum_c P_rc dP_rc (= dO_r . O_r),  dS = P * (dP - D),
      dQ = scale * dS K,  dK = scale * dS^T Q.
    ``heads`` optionally restricts the work to a list of (b, h); other heads stay zero.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    B, H, S, D = q.shape
    nb = S // N
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(H)]
    for b, h in heads:
        for i in range(nb):
            cols = _kept_tokens(mask[b, h, i], N)
            if cols.size == 0:
                continue
            rows = slice(i * N, (i + 1) * N)
            qi, doi = q[b, h, rows], dout[b, h, rows]
            kc, vc = k[b, h, cols], v[b, h, cols]
            s = (qi @ kc.T) * scale
            e = np.exp(s - s.max(axis=-1, keepdims=True))
            p = e / e.sum(axis=-1, keepdims=True)
            dv[b, h, cols] += p.T @ doi
            dp = doi @ vc.T
            drow = (p * dp).sum(axis=-1, keepdims=True)
            ds = p * (dp - drow)
            dq[b, h, rows] = scale * (ds @ kc)
            dk[b, h, cols] += scale * (ds.T @ qi)
    return dq, dk, dv
