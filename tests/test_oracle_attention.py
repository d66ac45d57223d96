"""Pins for the oracle's block-sparse attention forward and backward (CPU only)."""
import math

import numpy as np
import pytest
import torch

from oracle import (block_sparse_attention, block_sparse_attention_bwd,
                    block_sparse_attention_rows, nabla_mask, reorder, sta_mask)
from synth import WORKLOADS, make_qkv


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _sdpa(q, k, v, scale, attn_mask=None):
    t = [torch.tensor(a) for a in (q, k, v)]
    return torch.nn.functional.scaled_dot_product_attention(
        *t, attn_mask=attn_mask, scale=scale).numpy()


def _token_mask(mask, N):
    return np.repeat(np.repeat(mask, N, axis=-2), N, axis=-1)


def test_full_mask_equals_dense_library_attention():
    B, H, S, D, N = 1, 2, 256, 16, 64
    q, k, v = (_rand((B, H, S, D), s) for s in (1, 2, 3))
    mask = np.ones((B, H, S // N, S // N), dtype=bool)
    O, LSE = block_sparse_attention(q, k, v, mask, N, 0.3)
    np.testing.assert_allclose(O, _sdpa(q, k, v, 0.3), rtol=0, atol=1e-12)
    logits = np.einsum("bhsd,bhtd->bhst", q, k) * 0.3
    from scipy.special import logsumexp
    np.testing.assert_allclose(LSE, logsumexp(logits, axis=-1), rtol=0, atol=1e-12)


def test_random_mask_equals_library_attention_with_additive_mask():
    B, H, S, D, N = 1, 2, 320, 8, 64
    q, k, v = (_rand((B, H, S, D), s) for s in (4, 5, 6))
    rng = np.random.default_rng(7)
    mask = rng.random((B, H, S // N, S // N)) < 0.4
    mask[..., np.arange(S // N), np.arange(S // N)] = True   # no empty rows here
    O, _ = block_sparse_attention(q, k, v, mask, N, 0.5)
    add = torch.tensor(np.where(_token_mask(mask, N), 0.0, -np.inf))
    np.testing.assert_allclose(O, _sdpa(q, k, v, 0.5, add), rtol=0, atol=1e-12)


def test_block_diagonal_mask_is_independent_block_attention():
    B, H, S, D, N = 1, 1, 192, 8, 64
    q, k, v = (_rand((B, H, S, D), s) for s in (8, 9, 10))
    mask = np.eye(S // N, dtype=bool)[None, None]
    O, _ = block_sparse_attention(q, k, v, mask, N, 0.2)
    for i in range(S // N):
        sl = slice(i * N, (i + 1) * N)
        np.testing.assert_allclose(O[:, :, sl], _sdpa(q[:, :, sl], k[:, :, sl], v[:, :, sl], 0.2),
                                   rtol=0, atol=1e-12)


def test_per_token_brute_force_tiny_workload():
    """Scalar loops over every token pair of the tiny workload (one head, two rows/block)."""
    wl = WORKLOADS["tiny"]
    q, k, v = (reorder(t.double().numpy(), wl.T, wl.Hg, wl.W, wl.P) for t in make_qkv(wl))
    mask, _, _ = nabla_mask(q, k, wl.T, wl.Hg, wl.W, wl.P, 0.8)
    scale = 1 / math.sqrt(wl.D)
    O, LSE = block_sparse_attention(q, k, v, mask, wl.N, scale)
    h = 1
    for r in (0, 63, 64, 200, 511):
        logits = []
        for c in range(wl.S):
            if mask[0, h, r // wl.N, c // wl.N]:
                logits.append((c, sum(q[0, h, r, d] * k[0, h, c, d] for d in range(wl.D)) * scale))
        m = max(x for _, x in logits)
        w = [(c, math.exp(x - m)) for c, x in logits]
        l = math.fsum(x for _, x in w)
        for d in (0, 17, 63):
            o = math.fsum(x * v[0, h, c, d] for c, x in w) / l
            assert abs(O[0, h, r, d] - o) < 1e-11
        assert abs(LSE[0, h, r] - (m + math.log(l))) < 1e-11


def test_rows_variant_and_empty_rows():
    B, H, S, D, N = 1, 1, 256, 8, 64
    q, k, v = (_rand((B, H, S, D), s) for s in (11, 12, 13))
    mask = np.zeros((1, 1, 4, 4), dtype=bool)
    mask[0, 0, 0, [1, 3]] = True
    mask[0, 0, 2, 2] = True
    O, LSE = block_sparse_attention(q, k, v, mask, N, 0.4)
    rows = np.array([0, 5, 70, 130, 255])
    Or, Lr = block_sparse_attention_rows(q[0, 0], k[0, 0], v[0, 0], mask[0, 0], N, 0.4, rows)
    np.testing.assert_allclose(Or, O[0, 0, rows], rtol=0, atol=1e-14)
    np.testing.assert_allclose(Lr, LSE[0, 0, rows], rtol=0, atol=1e-14)
    assert np.all(O[0, 0, 64:128] == 0) and np.all(np.isneginf(LSE[0, 0, 64:128]))


def _autograd_ref(q, k, v, dout, mask, N, scale):
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    add = torch.tensor(np.where(_token_mask(mask, N), 0.0, -np.inf))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=add, scale=scale)
    o.backward(torch.tensor(dout))
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("full", [True, False])
def test_backward_matches_library_autograd(full):
    B, H, S, D, N = 1, 2, 256, 16, 64
    q, k, v, do = (_rand((B, H, S, D), s) for s in (21, 22, 23, 24))
    rng = np.random.default_rng(25)
    mask = np.ones((B, H, 4, 4), dtype=bool) if full else rng.random((B, H, 4, 4)) < 0.5
    mask[..., np.arange(4), np.arange(4)] = True
    got = block_sparse_attention_bwd(q, k, v, do, mask, N, 0.25)
    ref = _autograd_ref(q, k, v, do, mask, N, 0.25)
    for a, b in zip(got, ref):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-11)


def test_backward_finite_differences():
    B, H, S, D, N = 1, 1, 128, 4, 64
    q, k, v, do = (_rand((B, H, S, D), s, 0.7) for s in (31, 32, 33, 34))
    mask = np.array([[[[True, False], [True, True]]]])
    dq, dk, dv = block_sparse_attention_bwd(q, k, v, do, mask, N, 0.5)

    def loss(q_, k_, v_):
        return float(np.sum(block_sparse_attention(q_, k_, v_, mask, N, 0.5)[0] * do))

    eps = 1e-6
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in [(0, 0, 3, 1), (0, 0, 70, 2), (0, 0, 127, 0), (0, 0, 64, 3)]:
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args_p = {"q": (plus, k, v), "k": (q, plus, v), "v": (q, k, plus)}[name]
            args_m = {"q": (minus, k, v), "k": (q, minus, v), "v": (q, k, minus)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grad[idx]) < 1e-7, (name, idx, fd, grad[idx])


def test_mask_end_to_end_properties():
    wl = WORKLOADS["tiny"]
    q, k, v = (reorder(t.double().numpy(), wl.T, wl.Hg, wl.W, wl.P) for t in make_qkv(wl))
    full, _, _ = nabla_mask(q, k, wl.T, wl.Hg, wl.W, wl.P, 1.0)
    assert full.all()
    prev = None
    for thr in (0.2, 0.5, 0.8, 0.95):
        m, E, p = nabla_mask(q, k, wl.T, wl.Hg, wl.W, wl.P, thr)
        if prev is not None:
            assert np.all(prev <= m)
        assert np.all(m.sum(-1) >= 1)
        prev = m
    # union is a superset of both parts
    m_n, _, _ = nabla_mask(q, k, wl.T, wl.Hg, wl.W, wl.P, 0.5)
    m_u, _, _ = nabla_mask(q, k, wl.T, wl.Hg, wl.W, wl.P, 0.5, window=(1, 3, 1))
    sta = sta_mask(wl.T, wl.Hg // wl.P, wl.W // wl.P, (1, 3, 1))
    assert np.all(m_u >= m_n) and np.all(m_u >= sta[None, None])
    assert np.array_equal(m_u, m_n | sta[None, None])
    # thr -> 1 with full mask gives dense attention
    O, _ = block_sparse_attention(q, k, v, full, wl.N, 1 / math.sqrt(wl.D))
    np.testing.assert_allclose(O, _sdpa(q, k, v, 1 / math.sqrt(wl.D)), rtol=0, atol=1e-11)


def test_mask_closed_form_on_constant_blocks():
    """Blocks holding constant, mutually orthogonal vectors: the pooled map is known exactly."""
    T, Hg, W, P, D = 1, 16, 16, 8, 8
    N, nb = P * P, 4
    alpha = 3.0
    blocks = np.zeros((nb, D))
    blocks[np.arange(nb), np.arange(nb)] = alpha
    q = np.repeat(blocks, N, axis=0)[None, None]          # already in reordered order
    scale = 1 / math.sqrt(D)
    _, _, p = nabla_mask(q, q, T, Hg, W, P, 0.5)
    a = alpha * alpha * scale
    diag = math.exp(a) / (math.exp(a) + nb - 1)
    np.testing.assert_allclose(np.diagonal(p[0, 0]), diag, rtol=1e-14)
    for thr, expect in ((diag - 1e-3, 1), (diag + 1e-3, 2)):
        m, _, _ = nabla_mask(q, q, T, Hg, W, P, thr)
        assert np.all(m.sum(-1) == expect)
        assert np.all(np.diagonal(m[0, 0]))
    # with expect 2 the second block is the lowest other index (tie-break)
    m, _, _ = nabla_mask(q, q, T, Hg, W, P, diag + 1e-3)
    assert m[0, 0, 0].tolist() == [True, True, False, False]
    assert m[0, 0, 1].tolist() == [True, True, False, False]
    assert m[0, 0, 3].tolist() == [True, False, False, True]
