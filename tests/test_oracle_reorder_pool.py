"""Pins for the oracle's fractal-flatten reorder and block pooling (CPU only)."""
import math
import os

import numpy as np
import pytest

from oracle import fractal_permutation, inverse_reorder, pool_blocks, reorder

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


def test_reorder_hand_derived_indices():
    n = 0
    for line in _golden_rows("reorder_indices.txt"):
        T, Hg, W, P, t, h, w, r = (int(a) for a in line.split())
        perm = fractal_permutation(T, Hg, W, P)
        assert perm[r] == (t * Hg + h) * W + w, line
        n += 1
    assert n >= 10


def test_reorder_p1_is_identity():
    assert np.array_equal(fractal_permutation(3, 5, 7, 1), np.arange(105))


@pytest.mark.parametrize("shape", [(1, 16, 16, 8), (2, 16, 24, 8), (3, 8, 8, 4), (4, 32, 32, 8)])
def test_reorder_is_bijection_and_blocks_are_patches(shape):
    T, Hg, W, P = shape
    perm = fractal_permutation(T, Hg, W, P)
    assert np.array_equal(np.sort(perm), np.arange(T * Hg * W))
    t, rem = np.divmod(perm, Hg * W)
    h, w = np.divmod(rem, W)
    # frames stay in order: slot r lies in frame r // (Hg*W)
    assert np.array_equal(t, np.arange(T * Hg * W) // (Hg * W))
    # every run of P*P slots is one P x P spatial square of one frame
    N = P * P
    for blk in range(perm.size // N):
        sl = slice(blk * N, (blk + 1) * N)
        assert len(set(t[sl])) == 1
        assert h[sl].max() - h[sl].min() == P - 1 and w[sl].max() - w[sl].min() == P - 1
        assert h[sl].min() % P == 0 and w[sl].min() % P == 0


def test_inverse_roundtrip():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, 3, 2 * 16 * 24, 5))
    y = reorder(x, 2, 16, 24, 8)
    assert np.array_equal(inverse_reorder(y, 2, 16, 24, 8), x)
    assert not np.array_equal(y, x)


def test_pool_constant_and_token_index_closed_form():
    T, Hg, W, P = 2, 16, 24, 8
    N = P * P
    S = T * Hg * W
    c = np.full((1, 1, S, 3), 1.75)
    assert np.array_equal(pool_blocks(reorder(c, T, Hg, W, P), N), np.full((1, 1, S // N, 3), 1.75))
    # value = natural index; a block's mean is the index of its patch centre
    x = np.arange(S, dtype=np.float64)[None, None, :, None]
    got = pool_blocks(reorder(x, T, Hg, W, P), N)[0, 0, :, 0]
    Hb, Wb = Hg // P, W // P
    for blk in range(S // N):
        t, rem = divmod(blk, Hb * Wb)
        hb, wb = divmod(rem, Wb)
        centre = t * Hg * W + (hb * P + (P - 1) / 2) * W + wb * P + (P - 1) / 2
        assert got[blk] == centre


def test_pool_of_bf16_values_is_exact():
    import torch
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(1, 2, 256, 16, generator=g) * 3).to(torch.bfloat16).double().numpy()
    got = pool_blocks(x, 64)
    xb = x.reshape(1, 2, 4, 64, 16)
    for idx in np.ndindex(1, 2, 4, 16):
        b, h, i, d = idx
        assert got[b, h, i, d] == math.fsum(xb[b, h, i, :, d]) / 64
