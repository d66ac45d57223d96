"""Pins for the oracle's pooled softmax, CDF threshold and STA window (CPU only)."""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import (cdf_keep_row, cdf_mask, pack_mask_bits, pooled_logits, pooled_softmax,
                    sta_mask, unpack_mask_bits, row_lists, col_lists)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


def test_threshold_golden_rows():
    n = 0
    for line in _rows("threshold_rows.txt"):
        ps, thr, kept = (s.strip() for s in line.split(";"))
        p = np.array([float(a) for a in ps.split(",")])
        keep, _ = cdf_keep_row(p, float(thr))
        assert sorted(np.nonzero(keep)[0].tolist()) == [int(a) for a in kept.split(",")], line
        n += 1
    assert n >= 12


def test_pooled_softmax_matches_library_attention_weights():
    # softmax(Qp Kp^T * scale) read out of torch's attention with V = identity
    rng = np.random.default_rng(1)
    qp, kp = rng.standard_normal((7, 16)), rng.standard_normal((9, 16))
    ours = pooled_softmax(pooled_logits(qp, kp, 0.25))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(qp)[None], torch.tensor(kp)[None], torch.eye(9, dtype=torch.float64)[None],
        scale=0.25)[0].numpy()
    np.testing.assert_allclose(ours, ref, rtol=0, atol=1e-14)
    np.testing.assert_allclose(ours.sum(-1), 1.0, rtol=0, atol=1e-14)
    # two blocks: logistic closed form
    two = pooled_softmax(np.array([[1.5, -0.5]]))
    assert abs(two[0, 0] - 1 / (1 + math.exp(-2.0))) < 1e-15


def _dirichlet_rows(n_rows, nb, seed, alpha=0.7):
    rng = np.random.default_rng(seed)
    return rng.dirichlet(np.full(nb, alpha), size=n_rows)


def _literal_ascending_cdf(p, thr):
    """The page's literal wording: sort ascending, cumulate, keep CDF > 1 - thr."""
    order = np.argsort(p, kind="stable")
    cdf = np.cumsum(p[order])
    keep = np.zeros(p.size, dtype=bool)
    keep[order] = cdf > 1 - thr
    return keep


@pytest.mark.parametrize("thr", [0.3, 0.5, 0.8, 0.95])
def test_threshold_matches_literal_ascending_cdf_away_from_band(thr):
    rows = _dirichlet_rows(400, 12, seed=int(thr * 100))
    checked = 0
    for p in rows:
        keep, E = cdf_keep_row(p, thr)
        if np.min(np.abs(E - thr)) < 1e-9 or len(set(p.tolist())) < p.size:
            continue
        assert np.array_equal(keep, _literal_ascending_cdf(p, thr))
        checked += 1
    assert checked > 300


@pytest.mark.parametrize("nb", [3, 5, 8])
def test_threshold_brute_force_over_subsets(nb):
    """Kept set = the max-mass subset among the smallest subsets holding >= thr."""
    for seed in range(40):
        p = _dirichlet_rows(1, nb, seed=seed + 17 * nb)[0]
        for thr in (0.2, 0.5, 0.8, 0.9):
            keep, E = cdf_keep_row(p, thr)
            if np.min(np.abs(E - thr)) < 1e-9:
                continue
            best = None
            for m in range(1, nb + 1):
                cands = [c for c in itertools.combinations(range(nb), m) if p[list(c)].sum() >= thr]
                if cands:
                    best = max(cands, key=lambda c: p[list(c)].sum())
                    break
            assert sorted(np.nonzero(keep)[0].tolist()) == list(best)


def test_threshold_monotone_and_minimal():
    rows = _dirichlet_rows(200, 40, seed=5, alpha=0.3)
    thrs = [0.1, 0.3, 0.5, 0.7, 0.8, 0.9, 0.99]
    for p in rows:
        prev = np.zeros(p.size, dtype=bool)
        for thr in thrs:
            keep, _ = cdf_keep_row(p, thr)
            assert np.all(prev <= keep)            # nested in thr
            mass = p[keep].sum()
            assert mass >= thr - 1e-12             # holds at least thr of the mass
            assert mass - p[keep].min() < thr + 1e-12   # dropping any kept block falls short
            prev = keep
    keep, _ = cdf_keep_row(rows[0], 1.0)
    assert keep.all()
    keep, _ = cdf_keep_row(rows[0], 1e-9)
    assert np.nonzero(keep)[0].tolist() == [int(np.argmax(rows[0]))]


def test_cdf_mask_vectorised_equals_row_loop():
    p = _dirichlet_rows(64, 33, seed=9)
    keep, E = cdf_mask(p, 0.8)
    for r in range(64):
        k1, e1 = cdf_keep_row(p[r], 0.8)
        assert np.array_equal(keep[r], k1)
        assert np.array_equal(E[r], e1)


def test_sta_closed_form_counts():
    for line in _rows("sta_counts.txt"):
        T, Hb, Wb, wt, wh, ww, total = (int(a) for a in line.split())
        m = sta_mask(T, Hb, Wb, (wt, wh, ww))
        assert int(m.sum()) == total, line
        assert np.array_equal(m, m.T)
        assert m.diagonal().all()


def test_sta_full_window_and_identity():
    assert sta_mask(3, 4, 5, (5, 7, 9)).all()
    assert np.array_equal(sta_mask(3, 4, 5, (1, 1, 1)), np.eye(60, dtype=bool))
    assert not sta_mask(3, 4, 5, (0, 0, 0)).any()
    m = sta_mask(3, 3, 3, (3, 3, 3))
    assert m[0].sum() == 8 and m[13].sum() == 27   # corner and centre of a 3x3x3 grid


def test_bit_packing_and_lists():
    mask = np.zeros((2, 40), dtype=bool)
    mask[0, [0, 5, 33]] = True
    mask[1, [31, 32, 39]] = True
    bits = pack_mask_bits(mask)
    assert bits.tolist() == [[0x21, 0x2], [0x80000000, 0x81]]
    assert np.array_equal(unpack_mask_bits(bits, 40), mask)
    sq = np.zeros((3, 3), dtype=bool)
    sq[0, 2] = sq[2, 0] = sq[1, 1] = sq[2, 2] = True
    idx, cnt = row_lists(sq)
    assert cnt.tolist() == [1, 1, 2] and idx[2, :2].tolist() == [0, 2]
    cidx, ccnt = col_lists(sq)
    assert ccnt.tolist() == [1, 1, 2] and cidx[2, :2].tolist() == [0, 2]
