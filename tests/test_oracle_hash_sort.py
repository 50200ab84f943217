"""Pins for the oracle's hash and sort (CPU only).

The hash h(x) = argmax([xR; -xR]) and "sorted by bucket" come from
"Reformer: The Efficient Transformer" (research.elamur.ai summary page),
Summary and Key points ("LSH attention").
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import lsh_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_hash_hand_worked_examples():
    with open(os.path.join(GOLDEN, "hash_worked_examples.json")) as f:
        ex = json.load(f)["examples"]
    for e in ex:
        x = np.array([e["x"]], dtype=np.float64)
        R = np.array(e["R"], dtype=np.float64)
        b, gap = orc.hash_round(x, R)
        assert int(b[0]) == e["bucket"], e


def test_hash_identity_rotation_closed_form():
    # d = n_b/2 and R = I: u = [x, -x], so the bucket is the index of the
    # largest |x_k|, moved to the second half when that entry is negative.
    rng = np.random.default_rng(1)
    x = rng.standard_normal((500, 16))
    b, _ = orc.hash_round(x, np.eye(16))
    k = np.abs(x).argmax(axis=1)
    expect = np.where(x[np.arange(500), k] > 0, k, k + 16)
    np.testing.assert_array_equal(b, expect)


def test_hash_negation_swaps_halves():
    # -x swaps the two halves of [xR; -xR]: h(-x) = (h(x) + n_b/2) mod n_b,
    # wherever the top two entries are not (near-)tied.
    rng = np.random.default_rng(2)
    for n_half in (1, 16, 96, 512):
        x = rng.standard_normal((400, 64))
        R = rng.standard_normal((64, n_half))
        b, gap = orc.hash_round(x, R)
        bn, _ = orc.hash_round(-x, R)
        ok = gap >= 1e-5
        assert ok.mean() > 0.95
        np.testing.assert_array_equal(bn[ok], (b[ok] + n_half) % (2 * n_half))


def test_hash_positive_scaling_invariant():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((300, 64))
    R = rng.standard_normal((64, 32))
    b, gap = orc.hash_round(x, R)
    b2, _ = orc.hash_round(4.0 * x, R)   # power of two: exact in binary
    np.testing.assert_array_equal(b, b2)


def _exact_bucket(x_row, R):
    """Brute force in exact rational arithmetic: no rounding anywhere."""
    xs = [Fraction(float(t)) for t in x_row]
    d, nh = R.shape
    s = [sum(xs[c] * Fraction(float(R[c, k])) for c in range(d)) for k in range(nh)]
    u = s + [-t for t in s]
    best = max(u)
    idx = u.index(best)                 # lowest index on ties
    rest = sorted(u, reverse=True)
    second = rest[1]
    gap = (best - second) / best if best > 0 else Fraction(0)
    return idx, float(gap)


def test_hash_exact_rational_brute_force():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((60, 8))
    R = rng.standard_normal((8, 6))
    b, gap = orc.hash_round(x, R)
    for i in range(x.shape[0]):
        idx, g = _exact_bucket(x[i], R)
        if g >= 1e-9:
            assert b[i] == idx
        assert abs(gap[i] - g) < 1e-9


def test_hash_buckets_shapes_and_rounds():
    rng = np.random.default_rng(5)
    qk = rng.standard_normal((2, 3, 50, 8))
    R = rng.standard_normal((4, 8, 5))
    bk, gap = orc.hash_buckets(qk, R, row_block=16)
    assert bk.shape == (2, 3, 4, 50)
    for b in range(2):
        for h in range(3):
            for r in range(4):
                bb, _ = orc.hash_round(qk[b, h], R[r])
                np.testing.assert_array_equal(bk[b, h, r], bb)
    assert bk.min() >= 0 and bk.max() < 10


def _counting_sort(keys, n_buckets):
    """Independent stable counting sort (plain Python)."""
    count = [0] * n_buckets
    for k in keys:
        count[k] += 1
    start, acc = [0] * n_buckets, 0
    for b in range(n_buckets):
        start[b], acc = acc, acc + count[b]
    out = [0] * len(keys)
    for pos, k in enumerate(keys):
        out[start[k]] = pos
        start[k] += 1
    return out


def test_sort_is_stable_permutation():
    rng = np.random.default_rng(6)
    bucket = rng.integers(0, 12, size=(2, 2, 3, 257))
    perm = orc.sort_positions(bucket)
    for idx in np.ndindex(*bucket.shape[:-1]):
        p = perm[idx]
        assert sorted(p.tolist()) == list(range(257))
        kb = bucket[idx][p]
        assert np.all(np.diff(kb) >= 0)
        same = np.diff(kb) == 0
        assert np.all(np.diff(p)[same] > 0)
        assert p.tolist() == _counting_sort(bucket[idx].tolist(), 12)


def test_window_slots():
    assert list(orc.window_slots(0, 4)) == [0, 1, 2, 3]
    assert list(orc.window_slots(5, 4)) == list(range(0, 8))
    assert list(orc.window_slots(11, 4)) == list(range(4, 12))
    assert list(orc.window_slots(7, 8)) == list(range(0, 8))
