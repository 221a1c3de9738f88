"""Pins for the oracle's expert histogram / offsets / stable permutation (S3),
against numpy's bincount and Python's stable sort."""
import numpy as np

import oracle


def _check(idx, E):
    counts, offsets, perm, inv = oracle.permute(idx, E)
    flat = idx.reshape(-1)
    valid = (flat >= 0) & (flat < E)
    assert np.array_equal(counts, np.bincount(flat[valid], minlength=E))
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    order = sorted((i for i in range(flat.size) if valid[i]), key=lambda i: (flat[i], i))
    n = len(order)
    assert np.array_equal(perm[:n], np.array(order, np.int32))
    assert np.all(perm[n:] == -1)
    assert np.all(inv[~valid] == -1)
    assert np.array_equal(perm[inv[valid]], np.nonzero(valid)[0])


def test_uniform():
    rng = np.random.default_rng(0)
    _check(rng.integers(0, 64, (300, 6)).astype(np.int32), 64)


def test_skewed_with_empty_experts_and_invalid_ids():
    rng = np.random.default_rng(1)
    idx = (rng.zipf(1.5, (500, 8)) - 1).astype(np.int32)
    idx[::7, 3] = -1
    _check(np.minimum(idx, 300).astype(np.int32), 256)


def test_duplicates_and_empty():
    _check(np.array([[3, 3, 3], [0, 3, 1]], np.int32), 4)
    _check(np.zeros((0, 4), np.int32), 8)
