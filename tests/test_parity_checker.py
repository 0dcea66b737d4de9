"""The GPU parity checker (tests/helpers.py) on the CPU: it accepts the oracle's own
answers and near-tie flips within the stated budget, and rejects planted wrong
answers (a label that is not a near tie, too many near-tie flips, a centroid
outside the tolerance), in the plain, spherical and FP8 modes."""

import numpy as np
import pytest

from oracle import emeans_oracle as O
from tests.helpers import CENTROID_REL, FP8_GAP_REL, LabelBook, assert_centroids_close


def _rows_and_centroids(seed=4, n=100, d=6, k=9):
    g = np.random.default_rng(seed)
    return g.standard_normal((n, d)), g.standard_normal((k, d))


def _farthest(x, c):
    return O.squared_distances(x, c).argmax(axis=1)


def test_label_book_accepts_the_oracles_labels():
    x, c = _rows_and_centroids()
    book = LabelBook()
    lab, best = book.compare(O.assign(x, c)[0], x, c)
    book.finish()
    assert np.array_equal(lab, O.assign(x, c)[0]) and np.allclose(best, O.assign(x, c)[1])


def test_label_book_rejects_a_label_that_is_not_a_near_tie():
    x, c = _rows_and_centroids()
    wrong = O.assign(x, c)[0].copy()
    wrong[7] = _farthest(x, c)[7]
    with pytest.raises(AssertionError):
        LabelBook().compare(wrong, x, c)


def _near_tie_rows(n, flips):
    """n rows, each almost equidistant from two centroids (a gap of 2e-6 of the
    distance); the oracle picks centroid 0 for all of them."""
    c = np.array([[1.0, 0.0], [-1.0, 0.0]])
    x = np.column_stack([np.full(n, 1e-6), np.linspace(1.0, 2.0, n)])
    lab = np.zeros(n, dtype=np.int64)
    lab[:flips] = 1
    return x, c, lab


def test_label_book_allows_one_near_tie_flip_in_a_hundred_rows():
    x, c, lab = _near_tie_rows(100, 1)
    assert np.all(O.assign(x, c)[0] == 0)
    book = LabelBook()
    accepted, _ = book.compare(lab, x, c)
    book.finish()
    assert accepted[0] == 1


def test_label_book_rejects_two_near_tie_flips_in_a_hundred_rows():
    x, c, lab = _near_tie_rows(100, 2)
    book = LabelBook()
    book.compare(lab, x, c)
    with pytest.raises(AssertionError):
        book.finish()


def test_label_book_spherical_rejects_the_lowest_similarity():
    x, c = _rows_and_centroids(seed=5)
    x, c = O.unit_rows(x), O.unit_rows(c)
    lab = O.assign_dot(x, c)[0]
    book = LabelBook(spherical=True)
    book.compare(lab, x, c)
    book.finish()
    wrong = lab.copy()
    wrong[3] = (x @ c.T).argmin(axis=1)[3]
    with pytest.raises(AssertionError):
        LabelBook(spherical=True).compare(wrong, x, c)


def test_label_book_fp8_bound():
    # E4M3 codes: a label within the accumulation bound of the best passes, one
    # beyond it fails
    x = np.array([[16.0, 0.0], [0.0, 8.0]])
    c = np.array([[16.0, 0.0], [15.0, 0.0], [-16.0, 0.0], [0.0, 8.0]])
    book = LabelBook(fp8=True)
    lab, _ = book.compare(np.array([0, 3]), x, c)
    assert lab.tolist() == [0, 3]
    # row 0: centroid 1 is 1.0 away in squared distance; the bound is
    # 2 x FP8_GAP_REL x sum|x'c'| = 2 x 2^-11 x 240, about 0.23: rejected
    assert 1.0 > 2 * FP8_GAP_REL * 240.0
    with pytest.raises(AssertionError):
        LabelBook(fp8=True).compare(np.array([1, 3]), x, c)


def test_centroid_tolerance():
    c = np.random.default_rng(6).standard_normal((10, 8))
    direction = np.ones(8) / np.sqrt(8)
    ok = c.copy()
    ok[2] += 0.5 * CENTROID_REL * np.linalg.norm(c[2]) * direction
    assert_centroids_close(ok, c)
    bad = c.copy()
    bad[2] += 2.0 * CENTROID_REL * np.linalg.norm(c[2]) * direction
    with pytest.raises(AssertionError):
        assert_centroids_close(bad, c)
