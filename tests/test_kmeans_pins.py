"""Pins for the oracle's partition training (``oracle.kmeans_assign`` and
``oracle.kmeans_update``), against numpy and the k-means invariants:
* the assignment is numpy's fp64 brute-force argmin (where the two nearest
  centroids are not within rounding of each other) and its distance matches;
* points equal to a centroid go to it at distance 0, ties to the lower index;
* the update is numpy's mean of each cluster's members (within float32
  rounding), empty clusters keep their centroid, counts are numpy's bincount;
* a Lloyd step (assign then update) never raises the total squared error.
"""
import numpy as np

import oracle


def _data(n, d, k, seed):
    rng = np.random.default_rng(seed)
    C = rng.standard_normal((k, d)).astype(np.float32)
    X = (C[rng.integers(0, k, n)] + 0.4 * rng.standard_normal((n, d))).astype(np.float32)
    return X, C


def test_assign_is_bruteforce_argmin():
    X, C = _data(2000, 24, 50, 1)
    a, dist = oracle.kmeans_assign(X, C)
    D = ((X[:, None, :].astype(np.float64) - C[None, :, :].astype(np.float64)) ** 2).sum(-1)
    srt = np.sort(D, axis=1)
    clear = srt[:, 1] - srt[:, 0] > 1e-9 * (1 + srt[:, 0])
    assert clear.mean() > 0.99
    np.testing.assert_array_equal(a[clear], np.argmin(D, axis=1)[clear])
    np.testing.assert_allclose(dist, D[np.arange(len(a)), a], rtol=1e-12)


def test_points_on_centroids_and_ties():
    rng = np.random.default_rng(2)
    C = rng.standard_normal((10, 8)).astype(np.float32)
    C[7] = C[3]                                    # duplicate centroid: ties go to 3
    X = C[[0, 3, 7, 9]]
    a, dist = oracle.kmeans_assign(X, C)
    np.testing.assert_array_equal(a, [0, 3, 3, 9])
    np.testing.assert_array_equal(dist, 0.0)


def test_update_is_member_mean_and_empty_clusters_stay():
    X, C = _data(3000, 16, 40, 3)
    a, _ = oracle.kmeans_assign(X, C)
    a = a.copy()
    a[a == 5] = 6                                  # cluster 5 empty
    Cn, counts = oracle.kmeans_update(X, a, C)
    np.testing.assert_array_equal(counts, np.bincount(a, minlength=40))
    for c in range(40):
        if counts[c] == 0:
            np.testing.assert_array_equal(Cn[c], C[c])
        else:
            want = X[a == c].astype(np.float64).mean(axis=0)
            np.testing.assert_allclose(Cn[c], want, rtol=2e-7, atol=1e-7)


def test_lloyd_step_never_raises_the_error():
    X, C = _data(4000, 12, 30, 4)
    C = C + np.float32(0.5)                        # start away from the means
    prev = None
    for _ in range(5):
        a, dist = oracle.kmeans_assign(X, C)
        err = dist.sum()
        if prev is not None:
            assert err <= prev * (1 + 1e-12)
        C, _ = oracle.kmeans_update(X, a, C)
        # the error of the old assignment under the new centroids is no higher
        after = ((X.astype(np.float64) - C[a].astype(np.float64)) ** 2).sum()
        assert after <= err * (1 + 1e-6)
        prev = err
