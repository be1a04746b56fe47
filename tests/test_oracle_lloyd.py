"""Pins of the oracle's Lloyd iteration (the clustering the pages build on) that do not call its
formulas again: a hand-worked example, scikit-learn's Lloyd k-means, the fixed point of means,
an empty cluster, and the monotone decrease of the k-means objective."""
import numpy as np
import pytest

import oracle


def test_hand_example_one_step():
    # points 0, 1, 10, 11 on a line, centroids at 0 and 10: the means are 0.5 and 10.5
    K = np.array([[0.0], [1.0], [10.0], [11.0]])
    c, a = oracle.lloyd_step(K, np.array([[0.0], [10.0]]))
    assert a.tolist() == [0, 0, 1, 1]
    assert np.allclose(c, [[0.5], [10.5]])


def test_matches_scikit_learn_lloyd():
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(3)
    centres = rng.normal(size=(6, 8)) * 4
    K = centres[rng.integers(0, 6, size=400)] + rng.normal(size=(400, 8))
    init = K[:6].copy()
    ours, a = oracle.kmeans(K, init, 5)
    ref = KMeans(n_clusters=6, init=init, n_init=1, max_iter=5, tol=0.0, algorithm="lloyd").fit(K)
    # scikit-learn reports the centres after its last update and the labels of the last E-step
    assert np.allclose(ours, ref.cluster_centers_, atol=1e-9)


def test_means_are_a_fixed_point():
    rng = np.random.default_rng(5)
    K = rng.normal(size=(300, 4))
    c, _ = oracle.kmeans(K, K[:5], 60)          # converged
    c2, _ = oracle.lloyd_step(K, c)
    assert np.allclose(c2, c)


def test_empty_cluster_keeps_its_centroid():
    K = np.array([[0.0, 0.0], [0.1, 0.0], [0.0, 0.1]])
    far = np.array([[0.0, 0.0], [100.0, 100.0]])
    c, a = oracle.lloyd_step(K, far)
    assert (a == 0).all()
    assert np.array_equal(c[1], far[1])
    assert np.allclose(c[0], K.mean(axis=0))


def test_objective_never_increases():
    rng = np.random.default_rng(9)
    K = rng.normal(size=(500, 16))
    c = K[rng.choice(500, 12, replace=False)].copy()
    prev = np.inf
    for _ in range(8):
        a, _ = oracle.reassign(K, c)
        cur = oracle.sse(K, c, a)
        assert cur <= prev + 1e-9
        prev = cur
        c, _ = oracle.lloyd_step(K, c)


def test_objective_hand_value():
    # keys (0, 0) and (3, 4) on one centroid at the origin: 0 + 3^2 + 4^2 = 25
    assert oracle.sse(np.array([[0.0, 0.0], [3.0, 4.0]]), np.array([[0.0, 0.0]]), np.array([0, 0])) == 25.0
