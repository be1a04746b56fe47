"""Pins of the oracle's variance correction (ESTRA abstract: "a variance-based correction
further refines the attention weights of the cluster representatives").

Reading (the pages print no formula): the keys of cluster c are Gaussian about the
representative cbar_c with a diagonal second moment D_c, so the cluster logit gains
s^2/2 sum_t q_t^2 D_{c,t}.  These tests pin that reading against closed forms, without calling
the oracle's formulas again:

* keys offset from their centroid by a fixed vector b have D = b * b (about the representative,
  not about the keys' own mean, which would give 0);
* keys cbar +- delta e_t (symmetric along the axes): the exact log-sum-exp of the cluster is
  s q.cbar + ln(2 sum_t cosh(s q_t delta)), and the corrected logit must match it to O(delta^4)
  while the uncorrected one is off by O(delta^2);
* a zero second moment leaves the attention unchanged;
* moving keys and centroids by one vector leaves D unchanged.
"""
import math

import numpy as np
import pytest

import oracle


def test_offset_keys_give_the_squared_offset():
    rng = np.random.default_rng(1)
    d, C = 6, 3
    cent = rng.normal(size=(C, d))
    b = rng.normal(size=(C, d))
    reps = 5
    K = np.repeat(cent + b, reps, axis=0)                # every key of cluster c at cbar_c + b_c
    a = np.repeat(np.arange(C), reps)
    D = oracle.cluster_spread(K, cent, a, C)
    np.testing.assert_allclose(D, b * b, rtol=1e-12, atol=1e-14)


def test_empty_cluster_has_zero_spread():
    rng = np.random.default_rng(2)
    K = rng.normal(size=(10, 4))
    cent = rng.normal(size=(3, 4))
    a = np.array([0] * 5 + [2] * 5)
    D = oracle.cluster_spread(K, cent, a, 3)
    assert np.all(D[1] == 0.0)


@pytest.mark.parametrize("seed", [0, 1])
def test_corrected_logit_matches_the_cluster_log_sum_exp_to_fourth_order(seed):
    rng = np.random.default_rng(seed)
    d = 8
    cbar = rng.normal(size=(1, d))
    q = rng.normal(size=(1, d))
    s = 1.0 / math.sqrt(d)
    errs_c, errs_u = [], []
    for delta in (0.2, 0.1, 0.05):
        K = np.concatenate([cbar + delta * np.eye(d), cbar - delta * np.eye(d)])   # 2d keys
        a = np.zeros(2 * d, dtype=np.int64)
        D = oracle.cluster_spread(K, cbar, a, 1)
        V = rng.normal(size=(2 * d, d))
        exact = float(s * (q @ cbar.T)[0, 0] + math.log(2.0 * np.cosh(s * q[0] * delta).sum()))
        # one q-block holding only the query; the keys form a second block that is not selected,
        # so the single cluster column is the whole softmax and LSE is its logit
        Qa = np.concatenate([q, np.zeros((2 * d - 1, d))])
        Qfull = np.concatenate([Qa, np.zeros((2 * d, d))])
        Kfull = np.concatenate([np.zeros((2 * d, d)), K])
        Vfull = np.concatenate([np.zeros((2 * d, d)), V])
        afull = np.concatenate([np.zeros(2 * d, dtype=np.int64), a])
        # the first block's keys sit on the centroid, so they add zero second moment but count
        Dfull = oracle.cluster_spread(np.concatenate([np.repeat(cbar, 2 * d, axis=0), K]), cbar, afull, 1)
        _, lse_c = oracle.attention_qblock(Qfull, np.concatenate([np.repeat(cbar, 2 * d, axis=0), K]), Vfull, cbar,
                                           [], afull, 0, 2 * d, scale=s, return_lse=True, spread=Dfull)
        _, lse_u = oracle.attention_qblock(Qfull, np.concatenate([np.repeat(cbar, 2 * d, axis=0), K]), Vfull, cbar,
                                           [], afull, 0, 2 * d, scale=s, return_lse=True)
        # the 2d extra keys on the centroid add ln 2 (twice the keys) and halve the mean spread
        exact_full = math.log(math.exp(exact) + 2 * d * math.exp(float(s * (q @ cbar.T)[0, 0])))
        errs_c.append(abs(lse_c[0] - exact_full))
        errs_u.append(abs(lse_u[0] - exact_full))
        np.testing.assert_allclose(D, (delta ** 2 / d) * np.ones((1, d)), rtol=1e-12)
    # corrected: fourth order (halving delta divides the error by about 16); uncorrected: second
    assert errs_c[1] < errs_c[0] / 10 and errs_c[2] < errs_c[1] / 10
    assert errs_u[1] > errs_u[0] / 5
    assert all(c < u / 20 for c, u in zip(errs_c, errs_u))


def test_zero_spread_leaves_attention_unchanged():
    rng = np.random.default_rng(3)
    N, d, C, block = 48, 8, 4, 16
    Q = rng.normal(size=(N, d))
    cent = rng.normal(size=(C, d))
    a = rng.integers(0, C, size=N)
    K = cent[a]                                           # every key on its centroid
    V = rng.normal(size=(N, d))
    plan = [[0], [1, 2], []]
    D = oracle.cluster_spread(K, cent, a, C)
    assert np.all(D == 0.0)
    o1 = oracle.attention(Q, K, V, cent, plan, a, block)
    o2 = oracle.attention(Q, K, V, cent, plan, a, block, spread=D)
    np.testing.assert_array_equal(o1, o2)


def test_spread_is_translation_invariant():
    rng = np.random.default_rng(4)
    N, d, C = 60, 5, 4
    K = rng.normal(size=(N, d))
    cent = rng.normal(size=(C, d))
    a = rng.integers(0, C, size=N)
    shift = rng.normal(size=(1, d)) * 3.0
    D1 = oracle.cluster_spread(K, cent, a, C)
    D2 = oracle.cluster_spread(K + shift, cent + shift, a, C)
    np.testing.assert_allclose(D1, D2, rtol=1e-9, atol=1e-12)
