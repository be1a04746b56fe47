"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test checks the oracle against a library routine, a closed form, an
invariant the method must satisfy, brute force, or a hand-worked fixture.
None of them needs a GPU.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.spatial.distance import cdist

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _rand_case(seed, N=200, d=8, C=7, block=32, spread=1.0):
    rng = np.random.default_rng(seed)
    cent = rng.normal(size=(C, d)) * spread
    lab = rng.integers(0, C, size=N)
    K = cent[lab] + 0.4 * rng.normal(size=(N, d))
    V = rng.normal(size=(N, d))
    Q = rng.normal(size=(N, d))
    return Q, K, V, cent


def _dense_sdpa(Q, K, V, scale):
    """Textbook softmax attention from the library routine (fp64 on CPU)."""
    q = torch.from_numpy(np.asarray(Q, np.float64))[None, None]
    k = torch.from_numpy(np.asarray(K, np.float64))[None, None]
    v = torch.from_numpy(np.asarray(V, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=scale)[0, 0].numpy()


def _random_plan(rng, nB, p):
    return [sorted(int(j) for j in np.nonzero(rng.random(nB) < p)[0]) for _ in range(nB)]


# ---------------------------------------------------------------------------
# reassignment

def test_reassign_hand_fixture():
    g = _golden()["reassign_2d"]
    a, gap = oracle.reassign(np.array(g["keys"], float), np.array(g["centroids"], float))
    assert a.tolist() == g["assign"]
    np.testing.assert_allclose(gap, g["gap"], rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_reassign_matches_library_distance(seed):
    _, K, _, cent = _rand_case(seed, N=300, d=16, C=11)
    a, _ = oracle.reassign(K, cent)
    want = cdist(K, cent, "sqeuclidean").argmin(axis=1)
    assert np.array_equal(a, want)


def test_reassign_ties_go_to_lowest_index():
    cent = np.array([[1.0, 0.0], [-1.0, 0.0], [0.0, 1.0], [0.0, -1.0]])
    K = np.array([[0.0, 0.0], [0.0, 0.0], [5.0, 5.0]])
    a, gap = oracle.reassign(K, cent)
    assert a.tolist() == [0, 0, 0]      # (5,5): distances 41, 61, 41, 61 -> tie 0 vs 2
    assert gap[0] == 0.0


def test_reassign_keys_on_centroids_map_to_themselves():
    rng = np.random.default_rng(3)
    K = rng.normal(size=(64, 8))
    pick = rng.choice(64, size=9, replace=False)
    a, _ = oracle.reassign(K, K[pick])
    assert np.array_equal(a[pick], np.arange(9))


def test_reassign_permutation_and_translation():
    _, K, _, cent = _rand_case(5, N=256, d=12, C=9)
    a, gap = oracle.reassign(K, cent)
    perm = np.random.default_rng(1).permutation(9)
    a2, _ = oracle.reassign(K, cent[perm])
    ok = gap > 1e-9
    assert np.array_equal(perm[a2[ok]], a[ok])
    delta = np.random.default_rng(2).normal(size=12) * 3
    a3, _ = oracle.reassign(K + delta, cent + delta)
    assert np.array_equal(a3[ok], a[ok])


def test_reassign_single_centroid():
    _, K, _, cent = _rand_case(6, C=1)
    a, gap = oracle.reassign(K, cent[:1])
    assert (a == 0).all() and np.isinf(gap).all()


# ---------------------------------------------------------------------------
# block statistics

def test_stats_hand_fixture():
    g = _golden()["reassign_2d"]
    a = np.array(g["assign"])
    V = np.array(g["values"], float)
    N, C, bs = len(a), len(g["centroids"]), g["block"]
    assert oracle.block_histogram(a, C, N, bs).tolist() == g["hist"]
    for j, ent in enumerate(g["block_entries"]):
        c, n, S = oracle.block_entries(a, V, C, N, bs, j)
        assert c.tolist() == ent["clusters"] and n.tolist() == ent["counts"]
        np.testing.assert_array_equal(S, np.array(ent["sums"], float))
    n, S = oracle.cluster_totals(a, V, C)
    assert n.tolist() == g["n_tot"]
    np.testing.assert_array_equal(S, np.array(g["S_tot"], float))


@pytest.mark.parametrize("N,block", [(256, 64), (250, 64), (1, 64), (130, 128)])
def test_histogram_against_library_and_invariants(N, block):
    rng = np.random.default_rng(N)
    C = 13
    a = rng.integers(0, C, size=N)
    hist = oracle.block_histogram(a, C, N, block)
    nB = -(-N // block)
    blk = np.arange(N) // block
    want, _, _ = np.histogram2d(blk, a, bins=[np.arange(nB + 1) - 0.5, np.arange(C + 1) - 0.5])
    assert np.array_equal(hist, want.astype(np.int64))
    sizes = [min(block, N - j * block) for j in range(nB)]
    assert hist.sum(axis=1).tolist() == sizes          # every key of a block counted once
    n, _ = oracle.cluster_totals(a, np.zeros((N, 2)), C)
    assert np.array_equal(hist.sum(axis=0), n) and n.sum() == N


def test_block_sums_against_one_hot_matmul():
    rng = np.random.default_rng(11)
    N, C, d, block = 300, 9, 5, 64
    a = rng.integers(0, C, size=N)
    V = rng.normal(size=(N, d))
    n, S = oracle.cluster_totals(a, V, C)
    onehot = np.eye(C)[a]                        # [N, C]
    np.testing.assert_allclose(S, onehot.T @ V, atol=1e-12)
    np.testing.assert_allclose(S.sum(axis=0), V.sum(axis=0), atol=1e-12)
    acc = np.zeros((C, d))
    for j in range(-(-N // block)):
        c, cnt, sums = oracle.block_entries(a, V, C, N, block, j)
        assert list(c) == sorted(set(c)) and cnt.sum() == min(block, N - j * block)
        sl = slice(j * block, min(N, (j + 1) * block))
        np.testing.assert_allclose(sums, (np.eye(C)[a[sl]].T @ V[sl])[c], atol=1e-12)
        acc[c] += sums
    np.testing.assert_allclose(acc, S, atol=1e-12)


def test_block_stats_invariant_under_permutation_within_block():
    rng = np.random.default_rng(12)
    N, C, d, block = 256, 6, 4, 64
    a = rng.integers(0, C, size=N)
    V = rng.normal(size=(N, d))
    perm = np.concatenate([j * block + rng.permutation(block) for j in range(N // block)])
    for j in range(N // block):
        c1, n1, s1 = oracle.block_entries(a, V, C, N, block, j)
        c2, n2, s2 = oracle.block_entries(a[perm], V[perm], C, N, block, j)
        assert np.array_equal(c1, c2) and np.array_equal(n1, n2)
        np.testing.assert_allclose(s1, s2, atol=1e-12)


# ---------------------------------------------------------------------------
# attention

@pytest.mark.parametrize("name", ["attention_1d_a", "attention_1d_b"])
def test_attention_hand_fixture(name):
    g = _golden()[name]
    K = np.array(g["keys"], float)
    cent = np.array(g["centroids"], float)
    a, _ = oracle.reassign(K, cent)
    assert a.tolist() == g["assign"]
    out = oracle.attention(np.array(g["queries"], float), K, np.array(g["values"], float), cent,
                           g["plan"], a, g["block"], scale=g["scale"])
    np.testing.assert_allclose(out, np.array(g["expected"]), rtol=0, atol=1e-12)


def test_full_plan_is_dense_attention():
    Q, K, V, cent = _rand_case(21, N=250, d=16, C=5, block=64)
    block, nB = 64, 4
    a, _ = oracle.reassign(K, cent)
    plan = [list(range(nB))] * nB
    s = 1 / 4
    out = oracle.attention(Q, K, V, cent, plan, a, block, scale=s)
    np.testing.assert_allclose(out, _dense_sdpa(Q, K, V, s), atol=1e-12)


@pytest.mark.parametrize("p", [0.0, 0.3, 1.0])
def test_keys_on_centroids_compensation_is_exact(p):
    """When every key sits exactly on its centroid, each cluster term equals
    the sum of its compensated keys, so the result is dense attention for any plan."""
    rng = np.random.default_rng(22)
    N, d, C, block = 300, 8, 12, 32
    cent = rng.normal(size=(C, d))
    a = rng.integers(0, C, size=N)
    K = cent[a]
    V = rng.normal(size=(N, d))
    Q = rng.normal(size=(N, d))
    nB = -(-N // block)
    plan = _random_plan(rng, nB, p)
    got_a, _ = oracle.reassign(K, cent)
    assert np.array_equal(got_a, a)
    out = oracle.attention(Q, K, V, cent, plan, a, block, scale=0.7)
    np.testing.assert_allclose(out, _dense_sdpa(Q, K, V, 0.7), atol=1e-12)


def test_singleton_clusters_are_dense_attention():
    Q, K, V, _ = _rand_case(23, N=96, d=8, C=3)
    block = 16
    a, _ = oracle.reassign(K, K)
    assert np.array_equal(a, np.arange(96))
    plan = _random_plan(np.random.default_rng(4), 6, 0.4)
    out = oracle.attention(Q, K, V, K, plan, a, block)
    np.testing.assert_allclose(out, _dense_sdpa(Q, K, V, 1 / math.sqrt(8)), atol=1e-12)


def test_empty_plan_is_centroid_attention():
    Q, K, V, cent = _rand_case(24, N=200, d=8, C=6)
    block = 32
    a, _ = oracle.reassign(K, cent)
    s = 1 / math.sqrt(8)
    out = oracle.attention(Q, K, V, cent, [[]] * 7, a, block)
    # closed form: sum_c n_c e^{s q.c} vbar_c / sum_c n_c e^{s q.c}
    n = np.array([(a == c).sum() for c in range(6)], float)
    vbar = np.stack([V[a == c].mean(axis=0) if n[c] else np.zeros(8) for c in range(6)])
    w = n[None, :] * np.exp(s * Q @ cent.T)
    np.testing.assert_allclose(out, (w @ vbar) / w.sum(axis=1, keepdims=True), atol=1e-12)


def test_one_cluster_empty_plan_is_mean_value():
    Q, K, V, cent = _rand_case(25, N=150, d=8, C=1)
    a = np.zeros(150, dtype=np.int64)
    out = oracle.attention(Q, K, V, cent, [[]] * 5, a, 32)
    np.testing.assert_allclose(out, np.broadcast_to(V.mean(axis=0), out.shape), atol=1e-12)


def test_zero_queries_give_mean_value_for_any_plan():
    """q = 0 makes every logit equal, so each key counts once: O = mean(V)."""
    _, K, V, cent = _rand_case(26, N=220, d=8, C=9)
    block = 32
    a, _ = oracle.reassign(K, cent)
    plan = _random_plan(np.random.default_rng(9), 7, 0.35)
    out = oracle.attention(np.zeros((220, 8)), K, V, cent, plan, a, block)
    np.testing.assert_allclose(out, np.broadcast_to(V.mean(axis=0), out.shape), atol=1e-12)


def test_per_key_correction_form():
    """All keys by cluster, then each selected key's cluster term replaced by the key itself."""
    Q, K, V, cent = _rand_case(27, N=256, d=8, C=10, spread=1.5)
    block, nB = 32, 8
    rng = np.random.default_rng(5)
    a, _ = oracle.reassign(K, cent)
    plan = _random_plan(rng, nB, 0.3)
    s = 0.4
    out = oracle.attention(Q, K, V, cent, plan, a, block, scale=s)
    n = np.zeros(10)
    S = np.zeros((10, 8))
    np.add.at(n, a, 1.0)
    np.add.at(S, a, V)
    for i in range(nB):
        sel = np.concatenate([np.arange(j * block, (j + 1) * block) for j in plan[i]] + [np.zeros(0, int)])
        q = Q[i * block:(i + 1) * block]
        ex = np.exp(s * q @ K[sel].T)
        ec = np.exp(s * q @ cent.T)
        corr = ex - ec[:, a[sel]]
        num = corr @ V[sel] + ec @ S
        den = corr.sum(axis=1) + ec @ n
        np.testing.assert_allclose(out[i * block:(i + 1) * block], num / den[:, None], atol=1e-10)


def test_translation_and_key_permutation_invariance():
    Q, K, V, cent = _rand_case(28, N=192, d=8, C=6)
    block = 32
    plan = _random_plan(np.random.default_rng(6), 6, 0.4)
    a, _ = oracle.reassign(K, cent)
    out = oracle.attention(Q, K, V, cent, plan, a, block)
    delta = np.random.default_rng(7).normal(size=8)
    a2, _ = oracle.reassign(K + delta, cent + delta)
    assert np.array_equal(a, a2)
    np.testing.assert_allclose(oracle.attention(Q, K + delta, V, cent + delta, plan, a2, block), out, atol=1e-10)
    perm = np.concatenate([j * block + np.random.default_rng(j).permutation(block) for j in range(6)])
    np.testing.assert_allclose(oracle.attention(Q, K[perm], V[perm], cent, plan, a[perm], block), out, atol=1e-10)


def test_brute_force_tiny():
    """Plain loops over the definition on a tiny case: every compensated key
    contributes its cluster's centroid logit and its cluster's mean value."""
    Q, K, V, cent = _rand_case(29, N=20, d=3, C=3)
    block = 4
    a, _ = oracle.reassign(K, cent)
    plan = [[0], [1, 3], [], [0, 1, 2, 3, 4], [4]]
    out = oracle.attention(Q, K, V, cent, plan, a, block, scale=0.9)
    for i in range(5):
        sel = set()
        for j in plan[i]:
            sel.update(range(j * 4, j * 4 + 4))
        for r in range(i * 4, i * 4 + 4):
            num = np.zeros(3)
            den = 0.0
            for k in range(20):
                if k in sel:
                    w = math.exp(0.9 * float(Q[r] @ K[k]))
                    num += w * V[k]
                else:
                    c = a[k]
                    members = [u for u in range(20) if u not in sel and a[u] == c]
                    mean = sum(V[u] for u in members) / len(members)
                    w = math.exp(0.9 * float(Q[r] @ cent[c]))
                    num += w * mean
                den += w
            np.testing.assert_allclose(out[r], num / den, atol=1e-12)


def test_lse_matches_log_denominator():
    Q, K, V, cent = _rand_case(30, N=64, d=4, C=3)
    a, _ = oracle.reassign(K, cent)
    out, lse = oracle.attention_qblock(Q, K, V, cent, [0, 1], a, 0, 32, scale=1.0, return_lse=True)
    # full plan on 64 keys -> dense: lse = log sum_k e^{q.k}
    np.testing.assert_allclose(lse, np.log(np.exp(Q[:32] @ K.T).sum(axis=1)), atol=1e-12)
