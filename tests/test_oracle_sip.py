"""Pins of the oracle's inclusion-probability reweighting (AB-Attention abstract: blocks are
sampled and "reweighted by inverse inclusion probability, so that one pass estimates dense
attention").  Reading: each selected block j carries its inclusion probability pi_j; numerator
and denominator of the softmax sum (1 / pi_j) times the block's exact terms.  Pinned by:

* certain inclusion of every block (pi = 1, full plan): textbook dense softmax attention;
* unbiasedness of both sums (Horvitz-Thompson): under independent inclusion with probabilities
  pi_j, the expectation of exp(LSE) over all 2^nB subsets equals the dense exp(LSE), and the
  expectation of O * exp(LSE) equals the dense numerator (exact enumeration, tiny case);
* equal weights cancel: with one pi for all selected blocks the output is plain softmax
  attention over the selected keys.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle


def _dense(Q, K, V, s):
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None, None], torch.from_numpy(K)[None, None], torch.from_numpy(V)[None, None],
        scale=s)[0, 0].numpy()
    lg = s * (Q @ K.T)
    m = lg.max(axis=1)
    return out, m + np.log(np.exp(lg - m[:, None]).sum(axis=1))


def test_certain_inclusion_of_every_block_is_dense_attention():
    rng = np.random.default_rng(0)
    N, d, block = 96, 16, 32
    Q, K, V = (rng.normal(size=(N, d)) for _ in range(3))
    s = 1.0 / math.sqrt(d)
    ref, lref = _dense(Q, K, V, s)
    for i in range(3):
        out, lse = oracle.attention_sip_qblock(Q, K, V, [0, 1, 2], [1.0, 1.0, 1.0], i, block, return_lse=True)
        np.testing.assert_allclose(out, ref[32 * i:32 * (i + 1)], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lse, lref[32 * i:32 * (i + 1)], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed", [1, 2])
def test_sums_are_unbiased_over_all_subsets(seed):
    rng = np.random.default_rng(seed)
    nB, block, d = 4, 4, 6
    N = nB * block
    Q, K, V = (rng.normal(size=(N, d)) for _ in range(3))
    s = 1.0 / math.sqrt(d)
    pi = rng.uniform(0.2, 1.0, size=nB)
    _, lref = _dense(Q, K, V, s)
    ref, _ = _dense(Q, K, V, s)
    q0, q1 = 0, block
    e_den = np.zeros(block)
    e_num = np.zeros((block, d))
    for mask in itertools.product([0, 1], repeat=nB):
        prob = np.prod([pi[j] if mask[j] else 1.0 - pi[j] for j in range(nB)])
        sel = [j for j in range(nB) if mask[j]]
        out, lse = oracle.attention_sip_qblock(Q, K, V, sel, [pi[j] for j in sel], 0, block, return_lse=True)
        den = np.exp(lse)                     # -inf -> 0 for the empty subset
        e_den += prob * den
        e_num += prob * out * den[:, None]
    np.testing.assert_allclose(e_den, np.exp(lref[q0:q1]), rtol=1e-10)
    np.testing.assert_allclose(e_num, ref[q0:q1] * np.exp(lref[q0:q1])[:, None], rtol=1e-9, atol=1e-12)


def test_equal_weights_cancel():
    rng = np.random.default_rng(3)
    N, d, block = 80, 8, 16
    Q, K, V = (rng.normal(size=(N, d)) for _ in range(3))
    s = 1.0 / math.sqrt(d)
    sel = [0, 2, 4]
    keys = np.concatenate([np.arange(16 * j, 16 * j + 16) for j in sel])
    ref, _ = _dense(Q[16:32], K[keys], V[keys], s)
    out = oracle.attention_sip_qblock(Q, K, V, sel, [0.3, 0.3, 0.3], 1, block)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_empty_row_is_zero_with_minus_infinite_lse():
    rng = np.random.default_rng(4)
    Q, K, V = (rng.normal(size=(32, 4)) for _ in range(3))
    out, lse = oracle.attention_sip_qblock(Q, K, V, [], [], 0, 16, return_lse=True)
    assert np.all(out == 0) and np.all(np.isneginf(lse))
