"""Seeded input generators: shapes, determinism and the block-plan rule."""
import numpy as np
import torch

import workloads as W


def test_tiny_shapes_and_determinism():
    w = W.WORKLOADS["tiny"]
    a = W.make_inputs(w, seed=3)
    b = W.make_inputs(w, seed=3)
    assert a.Q.shape == (1, 2, 1024, 64) and a.Q.dtype == torch.float32
    assert a.centroids.shape == (1, 2, 32, 64)
    assert a.kv_idx.shape[:3] == (1, 2, 16) and a.kv_cnt.shape == (1, 2, 16)
    for x, y in [(a.Q, b.Q), (a.K, b.K), (a.V, b.V), (a.centroids, b.centroids), (a.kv_idx, b.kv_idx)]:
        assert torch.equal(x, y)
    c = W.make_inputs(w, seed=4)
    assert not torch.equal(a.K, c.K)


def test_head_regeneration_matches_full_tensor():
    w = W.scaled(W.WORKLOADS["wan13b"], H=3, T=3)
    full = W.make_inputs(w, seed=1)
    q, k, v, mu = W.head_qkv(w, 1, 0, 2)
    assert torch.equal(full.Q[0, 2], q) and torch.equal(full.K[0, 2], k)
    assert torch.equal(full.V[0, 2], v) and torch.equal(full.centroids[0, 2], mu)
    assert full.Q.dtype == torch.bfloat16


def test_plan_rule():
    w = W.WORKLOADS["wan14b"]
    rows = W.head_plan(w, 0, 0, 5)
    nB, Bs, frame = w.nB, w.block, w.Hs * w.Ws
    assert nB == 591 and len(rows) == nB
    for i, r in enumerate(rows):
        assert list(r) == sorted(set(r.tolist())) and r.min() >= 0 and r.max() < nB
        assert i in r
        m = min(i * Bs + Bs // 2, w.N - 1)
        for t in (m - frame, m + frame):
            if 0 <= t < w.N:
                assert t // Bs in r
        assert len(r) == 30              # round(0.05 * 591) = 30 >= mandatory 3


def test_plan_density_one_percent_keeps_mandatory():
    w = W.scaled(W.WORKLOADS["hunyuan"], T=5)      # nB = 141: round(0.01 * 141) = 1 < mandatory
    rows = W.head_plan(w, 0, 0, 0)
    frame = w.Hs * w.Ws
    for i, r in enumerate(rows):
        m = min(i * w.block + w.block // 2, w.N - 1)
        must = {i} | {t // w.block for t in (m - frame, m + frame) if 0 <= t < w.N}
        assert set(r.tolist()) == must


def test_loop_densities_in_range():
    w = W.WORKLOADS["loop"]
    ds = [W.head_density(w, 0, 0, h) for h in range(w.H)]
    assert all(0.01 <= x <= 0.20 for x in ds) and len(set(ds)) == w.H


def test_keys_cluster_around_centres():
    w = W.scaled(W.WORKLOADS["wan13b"], T=2)
    q, k, v, mu = W.head_qkv(w, 0, 0, 0)
    lab = W.head_labels(w, 0, 0, 0)
    resid = (k.float() - mu.float()[lab]).pow(2).mean().sqrt().item()
    assert abs(resid - 0.3) < 0.02


def test_drift_moves_keys_by_step():
    w = W.scaled(W.WORKLOADS["loop"], T=2)
    _, k0, _, mu0 = W.head_qkv(w, 0, 0, 0, step=0)
    _, k3, _, mu3 = W.head_qkv(w, 0, 0, 0, step=3)
    assert torch.equal(mu0, mu3)
    rms = (k3.float() - k0.float()).pow(2).mean().sqrt().item()
    assert abs(rms - 0.05 * np.sqrt(3)) < 0.01


def test_effective_flops_counts_real_keys():
    w = W.WORKLOADS["tiny"]
    x = W.make_inputs(w, seed=0)
    # N = 1024 = 16 full blocks of 64, 4 blocks kept per row, C = 32, d = 64
    assert W.effective_flops(w, x.kv_cnt, x.kv_idx) == 2 * 16 * 4 * 64 * (4 * 64 + 32) * 64
