"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the same seeded inputs."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

# Small cases the oracle finishes in seconds; each spans several tiles and ends in a ragged block.
SMALL = {
    # fp32, d=64, block 64, 16 full blocks, C=32 (the tiny workload itself)
    "tiny": W.WORKLOADS["tiny"],
    # fp32, d=128, block 128: N = 5*15*16 = 1200 -> 10 blocks, last one 48 keys
    "f32_d128_ragged": W.scaled(W.WORKLOADS["tiny"], d=128, block=128, T=5, Hs=15, C=64),
    # bf16 Wan2.1-1.3B shape cut to 3 frames: N = 4680, 37 blocks, last one 72 keys, C=256
    "wan13b_3f": W.scaled(W.WORKLOADS["wan13b"], H=2, T=3),
    # bf16 Wan2.1-14B shape cut to 2 frames: N = 7200, 57 blocks, last one 32 keys, C=512
    "wan14b_2f": W.scaled(W.WORKLOADS["wan14b"], H=2, T=2),
    # bf16 HunyuanVideo shape cut to 3 frames: N = 10800, 85 blocks, last one 48 keys, C=1024
    "hunyuan_3f": W.scaled(W.WORKLOADS["hunyuan"], H=1, T=3),
    # two batch entries: (batch, head) slices are flattened in every kernel
    "wan13b_b2": W.scaled(W.WORKLOADS["wan13b"], B=2, H=2, T=2),
    # C not a multiple of 128 on the tensor-core path: one partial chunk (C < 128), a partial last
    # chunk of 32 centroids, and of 32 again after three full ones (reassign, statistics, attention)
    "c96": W.scaled(W.WORKLOADS["wan14b"], H=2, T=2, C=96, cells=(2, 6, 8)),
    "c160": W.scaled(W.WORKLOADS["wan14b"], H=1, T=2, C=160, cells=(2, 8, 10)),
    "c416": W.scaled(W.WORKLOADS["wan14b"], H=1, T=2, C=416, cells=(2, 13, 16)),
    # bf16 shapes of the CUDA-core path: d = 64 with block 64, and d = 128 with block 64
    "bf16_d64": W.scaled(W.WORKLOADS["tiny"], dtype="bf16"),
    "bf16_block64": W.scaled(W.WORKLOADS["tiny"], d=128, block=64, T=5, Hs=15, C=64, dtype="bf16"),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_case_full_parity(name):
    w = SMALL[name]
    inp = W.make_inputs(w, seed=7)
    eng, O, lse = P.run_gpu(inp)
    assert eng.status() == 0
    st = eng.stats
    assign = st.assign.cpu().numpy()
    for b in range(w.B):
        for h in range(w.H):
            a = assign[b, h].astype(np.int64)
            P.check_assignment(inp, b, h, a)
            P.check_block_stats(inp, b, h, st, a)
            P.check_totals(inp, b, h, st, a)
            P.check_attention(inp, b, h, O, lse, a)


def test_drifted_keys_with_the_step0_plan():
    """Reassign-cache loop: step 3 of drifting keys, the plan prepared once from step 0 and the
    cached step-0 centroids; full parity on the drifted step."""
    w = W.scaled(W.WORKLOADS["loop"], H=2, T=3)
    inp0 = W.make_inputs(w, seed=31, step=0)
    inp = W.make_inputs(w, seed=31, step=3)
    assert torch.equal(inp.kv_idx, inp0.kv_idx) and not torch.equal(inp.K, inp0.K)
    eng, O, lse = P.run_gpu(inp)
    assert eng.status() == 0
    assign = eng.stats.assign.cpu().numpy()
    for h in range(w.H):
        a = assign[0, h].astype(np.int64)
        P.check_assignment(inp, 0, h, a)
        P.check_block_stats(inp, 0, h, eng.stats, a)
        P.check_totals(inp, 0, h, eng.stats, a)
        P.check_attention(inp, 0, h, O, lse, a)


def _edge_plan(w, rows):
    kv_idx, kv_cnt = W.pack_plan([[rows] * w.H] * w.B, w.nB)
    return kv_idx, kv_cnt


@pytest.mark.parametrize("name", ["tiny", "wan13b_3f"])
def test_empty_full_and_offset_rows(name):
    """Rows with no block (pure compensation), every block (dense), and plans without the own block."""
    w = SMALL[name]
    inp = W.make_inputs(w, seed=8)
    nB = w.nB
    rows = []
    for i in range(nB):
        if i % 3 == 0:
            rows.append(np.zeros(0, np.int32))
        elif i % 3 == 1:
            rows.append(np.arange(nB, dtype=np.int32))
        else:
            rows.append(np.array(sorted({(i + 5) % nB, (i + 9) % nB}), np.int32))
    inp.plans = [[rows] * w.H] * w.B
    inp.kv_idx, inp.kv_cnt = _edge_plan(w, rows)
    eng, O, lse = P.run_gpu(inp)
    assert eng.status() == 0
    a = eng.stats.assign.cpu().numpy()
    for h in range(w.H):
        P.check_attention(inp, 0, h, O, lse, a[0, h].astype(np.int64))


def test_full_plan_equals_dense_attention():
    w = SMALL["wan13b_3f"]
    inp = W.make_inputs(w, seed=9)
    rows = [np.arange(w.nB, dtype=np.int32)] * w.nB
    inp.kv_idx, inp.kv_cnt = _edge_plan(w, rows)
    _, O, _ = P.run_gpu(inp)
    q, k, v = (x.cuda().float() for x in (inp.Q, inp.K, inp.V))
    dense = torch.nn.functional.scaled_dot_product_attention(q, k, v)
    assert (O.float() - dense).abs().max().item() <= P.ATT_TOL["bf16"]


def test_singleton_clusters_equal_dense_attention():
    """C = N and the centroids are the keys: every cluster holds one key, so the result is dense."""
    w = W.scaled(W.WORKLOADS["tiny"], T=1, Hs=16, Ws=16, C=256, block=64)
    inp = W.make_inputs(w, seed=10)
    inp.centroids = inp.K.clone()
    eng, O, _ = P.run_gpu(inp)
    a = eng.stats.assign.cpu().numpy()
    assert np.array_equal(a[0, 0], np.arange(256))
    q, k, v = (x.double() for x in (inp.Q, inp.K, inp.V))
    dense = torch.nn.functional.scaled_dot_product_attention(q, k, v)
    assert (O.cpu().double() - dense).abs().max().item() <= P.ATT_TOL["f32"]


def test_explicit_scale_and_no_lse():
    import block_sparse_cluster_b200 as da
    w = SMALL["tiny"]
    inp = W.make_inputs(w, seed=11)
    dims = P.dims_of(w)
    eng = da.DecoupledAttention(dims)
    Q, K, V, cent = (x.cuda() for x in (inp.Q, inp.K, inp.V, inp.centroids))
    eng.prepare(inp.kv_idx.cuda(), inp.kv_cnt.cuda())
    O = torch.empty_like(Q)
    eng.step(Q, K, V, cent, O, None, scale=0.05)
    assert eng.status() == 0
    a = eng.stats.assign.cpu().numpy()
    for h in range(w.H):
        ref = oracle.attention(inp.Q[0, h], inp.K[0, h], inp.V[0, h], inp.centroids[0, h], inp.plans[0][h],
                               a[0, h], w.block, scale=0.05)
        assert np.abs(O[0, h].cpu().numpy() - ref).max() <= P.ATT_TOL["f32"]


def test_short_sequence_single_partial_block():
    w = W.scaled(W.WORKLOADS["tiny"], T=1, Hs=10, Ws=10, C=32)      # N = 100: blocks of 64 and 36
    inp = W.make_inputs(w, seed=12)
    eng, O, lse = P.run_gpu(inp)
    a = eng.stats.assign.cpu().numpy()
    for h in range(w.H):
        ah = a[0, h].astype(np.int64)
        P.check_assignment(inp, 0, h, ah)
        P.check_block_stats(inp, 0, h, eng.stats, ah)
        P.check_attention(inp, 0, h, O, lse, ah)


def test_repeat_calls_are_bitwise_identical():
    w = SMALL["wan13b_3f"]
    inp = W.make_inputs(w, seed=13)
    eng, O1, l1 = P.run_gpu(inp)
    s1 = {k: getattr(eng.stats, k).clone() for k in ("assign", "blk_hist", "seg_vsum", "S_tot", "n_tot")}
    Q, K, V, cent = (x.cuda() for x in (inp.Q, inp.K, inp.V, inp.centroids))
    O2 = torch.empty_like(O1)
    l2 = torch.empty_like(l1)
    eng.step(Q, K, V, cent, O2, l2)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(l1, l2)
    for k, v in s1.items():
        assert torch.equal(v, getattr(eng.stats, k)), k


def test_clusters_mostly_inside_the_selected_blocks():
    """Every q-block selects all blocks but three, and 64 clusters hold about 112 keys each, so a
    cluster keeps only a few of its keys outside the selection (n_c / n^U_c about 40 on average,
    up to 128, and n^U_c = 0 for many clusters): the complement sums S_c - sum_j S_{c,j} are small
    differences of large fp32 terms, and their means must still match the oracle within the bf16
    tolerance."""
    w = W.scaled(W.WORKLOADS["wan14b"], H=2, T=2, C=64, cells=(2, 4, 8))
    inp = W.make_inputs(w, seed=19)
    nB = w.nB
    rows = [np.array([j for j in range(nB) if j not in {(i + 7) % nB, (i + 19) % nB, (i + 31) % nB}], np.int32)
            for i in range(nB)]
    inp.plans = [[rows] * w.H] * w.B
    inp.kv_idx, inp.kv_cnt = _edge_plan(w, rows)
    eng, O, lse = P.run_gpu(inp)
    assert eng.status() == 0
    a = eng.stats.assign.cpu().numpy()
    n_tot = eng.stats.n_tot.cpu().numpy()
    ratios = []
    for h in range(w.H):
        ah = a[0, h].astype(np.int64)
        for i in range(0, nB, 7):
            out = [j for j in range(nB) if j not in set(rows[i].tolist())]
            n_u = np.bincount(np.concatenate([ah[j * w.block:(j + 1) * w.block] for j in out]), minlength=w.C)
            live = n_u > 0
            ratios.append(float((n_tot[0, h][live] / n_u[live]).mean()))
        P.check_attention(inp, 0, h, O, lse, ah)
    assert np.mean(ratios) > 20


def test_split_calls_equal_da_attention():
    """da_compensation followed by da_attention_prebuilt is da_attention, bit for bit."""
    import block_sparse_cluster_b200 as da
    w = SMALL["wan14b_2f"]
    inp = W.make_inputs(w, seed=17)
    eng, O1, l1 = P.run_gpu(inp)
    Q, K, V, cent = (x.cuda() for x in (inp.Q, inp.K, inp.V, inp.centroids))
    O2 = torch.empty_like(O1)
    l2 = torch.empty_like(l1)
    da.da_compensation(eng.dims, eng.mask, eng.stats, eng.ws)
    da.da_attention_prebuilt(eng.dims, Q, K, V, eng.mask, cent, eng.stats, 0.0, O2, l2, eng.ws)
    torch.cuda.synchronize()
    assert eng.status() == 0
    assert torch.equal(O1, O2) and torch.equal(l1, l2)


def test_malformed_plan_is_reported_without_fault():
    import block_sparse_cluster_b200 as da
    w = SMALL["tiny"]
    inp = W.make_inputs(w, seed=14)
    ki = inp.kv_idx.clone()
    kc = inp.kv_cnt.clone()
    ki[0, 0, 3, 0] = 10_000          # out of range
    ki[0, 1, 5, :2] = torch.tensor([7, 2], dtype=torch.int32)   # unsorted
    eng, O, _ = P.run_gpu(inp, kv_idx=ki, kv_cnt=kc)
    assert eng.status() == da.STATUS_NAMES.index("DA_ERR_DEVICE_INDEX")
    assert eng.status() == 0           # cleared by the read
    kc2 = inp.kv_cnt.clone()
    kc2[0, 0, 0] = 99                  # more than max_sel
    eng, _, _ = P.run_gpu(inp, kv_cnt=kc2)
    assert eng.status() == da.STATUS_NAMES.index("DA_ERR_DEVICE_INDEX")
    # the same plan without da_mask_prepare: da_attention validates it itself
    eng, _, _ = P.run_gpu(inp, kv_idx=ki, kv_cnt=kc, prepare=False)
    assert eng.status() == da.STATUS_NAMES.index("DA_ERR_DEVICE_INDEX")


def test_logits_far_above_the_first_steps_max_are_reported():
    """The tensor-core kernel exponentiates every step of a row against the row max of its
    q-block's first step.  Queries 30 e_1 against a first block of zero keys (logits 0) and a second
    block of keys 30 e_1 (about 115 in log2 units) exceed that reference by more than 2^96: the
    call reports DA_ERR_RANGE through the status word, and an ordinary step after it reports
    nothing."""
    import dataclasses
    import block_sparse_cluster_b200 as da
    w = W.scaled(W.WORKLOADS["wan13b"], H=1, T=1)      # bf16, d = block = 128, 13 blocks
    inp = W.make_inputs(w, seed=16)
    Q = torch.zeros_like(inp.Q)
    Q[..., 0] = 30.0
    K = torch.zeros_like(inp.K)
    K[0, 0, w.block:2 * w.block, 0] = 30.0
    far = dataclasses.replace(inp, Q=Q, K=K)
    ki = torch.empty(w.B, w.H, w.nB, 2, dtype=torch.int32)
    ki[..., 0], ki[..., 1] = 0, 1
    kc = torch.full_like(inp.kv_cnt, 2)
    eng, _, _ = P.run_gpu(far, kv_idx=ki, kv_cnt=kc)
    assert eng.status() == da.STATUS_NAMES.index("DA_ERR_RANGE")
    eng, _, _ = P.run_gpu(inp)
    assert eng.status() == 0


def test_plans_longer_than_one_staging_tile():
    """Rows with more selected blocks than the compensation pre-pass stages at a time (256): every
    block but every fifth (270), every block (338, dense), and all but the first 10 and last 20
    (308).  A 12-frame cut of the Wan2.1-14B shape: N = 43200, 338 blocks, the last one 64 keys."""
    w = W.scaled(W.WORKLOADS["wan14b"], H=1, T=12)
    assert w.nB == 338
    inp = W.make_inputs(w, seed=15)
    nB = w.nB
    kinds = [np.array([j for j in range(nB) if j % 5 != 0], np.int32),
             np.arange(nB, dtype=np.int32),
             np.arange(10, nB - 20, dtype=np.int32)]
    rows = [kinds[i % 3] for i in range(nB)]
    inp.plans = [[rows] * w.H] * w.B
    inp.kv_idx, inp.kv_cnt = _edge_plan(w, rows)
    eng, O, lse = P.run_gpu(inp)
    assert eng.status() == 0
    a = eng.stats.assign.cpu().numpy()[0, 0].astype(np.int64)
    P.check_attention(inp, 0, 0, O, lse, a, q_blocks=[0, 1, 2, 3, 4, 5, 166, 167, 168, nB - 3, nB - 2, nB - 1])
    dense_rows = [i for i in range(nB) if i % 3 == 1]
    q, k, v = (x[0, 0].cuda().float() for x in (inp.Q, inp.K, inp.V))
    dense = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None])[0]
    for i in dense_rows:
        s0, s1 = i * w.block, min(w.N, (i + 1) * w.block)
        assert (O[0, 0, s0:s1].float() - dense[s0:s1]).abs().max().item() <= P.ATT_TOL["bf16"]


# ---------------------------------------------------------------------------
# full-size workloads, in the launch configuration the benchmark times: sampled outputs

FULL = ["wan13b", "wan14b", "hunyuan"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled(name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=0)
    eng, O, lse = P.run_gpu(inp)
    assert eng.status() == 0
    st = eng.stats
    rng = np.random.default_rng(1)
    # properties over every head
    sizes = torch.full((w.nB,), w.block, dtype=torch.int64, device="cuda")
    sizes[-1] = w.N - (w.nB - 1) * w.block
    assert torch.equal(st.blk_hist.sum(-1).long(), sizes.expand(w.B, w.H, -1))
    assert torch.equal(st.blk_hist.sum(2), st.n_tot)
    assert (st.n_tot.sum(-1) == w.N).all()
    assert torch.isfinite(O.float()).all() and torch.isfinite(lse).all()
    assign = st.assign.cpu().numpy()
    heads = sorted(set([0, w.H - 1] + rng.choice(w.H, size=2, replace=False).tolist()))
    for h in heads:
        a = assign[0, h].astype(np.int64)
        keys = np.concatenate([rng.choice(w.N, size=512, replace=False), np.arange(w.N - 16, w.N)])
        P.check_assignment(inp, 0, h, a, keys=keys)
        blocks = sorted(set(rng.choice(w.nB, size=12, replace=False).tolist() + [w.nB - 1]))
        P.check_block_stats(inp, 0, h, st, a, blocks=blocks)
        P.check_totals(inp, 0, h, st, a)
        qbs = sorted(set(rng.choice(w.nB, size=6, replace=False).tolist() + [0, w.nB - 1]))
        P.check_attention(inp, 0, h, O, lse, a, q_blocks=qbs)
