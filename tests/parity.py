"""Helpers of the GPU parity tests: run the CUDA path through the C ABI, then compare its
outputs with the fp64 oracle on the same seeded inputs.

Tolerances
----------
* assignment: identical, except keys whose oracle top-2 relative distance gap is below 1e-4;
* counts, histograms, entry lists, entry indices: bit-exact given the GPU assignment;
* value sums: |dS| <= 1e-5 * sum|v| + 1e-6 per element (fp32 sums of at most N values);
* attention (against the oracle run on the GPU assignment): max-abs <= 2e-2 for bf16 inputs
  (P and the cluster means are rounded to bf16 for the tensor cores, fp32 accumulation),
  <= 1e-4 for the fp32 path.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads as W

GAP_TOL = 1e-4
ATT_TOL = {"bf16": 2e-2, "f32": 1e-4}
LSE_TOL = {"bf16": 2e-2, "f32": 1e-4}


def dims_of(w: W.Workload):
    import block_sparse_cluster_b200 as da
    return da.Dims(w.B, w.H, w.N, w.d, w.C, w.block, w.torch_dtype)


def run_gpu(inp: W.Inputs, scale: float = 0.0, prepare: bool = True, kv_idx=None, kv_cnt=None):
    """One reassign + attention step through the C ABI; returns (engine, O, lse) on the GPU."""
    import block_sparse_cluster_b200 as da
    w = inp.w
    dims = dims_of(w)
    eng = da.DecoupledAttention(dims)
    Q, K, V, cent = (x.cuda() for x in (inp.Q, inp.K, inp.V, inp.centroids))
    ki = (inp.kv_idx if kv_idx is None else kv_idx).cuda()
    kc = (inp.kv_cnt if kv_cnt is None else kv_cnt).cuda()
    if prepare:
        eng.prepare(ki, kc)
    else:
        eng.mask = da.BlockMask(ki, kc)
    O = torch.empty_like(Q)
    lse = torch.empty(w.B, w.H, w.N, dtype=torch.float32, device="cuda")
    eng.step(Q, K, V, cent, O, lse, scale=scale)
    torch.cuda.synchronize()
    return eng, O, lse


def check_assignment(inp, b, h, a_gpu, keys=None):
    """Returns the number of near-tie flips; asserts every other key matches the oracle."""
    K = inp.K[b, h]
    cent = inp.centroids[b, h]
    idx = np.arange(inp.w.N) if keys is None else np.asarray(keys)
    a_ref, gap = oracle.reassign(K[idx], cent)
    diff = a_ref != a_gpu[idx]
    bad = diff & (gap >= GAP_TOL)
    assert not bad.any(), f"head {b},{h}: {bad.sum()} assignments differ beyond near-ties, first key {idx[bad][0]}"
    return int(diff.sum())


def check_block_stats(inp, b, h, st, a_gpu, blocks=None):
    """Per-block histogram row, entry index row, entry list and value sums, from the GPU assignment."""
    w = inp.w
    N, C, bs = w.N, w.C, w.block
    Vh = inp.V[b, h]
    Vf = Vh.float().numpy().astype(np.float64)
    hist = st.blk_hist[b, h].cpu().numpy()
    sidx = st.seg_idx[b, h].cpu().numpy()
    segn = st.seg_n[b, h].cpu().numpy()
    segc = st.seg_c[b, h].cpu().numpy()
    segcnt = st.seg_cnt[b, h].cpu().numpy()
    vsum = st.seg_vsum[b, h].cpu().numpy()
    js = range(w.nB) if blocks is None else blocks
    for j in js:
        c, n, S = oracle.block_entries(a_gpu, Vh, C, N, bs, j)
        E = len(c)
        assert segn[j] == E, f"block {j}: seg_n {segn[j]} != {E}"
        assert np.array_equal(segc[j, :E], c) and np.array_equal(segcnt[j, :E], n), f"block {j} entries"
        row = np.zeros(C, dtype=np.int64)
        row[c] = n
        assert np.array_equal(hist[j], row), f"block {j} histogram"
        irow = np.full(C, 255, dtype=np.int64)
        irow[c] = np.arange(E)
        assert np.array_equal(sidx[j].astype(np.int64), irow), f"block {j} entry index"
        s0, s1 = j * bs, min(N, (j + 1) * bs)
        absv = np.zeros((E, w.d))
        aj = a_gpu[s0:s1]
        for e, cc in enumerate(c):
            absv[e] = np.abs(Vf[s0:s1][aj == cc]).sum(axis=0)
        assert (np.abs(vsum[j, :E] - S) <= 1e-5 * absv + 1e-6).all(), f"block {j} value sums"


def check_totals(inp, b, h, st, a_gpu):
    w = inp.w
    n, S = oracle.cluster_totals(a_gpu, inp.V[b, h], w.C)
    assert np.array_equal(st.n_tot[b, h].cpu().numpy(), n)
    Vf = inp.V[b, h].float().numpy().astype(np.float64)
    absS = np.zeros_like(S)
    np.add.at(absS, a_gpu, np.abs(Vf))
    got = st.S_tot[b, h].cpu().numpy()
    assert (np.abs(got - S) <= 1e-5 * absS + 1e-6).all()


def check_attention(inp, b, h, O, lse, a_gpu, q_blocks=None, scale=None):
    """Max-abs error of O (and lse) against the oracle on the GPU assignment; asserts the tolerance."""
    w = inp.w
    tol = ATT_TOL[w.dtype]
    qb = range(w.nB) if q_blocks is None else q_blocks
    Og = O[b, h].float().cpu().numpy()
    Lg = lse[b, h].cpu().numpy()
    worst = 0.0
    for i in qb:
        ref, lref = oracle.attention_qblock(inp.Q[b, h], inp.K[b, h], inp.V[b, h], inp.centroids[b, h],
                                            inp.plans[b][h][i], a_gpu, i, w.block, scale, return_lse=True)
        s0, s1 = i * w.block, min(w.N, (i + 1) * w.block)
        err = np.abs(Og[s0:s1] - ref).max()
        lerr = np.abs(Lg[s0:s1] - lref).max()
        assert err <= tol, f"head {b},{h} q-block {i}: max-abs {err:.3e} > {tol}"
        assert lerr <= LSE_TOL[w.dtype], f"head {b},{h} q-block {i}: lse error {lerr:.3e}"
        worst = max(worst, float(err))
    return worst

