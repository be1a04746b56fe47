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


def _unswizzle_rows(tile: np.ndarray, rows: int) -> np.ndarray:
    """An entry tile's operand (32 KB): 8-row groups of 2048 B holding panel 0 (columns 0-63) then
    panel 1 of their rows, 128 B per row, chunk k of row r stored at k ^ (r % 8) -> [rows][128]
    bf16 bits."""
    t = tile.reshape(16, 2, 8, 8, 16)[: rows // 8]          # [group][panel][row in group][chunk][byte]
    r = np.arange(8)[:, None]
    k = np.arange(8)[None, :]
    out = t[:, :, r, k ^ r]                                   # [group][panel][row][chunk][byte], logical chunks
    return np.ascontiguousarray(out.transpose(0, 2, 1, 3, 4)).reshape(rows, 256).view(np.uint16)


def _bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check_comp_tiles(inp, b, h, st, a_gpu, blocks=None):
    """The compensation tiles of the tensor-core path against the oracle's block entries and totals:
    centroid rows bit-exact, negated entry means and cluster means within one bf16 rounding of the
    fp64 values, log2 counts, zero rows and -inf bias past the entries."""
    import block_sparse_cluster_b200 as da
    w = inp.w
    dims = dims_of(w)
    if da.da_comp_tiles_bytes(dims) == 0:
        return
    N, C, bs, nB, d = w.N, w.C, w.block, w.nB, w.d
    up = lambda x: (x + 255) // 256 * 256
    BH = w.B * w.H
    bh = b * w.H + h
    comp = st.comp_tiles.cpu().numpy()
    tile_bytes = 66048
    cent_bits = inp.centroids[b, h].contiguous().view(torch.int16).numpy().view(np.uint16)
    js = range(nB) if blocks is None else blocks
    for j in js:
        c, n, S = oracle.block_entries(a_gpu, inp.V[b, h], C, N, bs, j)
        E = len(c)
        E8 = (E + 7) // 8 * 8
        t = comp[(bh * nB + j) * tile_bytes:(bh * nB + j + 1) * tile_bytes]
        kb = _unswizzle_rows(t[:32768], E8)
        vb = _unswizzle_rows(t[32768:65536], E8)
        bias = t[65536:].view(np.float32)[:E8]
        assert np.array_equal(kb[:E], cent_bits[c]), f"block {j}: entry centroid rows"
        want = -S / n[:, None]
        got = _bf16_bits_to_f64(vb[:E])
        assert (np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-6).all(), f"block {j}: entry means"
        assert np.allclose(bias[:E], np.log2(n), rtol=0, atol=1e-6), f"block {j}: entry bias"
        assert not kb[E:].any() and not vb[E:].any() and np.isneginf(bias[E:]).all(), f"block {j}: padding rows"
    cmean_off = up(BH * nB * tile_bytes)
    cbias_off = cmean_off + up(BH * C * d * 2)
    cpad = (C + 127) // 128 * 128
    nt, St = oracle.cluster_totals(a_gpu, inp.V[b, h], C)
    means = _bf16_bits_to_f64(comp[cmean_off + bh * C * d * 2:cmean_off + (bh + 1) * C * d * 2].view(np.uint16))
    means = means.reshape(C, d)
    want = np.where(nt[:, None] > 0, St / np.maximum(nt, 1)[:, None], 0.0)
    assert (np.abs(means - want) <= 2.0 ** -8 * np.abs(want) + 1e-6).all(), "cluster means"
    cb = comp[cbias_off + bh * cpad * 4:cbias_off + (bh + 1) * cpad * 4].view(np.float32)
    live = nt > 0
    assert np.allclose(cb[:C][live], np.log2(nt[live]), rtol=0, atol=1e-6), "cluster bias"
    assert np.isneginf(cb[:C][~live]).all() and np.isneginf(cb[C:]).all(), "cluster bias padding"
