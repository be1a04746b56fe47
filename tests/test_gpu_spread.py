"""GPU parity of the variance-corrected cluster logits (da_cluster_spread, da_attention_spread)
against the fp64 oracle (reading R6 of the oracle), on the GPU assignment.

bf16 with d = 128 and block = 128 runs on the tensor cores (a second contraction q o q . Dh into
every cluster column's score); the other cases on the CUDA cores.

Tolerances: the second moments within 1e-5 relative (fp32 sums of squares of exactly
representable differences); attention as in the other parity tests (1e-4 fp32, 2e-2 bf16).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": W.WORKLOADS["tiny"],
    "f32_d128_ragged": W.scaled(W.WORKLOADS["tiny"], d=128, block=128, T=5, Hs=15, C=64),
    "wan13b_3f": W.scaled(W.WORKLOADS["wan13b"], H=2, T=3),
    "hunyuan_3f": W.scaled(W.WORKLOADS["hunyuan"], H=1, T=3),
    # tensor cores, ragged last block, C = 160 (a short last chunk)
    "bf16_ragged_c160": W.scaled(W.WORKLOADS["tiny"], d=128, block=128, T=5, Hs=15, C=160, dtype="bf16"),
}


def _oracle_check(inp, O, lse, assign, spread_dev, q_blocks=None):
    w = inp.w
    tol = P.ATT_TOL[w.dtype]
    for b in range(w.B):
        for h in range(w.H):
            a = assign[b, h].astype(np.int64)
            D = oracle.cluster_spread(inp.K[b, h], inp.centroids[b, h], a, w.C)
            got = spread_dev[b, h].cpu().numpy()
            assert (np.abs(got - D) <= 1e-5 * D + 1e-7).all(), f"head {b},{h}: second moments"
            Og = O[b, h].float().cpu().numpy()
            Lg = lse[b, h].cpu().numpy()
            for i in (range(w.nB) if q_blocks is None else q_blocks):
                ref, lref = oracle.attention_qblock(inp.Q[b, h], inp.K[b, h], inp.V[b, h], inp.centroids[b, h],
                                                    inp.plans[b][h][i], a, i, w.block, return_lse=True, spread=D)
                s0, s1 = i * w.block, min(w.N, (i + 1) * w.block)
                assert np.abs(Og[s0:s1] - ref).max() <= tol, f"head {b},{h} q-block {i}"
                assert np.abs(Lg[s0:s1] - lref).max() <= P.LSE_TOL[w.dtype], f"head {b},{h} q-block {i} lse"


def _run(inp, zero_spread=False):
    import block_sparse_cluster_b200 as da
    w = inp.w
    eng, _, _ = P.run_gpu(inp)
    dims = P.dims_of(w)
    Q, K, V, cent = (x.cuda() for x in (inp.Q, inp.K, inp.V, inp.centroids))
    spread = torch.empty(w.B, w.H, w.C, w.d, dtype=torch.float32, device="cuda")
    da.da_cluster_spread(dims, K, cent, eng.stats, spread)
    if zero_spread:
        spread.zero_()
    O = torch.empty_like(Q)
    lse = torch.empty(w.B, w.H, w.N, dtype=torch.float32, device="cuda")
    da.da_attention_spread(dims, Q, K, V, eng.mask, cent, eng.stats, spread, 0.0, O, lse, eng.ws)
    torch.cuda.synchronize()
    assert eng.status() == 0
    return eng, spread, O, lse


@pytest.mark.parametrize("name", list(CASES))
def test_spread_and_corrected_attention(name):
    w = CASES[name]
    inp = W.make_inputs(w, seed=11)
    eng, spread, O, lse = _run(inp)
    _oracle_check(inp, O, lse, eng.stats.assign.cpu().numpy(), spread)


def test_spread_on_the_tensor_cores_with_several_items_per_cta():
    """Wan2.1-14B frame shape, 4 heads x 4 frames: 452 items over at most 148 CTAs, so every CTA
    carries the key ring, Q2 and the value ring across items; sampled q-blocks of every head."""
    w = W.scaled(W.WORKLOADS["wan14b"], H=4, T=4)
    inp = W.make_inputs(w, seed=14)
    eng, spread, O, lse = _run(inp)
    assert w.B * w.H * w.nB > 2 * 148
    _oracle_check(inp, O, lse, eng.stats.assign.cpu().numpy(), spread, q_blocks=[0, 1, w.nB // 2, w.nB - 1])


def test_zero_spread_equals_the_plain_tensor_core_path():
    """With D = 0 the second contraction adds exact zeros to every score, so the corrected mode
    (two key tiles per chunk step, Q2, a two-slot value ring) must reproduce da_attention's bits."""
    w = CASES["wan13b_3f"]
    inp = W.make_inputs(w, seed=15)
    _, O_plain, lse_plain = P.run_gpu(inp)
    _, _, O, lse = _run(inp, zero_spread=True)
    assert torch.equal(O, O_plain)
    assert torch.equal(lse, lse_plain)


def test_zero_spread_equals_the_plain_cuda_core_path():
    """fp32 runs the CUDA-core attention either way; a zero correction leaves only the chunking
    of the clusters (16 instead of 32 per pass) different."""
    w = CASES["f32_d128_ragged"]
    inp = W.make_inputs(w, seed=12)
    _, O_plain, _ = P.run_gpu(inp)
    _, _, O, _ = _run(inp, zero_spread=True)
    assert (O - O_plain).abs().max().item() <= 1e-5


def test_spread_is_bitwise_repeatable():
    import block_sparse_cluster_b200 as da
    w = CASES["wan13b_3f"]
    inp = W.make_inputs(w, seed=13)
    eng, s1, _, _ = _run(inp)
    s2 = torch.empty_like(s1)
    da.da_cluster_spread(P.dims_of(w), inp.K.cuda(), inp.centroids.cuda(), eng.stats, s2)
    torch.cuda.synchronize()
    assert torch.equal(s1, s2)
