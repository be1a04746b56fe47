"""GPU parity of inclusion-probability reweighting (da_attention_sip, the fused tensor-core kernel
with the weights as bias rows) against the fp64 oracle (reading R7), on seeded inclusion
probabilities; attention within the bf16 path's tolerance (2e-2)."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

CASES = {
    "wan13b_3f": W.scaled(W.WORKLOADS["wan13b"], H=2, T=3),
    "wan14b_2f": W.scaled(W.WORKLOADS["wan14b"], H=2, T=2),
    "hunyuan_3f": W.scaled(W.WORKLOADS["hunyuan"], H=1, T=3),
}


def _run(w, inp, incl, kv_idx=None, kv_cnt=None):
    import block_sparse_cluster_b200 as da
    dims = P.dims_of(w)
    ws = da.workspace(dims)
    Q, K, V = (x.cuda() for x in (inp.Q, inp.K, inp.V))
    ki = (inp.kv_idx if kv_idx is None else kv_idx).cuda()
    kc = (inp.kv_cnt if kv_cnt is None else kv_cnt).cuda()
    mask = da.BlockMask(ki, kc)
    O = torch.empty_like(Q)
    lse = torch.empty(w.B, w.H, w.N, dtype=torch.float32, device="cuda")
    da.da_attention_sip(dims, Q, K, V, mask, incl.cuda(), 0.0, O, lse, ws)
    torch.cuda.synchronize()
    assert da.da_device_status(ws) == 0
    return O, lse


def _check(w, inp, incl, O, lse, rows, q_blocks=None):
    tol = P.ATT_TOL[w.dtype]
    for b in range(w.B):
        for h in range(w.H):
            Og = O[b, h].float().cpu().numpy()
            Lg = lse[b, h].cpu().numpy()
            for i in (range(w.nB) if q_blocks is None else q_blocks):
                sel = [int(j) for j in rows[b][h][i]]
                pis = [float(incl[b, h, i, s]) for s in range(len(sel))]
                keep = [k for k, p in enumerate(pis) if p > 0]
                ref, lref = oracle.attention_sip_qblock(inp.Q[b, h], inp.K[b, h], inp.V[b, h],
                                                        [sel[k] for k in keep], [pis[k] for k in keep], i, w.block,
                                                        return_lse=True)
                s0, s1 = i * w.block, min(w.N, (i + 1) * w.block)
                assert np.abs(Og[s0:s1] - ref).max() <= tol, f"head {b},{h} q-block {i}"
                fin = np.isfinite(lref)
                assert np.array_equal(np.isfinite(Lg[s0:s1]), fin)
                assert np.abs(Lg[s0:s1][fin] - lref[fin]).max(initial=0.0) <= P.LSE_TOL[w.dtype]


@pytest.mark.parametrize("name", list(CASES))
def test_reweighted_attention(name):
    w = CASES[name]
    inp = W.make_inputs(w, seed=21)
    incl = W.inclusion_probabilities(w, 21, inp.kv_idx.shape[-1])
    O, lse = _run(w, inp, incl)
    _check(w, inp, incl, O, lse, inp.plans)


def test_empty_rows_and_excluded_slots():
    """Rows without selected blocks give O = 0 and LSE = -inf; a slot with pi = 0 drops its block."""
    w = CASES["wan13b_3f"]
    inp = W.make_inputs(w, seed=22)
    incl = W.inclusion_probabilities(w, 22, inp.kv_idx.shape[-1])
    kv_cnt = inp.kv_cnt.clone()
    kv_cnt[:, :, ::5] = 0                        # every fifth q-block: no blocks
    incl[:, :, 1::7, 0] = 0.0                     # some slots never included
    rows = [[[r if kv_cnt[b, h, i] > 0 else r[:0] for i, r in enumerate(inp.plans[b][h])]
             for h in range(w.H)] for b in range(w.B)]
    O, lse = _run(w, inp, incl, kv_cnt=kv_cnt)
    _check(w, inp, incl, O, lse, rows)
    assert torch.all(O[:, :, : w.block] == 0)


def test_certain_inclusion_of_every_block_is_dense_attention():
    w = CASES["wan13b_3f"]
    inp = W.make_inputs(w, seed=23)
    nB = w.nB
    kv_idx = torch.arange(nB, dtype=torch.int32).repeat(w.B, w.H, nB, 1).contiguous()
    kv_cnt = torch.full((w.B, w.H, nB), nB, dtype=torch.int32)
    incl = torch.ones(w.B, w.H, nB, nB, dtype=torch.float32)
    O, _ = _run(w, inp, incl, kv_idx=kv_idx, kv_cnt=kv_cnt)
    for h in range(w.H):
        q, k, v = (x[0, h].float()[None, None] for x in (inp.Q, inp.K, inp.V))
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v)[0, 0]
        assert (O[0, h].float().cpu() - ref).abs().max().item() <= 2e-2
