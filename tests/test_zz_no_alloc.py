"""da_reassign_noalloc: Reassign Cache for callers that cannot allocate device memory.

Such callers (a runtime whose device memory is planned once at start-up, an application whose
pool owns all device memory, a path where an allocation would synchronise the device) pass only
inputs and outputs; the library keeps the scratch in its own fixed device array.  The results
must match da_reassign's, which runs the same kernels with a caller workspace, on two calls in a
row (the array keeps the previous call's contents).
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
from tests import parity as P


def test_noalloc_rejects_dims_beyond_its_scratch():
    import block_sparse_cluster_b200 as da
    dims = da.Dims(B=1, H=512, N=4096, d=128, C=1024, block=128)       # B*H*C = 524288 > 262144
    s = da._Stats(*([0x1000] * 9))
    code = da._lib.da_reassign_noalloc(ctypes.byref(dims.c()), 0x1000, 0x1000, 0x1000, ctypes.byref(s), None)
    assert code == da.STATUS_NAMES.index("DA_ERR_WORKSPACE")


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["wan13b_3f", "tiny"])
def test_noalloc_matches_workspace_path_twice(name):
    import block_sparse_cluster_b200 as da
    w = {"wan13b_3f": W.scaled(W.WORKLOADS["wan13b"], H=2, T=3), "tiny": W.WORKLOADS["tiny"]}[name]
    inp = W.make_inputs(w, seed=21)
    dims = P.dims_of(w)
    K, V, cent = (x.cuda() for x in (inp.K, inp.V, inp.centroids))
    ref = da.ClusterStats.empty(dims)
    ws = da.workspace(dims)
    da.da_reassign(dims, K, V, cent, ref, ws)
    assert da.da_device_status(ws) == 0
    for _ in range(2):
        got = da.ClusterStats.empty(dims)
        da.da_reassign_noalloc(dims, K, V, cent, got)
        assert da.da_noalloc_device_status() == 0     # synchronises; no device-side problem
        assert torch.equal(got.assign, ref.assign)
        nB = dims.nB
        for f in ("blk_hist", "seg_idx", "seg_n", "n_tot"):
            assert torch.equal(getattr(got, f), getattr(ref, f)), f
        n = ref.seg_n.long()
        valid = torch.arange(dims.block, device="cuda")[None, None, None, :] < n[..., None]
        assert torch.equal(got.seg_c[valid], ref.seg_c[valid]) and torch.equal(got.seg_cnt[valid], ref.seg_cnt[valid])
        # value sums: the tolerance of the parity tests (|dS| <= 1e-5 * sum|v| + 1e-6; here both
        # sides are the same fp32 kernels)
        vs_ref = ref.seg_vsum[valid]
        assert (got.seg_vsum[valid] - vs_ref).abs().max().item() <= 1e-5 * vs_ref.abs().max().item() + 1e-6
        assert (got.S_tot - ref.S_tot).abs().max().item() <= 1e-5 * ref.S_tot.abs().max().item() + 1e-6
