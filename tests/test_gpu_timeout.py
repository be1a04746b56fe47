"""Bounded device waits: a wait that never completes ends in DA_ERR_TIMEOUT, not a hang.

The test build of the library (libda_fault.so: the same sources with DA_FAULT_INJECT) withholds
one plain software arrival in the fused attention kernel: the second softmax warpgroup of CTA 0
does not signal that its probabilities of step 5 are written.  Nothing else changes, so no copy or
product is left in flight.  The product issuer waiting for that arrival gives up after the
library's wait limit (2 s), records DA_ERR_TIMEOUT in the workspace status word and makes the
CTA's other roles leave (the producers drain their copies first, each drain wait bounded too).
The GPU context stays usable: the regular library then runs a step on the same process and
matches the oracle.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


def _fault_lib():
    import block_sparse_cluster_b200 as da
    path = os.path.join(os.path.dirname(da.LIB_PATH), "libda_fault.so")
    lib = ctypes.CDLL(path)
    for name in da.EXPORTS:
        getattr(lib, name).restype = getattr(da._lib, name).restype
        getattr(lib, name).argtypes = getattr(da._lib, name).argtypes
    return lib


def test_withheld_arrival_times_out_and_the_context_survives():
    import block_sparse_cluster_b200 as da
    w = W.scaled(W.WORKLOADS["wan14b"], H=2, T=2)
    inp = W.make_inputs(w, seed=41)
    dims = P.dims_of(w)
    eng = da.DecoupledAttention(dims)
    Q, K, V, cent = (x.cuda() for x in (inp.Q, inp.K, inp.V, inp.centroids))
    eng.prepare(inp.kv_idx.cuda(), inp.kv_cnt.cuda())
    O = torch.empty_like(Q)
    da.da_reassign(dims, K, V, cent, eng.stats, eng.ws)
    assert eng.status() == 0

    fault = _fault_lib()
    code = fault.da_attention(ctypes.byref(dims.c()), Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                              ctypes.byref(eng.mask.c()), cent.data_ptr(), ctypes.byref(eng.stats.c()), 0.0,
                              O.data_ptr(), None, eng.ws.data_ptr(), eng.ws.numel(),
                              torch.cuda.current_stream().cuda_stream)
    assert code == 0                              # the launch itself is fine
    assert eng.status() == da.STATUS_NAMES.index("DA_ERR_TIMEOUT")
    assert eng.status() == 0                      # cleared by the read

    # the same process, the regular library: a full step that matches the oracle
    lse = torch.empty(w.B, w.H, w.N, dtype=torch.float32, device="cuda")
    eng.step(Q, K, V, cent, O, lse)
    torch.cuda.synchronize()
    assert eng.status() == 0
    a = eng.stats.assign.cpu().numpy()
    for h in range(w.H):
        P.check_attention(inp, 0, h, O, lse, a[0, h].astype(np.int64), q_blocks=[0, 1, w.nB // 2, w.nB - 1])
