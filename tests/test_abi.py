"""The C ABI: every symbol include/da.h declares is exported, and the host-side argument
checks return their documented codes before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest
import torch

import block_sparse_cluster_b200 as da

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^DA_API\s+[\w\s\*]+?\b(da_\w+)\s*\(", src, flags=re.M)
    return names


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert set(names) >= {"da_reassign", "da_attention", "da_mask_prepare", "da_device_status"}
    lib = ctypes.CDLL(da.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(names) == sorted(set(names))
    assert set(da.EXPORTS) == set(names)


def test_version_and_strings():
    assert da.da_version() == 103
    for code in range(11):
        assert da.da_status_string(code) and da.da_status_string(code) != "unknown status"


def _dims(**kw):
    base = dict(B=1, H=12, N=32760, d=128, C=256, block=128, dtype=torch.bfloat16)
    base.update(kw)
    return da.Dims(**base)


def test_workspace_bytes():
    assert da.da_workspace_bytes(_dims()) > 12 * 256 * 4
    assert da.da_schedule_bytes(_dims()) == 12 * 256 * 4
    assert da.da_workspace_bytes(_dims(d=96)) == 0
    assert da.da_workspace_bytes(_dims(C=100)) == 0
    assert da.da_workspace_bytes(_dims(N=0)) == 0


def _call_reassign(dims, K=0x1000, V=0x1000, C=0x1000, stats=None, ws=0x1000, ws_bytes=1 << 30):
    s = stats if stats is not None else da._Stats(*([0x1000] * 9))
    return da._lib.da_reassign(ctypes.byref(dims.c()), K, V, C, ctypes.byref(s), ws, ws_bytes, None)


def _call_attention(dims, mask=None, O=0x1000, lse=None, ws_bytes=1 << 30):
    m = mask if mask is not None else da._Mask(0x1000, 0x1000, 4, None)
    s = da._Stats(*([0x1000] * 9))
    return da._lib.da_attention(ctypes.byref(dims.c()), 0x1000, 0x1000, 0x1000, ctypes.byref(m), 0x1000,
                                ctypes.byref(s), 0.0, O, lse, 0x1000, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=torch.float16), 3), (dict(d=96), 5), (dict(block=256), 5), (dict(C=48), 5), (dict(C=2048), 5),
    (dict(N=-1), 1), (dict(H=0), 1),
])
def test_reassign_rejects_dims(kw, code):
    assert _call_reassign(_dims(**kw)) == code


def test_reassign_rejects_pointers_and_workspace():
    d = _dims()
    assert _call_reassign(d, K=None) == 1
    assert _call_reassign(d, V=0x1008) == 4
    bad = da._Stats(*([0x1000] * 8 + [None]))
    assert _call_reassign(d, stats=bad) == 1
    bad = da._Stats(*([0x1000] * 7 + [0x1004, 0x1000]))
    assert _call_reassign(d, stats=bad) == 4
    assert _call_reassign(d, ws=None) == 1
    assert _call_reassign(d, ws_bytes=16) == 9


def test_attention_rejects_arguments():
    d = _dims()
    assert _call_attention(d, O=None) == 1
    assert _call_attention(d, O=0x1002) == 4
    assert _call_attention(d, lse=0x1001) == 4
    assert _call_attention(d, mask=da._Mask(0x1000, 0x1000, 0, None)) == 2
    assert _call_attention(d, mask=da._Mask(None, 0x1000, 4, None)) == 1
    assert _call_attention(d, mask=da._Mask(0x1000, 0x1000, 4, 0x1004)) == 4
    assert _call_attention(d, ws_bytes=0) == 9


def test_mask_prepare_rejects_small_schedule():
    d = _dims()
    m = da._Mask(0x1000, 0x1000, 4, None)
    assert da._lib.da_mask_prepare(ctypes.byref(d.c()), ctypes.byref(m), 0x1000, 16, 0x1000, 1 << 30, None) == 9
    assert da._lib.da_mask_prepare(ctypes.byref(d.c()), ctypes.byref(m), None, 1 << 20, 0x1000, 1 << 30, None) == 1


def test_shape_overflow_rejected():
    assert _call_reassign(_dims(B=64, H=1024, N=1 << 20)) == 2
    # one head whose lookup rows (nB x C) reach 2^31 entries
    big = _dims(B=1, H=1, N=1 << 28, C=1024)
    assert _call_reassign(big) == 2
    assert da.da_workspace_bytes(big) == 0
    assert da.da_workspace_bytes(_dims(B=1, H=1, N=(1 << 28) - 128, C=1024)) > 0


def test_split_attention_calls_reject_arguments():
    d = _dims()
    st = da._Stats(*([0x1000] * 9))
    m = da._Mask(0x1000, 0x1000, 4, None)
    assert da._lib.da_compensation(ctypes.byref(d.c()), ctypes.byref(m), ctypes.byref(st), 0x1000, 0, None) == 9
    assert da._lib.da_compensation(ctypes.byref(d.c()), ctypes.byref(da._Mask(None, 0x1000, 4, None)),
                                   ctypes.byref(st), 0x1000, 1 << 30, None) == 1
    assert da._lib.da_attention_prebuilt(ctypes.byref(d.c()), 0x1000, 0x1000, 0x1000, ctypes.byref(m), 0x1000,
                                         ctypes.byref(st), 0.0, None, None, 0x1000, 1 << 30, None) == 1
    assert da._lib.da_attention_prebuilt(ctypes.byref(d.c()), 0x1000, 0x1000, 0x1000, ctypes.byref(m), 0x1000,
                                         ctypes.byref(st), 0.0, 0x1002, None, 0x1000, 1 << 30, None) == 4


def test_centroid_update_rejects_arguments():
    d = _dims()
    st = da._Stats(*([0x1000] * 9))
    assert da._lib.da_centroid_update(ctypes.byref(d.c()), ctypes.byref(st), None, None) == 1
    assert da._lib.da_centroid_update(ctypes.byref(d.c()), ctypes.byref(st), 0x1004, None) == 4
    bad = da._Stats(*([0x1000] * 7 + [0x1004, 0x1000]))
    assert da._lib.da_centroid_update(ctypes.byref(d.c()), ctypes.byref(bad), 0x1000, None) == 4


def test_spread_calls_reject_arguments():
    d = _dims()
    st = da._Stats(*([0x1000] * 9))
    m = da._Mask(0x1000, 0x1000, 4, None)
    sp = da._lib.da_cluster_spread
    assert sp(ctypes.byref(d.c()), 0x1000, 0x1000, ctypes.byref(st), None, None) == 1
    assert sp(ctypes.byref(d.c()), None, 0x1000, ctypes.byref(st), 0x1000, None) == 1
    assert sp(ctypes.byref(d.c()), 0x1000, 0x1000, ctypes.byref(st), 0x1008, None) == 4
    bad = da._Stats(*([0x1000] * 7 + [0x1004, 0x1000]))
    assert sp(ctypes.byref(d.c()), 0x1000, 0x1000, ctypes.byref(bad), 0x1000, None) == 4
    at = da._lib.da_attention_spread
    ok = (0x1000, 0x1000, 0x1000, ctypes.byref(m), 0x1000, ctypes.byref(st))
    assert at(ctypes.byref(d.c()), *ok, None, 0.0, 0x1000, None, 0x1000, 1 << 30, None) == 1
    assert at(ctypes.byref(d.c()), *ok, 0x1004, 0.0, 0x1000, None, 0x1000, 1 << 30, None) == 4
    assert at(ctypes.byref(d.c()), *ok, 0x1000, 0.0, None, None, 0x1000, 1 << 30, None) == 1
    assert at(ctypes.byref(d.c()), *ok, 0x1000, 0.0, 0x1000, None, 0x1000, 0, None) == 9


def test_sip_call_rejects_arguments():
    d = _dims()
    m = da._Mask(0x1000, 0x1000, 4, None)
    f = da._lib.da_attention_sip
    ok = (0x1000, 0x1000, 0x1000, ctypes.byref(m))
    assert f(ctypes.byref(d.c()), *ok, None, 0.0, 0x1000, None, 0x1000, 1 << 30, None) == 1
    assert f(ctypes.byref(d.c()), *ok, 0x1004, 0.0, 0x1000, None, 0x1000, 1 << 30, None) == 4
    assert f(ctypes.byref(d.c()), *ok, 0x1000, 0.0, 0x1000, None, 0x1000, 0, None) == 9
    f32 = _dims(dtype=torch.float32)
    assert f(ctypes.byref(f32.c()), *ok, 0x1000, 0.0, 0x1000, None, 0x1000, 1 << 30, None) == 5


def test_noalloc_checks_match_da_reassign():
    """da_reassign_noalloc shares da_reassign's argument checks, so both accept the same dims and
    refuse the same ones with the same codes, the size limits of include/da.h included."""
    cases = [dict(dtype=torch.float16), dict(d=96), dict(C=48), dict(N=0),
             dict(B=64, H=1024, N=1 << 20),                       # B*H*nB >= 2^31
             dict(B=1, H=1, N=1 << 28, C=1024)]                   # nB*C >= 2^31 (one head's lookup rows)
    for kw in cases:
        d = _dims(**kw)
        s = da._Stats(*([0x1000] * 9))
        want = _call_reassign(d, stats=s)
        got = da._lib.da_reassign_noalloc(ctypes.byref(d.c()), 0x1000, 0x1000, 0x1000, ctypes.byref(s), None)
        assert want != 0 and got == want, (kw, want, got)
    d = _dims()
    for st in (da._Stats(*([0x1000] * 8 + [None])), da._Stats(*([0x1000] * 7 + [0x1004, 0x1000]))):
        want = _call_reassign(d, stats=st)
        got = da._lib.da_reassign_noalloc(ctypes.byref(d.c()), 0x1000, 0x1000, 0x1000, ctypes.byref(st), None)
        assert got == want, (want, got)
    assert da._lib.da_reassign_noalloc(ctypes.byref(d.c()), None, 0x1000, 0x1000,
                                       ctypes.byref(da._Stats(*([0x1000] * 9))), None) == 1
