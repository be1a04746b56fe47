"""Python binding of libda.so (decoupled sparse attention on B200).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libda.so.  The functions carry the names of the C ABI in
include/da.h and take torch CUDA tensors; they raise DAError when the library
returns a status other than DA_OK.  Importing this module loads libda.so and
fails loudly if it has not been built (``python block_sparse_cluster_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libda.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libda.so is not built ({LIB_PATH}); run python block_sparse_cluster_b200/build.py")
_lib = ctypes.CDLL(LIB_PATH)

DA_BF16, DA_F32 = 0, 1
STATUS_NAMES = ["DA_OK", "DA_ERR_INVALID_ARG", "DA_ERR_SHAPE", "DA_ERR_DTYPE", "DA_ERR_ALIGNMENT",
                "DA_ERR_UNSUPPORTED", "DA_ERR_CUDA", "DA_ERR_TIMEOUT", "DA_ERR_DEVICE_INDEX",
                "DA_ERR_WORKSPACE", "DA_ERR_RANGE"]
EXPORTS = ["da_version", "da_workspace_bytes", "da_schedule_bytes", "da_reassign", "da_mask_prepare",
           "da_attention", "da_device_status", "da_status_string", "da_reassign_noalloc", "da_compensation",
           "da_attention_prebuilt", "da_centroid_update", "da_cluster_spread", "da_attention_spread",
           "da_attention_sip", "da_noalloc_device_status"]


class DAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        name = STATUS_NAMES[code] if 0 <= code < len(STATUS_NAMES) else str(code)
        super().__init__(f"{where}: {name} ({da_status_string(code)})")


class _Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int),
                ("C", ctypes.c_int), ("block", ctypes.c_int), ("dtype", ctypes.c_int)]


class _Stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("assign", "blk_hist", "seg_idx", "seg_n", "seg_c", "seg_cnt", "seg_vsum", "n_tot", "S_tot")]


class _Mask(ctypes.Structure):
    _fields_ = [("kv_idx", ctypes.c_void_p), ("kv_cnt", ctypes.c_void_p), ("max_sel", ctypes.c_int),
                ("schedule", ctypes.c_void_p)]


_P = ctypes.c_void_p
_lib.da_version.restype = ctypes.c_int
_lib.da_workspace_bytes.restype = ctypes.c_size_t
_lib.da_workspace_bytes.argtypes = [ctypes.POINTER(_Dims)]
_lib.da_schedule_bytes.restype = ctypes.c_size_t
_lib.da_schedule_bytes.argtypes = [ctypes.POINTER(_Dims)]
_lib.da_reassign.restype = ctypes.c_int
_lib.da_reassign.argtypes = [ctypes.POINTER(_Dims), _P, _P, _P, ctypes.POINTER(_Stats), _P, ctypes.c_size_t, _P]
_lib.da_mask_prepare.restype = ctypes.c_int
_lib.da_mask_prepare.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Mask), _P, ctypes.c_size_t, _P,
                                 ctypes.c_size_t, _P]
_lib.da_attention.restype = ctypes.c_int
_lib.da_attention.argtypes = [ctypes.POINTER(_Dims), _P, _P, _P, ctypes.POINTER(_Mask), _P,
                              ctypes.POINTER(_Stats), ctypes.c_float, _P, _P, _P, ctypes.c_size_t, _P]
_lib.da_attention_prebuilt.restype = ctypes.c_int
_lib.da_attention_prebuilt.argtypes = _lib.da_attention.argtypes
_lib.da_compensation.restype = ctypes.c_int
_lib.da_compensation.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Mask), ctypes.POINTER(_Stats), _P,
                                 ctypes.c_size_t, _P]
_lib.da_centroid_update.restype = ctypes.c_int
_lib.da_centroid_update.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Stats), _P, _P]
_lib.da_cluster_spread.restype = ctypes.c_int
_lib.da_cluster_spread.argtypes = [ctypes.POINTER(_Dims), _P, _P, ctypes.POINTER(_Stats), _P, _P]
_lib.da_attention_spread.restype = ctypes.c_int
_lib.da_attention_spread.argtypes = [ctypes.POINTER(_Dims), _P, _P, _P, ctypes.POINTER(_Mask), _P,
                                     ctypes.POINTER(_Stats), _P, ctypes.c_float, _P, _P, _P, ctypes.c_size_t, _P]
_lib.da_attention_sip.restype = ctypes.c_int
_lib.da_attention_sip.argtypes = [ctypes.POINTER(_Dims), _P, _P, _P, ctypes.POINTER(_Mask), _P, ctypes.c_float, _P,
                                  _P, _P, ctypes.c_size_t, _P]
_lib.da_reassign_noalloc.restype = ctypes.c_int
_lib.da_reassign_noalloc.argtypes = [ctypes.POINTER(_Dims), _P, _P, _P, ctypes.POINTER(_Stats), _P]
_lib.da_noalloc_device_status.restype = ctypes.c_int
_lib.da_noalloc_device_status.argtypes = [_P]
_lib.da_device_status.restype = ctypes.c_int
_lib.da_device_status.argtypes = [_P, _P]
_lib.da_status_string.restype = ctypes.c_char_p
_lib.da_status_string.argtypes = [ctypes.c_int]


@dataclass(frozen=True)
class Dims:
    B: int
    H: int
    N: int
    d: int
    C: int
    block: int
    dtype: torch.dtype = torch.bfloat16

    @property
    def nB(self) -> int:
        return -(-self.N // self.block)

    def c(self) -> _Dims:
        code = DA_BF16 if self.dtype == torch.bfloat16 else DA_F32 if self.dtype == torch.float32 else -1
        return _Dims(self.B, self.H, self.N, self.d, self.C, self.block, code)


@dataclass
class ClusterStats:
    """Caller-owned Reassign Cache output (layouts in include/da.h)."""
    assign: torch.Tensor
    blk_hist: torch.Tensor
    seg_idx: torch.Tensor
    seg_n: torch.Tensor
    seg_c: torch.Tensor
    seg_cnt: torch.Tensor
    seg_vsum: torch.Tensor
    n_tot: torch.Tensor
    S_tot: torch.Tensor

    @staticmethod
    def empty(dims: Dims, device="cuda") -> "ClusterStats":
        B, H, N, d, C, bs, nB = dims.B, dims.H, dims.N, dims.d, dims.C, dims.block, dims.nB
        i32 = dict(dtype=torch.int32, device=device)
        return ClusterStats(
            assign=torch.empty(B, H, N, **i32),
            blk_hist=torch.empty(B, H, nB, C, **i32),
            seg_idx=torch.empty(B, H, nB, C, dtype=torch.uint8, device=device),
            seg_n=torch.empty(B, H, nB, **i32),
            seg_c=torch.empty(B, H, nB, bs, **i32),
            seg_cnt=torch.empty(B, H, nB, bs, **i32),
            seg_vsum=torch.empty(B, H, nB, bs, d, dtype=torch.float32, device=device),
            n_tot=torch.empty(B, H, C, **i32),
            S_tot=torch.empty(B, H, C, d, dtype=torch.float32, device=device),
        )

    def c(self) -> _Stats:
        return _Stats(*[getattr(self, n).data_ptr() for n, _ in _Stats._fields_])


@dataclass
class BlockMask:
    kv_idx: torch.Tensor                    # [B,H,nB,max_sel] int32
    kv_cnt: torch.Tensor                    # [B,H,nB] int32
    schedule: Optional[torch.Tensor] = None  # [B*H*nB] int32 from da_mask_prepare

    def c(self) -> _Mask:
        return _Mask(self.kv_idx.data_ptr(), self.kv_cnt.data_ptr(), int(self.kv_idx.shape[-1]),
                     self.schedule.data_ptr() if self.schedule is not None else None)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(code: int, where: str):
    if code != 0:
        raise DAError(code, where)


def da_version() -> int:
    return _lib.da_version()


def da_status_string(code: int) -> str:
    return _lib.da_status_string(int(code)).decode()


def da_workspace_bytes(dims: Dims) -> int:
    return _lib.da_workspace_bytes(ctypes.byref(dims.c()))


def da_schedule_bytes(dims: Dims) -> int:
    return _lib.da_schedule_bytes(ctypes.byref(dims.c()))


def workspace(dims: Dims, device="cuda") -> torch.Tensor:
    """A zero-filled workspace of da_workspace_bytes(dims) bytes."""
    n = da_workspace_bytes(dims)
    if n == 0:
        raise DAError(1, "da_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def da_reassign(dims: Dims, K: torch.Tensor, V: torch.Tensor, centroids: torch.Tensor, stats: ClusterStats,
                ws: torch.Tensor, stream=None) -> ClusterStats:
    _check(_lib.da_reassign(ctypes.byref(dims.c()), K.data_ptr(), V.data_ptr(), centroids.data_ptr(),
                            ctypes.byref(stats.c()), ws.data_ptr(), ws.numel(), _stream(stream)), "da_reassign")
    return stats


def da_reassign_noalloc(dims: Dims, K: torch.Tensor, V: torch.Tensor, centroids: torch.Tensor,
                        stats: ClusterStats, stream=None) -> ClusterStats:
    """da_reassign for callers that cannot allocate device memory: no workspace argument; the
    library's own fixed device scratch (about 1 MiB, B*H*C <= 262144) is used instead."""
    _check(_lib.da_reassign_noalloc(ctypes.byref(dims.c()), K.data_ptr(), V.data_ptr(), centroids.data_ptr(),
                                    ctypes.byref(stats.c()), _stream(stream)), "da_reassign_noalloc")
    return stats


def da_mask_prepare(dims: Dims, mask: BlockMask, schedule: torch.Tensor, ws: torch.Tensor, stream=None) -> BlockMask:
    _check(_lib.da_mask_prepare(ctypes.byref(dims.c()), ctypes.byref(mask.c()), schedule.data_ptr(),
                                schedule.numel() * schedule.element_size(), ws.data_ptr(), ws.numel(),
                                _stream(stream)), "da_mask_prepare")
    return BlockMask(mask.kv_idx, mask.kv_cnt, schedule)


def da_attention(dims: Dims, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, mask: BlockMask,
                 centroids: torch.Tensor, stats: ClusterStats, scale: float, O: torch.Tensor,
                 lse: Optional[torch.Tensor], ws: torch.Tensor, stream=None) -> torch.Tensor:
    _check(_lib.da_attention(ctypes.byref(dims.c()), Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                             ctypes.byref(mask.c()), centroids.data_ptr(), ctypes.byref(stats.c()),
                             float(scale), O.data_ptr(), lse.data_ptr() if lse is not None else None,
                             ws.data_ptr(), ws.numel(), _stream(stream)), "da_attention")
    return O


def da_compensation(dims: Dims, mask: BlockMask, stats: ClusterStats, ws: torch.Tensor, stream=None) -> None:
    """First half of da_attention: the compensation values of every q-block, into ws."""
    _check(_lib.da_compensation(ctypes.byref(dims.c()), ctypes.byref(mask.c()), ctypes.byref(stats.c()),
                                ws.data_ptr(), ws.numel(), _stream(stream)), "da_compensation")


def da_attention_prebuilt(dims: Dims, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, mask: BlockMask,
                          centroids: torch.Tensor, stats: ClusterStats, scale: float, O: torch.Tensor,
                          lse: Optional[torch.Tensor], ws: torch.Tensor, stream=None) -> torch.Tensor:
    """Second half of da_attention: the fused kernel on the values da_compensation left in ws."""
    _check(_lib.da_attention_prebuilt(ctypes.byref(dims.c()), Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                      ctypes.byref(mask.c()), centroids.data_ptr(), ctypes.byref(stats.c()),
                                      float(scale), O.data_ptr(), lse.data_ptr() if lse is not None else None,
                                      ws.data_ptr(), ws.numel(), _stream(stream)), "da_attention_prebuilt")
    return O


def da_centroid_update(dims: Dims, stats: ClusterStats, centroids: torch.Tensor, stream=None) -> torch.Tensor:
    """Lloyd update: centroids <- S_c / n_c from stats taken with the keys as the values."""
    _check(_lib.da_centroid_update(ctypes.byref(dims.c()), ctypes.byref(stats.c()), centroids.data_ptr(),
                                   _stream(stream)), "da_centroid_update")
    return centroids


def da_cluster_spread(dims: Dims, K: torch.Tensor, centroids: torch.Tensor, stats: ClusterStats,
                      spread: torch.Tensor, stream=None) -> torch.Tensor:
    """Second moment of each cluster's keys about its centroid, [B,H,C,d] fp32 (variance
    correction); stats from da_reassign on the same keys and centroids."""
    _check(_lib.da_cluster_spread(ctypes.byref(dims.c()), K.data_ptr(), centroids.data_ptr(),
                                  ctypes.byref(stats.c()), spread.data_ptr(), _stream(stream)), "da_cluster_spread")
    return spread


def da_attention_spread(dims: Dims, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, mask: BlockMask,
                        centroids: torch.Tensor, stats: ClusterStats, spread: torch.Tensor, scale: float,
                        O: torch.Tensor, lse: Optional[torch.Tensor], ws: torch.Tensor, stream=None) -> torch.Tensor:
    """da_attention with the variance-corrected cluster logits (CUDA-core path)."""
    _check(_lib.da_attention_spread(ctypes.byref(dims.c()), Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                    ctypes.byref(mask.c()), centroids.data_ptr(), ctypes.byref(stats.c()),
                                    spread.data_ptr(), float(scale), O.data_ptr(),
                                    lse.data_ptr() if lse is not None else None, ws.data_ptr(), ws.numel(),
                                    _stream(stream)), "da_attention_spread")
    return O


def da_attention_sip(dims: Dims, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, mask: BlockMask,
                     incl: torch.Tensor, scale: float, O: torch.Tensor, lse: Optional[torch.Tensor], ws: torch.Tensor,
                     stream=None) -> torch.Tensor:
    """Block-sparse attention with every selected block weighted by 1 / its inclusion probability
    (incl [B,H,nB,max_sel] fp32, aligned with the plan's slots); no cluster compensation."""
    _check(_lib.da_attention_sip(ctypes.byref(dims.c()), Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                 ctypes.byref(mask.c()), incl.data_ptr(), float(scale), O.data_ptr(),
                                 lse.data_ptr() if lse is not None else None, ws.data_ptr(), ws.numel(),
                                 _stream(stream)), "da_attention_sip")
    return O


def kmeans(dims: Dims, K: torch.Tensor, centroids: torch.Tensor, iters: int, stats: ClusterStats,
           ws: torch.Tensor, stream=None) -> torch.Tensor:
    """`iters` Lloyd iterations on the GPU, updating `centroids` in place.  Each iteration is
    da_reassign with the keys as the values (so S_c sums the keys of cluster c) followed by
    da_centroid_update; `stats` holds the last iteration's assignment afterwards."""
    for _ in range(iters):
        da_reassign(dims, K, K, centroids, stats, ws, stream)
        da_centroid_update(dims, stats, centroids, stream)
    return centroids


def da_device_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronise and return (and clear) the device status word as a status code."""
    return _lib.da_device_status(ws.data_ptr(), _stream(stream))


def da_noalloc_device_status(stream=None) -> int:
    """Synchronise and return (and clear) the status word of da_reassign_noalloc's scratch."""
    return _lib.da_noalloc_device_status(_stream(stream))


class DecoupledAttention:
    """Buffers of one workload shape plus the two calls of a step.

    One step = Reassign Cache (da_reassign) then the fused decoupled attention
    (da_attention).  The plan is fixed across steps, so its work order is
    prepared once (da_mask_prepare).
    """

    def __init__(self, dims: Dims, device="cuda"):
        self.dims = dims
        self.device = device
        self.stats = ClusterStats.empty(dims, device)
        self.ws = workspace(dims, device)
        self.mask: Optional[BlockMask] = None

    def prepare(self, kv_idx: torch.Tensor, kv_cnt: torch.Tensor, stream=None) -> BlockMask:
        sched = torch.empty(da_schedule_bytes(self.dims) // 4, dtype=torch.int32, device=self.device)
        self.mask = da_mask_prepare(self.dims, BlockMask(kv_idx, kv_cnt), sched, self.ws, stream)
        return self.mask

    def step(self, Q, K, V, centroids, O, lse=None, scale: float = 0.0, stream=None) -> torch.Tensor:
        if self.mask is None:
            raise RuntimeError("call prepare(kv_idx, kv_cnt) first")
        da_reassign(self.dims, K, V, centroids, self.stats, self.ws, stream)
        return da_attention(self.dims, Q, K, V, self.mask, centroids, self.stats, scale, O, lse, self.ws, stream)

    def status(self, stream=None) -> int:
        return da_device_status(self.ws, stream)
