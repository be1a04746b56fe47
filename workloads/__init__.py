"""Seeded synthetic inputs for decoupled sparse attention.

This module draws random numbers and lays out the fixed block plan. It holds
none of the method's arithmetic (no distances, no assignment, no statistics,
no attention), so that the fp64 oracle and the CUDA path can both take their
inputs from it without sharing any computation.

Every tensor is produced per (batch, head) from its own seed, so a test can
regenerate one head of a full-size workload without building the others.

Workloads (shapes of the video diffusion transformers named on the pages:
Wan2.1 and HunyuanVideo, "AB-Attention" abstract and "ESTRA" abstract):

* keys: a per-head mixture of C Gaussian centres mu_c ~ N(0, I_d) with
  isotropic noise (sigma 0.3); in the video-shaped workloads a token takes the
  cluster of its cell of the (T, Hs, Ws) latent grid with probability 0.9 and a
  uniformly random cluster otherwise, so clusters are correlated with 3-D
  position;
* queries and values ~ N(0, 1);
* cached centroids = the generating centres, rounded to the input dtype;
* block plan ("blocks fixed once offline by position", DecoupAttn abstract):
  for q-block i the own block, the blocks holding the same spatial position in
  the previous and next frame, then seeded random blocks up to the density.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, Optional, Sequence, Tuple

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int            # latent frames
    Hs: int           # latent height
    Ws: int           # latent width
    d: int
    block: int
    C: int
    density: float    # target fraction of kv blocks kept per q-block
    dtype: str        # "bf16" or "f32"
    cells: Optional[Tuple[int, int, int]] = None   # (ct, cy, cx) cluster grid; None = uniform clusters
    noise: float = 0.3
    p_cell: float = 0.9
    density_range: Optional[Tuple[float, float]] = None  # per-head densities (reassign-cache loop)
    steps: int = 1
    drift: float = 0.0

    @property
    def N(self) -> int:
        return self.T * self.Hs * self.Ws

    @property
    def nB(self) -> int:
        return -(-self.N // self.block)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


WORKLOADS: Dict[str, Workload] = {
    # tiny fp32 case the oracle finishes in well under a second
    "tiny": Workload("tiny", B=1, H=2, T=4, Hs=16, Ws=16, d=64, block=64, C=32,
                     density=0.25, dtype="f32", cells=None),
    # Wan2.1-1.3B latent (21 x 30 x 52), 10 % of blocks, 256 clusters
    "wan13b": Workload("wan13b", B=1, H=12, T=21, Hs=30, Ws=52, d=128, block=128, C=256,
                       density=0.10, dtype="bf16", cells=(4, 8, 8)),
    # Wan2.1-14B latent (21 x 45 x 80), 5 % of blocks, 512 clusters
    "wan14b": Workload("wan14b", B=1, H=40, T=21, Hs=45, Ws=80, d=128, block=128, C=512,
                       density=0.05, dtype="bf16", cells=(4, 8, 16)),
    # HunyuanVideo-13B latent (33 x 45 x 80), 1 % of blocks, 1024 clusters
    "hunyuan": Workload("hunyuan", B=1, H=24, T=33, Hs=45, Ws=80, d=128, block=128, C=1024,
                        density=0.01, dtype="bf16", cells=(8, 8, 16)),
    # reassign-cache loop: Wan2.1-1.3B shape, per-head density in [1 %, 20 %], 8 drifting steps
    "loop": Workload("loop", B=1, H=12, T=21, Hs=30, Ws=52, d=128, block=128, C=256,
                     density=0.10, dtype="bf16", cells=(4, 8, 8),
                     density_range=(0.01, 0.20), steps=8, drift=0.05),
}


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (smaller test cases)."""
    return replace(w, **kw)


# ---------------------------------------------------------------------------
# seeding

_TAGS = {"q": 1, "k": 2, "v": 3, "mu": 4, "label": 5, "mask": 6, "density": 7, "drift": 8,
         "perm": 9, "incl": 10}


def _seed(seed: int, tag: str, *idx: int) -> int:
    ss = np.random.SeedSequence([int(seed) & 0xFFFFFFFF, _TAGS[tag]] + [int(i) for i in idx])
    return int(ss.generate_state(1, dtype=np.uint64)[0] & ((1 << 63) - 1))


def _gen(seed: int, tag: str, *idx: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(_seed(seed, tag, *idx))
    return g


# ---------------------------------------------------------------------------
# per-head tensors (float32 before rounding to the workload dtype)

def head_centres(w: Workload, seed: int, b: int, h: int) -> torch.Tensor:
    """Generating centres mu [C, d] ~ N(0, I_d)."""
    return torch.randn(w.C, w.d, generator=_gen(seed, "mu", b, h))


def head_labels(w: Workload, seed: int, b: int, h: int) -> torch.Tensor:
    """Generating cluster of every token, int64 [N] (tokens flattened frame-major)."""
    N = w.N
    g = _gen(seed, "label", b, h)
    uniform = torch.randint(0, w.C, (N,), generator=g)
    if w.cells is None:
        return uniform
    ct, cy, cx = w.cells
    assert ct * cy * cx == w.C, "cell grid must have C cells"
    t = torch.arange(w.T).repeat_interleave(w.Hs * w.Ws)
    y = torch.arange(w.Hs).repeat_interleave(w.Ws).repeat(w.T)
    x = torch.arange(w.Ws).repeat(w.T * w.Hs)
    cell = ((t * ct // w.T) * cy + (y * cy // w.Hs)) * cx + (x * cx // w.Ws)
    perm = torch.randperm(w.C, generator=_gen(seed, "perm", b, h))
    by_cell = perm[cell]
    keep = torch.rand(N, generator=g) < w.p_cell
    return torch.where(keep, by_cell, uniform)


def head_qkv(w: Workload, seed: int, b: int, h: int, step: int = 0):
    """(Q, K, V, centroids) of one head in the workload dtype (CPU tensors).

    At step s > 0 of the reassign-cache loop the keys have drifted by s
    additive N(0, drift^2) increments; queries and values are redrawn per step;
    the cached centroids stay the step-0 generating centres.
    """
    N, d = w.N, w.d
    mu = head_centres(w, seed, b, h)
    lab = head_labels(w, seed, b, h)
    k = mu[lab] + w.noise * torch.randn(N, d, generator=_gen(seed, "k", b, h))
    for s in range(1, step + 1):
        k = k + w.drift * torch.randn(N, d, generator=_gen(seed, "drift", b, h, s))
    q = torch.randn(N, d, generator=_gen(seed, "q", b, h, step))
    v = torch.randn(N, d, generator=_gen(seed, "v", b, h, step))
    dt = w.torch_dtype
    return q.to(dt), k.to(dt), v.to(dt), mu.to(dt)


def head_density(w: Workload, seed: int, b: int, h: int) -> float:
    if w.density_range is None:
        return w.density
    lo, hi = w.density_range
    u = torch.rand(1, generator=_gen(seed, "density", b, h)).item()
    return lo + (hi - lo) * u


def head_plan(w: Workload, seed: int, b: int, h: int) -> list:
    """Fixed block plan of one head: a list of nB sorted int32 arrays of kv blocks.

    Mandatory blocks of q-block i: i itself and the blocks that hold the token
    one frame before and one frame after the block's centre token.  Seeded
    random other blocks are added until the row holds
    max(#mandatory, round(density * nB)) blocks.
    """
    nB, Bs, N = w.nB, w.block, w.N
    frame = w.Hs * w.Ws
    k_row = int(math.floor(head_density(w, seed, b, h) * nB + 0.5))
    rng = np.random.default_rng(_seed(seed, "mask", b, h))
    rows = []
    for i in range(nB):
        m = min(i * Bs + Bs // 2, N - 1)
        must = {i}
        for t in (m - frame, m + frame):
            if 0 <= t < N:
                must.add(t // Bs)
        want = max(len(must), min(k_row, nB))
        chosen = set(must)
        if want > len(chosen):
            others = np.array([j for j in range(nB) if j not in chosen], dtype=np.int64)
            extra = rng.choice(others, size=want - len(chosen), replace=False)
            chosen.update(int(j) for j in extra)
        rows.append(np.array(sorted(chosen), dtype=np.int32))
    return rows


def pack_plan(rows_per_head: Sequence[Sequence[np.ndarray]], nB: int, max_sel: Optional[int] = None):
    """Pack per-(b,h) row lists into kv_idx [B,H,nB,max_sel] (pad -1) and kv_cnt [B,H,nB]."""
    B = len(rows_per_head)
    H = len(rows_per_head[0])
    if max_sel is None:
        max_sel = max(len(r) for hp in rows_per_head for rows in hp for r in rows)
    ms = max(max_sel, 1)
    kv_idx = np.full((B, H, nB, ms), -1, dtype=np.int32)
    kv_cnt = np.zeros((B, H, nB), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i, r in enumerate(rows_per_head[b][h]):
                kv_idx[b, h, i, : len(r)] = r
                kv_cnt[b, h, i] = len(r)
    return torch.from_numpy(kv_idx), torch.from_numpy(kv_cnt)


@dataclass
class Inputs:
    w: Workload
    seed: int
    Q: torch.Tensor          # [B,H,N,d]
    K: torch.Tensor
    V: torch.Tensor
    centroids: torch.Tensor  # [B,H,C,d]
    kv_idx: torch.Tensor     # [B,H,nB,max_sel] int32, -1 padded
    kv_cnt: torch.Tensor     # [B,H,nB] int32
    plans: list = field(default_factory=list)   # [B][H] lists of row arrays


def make_inputs(w: Workload, seed: int = 0, step: int = 0, heads: Optional[Sequence[int]] = None) -> Inputs:
    """Inputs of a workload on the CPU: every head, or the given heads (global indices, so that a
    slice holds exactly the same tensors as those heads of the full workload).  The returned
    Inputs' workload has H = the number of heads returned."""
    heads = list(range(w.H)) if heads is None else [int(h) for h in heads]
    B, H, N, d, C = w.B, len(heads), w.N, w.d, w.C
    dt = w.torch_dtype
    Q = torch.empty(B, H, N, d, dtype=dt)
    K = torch.empty_like(Q)
    V = torch.empty_like(Q)
    cent = torch.empty(B, H, C, d, dtype=dt)
    plans = []
    for b in range(B):
        hp = []
        for i, h in enumerate(heads):
            q, k, v, mu = head_qkv(w, seed, b, h, step)
            Q[b, i], K[b, i], V[b, i], cent[b, i] = q, k, v, mu
            hp.append(head_plan(w, seed, b, h))
        plans.append(hp)
    kv_idx, kv_cnt = pack_plan(plans, w.nB)
    return Inputs(replace(w, H=H), seed, Q, K, V, cent, kv_idx, kv_cnt, plans)


def effective_flops(w: Workload, kv_cnt: torch.Tensor, kv_idx: torch.Tensor) -> float:
    """Effective FLOPs of one attention call: sum over heads and q-blocks of
    4 * |q-block| * (kept keys + C) * d, kept keys counting only real keys."""
    N, Bs, C, d = w.N, w.block, w.C, w.d
    nB = w.nB
    blk_len = np.full(nB, Bs, dtype=np.int64)
    blk_len[-1] = N - (nB - 1) * Bs
    idx = kv_idx.numpy().astype(np.int64)
    cnt = kv_cnt.numpy().astype(np.int64)
    valid = np.arange(idx.shape[-1])[None, None, None, :] < cnt[..., None]
    kept = np.where(valid, blk_len[np.clip(idx, 0, nB - 1)], 0).sum(-1)      # [B,H,nB]
    qlen = blk_len[None, None, :]
    return float((4 * qlen * (kept + C) * d).sum())


def inclusion_probabilities(w: Workload, seed: int, max_sel: int, lo: float = 0.2) -> torch.Tensor:
    """Seeded inclusion probabilities for the plan's slots, [B,H,nB,max_sel] fp32 drawn uniformly
    from [lo, 1) per (batch, head); numbers only (the reweighting itself lives elsewhere)."""
    out = torch.empty(w.B, w.H, w.nB, max_sel, dtype=torch.float32)
    for b in range(w.B):
        for h in range(w.H):
            u = torch.rand(w.nB, max_sel, generator=_gen(seed, "incl", b, h))
            out[b, h] = lo + (1.0 - lo) * u
    return out
