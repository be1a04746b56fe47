"""fp64 CPU oracle for decoupled sparse attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, the package entry's smoke check and the benchmark's CPU
baseline leg may import this module.  The product path (the CUDA library and
its Python binding) never calls it, and this module imports nothing from the
product path: the two share no code.  Inputs reach both sides from the seeded
generators in ``workloads``, which hold none of the method's arithmetic.

What is computed, and where it is stated
----------------------------------------
The pages state the method in words only ("DecoupAttn: Decoupled Sparse
Attention for Training-Free Acceleration of Video Diffusion", abstract):

* semantic clusters compensate every key, and exact attention corrects their
  error on a few key blocks that are fixed once, offline, by position;
* Reassign Cache: each step reassigns the drifting keys to cached centroids
  and refreshes the compensation while the budgeted blocks stay fixed;
* the clustering is Lloyd's least-squares quantisation (the same page lists
  "Least squares quantization in PCM" among the works it builds on), hence the
  squared Euclidean distance.

Readings taken where the pages are silent (each is listed in the design notes):

* R1 distance: squared Euclidean, written as the explicit difference
  sum_t (k_t - c_t)^2; ties go to the lowest centroid index.
* R2 blocks: key block j holds tokens [j*Bs, min((j+1)*Bs, N)); the last block
  may be short; there are no padding keys.
* R3 compensated keys: the keys outside the selected blocks of the q-block
  (the complement U).  Cluster c enters the softmax as n^U_c copies of one key
  at the cached centroid with the mean complement value:
  logit s*q.cbar_c + ln n^U_c (natural log) and value vbar^U_c; a cluster with
  n^U_c = 0 is left out.  The complement statistics are counted directly over
  U here, not obtained by subtraction.
* R4 the cached centroid is used as given; it is not re-estimated from the
  keys assigned to it.
* R5 scale s = 1/sqrt(d) unless given.
* R6 (variance correction, optional) the pages' ESTRA abstract refines the
  weights of the cluster representatives with "a variance-based correction"
  and prints no formula.  Reading: the cluster's keys are treated as Gaussian
  about the representative with a diagonal second moment D_c (per dimension,
  the mean of (k_t - cbar_{c,t})^2 over all keys assigned to c), so that
  mean_k exp(s q.k) = exp(s q.cbar_c + s^2/2 sum_t q_t^2 D_{c,t}) up to higher
  cumulants; the cluster logit gains the term s^2/2 sum_t q_t^2 D_{c,t}.
* R7 (inclusion-probability reweighting, optional) the AB-Attention abstract
  samples blocks and "reweights them by inverse inclusion probability, so that
  one pass estimates dense attention".  Reading: the q-block's selected blocks
  carry inclusion probabilities pi_j in (0, 1]; numerator and denominator of
  the softmax each sum (1 / pi_j) times the block's exact terms (Horvitz-
  Thompson), with no cluster compensation; a row without selected blocks
  gives O = 0 and LSE = -inf.

Parity status: reassignment, block statistics and attention are each pinned
by tests that do not call this module's formulas again (library routines,
closed forms, invariants, brute force and hand-worked fixtures).  The choice
of the complement set and of ln n^U (R3) is pinned only as far as the pages'
own statement goes ("every key is compensated"): when every key sits exactly
on its centroid, compensation is exact and the result must equal dense
attention for any block plan; the tests check that.
"""
from __future__ import annotations

import math
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "reassign", "block_ranges", "block_histogram", "block_entries", "cluster_totals",
    "complement_stats", "attention_qblock", "attention", "lloyd_step", "kmeans", "sse",
    "cluster_spread", "attention_sip_qblock",
]


def _f64(x) -> np.ndarray:
    """Upcast a numpy array or a CPU torch tensor (any float dtype) to float64."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        if str(x.dtype) in ("torch.bfloat16", "torch.float16"):
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def _i64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.asarray(x, dtype=np.int64)


# ---------------------------------------------------------------------------
# Reassign Cache, step 1: reassign every key to its nearest cached centroid

def reassign(K, centroids, chunk: int = 64) -> Tuple[np.ndarray, np.ndarray]:
    """Nearest cached centroid of every key (DecoupAttn abstract, Reassign Cache).

    K [N, d], centroids [C, d].  Returns (assign int64 [N], gap float64 [N]),
    where gap is the relative distance gap to the runner-up centroid,
    (d2 - d1) / max(d1, 1e-12); gap is +inf when C == 1.
    """
    K = _f64(K)
    Cn = _f64(centroids)
    N = K.shape[0]
    C = Cn.shape[0]
    assign = np.empty(N, dtype=np.int64)
    gap = np.empty(N, dtype=np.float64)
    for s in range(0, N, chunk):
        e = min(N, s + chunk)
        diff = K[s:e, None, :] - Cn[None, :, :]
        dist = np.einsum("nct,nct->nc", diff, diff)
        a = np.argmin(dist, axis=1)          # first minimum = lowest index on ties
        rows = np.arange(e - s)
        d1 = dist[rows, a]
        assign[s:e] = a
        if C > 1:
            dist[rows, a] = np.inf
            d2 = dist.min(axis=1)
            gap[s:e] = (d2 - d1) / np.maximum(d1, 1e-12)
        else:
            gap[s:e] = np.inf
    return assign, gap


# ---------------------------------------------------------------------------
# Reassign Cache, step 2: refresh the per-(key block, cluster) statistics

def block_ranges(N: int, block: int) -> List[Tuple[int, int]]:
    """Token range [start, end) of every key block; the last one may be short."""
    return [(j, min(j + block, N)) for j in range(0, N, block)]


def block_histogram(assign, C: int, N: int, block: int) -> np.ndarray:
    """n_{c,j}: number of keys of block j assigned to cluster c, int64 [nB, C]."""
    a = _i64(assign)
    rng = block_ranges(N, block)
    hist = np.zeros((len(rng), C), dtype=np.int64)
    for j, (s, e) in enumerate(rng):
        for k in range(s, e):
            hist[j, a[k]] += 1
    return hist


def block_entries(assign, V, C: int, N: int, block: int, j: int):
    """Statistics of one key block j, one entry per cluster present in it.

    Returns (clusters int64 [E] ascending, counts int64 [E], sums float64 [E, d])
    with sums[e] = sum of the value rows of the block's keys in clusters[e].
    """
    a = _i64(assign)
    Vf = _f64(V)
    s, e = block_ranges(N, block)[j]
    present = sorted(set(int(c) for c in a[s:e]))
    d = Vf.shape[1]
    counts = np.zeros(len(present), dtype=np.int64)
    sums = np.zeros((len(present), d), dtype=np.float64)
    pos = {c: i for i, c in enumerate(present)}
    for k in range(s, e):
        i = pos[int(a[k])]
        counts[i] += 1
        sums[i] += Vf[k]
    return np.array(present, dtype=np.int64), counts, sums


def cluster_totals(assign, V, C: int) -> Tuple[np.ndarray, np.ndarray]:
    """Per-head totals n_c (int64 [C]) and S_c = sum of value rows (float64 [C, d])."""
    a = _i64(assign)
    Vf = _f64(V)
    n = np.bincount(a, minlength=C).astype(np.int64)
    S = np.stack([np.bincount(a, weights=Vf[:, t], minlength=C) for t in range(Vf.shape[1])], axis=1)
    return n, S


def cluster_spread(K, centroids, assign, C: int) -> np.ndarray:
    """Second moment of each cluster's keys about its representative (reading R6):
    D[c, t] = mean over the keys k with a(k) = c of (k_t - cbar_{c,t})^2; zero for an empty
    cluster.  float64 [C, d]."""
    a = _i64(assign)
    Kf = _f64(K)
    Cf = _f64(centroids)
    dev2 = (Kf - Cf[a]) ** 2
    n = np.bincount(a, minlength=C).astype(np.float64)
    tot = np.stack([np.bincount(a, weights=dev2[:, t], minlength=C) for t in range(Kf.shape[1])], axis=1)
    D = np.zeros_like(tot)
    nz = n > 0
    D[nz] = tot[nz] / n[nz, None]
    return D


# ---------------------------------------------------------------------------
# Decoupled attention for one q-block

def complement_stats(assign, V, C: int, in_sel: np.ndarray):
    """Counts and mean values of the keys outside the selected blocks (reading R3).

    in_sel: bool [N], True for keys in the q-block's selected blocks.
    Returns (nU int64 [C], vbarU float64 [C, d]; rows with nU == 0 are zero).
    """
    a = _i64(assign)
    Vf = _f64(V)
    U = ~in_sel
    aU = a[U]
    VU = Vf[U]
    nU = np.bincount(aU, minlength=C).astype(np.int64)
    SU = np.stack([np.bincount(aU, weights=VU[:, t], minlength=C) for t in range(Vf.shape[1])], axis=1)
    vbar = np.zeros_like(SU)
    nz = nU > 0
    vbar[nz] = SU[nz] / nU[nz, None]
    return nU, vbar


def attention_qblock(Q, K, V, centroids, sel_blocks: Sequence[int], assign, i: int,
                     block: int, scale: Optional[float] = None, return_lse: bool = False,
                     spread=None):
    """Output rows of q-block i (DecoupAttn abstract: exact attention on the
    fixed blocks, every other key compensated through its cluster).

    Logits: s*q.k for keys in the selected blocks, s*q.cbar_c + ln n^U_c for
    the clusters with n^U_c > 0; one softmax over both; the clusters carry the
    mean complement value vbar^U_c.  With `spread` (D of cluster_spread, reading
    R6) each cluster logit gains s^2/2 sum_t q_t^2 D_{c,t}.
    """
    Qf = _f64(Q)
    Kf = _f64(K)
    Vf = _f64(V)
    Cf = _f64(centroids)
    N, d = Kf.shape
    C = Cf.shape[0]
    s = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rng = block_ranges(N, block)
    qs, qe = rng[i]
    in_sel = np.zeros(N, dtype=bool)
    for j in sel_blocks:
        bs, be = rng[int(j)]
        in_sel[bs:be] = True
    nU, vbar = complement_stats(assign, Vf, C, in_sel)
    live = nU > 0
    q = Qf[qs:qe]
    ell = s * (q @ Kf[in_sel].T)                               # [nq, |Sel|]
    lam = s * (q @ Cf[live].T) + np.log(nU[live])[None, :]    # [nq, #live]
    if spread is not None:
        lam = lam + 0.5 * s * s * ((q * q) @ _f64(spread)[live].T)
    m = np.maximum(ell.max(axis=1, initial=-np.inf), lam.max(axis=1, initial=-np.inf))
    pe = np.exp(ell - m[:, None])
    pl = np.exp(lam - m[:, None])
    num = pe @ Vf[in_sel] + pl @ vbar[live]
    den = pe.sum(axis=1) + pl.sum(axis=1)
    out = num / den[:, None]
    if return_lse:
        return out, m + np.log(den)
    return out


def attention_sip_qblock(Q, K, V, sel_blocks: Sequence[int], incl: Sequence[float], i: int, block: int,
                         scale: Optional[float] = None, return_lse: bool = False):
    """Output rows of q-block i under inclusion-probability reweighting (reading R7): block j of
    the selection, included with probability incl[j], enters numerator and denominator with the
    weight 1 / incl[j]."""
    Qf = _f64(Q)
    Kf = _f64(K)
    Vf = _f64(V)
    N, d = Kf.shape
    s = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rng = block_ranges(N, block)
    qs, qe = rng[i]
    q = Qf[qs:qe]
    nq = qe - qs
    if len(sel_blocks) == 0:
        out = np.zeros((nq, d))
        return (out, np.full(nq, -np.inf)) if return_lse else out
    logits, vals = [], []
    for j, p in zip(sel_blocks, incl):
        bs, be = rng[int(j)]
        logits.append(s * (q @ Kf[bs:be].T) - math.log(float(p)))   # weight 1/p as a log
        vals.append(Vf[bs:be])
    ell = np.concatenate(logits, axis=1)
    vv = np.concatenate(vals, axis=0)
    m = ell.max(axis=1)
    pe = np.exp(ell - m[:, None])
    den = pe.sum(axis=1)
    out = (pe @ vv) / den[:, None]
    if return_lse:
        return out, m + np.log(den)
    return out


def attention(Q, K, V, centroids, plan: Sequence[Sequence[int]], assign, block: int,
              scale: Optional[float] = None, q_blocks: Optional[Iterable[int]] = None, spread=None):
    """Output [N, d] of one head (rows of q-blocks not requested stay NaN)."""
    Qf = _f64(Q)
    N, d = Qf.shape
    out = np.full((N, d), np.nan)
    rng = block_ranges(N, block)
    qb = range(len(rng)) if q_blocks is None else q_blocks
    for i in qb:
        s, e = rng[i]
        out[s:e] = attention_qblock(Qf, K, V, centroids, plan[i], assign, i, block, scale, spread=spread)
    return out


# ---------------------------------------------------------------------------------------------
# Lloyd's algorithm (the clustering the pages build on: "Least squares quantization in PCM"), used
# for the initial centroids and for the comparison with fresh clusters in the reassign-cache loop.

def sse(K, centroids, assign) -> float:
    """Sum of squared distances of every key to its assigned centroid (the k-means objective)."""
    Kf, Cf = _f64(K), _f64(centroids)
    a = _i64(assign)
    return float(((Kf - Cf[a]) ** 2).sum())


def lloyd_update(K, centroids, assign) -> np.ndarray:
    """The update half of a Lloyd iteration for a given assignment: each centroid moves to the
    mean of its keys; a centroid without keys stays where it is.  Returns float64 [C, d]."""
    Kf, Cf = _f64(K), _f64(centroids)
    a = _i64(assign)
    C = Cf.shape[0]
    n = np.bincount(a, minlength=C)
    S = np.zeros_like(Cf)
    np.add.at(S, a, Kf)
    new = Cf.copy()
    live = n > 0
    new[live] = S[live] / n[live][:, None]
    return new


def lloyd_step(K, centroids) -> Tuple[np.ndarray, np.ndarray]:
    """One Lloyd iteration: assign every key to its nearest centroid (reassign, reading R1), then
    move each centroid to the mean of its keys (lloyd_update).
    Returns (new centroids float64 [C, d], assignment int64 [N])."""
    a, _ = reassign(_f64(K), _f64(centroids))
    return lloyd_update(K, centroids, a), a


def kmeans(K, init, iters: int) -> Tuple[np.ndarray, np.ndarray]:
    """`iters` Lloyd iterations from `init`; returns (centroids, assignment of the last step)."""
    c = _f64(init)
    a = None
    for _ in range(iters):
        c, a = lloyd_step(K, c)
    return c, a
