// CUDA-core reassignment and decoupled attention kernels (templates).
//
// The fp32 path is exact fp32 arithmetic on the CUDA cores (no TF32), so it can be held to a
// 1e-4 tolerance.  simt_f32.cu and simt_bf16.cu instantiate them.
#pragma once
#include <math.h>

#include "da_common.cuh"
#include "da_internal.h"

namespace da {

// Reassignment on CUDA cores: a(k) = argmin_c sum_t (k_t - cbar_{c,t})^2, ties to the lowest c.
// One thread per key; centroids staged through shared memory 32 at a time.
template <typename T, int D>
__global__ void __launch_bounds__(128) assign_simt_kernel(const T* __restrict__ K, const T* __restrict__ cent,
                                                          int32_t* __restrict__ assign, int N, int C) {
  __shared__ float cs[32][D];
  const int bh = blockIdx.x;
  const int k = blockIdx.y * 128 + threadIdx.x;
  const bool live = k < N;
  float kr[D];
  if (live) {
    const T* kp = K + ((size_t)bh * N + k) * D;
#pragma unroll
    for (int t = 0; t < D; t += 4) load_vec(kp + t, &kr[t], 4);
  }
  float best = INFINITY;
  int arg = 0;
  for (int c0 = 0; c0 < C; c0 += 32) {
    __syncthreads();
    for (int x = threadIdx.x; x < 32 * D; x += 128) cs[x / D][x % D] = to_f32(cent[((size_t)bh * C + c0) * D + x]);
    __syncthreads();
    if (live) {
      for (int cc = 0; cc < 32; ++cc) {
        float dist = 0.f;
#pragma unroll
        for (int t = 0; t < D; ++t) {
          const float df = kr[t] - cs[cc][t];
          dist = fmaf(df, df, dist);
        }
        if (dist < best) {
          best = dist;
          arg = c0 + cc;
        }
      }
    }
  }
  if (live) assign[(size_t)bh * N + k] = arg;
}

// fp32 decoupled attention on CUDA cores.  One CTA per (head, q-block); four threads per query
// row, each holding a quarter of q and of the output (dot products finished with two lane
// shuffles), so everything stays in registers.  Exact part over the selected blocks, then the
// clusters in chunks of 32 with the complement statistics built in shared memory:
//   n^U_c = n_c - sum_{j in sel} n_{c,j},  vbar^U_c = (S_c - sum_{j in sel} S_{c,j}) / n^U_c,
//   logit = s q.cbar_c + ln n^U_c  (left out when n^U_c = 0).
// With `spread` (the second moment D_c of each cluster's keys about its representative), the
// variance-corrected logit of the ESTRA abstract's reading: + s^2/2 sum_t q_t^2 D_{c,t}; the
// clusters then go in chunks of 16, their D rows in the upper half of ks.
// Logits are kept in log2 units (q pre-scaled by s*log2(e), bias log2 n^U_c; the correction is
// then ln(2)/2 sum_t q_t^2 D_{c,t} in those units).
constexpr int kSimtTPR = 4;                     // threads per query row
constexpr int kSimtThreads = 128 * kSimtTPR;    // one CTA covers a q-block of up to 128 rows

template <typename T, int D>
__global__ void __launch_bounds__(kSimtThreads) attention_simt_kernel(
    const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V, const int32_t* __restrict__ kv_idx,
    const int32_t* __restrict__ kv_cnt, int max_sel, const int32_t* __restrict__ schedule,
    const T* __restrict__ cent, StatsPtrs st, const float* __restrict__ spread, float scale_log2,
    T* __restrict__ O, float* __restrict__ lse, int* status, int N, int C, int block, int nB) {
  constexpr int DP = D / kSimtTPR;              // columns per thread
  // staged rows: the four quarters of a row each followed by 4 floats of padding, so that the
  // four threads of a query row (one quarter each) read distinct banks
  constexpr int SEG = DP + 4;
  constexpr int ROW = kSimtTPR * SEG;
  __shared__ __align__(16) float ks[32][ROW];
  __shared__ __align__(16) float vs[32][ROW];
  auto col = [](int c) { return c / DP * SEG + c % DP; };   // column c of a staged row
  __shared__ float beta[32];
  const int item = schedule ? schedule[blockIdx.x] : (int)blockIdx.x;
  if (item < 0 || item >= (int)gridDim.x) {   // a schedule not written by da_mask_prepare
    if (threadIdx.x == 0) set_status(status, DA_ERR_DEVICE_INDEX);
    return;
  }
  const int bh = item / nB, i = item % nB;
  const int q0 = i * block;
  const int qlen = min(block, N - q0);
  const int t = threadIdx.x;
  const int row = t / kSimtTPR, part = t % kSimtTPR;
  const int c0l = part * DP;                    // first column of this thread
  const int s0l = part * SEG;                   // its quarter in a staged row
  const bool active = row < qlen;

  float q[DP], o[DP];
  if (active) {
    const T* qp = Q + ((size_t)bh * N + q0 + row) * D + c0l;
#pragma unroll
    for (int x = 0; x < DP; x += 4) load_vec(qp + x, &q[x], 4);
#pragma unroll
    for (int x = 0; x < DP; ++x) q[x] *= scale_log2;
  } else {
#pragma unroll
    for (int x = 0; x < DP; ++x) q[x] = 0.f;
  }
#pragma unroll
  for (int x = 0; x < DP; ++x) o[x] = 0.f;
  float m = -INFINITY, l = 0.f;

  int cnt = kv_cnt[item];
  if (cnt < 0 || cnt > max_sel) cnt = 0;   // reported by the schedule pass
  const int32_t* rowp = kv_idx + (size_t)item * max_sel;

  // sum over the row's four threads (adjacent lanes)
  auto rowsum = [&](float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    return v;
  };
  // online softmax over shared rows [r0, r0 + 8) of ks/vs, of which the first `valid` are real;
  // `corr`: ks row 16 + r holds the second moment of cluster row r (variance correction).
  // Every thread of the CTA calls this (the shuffles need whole warps).
  auto absorb8 = [&](int r0, int valid, bool corr) {
    float x[8];
    float cm = -INFINITY;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      float dot = 0.f, c2 = 0.f;
#pragma unroll
      for (int u = 0; u < DP; ++u) dot = fmaf(q[u], ks[r0 + kk][s0l + u], dot);
      if (corr) {
#pragma unroll
        for (int u = 0; u < DP; ++u) c2 = fmaf(q[u] * q[u], ks[16 + r0 + kk][s0l + u], c2);
      }
      dot = rowsum(dot);
      if (corr) dot = fmaf(0.34657359027997264f, rowsum(c2), dot);   // ln(2) / 2
      x[kk] = kk < valid ? dot + beta[r0 + kk] : -INFINITY;
      cm = fmaxf(cm, x[kk]);
    }
    const float mn = fmaxf(m, cm);
    if (mn == -INFINITY) return;
    const float alpha = exp2f(m - mn);
    l *= alpha;
#pragma unroll
    for (int u = 0; u < DP; ++u) o[u] *= alpha;
    m = mn;
#pragma unroll 4
    for (int kk = 0; kk < 8; ++kk) {
      const float pw = exp2f(x[kk] - m);
      l += pw;
#pragma unroll
      for (int u = 0; u < DP; ++u) o[u] = fmaf(pw, vs[r0 + kk][s0l + u], o[u]);
    }
  };
  auto absorb = [&](int valid) {   // rows [0, valid) of the 32 staged
    for (int r0 = 0; r0 < valid; r0 += 8) absorb8(r0, min(8, valid - r0), false);
  };

  // exact attention on the selected blocks
  for (int s = 0; s < cnt; ++s) {
    const int j = rowp[s];
    if (j < 0 || j >= nB) {
      if (t == 0) set_status(status, DA_ERR_DEVICE_INDEX);
      continue;
    }
    const int k0 = j * block;
    const int klen = min(block, N - k0);
    for (int kc = 0; kc < klen; kc += 32) {
      const int valid = min(32, klen - kc);
      __syncthreads();
      for (int x = t; x < 32 * D; x += kSimtThreads) {
        const int r = x / D, u = x % D;
        float kv = 0.f, vv = 0.f;
        if (r < valid) {
          const size_t off = ((size_t)bh * N + k0 + kc + r) * D + u;
          kv = to_f32(K[off]);
          vv = to_f32(V[off]);
        }
        ks[r][col(u)] = kv;
        vs[r][col(u)] = vv;
      }
      if (t < 32) beta[t] = 0.f;
      __syncthreads();
      absorb(valid);
    }
  }

  // compensation: clusters in chunks of 32 (16 with the variance correction)
  const int CH = spread ? 16 : 32;
  for (int cb = 0; cb < C; cb += CH) {
    __syncthreads();
    if ((t >> 2) < CH) {                        // 4 threads per cluster, D/4 columns each
      const int cl = t >> 2, qpart = t & 3;
      const int c = cb + cl;
      constexpr int W = D / 4;
      int nU = st.n_tot[(size_t)bh * C + c];
      float acc[W];
      const float* tot = st.S_tot + ((size_t)bh * C + c) * D + qpart * W;
#pragma unroll
      for (int u = 0; u < W; ++u) acc[u] = tot[u];
      for (int s = 0; s < cnt; ++s) {
        const int j = rowp[s];
        if (j < 0 || j >= nB) continue;
        const size_t bj = (size_t)bh * nB + j;
        const int e = st.seg_idx[bj * C + c];
        if (e == 0xFF) continue;
        nU -= st.seg_cnt[bj * block + e];
        const float* sv = st.seg_vsum + (bj * block + e) * D + qpart * W;
#pragma unroll
        for (int u = 0; u < W; ++u) acc[u] -= sv[u];
      }
      const float inv = nU > 0 ? 1.f / (float)nU : 0.f;
#pragma unroll
      for (int u = 0; u < W; ++u) vs[cl][col(qpart * W + u)] = acc[u] * inv;
      if (qpart == 0) beta[cl] = nU > 0 ? log2f((float)nU) : -INFINITY;
    }
    for (int x = t; x < CH * D; x += kSimtThreads)
      ks[x / D][col(x % D)] = to_f32(cent[((size_t)bh * C + cb) * D + x]);
    if (spread)
      for (int x = t; x < 16 * D; x += kSimtThreads) ks[16 + x / D][col(x % D)] = spread[((size_t)bh * C + cb) * D + x];
    __syncthreads();
    if (spread) {
      absorb8(0, 8, true);
      absorb8(8, 8, true);
    } else {
      absorb(32);
    }
  }

  if (active) {
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    T* op = O + ((size_t)bh * N + q0 + row) * D + c0l;
#pragma unroll
    for (int u = 0; u < DP; ++u) store_out(op + u, o[u] * inv_l);
    if (lse && part == 0) lse[(size_t)bh * N + q0 + row] = (m + log2f(l)) * 0.69314718055994531f;
  }
}

}  // namespace da
