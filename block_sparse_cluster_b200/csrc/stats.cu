// Reassign Cache statistics and plan kernels shared by the fp32 and bf16 paths: centroid norms,
// per-block statistics, per-head totals, plan validation and work order.
#include <math.h>

#include "block_stats.cuh"
#include "da_common.cuh"
#include "da_internal.h"

#include <type_traits>

namespace da {

WsLayout ws_layout(const Dims& g) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  WsLayout L;
  const size_t BH = (size_t)g.B * g.H;
  L.status = 0;
  L.norms = 256;
  L.sched = L.norms + up(BH * g.C * sizeof(float));
  L.comp = L.sched + up(BH * g.nB * sizeof(int32_t));
  L.spread = L.comp + up(attention_tc_scratch_bytes(g));
  // Dh of the variance-corrected mode on the tensor cores (bf16 [B*H][C][d])
  L.total = L.spread + (attention_tc_supported(g) ? up(BH * g.C * g.d * 2) : 0);
  return L;
}

// ||cbar_c||^2 in fp32 from the stored centroids; one warp per centroid, fixed reduction order.
template <typename T>
__global__ void centroid_norms_kernel(const T* __restrict__ cent, float* __restrict__ norms, long long rows, int d) {
  const long long r = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const T* c = cent + r * d;
  float s = 0.f;
  for (int t = lane; t < d; t += 32) {
    const float x = to_f32(c[t]);
    s = fmaf(x, x, s);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) norms[r] = s;
}

// Per-block statistics from an existing assignment: one CTA of 128 threads per (head, block).
template <typename T, int D>
__global__ void __launch_bounds__(128) block_stats_kernel(const T* __restrict__ V, StatsPtrs st, int N, int C,
                                                          int block, int nB) {
  __shared__ StatsSmem sm;
  __shared__ int s_assign[128];
  const int bh = blockIdx.y, j = blockIdx.x;
  const int k0 = j * block;
  const int nk = min(block, N - k0);
  const int t = threadIdx.x;
  if (t < nk) s_assign[t] = st.assign[(size_t)bh * N + k0 + t];
  __syncthreads();
  const size_t bj = (size_t)bh * nB + j;
  block_stats_group<T, D>(t, 1, s_assign, nk, V + ((size_t)bh * N + k0) * D, C, st.blk_hist + bj * C,
                          st.seg_idx + bj * C, st.seg_n + bj, st.seg_c + bj * block, st.seg_cnt + bj * block,
                          st.seg_vsum + bj * block * D, sm);
}

// Per-head totals n_c, S_c = sum over blocks of the block entries, in a fixed order.
// A warp per (head, 8 clusters), lanes over the value columns.  Per batch of 32 blocks, lane u
// looks up the 8 clusters' entries in block j0 + u (one 8-byte load of seg_idx); the present
// (block, cluster) pairs are compacted into a per-warp list ordered by block, then cluster; the
// list's entry rows are loaded 8 at a time and added, in list order, into the clusters'
// accumulators in shared memory.  Every cluster's sum therefore takes its blocks' entries in block
// order, the same fp32 additions in the same order as a walk over one cluster's blocks:
// deterministic bits, with 8 lookups per load and 8 row loads in flight.
template <int D>
__global__ void __launch_bounds__(128) totals_kernel(StatsPtrs st, int C, int block, int nB) {
  constexpr int NS = D / 32;              // columns per lane
  constexpr int G = 8;                    // clusters per warp
  constexpr int kWarps = 4;
  constexpr int kInFlight = 8;            // entry rows loaded per group
  __shared__ __align__(16) float s_acc[kWarps][G][D];
  __shared__ int s_list[kWarps][32 * G];  // (u << 11) | (g << 8) | entry
  __shared__ int s_n[kWarps][G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int c0 = (blockIdx.y * kWarps + warp) * G;
  if (c0 >= C) return;                    // (C is a multiple of 32: whole warps)
  float(*acc)[D] = s_acc[warp];
  int* list = s_list[warp];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int i = 0; i < NS; ++i) acc[g][lane * NS + i] = 0.f;
  if (lane < G) s_n[warp][lane] = 0;
  __syncwarp();
  const size_t hb = (size_t)bh * nB;
  for (int j0 = 0; j0 < nB; j0 += 32) {
    // lookups: the 8 entry indices of block j0 + lane
    uint2 w = make_uint2(0xFFFFFFFFu, 0xFFFFFFFFu);
    if (j0 + lane < nB) w = *reinterpret_cast<const uint2*>(st.seg_idx + (hb + j0 + lane) * C + c0);
    unsigned present = 0;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const unsigned e = ((g < 4 ? w.x : w.y) >> (8 * (g & 3))) & 0xFFu;
      present |= (e != 0xFFu ? 1u : 0u) << g;
    }
    // exclusive prefix of the counts over the lanes (blocks in order)
    const int cnt = __popc(present);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    int pos = incl - cnt;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (present & (1u << g)) {
        const unsigned e = ((g < 4 ? w.x : w.y) >> (8 * (g & 3))) & 0xFFu;
        list[pos++] = (lane << 11) | (g << 8) | (int)e;
      }
    }
    __syncwarp();
    for (int i0 = 0; i0 < total; i0 += kInFlight) {
      float y[kInFlight][NS];
      int cnt_k[kInFlight] = {};
      int item[kInFlight];
#pragma unroll
      for (int k = 0; k < kInFlight; ++k) {
        item[k] = i0 + k < total ? list[i0 + k] : -1;
        if (item[k] >= 0) {
          const size_t row = (hb + j0 + (item[k] >> 11)) * block + (item[k] & 0xFF);
          load_vec(st.seg_vsum + row * D + lane * NS, y[k], NS);
          cnt_k[k] = lane == 0 ? st.seg_cnt[row] : 0;
        }
      }
#pragma unroll
      for (int k = 0; k < kInFlight; ++k) {
        if (item[k] >= 0) {                 // warp-uniform
          const int g = (item[k] >> 8) & 7;
#pragma unroll
          for (int i = 0; i < NS; ++i) acc[g][lane * NS + i] += y[k][i];
          if (lane == 0) s_n[warp][g] += cnt_k[k];
        }
      }
    }
    __syncwarp();                           // the list is rewritten by the next batch
  }
  __syncwarp();
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float* dst = st.S_tot + ((size_t)bh * C + c0 + g) * D + lane * NS;
    if constexpr (NS == 4) {
      *reinterpret_cast<float4*>(dst) = *reinterpret_cast<const float4*>(&acc[g][lane * NS]);
    } else {
#pragma unroll
      for (int i = 0; i < NS; ++i) dst[i] = acc[g][lane * NS + i];
    }
  }
  if (lane < G) st.n_tot[(size_t)bh * C + c0 + lane] = s_n[warp][lane];
}

// Second moment of each cluster's keys about its representative (the variance correction of
// the ESTRA abstract, read as a diagonal Gaussian about cbar_c):
//   D[c, t] = (1 / n_c) sum over the keys k with a(k) = c of (k_t - cbar_{c,t})^2  (0 when n_c = 0).
// A warp per (head, cluster), lanes over the columns: it walks the blocks that hold the cluster
// (seg_idx) in order and, in each, the block's keys of the cluster in index order (a ballot over
// the assignments), so the sums are taken in a fixed order: deterministic bits.
template <typename T, int D>
__global__ void __launch_bounds__(128) cluster_spread_kernel(const T* __restrict__ K, const T* __restrict__ cent,
                                                             StatsPtrs st, float* __restrict__ spread, int N, int C,
                                                             int block, int nB) {
  constexpr int NS = D / 32;              // columns per lane
  const int bh = blockIdx.x;
  const int c = blockIdx.y * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (c >= C) return;                     // (C is a multiple of 32)
  float cb[NS], acc[NS];
  load_vec(cent + ((size_t)bh * C + c) * D + lane * NS, cb, NS);
#pragma unroll
  for (int i = 0; i < NS; ++i) acc[i] = 0.f;
  const size_t hb = (size_t)bh * nB;
  const int32_t* arow = st.assign + (size_t)bh * N;
  const T* krow = K + (size_t)bh * N * D + lane * NS;
  // Blocks are looked up 32 at a time (lane u: block j0 + u); in each block holding the cluster,
  // its keys are found from the block's assignments (four independent loads) and their rows are
  // loaded up to eight at a time, then added in key order: the order of a plain walk over the
  // blocks and their keys.
  constexpr int kRows = 8;
  for (int j0 = 0; j0 < nB; j0 += 32) {
    const int jl = j0 + lane;
    unsigned pm = __ballot_sync(0xffffffffu, jl < nB && st.seg_idx[(hb + jl) * C + c] != 0xFF);
    while (pm) {
      const int j = j0 + __ffs(pm) - 1;
      pm &= pm - 1u;
      const int k0 = j * block;
      const int nk = min(block, N - k0);
      unsigned km[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int kk = 32 * q + lane;
        km[q] = __ballot_sync(0xffffffffu, kk < nk && arow[k0 + kk] == c);
      }
      // the cluster's keys of the block, in index order: keys 0-63 in lo, 64-127 in hi
      unsigned long long lo = (unsigned long long)km[0] | ((unsigned long long)km[1] << 32);
      unsigned long long hi = (unsigned long long)km[2] | ((unsigned long long)km[3] << 32);
      while (lo | hi) {
        int idx[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          int k = -1;
          if (lo) {
            k = __ffsll((long long)lo) - 1;
            lo &= lo - 1ull;
          } else if (hi) {
            k = 64 + __ffsll((long long)hi) - 1;
            hi &= hi - 1ull;
          }
          idx[r] = k;
        }
        float kv[kRows][NS];
#pragma unroll
        for (int r = 0; r < kRows; ++r)
          if (idx[r] >= 0) load_vec(krow + (size_t)(k0 + idx[r]) * D, kv[r], NS);
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          if (idx[r] >= 0) {
#pragma unroll
            for (int i = 0; i < NS; ++i) {
              const float dv = kv[r][i] - cb[i];
              acc[i] = fmaf(dv, dv, acc[i]);
            }
          }
        }
      }
    }
  }
  const int n = st.n_tot[(size_t)bh * C + c];
  const float inv = n > 0 ? 1.f / (float)n : 0.f;
  float* dst = spread + ((size_t)bh * C + c) * D + lane * NS;
#pragma unroll
  for (int i = 0; i < NS; ++i) dst[i] = acc[i] * inv;
}

// Plan validation and work order: items of a head ordered by descending row length
// (ties by q-block index); heads in order.  A malformed row is reported and scheduled with
// cost 0 (the attention kernels skip its invalid entries).
__global__ void schedule_kernel(const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ kv_cnt,
                                int max_sel, int nB, int32_t* __restrict__ schedule, int* status) {
  extern __shared__ int cost[];
  const int bh = blockIdx.x;
  for (int i = threadIdx.x; i < nB; i += blockDim.x) {
    const size_t item = (size_t)bh * nB + i;
    const int cnt = kv_cnt[item];
    bool ok = cnt >= 0 && cnt <= max_sel;
    if (ok) {
      int prev = -1;
      const int32_t* row = kv_idx + item * max_sel;
      for (int s = 0; s < cnt; ++s) {
        const int j = row[s];
        if (j <= prev || j >= nB) { ok = false; break; }
        prev = j;
      }
    }
    if (!ok) set_status(status, DA_ERR_DEVICE_INDEX);
    cost[i] = ok ? cnt : 0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nB; i += blockDim.x) {
    const int ci = cost[i];
    int rank = 0;
    for (int i2 = 0; i2 < nB; ++i2) {
      const int c2 = cost[i2];
      rank += (c2 > ci) || (c2 == ci && i2 < i);
    }
    schedule[(size_t)bh * nB + rank] = bh * nB + i;
  }
}

// Dh = (scale / 2) D rounded to bf16; one thread per 4 values (C * d is a multiple of 4).
__global__ void spread_half_kernel(const float4* __restrict__ D, float half_scale, uint2* __restrict__ out,
                                   long long n4) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 v = D[i];
  out[i] = make_uint2(pack_bf16x2(v.x * half_scale, v.y * half_scale), pack_bf16x2(v.z * half_scale, v.w * half_scale));
}

// ------------------------------------------------------------------------------------------
// launches

cudaError_t launch_centroid_norms(const Dims& g, const void* cent, float* norms, cudaStream_t s) {
  const long long rows = (long long)g.B * g.H * g.C;
  const unsigned grid = (unsigned)((rows + 3) / 4);
  if (g.bf16)
    centroid_norms_kernel<<<grid, 128, 0, s>>>((const __nv_bfloat16*)cent, norms, rows, g.d);
  else
    centroid_norms_kernel<<<grid, 128, 0, s>>>((const float*)cent, norms, rows, g.d);
  return cudaGetLastError();
}

cudaError_t launch_block_stats(const Dims& g, const void* V, const StatsPtrs& st, cudaStream_t s) {
  dim3 grid(g.nB, g.B * g.H);
#define DA_STATS(T, DD) block_stats_kernel<T, DD><<<grid, 128, 0, s>>>((const T*)V, st, g.N, g.C, g.block, g.nB)
  if (g.bf16) {
    if (g.d == 128) DA_STATS(__nv_bfloat16, 128); else DA_STATS(__nv_bfloat16, 64);
  } else {
    if (g.d == 128) DA_STATS(float, 128); else DA_STATS(float, 64);
  }
#undef DA_STATS
  return cudaGetLastError();
}

// Lloyd update (least-squares quantisation): centroid c <- S_c / n_c, where the totals were taken
// with the keys as values; a centroid without keys stays where it is.  One thread per (row, column).
template <typename T>
__global__ void centroid_update_kernel(const float* __restrict__ S, const int32_t* __restrict__ n, T* cent,
                                       long long rows, int d) {
  const long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= rows * d) return;
  const long long r = x / d;
  const int cnt = n[r];
  if (cnt <= 0) return;
  const float v = S[x] / (float)cnt;
  if constexpr (std::is_same<T, float>::value) cent[x] = v;
  else cent[x] = __float2bfloat16_rn(v);
}

cudaError_t launch_centroid_update(const Dims& g, const StatsPtrs& st, void* cent, cudaStream_t s) {
  const long long rows = (long long)g.B * g.H * g.C;
  const long long total = rows * g.d;
  const unsigned grid = (unsigned)((total + 255) / 256);
  if (g.bf16)
    centroid_update_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(st.S_tot, st.n_tot, (__nv_bfloat16*)cent, rows, g.d);
  else
    centroid_update_kernel<float><<<grid, 256, 0, s>>>(st.S_tot, st.n_tot, (float*)cent, rows, g.d);
  return cudaGetLastError();
}

cudaError_t launch_totals(const Dims& g, const StatsPtrs& st, cudaStream_t s) {
  dim3 grid(g.B * g.H, (g.C + 31) / 32);                // 4 warps of 8 clusters per CTA
  if (g.d == 128) totals_kernel<128><<<grid, 128, 0, s>>>(st, g.C, g.block, g.nB);
  else totals_kernel<64><<<grid, 128, 0, s>>>(st, g.C, g.block, g.nB);
  return cudaGetLastError();
}

cudaError_t launch_cluster_spread(const Dims& g, const void* K, const void* cent, const StatsPtrs& st, float* spread,
                                  cudaStream_t s) {
  dim3 grid(g.B * g.H, (g.C + 3) / 4);                  // 4 clusters (warps) per CTA
#define DA_SPREAD(T, DD) \
  cluster_spread_kernel<T, DD><<<grid, 128, 0, s>>>((const T*)K, (const T*)cent, st, spread, g.N, g.C, g.block, g.nB)
  if (g.bf16) {
    if (g.d == 128) DA_SPREAD(__nv_bfloat16, 128); else DA_SPREAD(__nv_bfloat16, 64);
  } else {
    if (g.d == 128) DA_SPREAD(float, 128); else DA_SPREAD(float, 64);
  }
#undef DA_SPREAD
  return cudaGetLastError();
}

cudaError_t launch_spread_half(const Dims& g, const float* spread, float scale, void* out, cudaStream_t s) {
  const long long n4 = (long long)g.B * g.H * g.C * g.d / 4;
  const unsigned grid = (unsigned)((n4 + 255) / 256);
  spread_half_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float4*>(spread), 0.5f * scale,
                                           static_cast<uint2*>(out), n4);
  return cudaGetLastError();
}

cudaError_t launch_schedule(const Dims& g, const int32_t* kv_idx, const int32_t* kv_cnt, int max_sel,
                            int32_t* schedule, int* status, cudaStream_t s) {
  const size_t smem = (size_t)g.nB * sizeof(int);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(schedule_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  schedule_kernel<<<g.B * g.H, 256, smem, s>>>(kv_idx, kv_cnt, max_sel, g.nB, schedule, status);
  return cudaGetLastError();
}

}  // namespace da
