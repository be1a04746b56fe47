// Reassign Cache on the tensor cores (bf16, d = 128, block = 128).
//
// "each step reassigns the drifting keys to cached centroids and refreshes compensation"
// (DecoupAttn abstract).  One CTA per (head, key block of 128 keys):
//   1. TMA loads the key tile (128 x 128 bf16, 128-byte swizzle) and the centroid chunks
//      (128 x 128 bf16 each, double buffered).
//   2. One thread issues tcgen05.mma: D[key, c] = k . cbar_c into TMEM (fp32, 128 columns per
//      chunk, two TMEM buffers so the next chunk's contraction overlaps this chunk's epilogue).
//   3. Every thread owns one key (= one TMEM lane) and keeps the running argmin of
//      ||cbar_c||^2 - 2 k.cbar_c (ties to the lowest c; the key's own norm is the same for
//      every c and is dropped).
//   4. The same 128 threads refresh the block's statistics (block_stats.cuh): sorted entry list,
//      histogram row, entry index row and fp32 value sums, reading the block's value rows from
//      shared memory (copied with cp.async into centroid buffer 0 once the last MMA reading it is
//      done, overlapping the remaining epilogues).
// The CTA takes about 109 KB of shared memory and 256 TMEM columns, so two CTAs share an SM and
// one's contraction overlaps the other's argmin and statistics.
#include "block_stats.cuh"
#include "da_common.cuh"
#include "da_internal.h"
#include "tma_host.h"

namespace da {

namespace {

constexpr int kKeys = 128;           // keys per tile (= block)
constexpr int kD = 128;              // head dimension
constexpr int kChunk = 128;          // centroids per MMA chunk (N of the MMA)
constexpr int kMaxC = 1024;          // centroid norms staged in shared memory
constexpr int kKTileBytes = kKeys * kD * 2;        // 32 KB
constexpr int kCTileBytes = kChunk * kD * 2;       // 32 KB
constexpr int kPanelK = kKeys * 128;               // one 64-column panel of the key tile
constexpr int kPanelC = kChunk * 128;              // one 64-column panel of a centroid chunk
constexpr int kThreads = 256;                      // two warpgroups: each half of every chunk's columns

struct __align__(8) Bars {
  uint64_t kfull;
  uint64_t cfull[2];
  uint64_t mdone[2];
  uint64_t tfree[2];      // TMEM buffer read out by all 8 warps (one arrival per warp)
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes = 1024 /*align slack*/ + kKTileBytes /*K*/ + 2 * kCTileBytes + kMaxC * 4 /*norms*/ +
                              sizeof(StatsSmem) + 512 /*assign*/ + 1024 /*second half's minima*/ + 128 /*bars*/;
static_assert(sizeof(Bars) <= 128, "barrier block");
static_assert(2 * (kSmemBytes + 1024) <= 233472, "two CTAs per SM");

__global__ void __launch_bounds__(kThreads, 2)
reassign_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_c,
                   const __nv_bfloat16* __restrict__ V, const float* __restrict__ norms, StatsPtrs st, int N,
                   int C, int nB, int* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sK = base;
  uint8_t* sC0 = sK + kKTileBytes;
  float* s_norm = reinterpret_cast<float*>(sC0 + 2 * kCTileBytes);
  StatsSmem* ssm = reinterpret_cast<StatsSmem*>(s_norm + kMaxC);
  int* s_assign = reinterpret_cast<int*>(ssm + 1);
  float* s_hbest = reinterpret_cast<float*>(s_assign + 128);   // warpgroup 1's (distance, cluster)
  int* s_harg = reinterpret_cast<int*>(s_hbest + 128);
  Bars* bars = reinterpret_cast<Bars*>(s_harg + 128);

  const int t = threadIdx.x;
  const int warp = t >> 5;
  const int half = t >> 7;                           // columns [64 half, 64 half + 64) of each chunk
  const int row = t & 127;                           // key = TMEM lane
  const int j = blockIdx.x;
  const int bh = blockIdx.y;
  const int k0 = j * kKeys;
  const int nk = min(kKeys, N - k0);
  const int nchunks = (C + kChunk - 1) / kChunk;

  if (t == 0) {
    mbar_init(&bars->kfull, 1);
    mbar_init(&bars->cfull[0], 1);
    mbar_init(&bars->cfull[1], 1);
    mbar_init(&bars->mdone[0], 1);
    mbar_init(&bars->mdone[1], 1);
    mbar_init(&bars->tfree[0], kThreads / 32);
    mbar_init(&bars->tfree[1], kThreads / 32);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&bars->tmem_base, 2 * kChunk);
    tmem_relinquish();
  }
  for (int c = t; c < C; c += kThreads) s_norm[c] = norms[(size_t)bh * C + c];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  auto load_chunk = [&](int c) {
    uint8_t* dst = sC0 + (c & 1) * kCTileBytes;
    mbar_expect_tx(&bars->cfull[c & 1], kCTileBytes);
    tma_load_3d(dst, &tm_c, &bars->cfull[c & 1], 0, c * kChunk, bh);
    tma_load_3d(dst + kPanelC, &tm_c, &bars->cfull[c & 1], 64, c * kChunk, bh);
  };
  auto issue_mma = [&](int c) -> bool {
    // TMEM buffer c & 1 was last written for chunk c - 2: every warp must have read it out
    if (c >= 2 && !mbar_wait(&bars->tfree[c & 1], ((c - 2) >> 1) & 1, abort, status)) return false;
    if (!mbar_wait(&bars->cfull[c & 1], (c >> 1) & 1, abort, status)) return false;
    tc_fence_after();
    const int n = min(kChunk, C - c * kChunk);
    const uint32_t idesc = idesc_bf16(128, n, 0, 0);
    const uint32_t a0 = smem_u32(sK), b0 = smem_u32(sC0 + (c & 1) * kCTileBytes);
#pragma unroll
    for (int ks = 0; ks < kD / 16; ++ks) {
      const uint32_t koff = (ks & 3) * 32;
      const uint64_t ad = sdesc_sw128(a0 + (ks >> 2) * kPanelK + koff, 16, 1024);
      const uint64_t bd = sdesc_sw128(b0 + (ks >> 2) * kPanelC + koff, 16, 1024);
      umma_ss(tmem + (c & 1) * kChunk, ad, bd, idesc, ks > 0 ? 1u : 0u);
    }
    umma_commit(&bars->mdone[c & 1]);
    return true;
  };

  if (t == 0) {
    tma_prefetch(&tm_k);
    tma_prefetch(&tm_c);
    mbar_expect_tx(&bars->kfull, kKTileBytes);
    tma_load_3d(sK, &tm_k, &bars->kfull, 0, k0, bh);
    tma_load_3d(sK + kPanelK, &tm_k, &bars->kfull, 64, k0, bh);
    load_chunk(0);
    if (nchunks > 1) load_chunk(1);
    if (mbar_wait(&bars->kfull, 0, abort, status)) issue_mma(0);
  }

  // four running minima per thread over disjoint groups of 16 columns (shorter dependency
  // chains); each visits its columns in ascending c and keeps the first of equal distances
  float best[4];
  int arg[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    best[a] = INFINITY;
    arg[a] = 0;
  }
  const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  for (int c = 0; c < nchunks; ++c) {
    if (t == 0 && c + 1 < nchunks && !*abort) issue_mma(c + 1);
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars->mdone[c & 1], (c >> 1) & 1, abort, status));
    tc_fence_after();
    // MMA(c) is done, so its centroid buffer is free: the next chunk for it loads during this epilogue
    if (t == 0 && c + 2 < nchunks && !*abort) load_chunk(c + 2);
    // buffer 0 after its last chunk: the block's value rows for the statistics
    if ((c & 1) == 0 && c + 2 >= nchunks && ok) {
      const __nv_bfloat16* Vg = V + ((size_t)bh * N + k0) * kD;
      for (int i = t; i < nk * kD / 8; i += kThreads) cp_async16(sC0 + (size_t)i * 16, Vg + (size_t)i * 8);
      cp_async_commit();
    }
    // C is a multiple of 32: the chunk has n / 32 full groups of 32 columns
    const int ngroups = ok ? min(kChunk, C - c * kChunk) >> 5 : 0;
    if (ngroups > 2 * half) {                         // warp-uniform
      uint32_t r[2][32];
#pragma unroll
      for (int q = 0; q < 2; ++q) tmem_ld32(lane_base + (c & 1) * kChunk + 64 * half + 32 * q, r[q]);
      tmem_wait_ld();
      const float4* nv = reinterpret_cast<const float4*>(s_norm + c * kChunk + 64 * half);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (2 * half + q < ngroups) {                 // warp-uniform
          int loc[2] = {-1, -1};                      // column (in the chunk) of a new minimum
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 nn = nv[8 * q + q4];
            const float nq[4] = {nn.x, nn.y, nn.z, nn.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int h = q4 >> 2;
              const float dist = fmaf(-2.f, __uint_as_float(r[q][4 * q4 + u]), nq[u]);
              if (dist < best[2 * q + h]) {
                best[2 * q + h] = dist;
                loc[h] = 32 * q + 4 * q4 + u;
              }
            }
          }
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (loc[h] >= 0) arg[2 * q + h] = c * kChunk + 64 * half + loc[h];
        }
      }
    }
    // this warp has read TMEM buffer c & 1: the MMA of chunk c + 2 may overwrite it
    tc_fence_before();
    __syncwarp();
    if ((t & 31) == 0) mbar_arrive(&bars->tfree[c & 1]);
  }
  // merge: the smallest distance, the lowest cluster among equal ones; warpgroup 1 hands its
  // minimum to warpgroup 0 through shared memory
  float bd = best[0];
  int ba = arg[0];
#pragma unroll
  for (int a = 1; a < 4; ++a) {
    if (best[a] < bd || (best[a] == bd && arg[a] < ba)) {
      bd = best[a];
      ba = arg[a];
    }
  }
  if (half == 1) {
    s_hbest[row] = bd;
    s_harg[row] = ba;
  }
  __syncthreads();
  if (half == 0) {
    const float b1 = s_hbest[row];
    const int a1 = s_harg[row];
    if (b1 < bd || (b1 == bd && a1 < ba)) {
      bd = b1;
      ba = a1;
    }
  }
  if (!*abort) {
    if (t < nk) {
      s_assign[t] = ba;
      st.assign[(size_t)bh * N + k0 + t] = ba;
    }
    cp_async_wait<0>();
    __syncthreads();
    const size_t bj = (size_t)bh * nB + j;
    block_stats_group<__nv_bfloat16, kD, kThreads>(t, 1, s_assign, nk, reinterpret_cast<const __nv_bfloat16*>(sC0), C,
                                                   st.blk_hist + bj * C, st.seg_idx + bj * C, st.seg_n + bj,
                                                   st.seg_c + bj * kKeys, st.seg_cnt + bj * kKeys,
                                                   st.seg_vsum + bj * kKeys * kD, *ssm);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kChunk);
  }
}

}  // namespace

bool reassign_tc_supported(const Dims& g) { return g.bf16 && g.d == kD && g.block == kKeys && g.C <= kMaxC; }

cudaError_t launch_reassign_tc(const Dims& g, const void* K, const void* V, const void* cent, const float* norms,
                               const StatsPtrs& st, int* status, cudaStream_t s) {
  CUtensorMap tk, tc;
  const unsigned long long BH = (unsigned long long)g.B * g.H;
  if (!make_tmap_bf16_3d(&tk, K, kD, g.N, BH, 64, kKeys)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_3d(&tc, cent, kD, g.C, BH, 64, kChunk)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(reassign_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(g.nB, (unsigned)BH);
  reassign_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(tk, tc, static_cast<const __nv_bfloat16*>(V), norms, st, g.N,
                                                   g.C, g.nB, status);
  return cudaGetLastError();
}

}  // namespace da
