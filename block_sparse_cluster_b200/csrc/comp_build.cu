// Compensation chunks of every work item (the "compensation" half of decoupled sparse attention).
//
// DecoupAttn abstract: every key outside the q-block's exact blocks is compensated through its
// semantic cluster.  For work item (head, q-block i) with selected blocks sel(i) and cluster c:
//   n^U_c    = n_c - sum_{j in sel} n_{c,j}                      (keys of c outside sel(i))
//   vbar^U_c = (S_c - sum_{j in sel} S_{c,j}) / n^U_c            (their mean value, fp32 -> bf16)
//   beta_c   = log2 n^U_c  (-inf when n^U_c = 0)                 (the count weight, log2 units)
// One CTA per (item, 128-cluster chunk) writes the chunk as 128 bf16 rows of d = 128 (the layout a
// TMA tile load reads) followed by the 128 fp32 beta values.
//
// Phase 1: thread t <-> cluster row t of the chunk looks the row up in every selected block
// (seg_idx: the entry of the cluster in the block, or 0xFF) with independent loads, keeping the
// first kSlots entries in block order and the selected count.  Phase 2: each warp builds 16 rows
// with lanes over d (coalesced 512-byte rows): S_c minus the entries' value sums, summed in block
// order, times 1 / n^U_c.
#include "da_common.cuh"
#include "da_internal.h"

namespace da {

namespace {

constexpr int kD = 128;
constexpr int kRows = 128;               // clusters per chunk
constexpr int kSlots = 8;                // entries per row kept from phase 1
constexpr int kThreads = 256;            // 8 warps: 16 rows each in phase 2
constexpr int kChunkBytes = kRows * kD * 2 + kRows * 4;

struct Smem {
  uint32_t ptr[kRows][kSlots];           // entry rows (block row * block + entry), block order
  int nm[kRows];                         // entries of the row in the selected blocks
  float inv[kRows];                      // 1 / n^U (0 when n^U = 0)
};

__device__ __forceinline__ float4 ldg4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }

__global__ void __launch_bounds__(kThreads)
comp_build_kernel(StatsPtrs st, const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ kv_cnt,
                  int max_sel, int N, int C, int nB, int block, int nchunk, uint8_t* __restrict__ out) {
  __shared__ Smem sm;
  const int item = blockIdx.x / nchunk;
  const int c = blockIdx.x - item * nchunk;
  const int bh = item / nB;
  const int t = threadIdx.x;
  int nsel = kv_cnt[item];
  if (nsel < 0 || nsel > max_sel) nsel = 0;            // reported by the schedule pass
  const int32_t* row = kv_idx + (size_t)item * max_sel;
  const size_t hb = (size_t)bh * nB;                   // first block row of the head
  const size_t hc = (size_t)bh * C;                    // first cluster row of the head
  uint8_t* chunk = out + (size_t)blockIdx.x * kChunkBytes;

  if (t < kRows) {
    const int r = c * kRows + t;
    const bool rl = r < C;
    int nm = 0, csel = 0;
    uint32_t mp[kSlots];
#pragma unroll
    for (int k = 0; k < kSlots; ++k) mp[k] = 0;
#pragma unroll 8
    for (int s = 0; s < nsel; ++s) {
      const int jr = row[s];
      const bool ok = rl && jr >= 0 && jr < nB;
      const size_t bj = hb + (ok ? jr : 0);
      const int e = ok ? (int)st.seg_idx[bj * C + r] : 0xFF;
      const bool hit = e != 0xFF;
      csel += hit ? st.blk_hist[bj * C + r] : 0;
      const uint32_t ptr = (uint32_t)(bj * block + (hit ? e : 0));
#pragma unroll
      for (int k = 0; k < kSlots; ++k) mp[k] = (hit && nm == k) ? ptr : mp[k];
      nm += hit ? 1 : 0;
    }
    const int nU = rl ? st.n_tot[hc + r] - csel : 0;
#pragma unroll
    for (int k = 0; k < kSlots; ++k) sm.ptr[t][k] = mp[k];
    sm.nm[t] = nm;
    sm.inv[t] = nU > 0 ? 1.f / (float)nU : 0.f;
    reinterpret_cast<float*>(chunk + kRows * kD * 2)[t] = nU > 0 ? log2f((float)nU) : -INFINITY;
  }
  __syncthreads();

  const int w = t >> 5, lane = t & 31;
  for (int i0 = 0; i0 < 16; i0 += 4) {
    float4 a[4];
    int nmq[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = 16 * w + i0 + q;
      const int r = c * kRows + i;
      nmq[q] = sm.nm[i];
      a[q] = r < C ? ldg4(st.S_tot + (hc + r) * kD + 4 * lane) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float4 acc[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kSlots; ++k) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (nmq[q] > k) {                               // warp-uniform
          const float4 y = ldg4(st.seg_vsum + (size_t)sm.ptr[16 * w + i0 + q][k] * kD + 4 * lane);
          acc[q].x += y.x; acc[q].y += y.y; acc[q].z += y.z; acc[q].w += y.w;
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = 16 * w + i0 + q;
      const int r = c * kRows + i;
      if (nmq[q] > kSlots) {
        // rare: the cluster sits in more than kSlots selected blocks; the remaining entries, in
        // block order
        int seen = 0;
        for (int s = 0; s < nsel; ++s) {
          const int jr = row[s];
          if (jr < 0 || jr >= nB) continue;
          const size_t bj = hb + jr;
          const int e = st.seg_idx[bj * C + r];
          if (e == 0xFF) continue;
          if (seen++ >= kSlots) {
            const float4 y = ldg4(st.seg_vsum + (bj * block + e) * kD + 4 * lane);
            acc[q].x += y.x; acc[q].y += y.y; acc[q].z += y.z; acc[q].w += y.w;
          }
        }
      }
      const float iv = sm.inv[i];
      const float4 v = make_float4((a[q].x - acc[q].x) * iv, (a[q].y - acc[q].y) * iv, (a[q].z - acc[q].z) * iv,
                                   (a[q].w - acc[q].w) * iv);
      uint2 o;
      o.x = pack_bf16x2(v.x, v.y);
      o.y = pack_bf16x2(v.z, v.w);
      *reinterpret_cast<uint2*>(chunk + (size_t)i * (kD * 2) + lane * 8) = o;
    }
  }
}

}  // namespace

size_t comp_chunk_bytes() { return kChunkBytes; }

cudaError_t launch_comp_build(const Dims& g, const int32_t* kv_idx, const int32_t* kv_cnt, int max_sel,
                              const StatsPtrs& st, void* out, cudaStream_t s) {
  const int nchunk = (g.C + kRows - 1) / kRows;
  const long long ctas = (long long)g.B * g.H * g.nB * nchunk;
  if (ctas >= (1LL << 31)) return cudaErrorInvalidValue;
  comp_build_kernel<<<(unsigned)ctas, kThreads, 0, s>>>(st, kv_idx, kv_cnt, max_sel, g.N, g.C, g.nB, g.block, nchunk,
                                                        static_cast<uint8_t*>(out));
  return cudaGetLastError();
}

}  // namespace da
