// Compensation chunks of every work item (the "compensation" half of decoupled sparse attention).
//
// DecoupAttn abstract: every key outside the q-block's exact blocks is compensated through its
// semantic cluster.  For work item (head, q-block i) with selected blocks sel(i) and cluster c:
//   n^U_c    = n_c - sum_{j in sel} n_{c,j}                      (keys of c outside sel(i))
//   vbar^U_c = (S_c - sum_{j in sel} S_{c,j}) / n^U_c            (their mean value, fp32 -> bf16)
//   beta_c   = log2 n^U_c  (-inf when n^U_c = 0)                 (the count weight, log2 units)
// One CTA per (item, 128-cluster chunk), in chunk-major order, writes the chunk as 128 bf16 rows
// of d = 128 (the layout a TMA tile load reads) followed by the 128 fp32 beta values.
//
// Phase 0: the item's selected blocks are validated once into shared memory (tiles of kThreads).
// Phase 1: thread (row, h) looks the row up in half h of the selected blocks (seg_idx: the entry
// of the cluster in the block, or 0xFF) with batches of independent loads, keeping the first
// kSlots entries of its half in block order and the half's selected count.  The two halves'
// entries are then merged per row, slot k of both halves before slot k + 1 (a fixed order).
// Phase 2: each warp builds 16 rows with lanes over d (coalesced 512-byte rows): S_c minus the
// entries' value sums in merged order, times 1 / n^U_c.
#include "da_common.cuh"
#include "da_internal.h"

namespace da {

namespace {

constexpr int kD = 128;
constexpr int kRows = 128;               // clusters per chunk
constexpr int kSlots = 4;                // entries per (row, half) kept from phase 1
constexpr int kThreads = 256;            // phase 1: (row, half); phase 2: 8 warps x 16 rows
constexpr int kBatch = 4;                // lookups in flight per thread
constexpr int kGroup = 2;                // rows whose loads a warp issues together in phase 2
constexpr int kChunkBytes = kRows * kD * 2 + kRows * 4;

struct Smem {
  uint32_t ptr[2][kRows][kSlots];        // entry rows (block row * block + entry), block order
  uint32_t lst[kRows][2 * kSlots];       // both halves' kept entries, merged slot-major
  int nm[2][kRows];                      // entries of the row in each half of the selected blocks
  int csel[2][kRows];                    // selected keys of the cluster in each half
  int ne[kRows];                         // merged entries of the row
  float inv[kRows];                      // 1 / n^U (0 when n^U = 0)
  int jsel[kThreads];                    // a tile of the selected blocks, -1 where out of range
};

__device__ __forceinline__ float4 ldg4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }

__device__ __forceinline__ void add4(float4& a, const float4& y) {
  a.x += y.x; a.y += y.y; a.z += y.z; a.w += y.w;
}

__global__ void __launch_bounds__(kThreads, 4)
comp_build_kernel(StatsPtrs st, const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ kv_cnt,
                  int max_sel, int N, int C, int nB, int block, int nchunk, uint8_t* __restrict__ out) {
  __shared__ Smem sm;
  // chunk-major order: the CTAs resident at one time share the chunk, so its S_c rows and the
  // blocks' lookup rows are served from L1
  const int n_items = gridDim.x / nchunk;
  const int c = blockIdx.x / n_items;
  const int item = blockIdx.x - c * n_items;
  const int bh = item / nB;
  const int t = threadIdx.x;
  int nsel = kv_cnt[item];
  if (nsel < 0 || nsel > max_sel) nsel = 0;            // reported by the schedule pass
  const int32_t* row = kv_idx + (size_t)item * max_sel;
  const size_t hb = (size_t)bh * nB;                   // first block row of the head
  const size_t hc = (size_t)bh * C;                    // first cluster row of the head
  const uint8_t* seg_idx_h = st.seg_idx + hb * C;      // the head's lookup rows (nB * C < 2^31)
  const int32_t* blk_hist_h = st.blk_hist + hb * C;
  const uint32_t eb = (uint32_t)(hb * block);          // first entry row of the head
  uint8_t* chunk = out + ((size_t)item * nchunk + c) * kChunkBytes;

  const int rr = t & (kRows - 1), h = t / kRows;
  const int r = c * kRows + rr;
  const bool rl = r < C;
  const int mid = (nsel + 1) >> 1;
  const int sb = h ? mid : 0, se = h ? nsel : mid;
  int nm = 0, cs = 0;
  for (int t0 = 0; t0 < nsel; t0 += kThreads) {        // CTA-uniform
    __syncthreads();                                   // the previous tile has been read
    if (t0 + t < nsel) {
      const int jr = __ldg(row + t0 + t);
      sm.jsel[t] = (jr >= 0 && jr < nB) ? jr : -1;
    }
    __syncthreads();
    const int lo = max(sb, t0), hi = min(se, t0 + kThreads);
    for (int s0 = lo; s0 < hi; s0 += kBatch) {
      int e[kBatch], hv[kBatch];
      uint32_t bb[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int sidx = s0 + u;
        const int jr = sidx < hi ? sm.jsel[sidx - t0] : -1;
        const bool ok = rl && jr >= 0;
        const int o = ok ? jr * C + r : 0;
        bb[u] = eb + (uint32_t)(jr * block);
        e[u] = ok ? (int)__ldg(seg_idx_h + o) : 0xFF;
        hv[u] = ok ? __ldg(blk_hist_h + o) : 0;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        if (e[u] != 0xFF) {
          if (nm < kSlots) sm.ptr[h][rr][nm] = bb[u] + (uint32_t)e[u];
          ++nm;
        }
        cs += hv[u];                                     // zero where the cluster is absent
      }
    }
  }
  sm.nm[h][rr] = nm;
  sm.csel[h][rr] = cs;
  __syncthreads();
  if (t < kRows) {
    const int rc = c * kRows + t;
    const int nU = rc < C ? st.n_tot[hc + rc] - sm.csel[0][t] - sm.csel[1][t] : 0;
    sm.inv[t] = nU > 0 ? 1.f / (float)nU : 0.f;
    reinterpret_cast<float*>(chunk + kRows * kD * 2)[t] = nU > 0 ? log2f((float)nU) : -INFINITY;
    const int a0 = min(sm.nm[0][t], kSlots), a1 = min(sm.nm[1][t], kSlots);
    int n = 0;
#pragma unroll
    for (int k = 0; k < kSlots; ++k) {
      if (k < a0) sm.lst[t][n++] = sm.ptr[0][t][k];
      if (k < a1) sm.lst[t][n++] = sm.ptr[1][t][k];
    }
    sm.ne[t] = n;
  }
  __syncthreads();

  const int w = t >> 5, lane = t & 31;
  const float* vs = st.seg_vsum + 4 * lane;
  for (int i0 = 0; i0 < 16; i0 += kGroup) {
    float4 a[kGroup], acc[kGroup];
    int ne[kGroup];
    int emax = 0;
#pragma unroll
    for (int q = 0; q < kGroup; ++q) {
      const int i = 16 * w + i0 + q;
      const int rc = c * kRows + i;
      ne[q] = sm.ne[i];
      emax = max(emax, ne[q]);
      a[q] = rc < C ? ldg4(st.S_tot + (hc + rc) * kD + 4 * lane) : make_float4(0.f, 0.f, 0.f, 0.f);
      acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int e = 0; e < emax; ++e) {                     // warp-uniform
      float4 y[kGroup];
#pragma unroll
      for (int q = 0; q < kGroup; ++q)
        if (e < ne[q]) y[q] = ldg4(vs + (size_t)sm.lst[16 * w + i0 + q][e] * kD);
#pragma unroll
      for (int q = 0; q < kGroup; ++q)
        if (e < ne[q]) add4(acc[q], y[q]);
    }
#pragma unroll
    for (int q = 0; q < kGroup; ++q) {
      const int i = 16 * w + i0 + q;
      const int rc = c * kRows + i;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (sm.nm[hh][i] <= kSlots) continue;            // warp-uniform
        // rare: the cluster sits in more than kSlots blocks of this half; the rest, in block order
        const int hb0 = hh ? mid : 0, he = hh ? nsel : mid;
        int seen = 0;
        for (int sidx = hb0; sidx < he; ++sidx) {
          const int jr = row[sidx];
          if (jr < 0 || jr >= nB) continue;
          const int ei = seg_idx_h[jr * C + rc];
          if (ei == 0xFF) continue;
          if (seen++ >= kSlots) add4(acc[q], ldg4(vs + (size_t)(eb + (uint32_t)(jr * block + ei)) * kD));
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
  if (ctas >= (1LL << 31) || (long long)g.nB * g.C >= (1LL << 31)) return cudaErrorInvalidValue;   // also refused by the ABI
  comp_build_kernel<<<(unsigned)ctas, kThreads, 0, s>>>(st, kv_idx, kv_cnt, max_sel, g.N, g.C, g.nB, g.block, nchunk,
                                                        static_cast<uint8_t*>(out));
  return cudaGetLastError();
}

}  // namespace da
