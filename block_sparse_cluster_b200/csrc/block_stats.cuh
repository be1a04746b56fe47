// Per-block refresh of the compensation statistics (Reassign Cache, second half).
//
// "each step reassigns the drifting keys to cached centroids and refreshes compensation"
// (DecoupAttn abstract).  Given the cluster of every key of one key block, one group of 128
// threads writes that block's
//   - dense histogram row  n_{c,j}            (blk_hist[j][0..C))
//   - entry index row      e(c) or 0xFF        (seg_idx[j][0..C))
//   - sorted entry list    (c, n_{c,j})        (seg_c, seg_cnt, seg_n)
//   - value sum per entry  S_{c,j} = sum v_k   (seg_vsum, fp32, keys summed in index order)
// The block's keys are ranked by (cluster, key index), so every entry is a contiguous run and
// the sums are reduced in a fixed order: no atomics, deterministic bits.
#pragma once

#include "da_common.cuh"

namespace da {

struct StatsSmem {
  int sorted_key[128];
  int sorted_c[128];
  int start_pos[132];
  int warp_cnt[4];
  int hist_row[1024];
  uint8_t idx_row[1024];
};

// Synchronise the 128 threads of named barrier `bar_id` (1..15).
__device__ __forceinline__ void group_sync(int bar_id) {
  asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
}

// t: thread index within the group (0..127); every thread of the group must call this.
// s_assign: the block's clusters in shared memory (nk <= 128 entries, each in [0, C)).
// Vblk: value rows of the block (row k at Vblk + k*D).  Output pointers are already offset to
// this block.
template <typename T, int D>
__device__ void block_stats_group(int t, int bar_id, const int* s_assign, int nk, const T* __restrict__ Vblk,
                                  int C, int32_t* __restrict__ hist_out, uint8_t* __restrict__ idx_out,
                                  int32_t* __restrict__ segn_out, int32_t* __restrict__ segc_out,
                                  int32_t* __restrict__ segcnt_out, float* __restrict__ vsum_out,
                                  StatsSmem& sm) {
  const int warp = t >> 5, lane = t & 31;
  if (t < nk) {
    const int a_t = s_assign[t];
    int rank = 0;
    for (int k = 0; k < nk; ++k) {
      const int ak = s_assign[k];
      rank += (ak < a_t) || (ak == a_t && k < t);
    }
    sm.sorted_key[rank] = t;
    sm.sorted_c[rank] = a_t;
  }
  for (int c = t; c < C; c += 128) {
    sm.hist_row[c] = 0;
    sm.idx_row[c] = 0xFF;
  }
  group_sync(bar_id);

  const bool start = (t < nk) && (t == 0 || sm.sorted_c[t] != sm.sorted_c[t - 1]);
  const unsigned ballot = __ballot_sync(0xffffffffu, start);
  if (lane == 0) sm.warp_cnt[warp] = __popc(ballot);
  group_sync(bar_id);
  int before = 0, E = 0;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int c = sm.warp_cnt[w];
    before += (w < warp) ? c : 0;
    E += c;
  }
  const int e = before + __popc(ballot & ((1u << lane) - 1u));
  if (start) sm.start_pos[e] = t;
  if (t == 0) sm.start_pos[E] = nk;
  group_sync(bar_id);

  if (t < E) {
    const int p0 = sm.start_pos[t], p1 = sm.start_pos[t + 1];
    const int c = sm.sorted_c[p0];
    segc_out[t] = c;
    segcnt_out[t] = p1 - p0;
    sm.hist_row[c] = p1 - p0;
    sm.idx_row[c] = (uint8_t)t;
  }
  if (t == 0) *segn_out = E;
  group_sync(bar_id);

  for (int c = t; c < C; c += 128) hist_out[c] = sm.hist_row[c];
  {
    uint32_t* dst = reinterpret_cast<uint32_t*>(idx_out);
    const uint32_t* src = reinterpret_cast<const uint32_t*>(sm.idx_row);
    for (int w4 = t; w4 < C / 4; w4 += 128) dst[w4] = src[w4];
  }

  constexpr int NE = D / 32;
  for (int ee = warp; ee < E; ee += 4) {
    const int p0 = sm.start_pos[ee], p1 = sm.start_pos[ee + 1];
    float acc[NE];
#pragma unroll
    for (int i = 0; i < NE; ++i) acc[i] = 0.f;
    for (int p = p0; p < p1; ++p) {
      const int k = sm.sorted_key[p];
      float v[NE];
      load_vec(Vblk + (size_t)k * D + lane * NE, v, NE);
#pragma unroll
      for (int i = 0; i < NE; ++i) acc[i] += v[i];
    }
    float* dst = vsum_out + (size_t)ee * D + lane * NE;
    if constexpr (NE == 4) {
      *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    } else {
#pragma unroll
      for (int i = 0; i < NE; ++i) dst[i] = acc[i];
    }
  }
  group_sync(bar_id);
}

}  // namespace da
