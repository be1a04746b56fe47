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
  int sorted_key[128];     // the block's keys ranked by (cluster, key index)
  int start_pos[132];      // first rank of each entry; start_pos[E] = nk
  int scan_c[8], scan_f[8];
  int hist_row[1024];      // n_{c,j}; then, for a cluster present in the block, its first rank
  uint8_t idx_row[1024];
};

// Synchronise the NT threads of named barrier `bar_id` (1..15).
template <int NT>
__device__ __forceinline__ void group_sync(int bar_id) {
  asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "n"(NT) : "memory");
}

// t: thread index within the group of NT = 128 or 256 threads; every thread of the group must
// call this.
// s_assign: the block's clusters in shared memory (nk <= 128 entries, each in [0, C)).
// Vblk: value rows of the block (row k at Vblk + k*D).  Output pointers are already offset to
// this block.
//   1. Keys with equal clusters are grouped per warp (match_any); the warps, in order, add their
//      groups to the histogram row, so a key's rank among its cluster's keys is its key-index
//      rank, without atomics.
//   2. One scan over the clusters gives each present cluster its entry index and its first rank.
//   3. A warp per entry sums the run's value rows in rank order, lanes over the columns.
template <typename T, int D, int NT = 128>
__device__ void block_stats_group(int t, int bar_id, const int* s_assign, int nk, const T* __restrict__ Vblk,
                                  int C, int32_t* __restrict__ hist_out, uint8_t* __restrict__ idx_out,
                                  int32_t* __restrict__ segn_out, int32_t* __restrict__ segc_out,
                                  int32_t* __restrict__ segcnt_out, float* __restrict__ vsum_out,
                                  StatsSmem& sm) {
  const int warp = t >> 5, lane = t & 31;
  const unsigned below = (1u << lane) - 1u;
  static_assert(NT == 128 || NT == 256, "a group of 4 or 8 warps");
  const int a_t = t < nk ? s_assign[t] : C;          // C: no key (also every thread t >= 128)
  const unsigned peers = __match_any_sync(0xffffffffu, a_t);
  const int r_in = __popc(peers & below);
  const bool leader = (peers & below) == 0u;
  for (int c = t; c < C; c += NT) sm.hist_row[c] = 0;
  group_sync<NT>(bar_id);
  int before = 0;                                     // keys of the cluster in earlier warps
#pragma unroll 1
  for (int w = 0; w < 4; ++w) {
    if (warp == w && leader && a_t < C) {
      before = sm.hist_row[a_t];
      sm.hist_row[a_t] = before + __popc(peers);
    }
    group_sync<NT>(bar_id);
  }
  before = __shfl_sync(0xffffffffu, before, __ffs(peers) - 1);

  // exclusive scan over the clusters of (count, present): thread t owns clusters [t*cp, t*cp + cp)
  const int cp = (C + NT - 1) / NT;
  const int c0 = t * cp;
  int cnt = 0, flg = 0;
  for (int i = 0; i < cp; ++i) {
    const int c = c0 + i;
    if (c < C) {
      const int h = sm.hist_row[c];
      cnt += h;
      flg += h > 0 ? 1 : 0;
    }
  }
  int ic = cnt, ifl = flg;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int yc = __shfl_up_sync(0xffffffffu, ic, o);
    const int yf = __shfl_up_sync(0xffffffffu, ifl, o);
    if (lane >= o) {
      ic += yc;
      ifl += yf;
    }
  }
  if (lane == 31) {
    sm.scan_c[warp] = ic;
    sm.scan_f[warp] = ifl;
  }
  group_sync<NT>(bar_id);
  int run_c = ic - cnt, run_f = ifl - flg, E = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    run_c += w < warp ? sm.scan_c[w] : 0;
    run_f += w < warp ? sm.scan_f[w] : 0;
    E += sm.scan_f[w];
  }
  for (int i = 0; i < cp; ++i) {
    const int c = c0 + i;
    if (c < C) {
      const int h = sm.hist_row[c];
      hist_out[c] = h;
      if (h > 0) {
        sm.idx_row[c] = (uint8_t)run_f;
        sm.start_pos[run_f] = run_c;
        segc_out[run_f] = c;
        segcnt_out[run_f] = h;
        sm.hist_row[c] = run_c;                       // from here on: the cluster's first rank
        run_c += h;
        ++run_f;
      } else {
        sm.idx_row[c] = 0xFF;
      }
    }
  }
  if (t == 0) {
    *segn_out = E;
    sm.start_pos[E] = nk;
  }
  group_sync<NT>(bar_id);

  if (t < nk) sm.sorted_key[sm.hist_row[a_t] + before + r_in] = t;
  {
    uint32_t* dst = reinterpret_cast<uint32_t*>(idx_out);
    const uint32_t* src = reinterpret_cast<const uint32_t*>(sm.idx_row);
    for (int w4 = t; w4 < C / 4; w4 += NT) dst[w4] = src[w4];
  }
  group_sync<NT>(bar_id);

  // value sums: warp w takes entries w, w + NT/32, ...; lane l holds columns [l*D/32, (l+1)*D/32);
  // the run's keys are added in rank order, two rows in flight at a time
  constexpr int NE = D / 32;
  for (int ee = warp; ee < E; ee += NT / 32) {
    const int p0 = sm.start_pos[ee], p1 = sm.start_pos[ee + 1];
    float acc[NE];
#pragma unroll
    for (int i = 0; i < NE; ++i) acc[i] = 0.f;
    int p = p0;
    for (; p + 1 < p1; p += 2) {
      const int ka = sm.sorted_key[p], kb = sm.sorted_key[p + 1];
      float va[NE], vb[NE];
      load_vec(Vblk + (size_t)ka * D + lane * NE, va, NE);
      load_vec(Vblk + (size_t)kb * D + lane * NE, vb, NE);
#pragma unroll
      for (int i = 0; i < NE; ++i) acc[i] += va[i];
#pragma unroll
      for (int i = 0; i < NE; ++i) acc[i] += vb[i];
    }
    if (p < p1) {
      float va[NE];
      load_vec(Vblk + (size_t)sm.sorted_key[p] * D + lane * NE, va, NE);
#pragma unroll
      for (int i = 0; i < NE; ++i) acc[i] += va[i];
    }
    float* dst = vsum_out + (size_t)ee * D + lane * NE;
    if constexpr (NE == 4) {
      *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    } else {
#pragma unroll
      for (int i = 0; i < NE; ++i) dst[i] = acc[i];
    }
  }
  group_sync<NT>(bar_id);
}

}  // namespace da
