// Fused decoupled sparse attention on the tensor cores (bf16, d = 128, block = 128).
//
// DecoupAttn abstract: exact attention runs on a few key blocks fixed by position, and every
// other key is compensated through its semantic cluster, with "one fused compensation kernel".
// For q-block i with selected blocks sel(i), the kernel runs one online softmax over
//   - the keys of the selected blocks:            logit s q.k,  value v_k;
//   - one column per cluster with n^U_c > 0:     logit s q.cbar_c + ln n^U_c,  value vbar^U_c,
// where n^U_c = n_c - sum_{j in sel} n_{c,j} and vbar^U_c = (S_c - sum_{j in sel} S_{c,j}) / n^U_c
// are the count and mean value of the cluster's keys outside the selected blocks.
//
// Work: items (head, q-block) from the plan's work order; a persistent CTA per SM walks
// items blockIdx.x, blockIdx.x + gridDim.x, ...  An item is a sequence of steps: one per selected
// block, then one per 128-cluster chunk.  Every step is a 128 x 128 score tile S = Q K^T (K a
// key block or a centroid chunk) and a P V product (V a value block or the chunk's vbar^U rows).
//
// Roles (384 threads, three warpgroups):
//   warps 0-3  softmax: thread t owns query row t = TMEM lane t; online softmax with lazy
//              rescaling (the running max only moves when it grows by more than 2^8), P written
//              back to TMEM as bf16, final normalisation and store of O;
//   warps 4-7  builder: thread t owns cluster row t of a chunk; builds vbar^U (bf16, in the
//              swizzled operand layout) and log2 n^U in shared memory;
//   warp 8     producer: TMA loads of Q, K / V blocks and centroid chunks into a 3-stage ring;
//   warp 9     MMA: allocates TMEM, issues tcgen05.mma S(g+1) = Q K^T ahead of O += P(g) V(g);
//   warps 10-11 idle.
// TMEM columns: S double buffer [0,128) and [128,256), O [256,384).
#include "da_common.cuh"
#include "da_internal.h"
#include "tma_host.h"

namespace da {

namespace {

constexpr int kD = 128;
constexpr int kBM = 128;                 // query rows per item
constexpr int kBN = 128;                 // keys per block / clusters per chunk
constexpr int kStages = 3;
constexpr int kTile = kBN * kD * 2;      // 32 KB bf16 tile
constexpr int kPanel = kBN * 128;        // one 64-column panel (128 rows x 128 B)
constexpr float kRescaleLog2 = 8.0f;     // lazy rescale threshold (factor 256)
constexpr int kThreads = 384;            // three warpgroups
constexpr int kWarpProducer = 8;
constexpr int kWarpMMA = 9;
// Register split (setmaxnreg): the launch holds 384 x 168 registers; the softmax and builder
// warpgroups grow, the producer / MMA warpgroup shrinks.
constexpr int kRegSoftmax = 240, kRegBuilder = 200, kRegIssue = 56;
static_assert(128 * (kRegSoftmax + kRegBuilder + kRegIssue) <= kThreads * 168, "register split above the launch");
constexpr int kBatch = 16;               // selected blocks looked up per round by the builder

struct __align__(8) Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kStages], v_full[kStages], st_empty[kStages], bfree[kStages];
  uint64_t s_full[2], p_ready[2];
  uint64_t o_done, o_free, drain;
  uint32_t tmem_base;
  int abort;
  volatile int bld_ok[2];
};

constexpr size_t kSmemBytes =
    1024 + kTile /*Q*/ + 2 * kStages * kTile /*K,V*/ + kStages * kBN * sizeof(float) /*beta*/ + sizeof(Bars);
static_assert(kSmemBytes <= 232448, "shared memory above the 227 KB per-block limit");

struct Params {
  const int32_t* kv_idx;
  const int32_t* kv_cnt;
  const int32_t* schedule;
  int max_sel;
  StatsPtrs st;
  __nv_bfloat16* O;
  float* lse;
  int* status;
  int N, C, nB, n_items, nchunk;
  float scale_log2;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Item geometry shared by every role.
struct Item {
  int bh, i, q0, qlen, nsel, T;
  const int32_t* row;
};

__device__ __forceinline__ Item item_at(const Params& p, int k) {
  Item it;
  int item = p.schedule[k];
  if (item < 0 || item >= p.n_items) item = 0;      // reported by the schedule pass
  it.bh = item / p.nB;
  it.i = item - it.bh * p.nB;
  it.q0 = it.i * kBM;
  it.qlen = min(kBM, p.N - it.q0);
  int cnt = p.kv_cnt[item];
  if (cnt < 0 || cnt > p.max_sel) cnt = 0;
  it.nsel = cnt;
  it.T = cnt + p.nchunk;
  it.row = p.kv_idx + (size_t)item * p.max_sel;
  return it;
}

// Key block of exact step s; an out-of-range index becomes a fully masked block 0.
__device__ __forceinline__ int block_of(const Params& p, const Item& it, int s, bool* valid) {
  const int j = it.row[s];
  *valid = (j >= 0 && j < p.nB);
  return *valid ? j : 0;
}

// One row of a compensation chunk: cluster cl of the item's head.  Packs
// vbar^U = (S_c - sum_{j in sel} S_{c,j}) / n^U_c as bf16 pairs and returns log2 n^U_c
// (-inf when the cluster has no key outside the selected blocks or cl >= C).  The selected
// blocks are looked up kBatch at a time with independent loads (the entry index of cluster cl in
// block j is seg_idx[j][cl]); a hit subtracts that entry's value sum and count.
__device__ __forceinline__ void build_row(const Params& p, const Item& it, int cl, uint32_t (&packed)[64],
                                          float* beta) {
  if (cl >= p.C) {
#pragma unroll
    for (int v = 0; v < 64; ++v) packed[v] = 0u;
    *beta = -INFINITY;
    return;
  }
  const size_t hc = (size_t)it.bh * p.C + cl;
  float acc[kD];
  {
    const float4* tot = reinterpret_cast<const float4*>(p.st.S_tot + hc * kD);
#pragma unroll
    for (int v = 0; v < kD / 4; ++v) {
      const float4 x = tot[v];
      acc[4 * v] = x.x; acc[4 * v + 1] = x.y; acc[4 * v + 2] = x.z; acc[4 * v + 3] = x.w;
    }
  }
  int nU = p.st.n_tot[hc];
  const size_t head_blk = (size_t)it.bh * p.nB;
  for (int s0 = 0; s0 < it.nsel; s0 += kBatch) {
    int jb[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = s0 + u < it.nsel ? it.row[s0 + u] : -1;
      jb[u] = (j >= 0 && j < p.nB) ? j : -1;
    }
    int eb[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) eb[u] = jb[u] >= 0 ? (int)p.st.seg_idx[(head_blk + jb[u]) * p.C + cl] : 0xFF;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (eb[u] != 0xFF) {
        const size_t ent = (head_blk + jb[u]) * kBN + eb[u];
        nU -= p.st.seg_cnt[ent];
        const float4* sv = reinterpret_cast<const float4*>(p.st.seg_vsum + ent * kD);
#pragma unroll
        for (int v = 0; v < kD / 4; ++v) {
          const float4 x = sv[v];
          acc[4 * v] -= x.x; acc[4 * v + 1] -= x.y; acc[4 * v + 2] -= x.z; acc[4 * v + 3] -= x.w;
        }
      }
    }
  }
  const float inv = nU > 0 ? 1.f / (float)nU : 0.f;
  *beta = nU > 0 ? log2f((float)nU) : -INFINITY;
#pragma unroll
  for (int v = 0; v < 64; ++v) packed[v] = pack_bf16x2(acc[2 * v] * inv, acc[2 * v + 1] * inv);
}

__global__ void __launch_bounds__(kThreads, 1)
attention_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_c,
                    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = base;
  uint8_t* sK = sQ + kTile;                       // kStages tiles
  uint8_t* sV = sK + kStages * kTile;             // kStages tiles
  float* sBeta = reinterpret_cast<float*>(sV + kStages * kTile);   // [kStages][kBN]
  Bars* bars = reinterpret_cast<Bars*>(sBeta + kStages * kBN);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->st_empty[s], 1);
      mbar_init(&bars->bfree[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->p_ready[b], 128);
    }
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->o_free, 128);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMMA) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;
  int* status = p.status;

  if (warp >= 8) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegIssue));
  if (warp == kWarpProducer) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch(&tm_q);
      tma_prefetch(&tm_k);
      tma_prefetch(&tm_v);
      tma_prefetch(&tm_c);
      uint32_t g = 0;
      uint32_t exact_bits = 0;           // bit x: the last load into slot x carried a value block
      int n = 0, nq = 0;                 // items walked, query tiles loaded
      for (int k = blockIdx.x; k < p.n_items && !*abort; k += gridDim.x, ++n) {
        const Item it = item_at(p, k);
        if (!mbar_wait(&bars->q_empty, (n & 1) ^ 1, abort, status)) break;
        ++nq;
        mbar_expect_tx(&bars->q_full, kTile);
        tma_load_3d(sQ, &tm_q, &bars->q_full, 0, it.q0, it.bh);
        tma_load_3d(sQ + kPanel, &tm_q, &bars->q_full, 64, it.q0, it.bh);
        bool ok = true;
        for (int s = 0; s < it.T; ++s, ++g) {
          const int slot = g % kStages;
          const uint32_t u = g / kStages;
          if (!mbar_wait(&bars->st_empty[slot], (u & 1) ^ 1, abort, status)) { ok = false; break; }
          uint8_t* dk = sK + slot * kTile;
          if (s < it.nsel) {
            bool valid;
            const int j = block_of(p, it, s, &valid);
            uint8_t* dv = sV + slot * kTile;
            mbar_expect_tx(&bars->k_full[slot], kTile);
            tma_load_3d(dk, &tm_k, &bars->k_full[slot], 0, j * kBN, it.bh);
            tma_load_3d(dk + kPanel, &tm_k, &bars->k_full[slot], 64, j * kBN, it.bh);
            mbar_expect_tx(&bars->v_full[slot], kTile);
            tma_load_3d(dv, &tm_v, &bars->v_full[slot], 0, j * kBN, it.bh);
            tma_load_3d(dv + kPanel, &tm_v, &bars->v_full[slot], 64, j * kBN, it.bh);
            exact_bits |= 1u << slot;
          } else {
            exact_bits &= ~(1u << slot);
            const int c = s - it.nsel;
            mbar_arrive(&bars->bfree[slot]);        // hand the value half of the slot to the builder
            mbar_expect_tx(&bars->k_full[slot], kTile);
            tma_load_3d(dk, &tm_c, &bars->k_full[slot], 0, c * kBN, it.bh);
            tma_load_3d(dk + kPanel, &tm_c, &bars->k_full[slot], 64, c * kBN, it.bh);
          }
        }
        if (!ok) break;
      }
      // no copy may still be in flight when the CTA leaves (this matters only after an abort:
      // otherwise the MMA issuer has consumed every load)
      if (nq > 0) mbar_wait_drain(&bars->q_full, (nq - 1) & 1);
      for (uint32_t gd = g >= kStages ? g - kStages : 0; gd < g; ++gd) {
        const int slot = gd % kStages;
        mbar_wait_drain(&bars->k_full[slot], (gd / kStages) & 1);
        if ((exact_bits >> slot) & 1u) mbar_wait_drain(&bars->v_full[slot], (gd / kStages) & 1);
      }
    }
  } else if (warp == kWarpMMA) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16(kBM, kBN, 0, 0);   // Q, K both K-major
      const uint32_t idesc_pv = idesc_bf16(kBM, kD, 0, 1);    // P from TMEM, V MN-major
      const uint32_t q0 = smem_u32(sQ);
      uint32_t g = 0;
      int n = 0;
      auto issue_s = [&](uint32_t gs) {
        const int slot = gs % kStages;
        const uint32_t kb = smem_u32(sK + slot * kTile);
        const uint32_t d = tmem + (gs & 1) * kBN;
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kPanel + (ks & 3) * 32;
          umma_ss(d, sdesc_sw128(q0 + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024), idesc_qk, ks > 0);
        }
        umma_commit(&bars->s_full[gs & 1]);
      };
      bool ok = true;
      for (int k = blockIdx.x; k < p.n_items && ok; k += gridDim.x, ++n) {
        const Item it = item_at(p, k);
        if (!mbar_wait(&bars->q_full, n & 1, abort, status)) break;
        tc_fence_after();
        const uint32_t g0 = g;
        if (!mbar_wait(&bars->k_full[g0 % kStages], (g0 / kStages) & 1, abort, status)) break;
        tc_fence_after();
        issue_s(g0);
        for (int s = 0; s < it.T; ++s, ++g) {
          if (s + 1 < it.T) {
            const uint32_t gn = g + 1;
            if (!mbar_wait(&bars->k_full[gn % kStages], (gn / kStages) & 1, abort, status)) { ok = false; break; }
            tc_fence_after();
            issue_s(gn);
          } else {
            umma_commit(&bars->q_empty);
          }
          const int slot = g % kStages;
          if (!mbar_wait(&bars->p_ready[g & 1], (g >> 1) & 1, abort, status)) { ok = false; break; }
          if (!mbar_wait(&bars->v_full[slot], (g / kStages) & 1, abort, status)) { ok = false; break; }
          if (s == 0 && !mbar_wait(&bars->o_free, (n & 1) ^ 1, abort, status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t vb = smem_u32(sV + slot * kTile);
          const uint32_t pt = tmem + (g & 1) * kBN;       // P: bf16 pairs in the S buffer's first 64 columns
#pragma unroll
          for (int ks = 0; ks < kBN / 16; ++ks) {
            // V rows (keys) 16*ks .. 16*ks+15: two 8-row groups of 1024 B
            umma_ts(tmem + 2 * kBN, pt + ks * 8, sdesc_sw128(vb + ks * 2048, kPanel, 1024), idesc_pv,
                    (s > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(&bars->st_empty[slot]);
          umma_commit(&bars->o_done);
        }
      }
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0);
    }
  } else if (warp >= 8) {
    // warps 10-11: idle
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ builder
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegBuilder));
    const int t = tid - 128;                  // row t of every chunk
    uint32_t g = 0, nb = 0;                   // global step, chunks built so far
    uint32_t use_par = 0;                     // bit x: parity of the chunks built into slot x so far
    // (no abort test in the loop condition: the builders leave together, on bld_ok)
    for (int k = blockIdx.x; k < p.n_items; k += gridDim.x) {
      const Item it = item_at(p, k);
      g += it.nsel;
      bool ok = true;
      for (int c = 0; c < p.nchunk; ++c, ++g) {
        uint32_t packed[64];
        float beta;
        build_row(p, it, c * kBN + t, packed, &beta);
        const int slot = g % kStages;
        // The producer, which follows every phase of the ring, releases the slot's value half
        // through bfree[slot] once the slot is empty; its phases are this builder's uses of the
        // slot, in order.  One thread waits; the decision reaches every builder warp through a
        // named barrier so that they leave (or go on) together.
        const uint32_t use = (use_par >> slot) & 1u;
        use_par ^= 1u << slot;
        if (t == 0) bars->bld_ok[nb & 1] = mbar_wait(&bars->bfree[slot], use, abort, status);
        asm volatile("bar.sync 2, 128;" ::: "memory");
        if (!bars->bld_ok[(nb++) & 1]) { ok = false; break; }
        // row t of the value operand: panel d / 64, 16-byte chunk (d % 64) / 8, 128-byte swizzle
        uint8_t* rowp = sV + slot * kTile + t * 128;
#pragma unroll
        for (int ch = 0; ch < 16; ++ch) {
          const int panel = ch >> 3, cc = ch & 7;
          const uint4 v = make_uint4(packed[4 * ch], packed[4 * ch + 1], packed[4 * ch + 2], packed[4 * ch + 3]);
          *reinterpret_cast<uint4*>(rowp + panel * kPanel + ((cc ^ (t & 7)) << 4)) = v;
        }
        sBeta[slot * kBN + t] = beta;
        fence_async_smem();
        asm volatile("bar.sync 2, 128;" ::: "memory");
        if (t == 0) mbar_arrive(&bars->v_full[slot]);
      }
      if (!ok) break;
    }
  } else {
    // ------------------------------------------------------------------ softmax (warps 0-3)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegSoftmax));
    const int r = tid;                                        // query row = TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    uint32_t g = 0;
    // (no abort test in the loop condition: a warp leaves as a whole, on its __all_sync'd waits)
    for (int k = blockIdx.x; k < p.n_items; k += gridDim.x) {
      const Item it = item_at(p, k);
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int s = 0; s < it.T; ++s, ++g) {
        const int b = g & 1;
        const int slot = g % kStages;
        const bool comp = s >= it.nsel;
        int ncol = kBN;                       // valid columns of this tile
        if (!comp) {
          bool valid;
          const int j = block_of(p, it, s, &valid);
          ncol = valid ? min(kBN, p.N - j * kBN) : 0;
        }
        // every phase of v_full and s_full is waited, in order (the value half of a compensation
        // step carries the chunk's log2 n^U in sBeta)
        bool w_ok = mbar_wait(&bars->v_full[slot], (g / kStages) & 1, abort, status);
        w_ok = w_ok && mbar_wait(&bars->s_full[b], (g >> 1) & 1, abort, status);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        tc_fence_after();
        float x[kBN];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t rr[32];
          tmem_ld32(lane_addr + b * kBN + q * 32, rr);
          tmem_wait_ld();
#pragma unroll
          for (int v = 0; v < 32; ++v) x[q * 32 + v] = __uint_as_float(rr[v]);
        }
        float mx = -INFINITY;
        if (comp) {
          const float* bt = sBeta + slot * kBN;
#pragma unroll
          for (int c = 0; c < kBN; ++c) {
            x[c] = fmaf(x[c], p.scale_log2, bt[c]);
            mx = fmaxf(mx, x[c]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < kBN; ++c) {
            x[c] = c < ncol ? x[c] * p.scale_log2 : -INFINITY;
            mx = fmaxf(mx, x[c]);
          }
        }
        // lazy rescaling: the running max moves only when it grows by more than 2^8
        const bool grow = mx > m + kRescaleLog2 || (m == -INFINITY && mx > -INFINITY);
        const bool need_o = grow && s > 0 && m > -INFINITY;
        const float m_new = grow ? mx : m;
        const float mu = (m_new == -INFINITY) ? 0.f : m_new;
        float rs = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t pk[16];
#pragma unroll
          for (int v = 0; v < 16; ++v) {
            const float p0 = ex2(x[q * 32 + 2 * v] - mu);
            const float p1 = ex2(x[q * 32 + 2 * v + 1] - mu);
            rs += p0 + p1;
            pk[v] = pack_bf16x2(p0, p1);
          }
          tmem_st16(lane_addr + b * kBN + q * 16, pk);
        }
        if (s > 0) {
          // PV(g-1) has landed in O: every phase of o_done is waited, in order; a row whose max
          // moved rescales its O (warp-uniform, as tcgen05.ld/st are)
          const bool d_ok = mbar_wait(&bars->o_done, (g - 1) & 1, abort, status);
          if (!__all_sync(0xffffffffu, d_ok)) { ok = false; break; }
          tc_fence_after();
          if (__any_sync(0xffffffffu, need_o)) {
            const float alpha = need_o ? ex2(m - m_new) : 1.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t rr[32];
              tmem_ld32(lane_addr + 2 * kBN + q * 32, rr);
              tmem_wait_ld();
#pragma unroll
              for (int v = 0; v < 32; ++v) rr[v] = __float_as_uint(__uint_as_float(rr[v]) * alpha);
              tmem_st32(lane_addr + 2 * kBN + q * 32, rr);
            }
            if (need_o) l *= alpha;
          }
        }
        m = m_new;
        l += rs;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_ready[b]);
      }
      if (!ok) break;
      // epilogue: O / l once the item's last PV has landed
      const uint32_t glast = g - 1;
      const bool e_ok = mbar_wait(&bars->o_done, glast & 1, abort, status);
      if (!__all_sync(0xffffffffu, e_ok)) break;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const bool live = r < it.qlen;
      __nv_bfloat16* op = p.O + ((size_t)it.bh * p.N + it.q0 + r) * kD;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t rr[32];
        tmem_ld32(lane_addr + 2 * kBN + q * 32, rr);
        tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(rr[8 * v + 0]) * inv, __uint_as_float(rr[8 * v + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(rr[8 * v + 2]) * inv, __uint_as_float(rr[8 * v + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(rr[8 * v + 4]) * inv, __uint_as_float(rr[8 * v + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(rr[8 * v + 6]) * inv, __uint_as_float(rr[8 * v + 7]) * inv);
            *reinterpret_cast<uint4*>(op + q * 32 + v * 8) = w;
          }
        }
      }
      if (live && p.lse) p.lse[(size_t)it.bh * p.N + it.q0 + r] = (m + __log2f(l)) * 0.69314718055994531f;
      tc_fence_before();
      mbar_arrive(&bars->o_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool attention_tc_supported(const Dims& g) { return g.bf16 && g.d == kD && g.block == kBN; }

cudaError_t launch_attention_tc(const Dims& g, const void* Q, const void* K, const void* V,
                                const int32_t* kv_idx, const int32_t* kv_cnt, int max_sel,
                                const int32_t* schedule, const void* cent, const StatsPtrs& st, float scale,
                                void* O, float* lse, int* status, cudaStream_t s) {
  CUtensorMap tq, tk, tv, tc;
  const unsigned long long BH = (unsigned long long)g.B * g.H;
  if (!make_tmap_bf16_3d(&tq, Q, kD, g.N, BH, 64, kBM) || !make_tmap_bf16_3d(&tk, K, kD, g.N, BH, 64, kBN) ||
      !make_tmap_bf16_3d(&tv, V, kD, g.N, BH, 64, kBN) || !make_tmap_bf16_3d(&tc, cent, kD, g.C, BH, 64, kBN))
    return cudaErrorInvalidValue;
  Params p;
  p.kv_idx = kv_idx;
  p.kv_cnt = kv_cnt;
  p.schedule = schedule;
  p.max_sel = max_sel;
  p.st = st;
  p.O = (__nv_bfloat16*)O;
  p.lse = lse;
  p.status = status;
  p.N = g.N;
  p.C = g.C;
  p.nB = g.nB;
  p.n_items = (int)(BH * g.nB);
  p.nchunk = (g.C + kBN - 1) / kBN;
  p.scale_log2 = scale * 1.4426950408889634f;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaError_t e = cudaFuncSetAttribute(attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = min(sms, p.n_items);
  attention_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, tc, p);
  return cudaGetLastError();
}

}  // namespace da
