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
// The cluster columns are taken in the per-key correction form, which needs no per-q-block table:
//   e^{s q.cbar_c} n^U_c vbar^U_c = e^{s q.cbar_c + ln n_c} (S_c / n_c)
//                                   - sum_{j in sel} e^{s q.cbar_c + ln n_{c,j}} (S_{c,j} / n_{c,j}),
// and the same with the counts alone for the denominator.  So an item's steps are
//   - one per selected block (exact keys);
//   - one per 128-cluster chunk of the head (centroid rows, bias log2 n_c, head-wide means);
//   - its entry tiles: the entries of its selected blocks, 128 rows at a time (centroid rows,
//     bias log2 n_e, negated entry means), whose weights leave the running sum.
// The Reassign Cache writes the chunk and entry operands (compensation tiles, include/da.h);
// the entry tiles are copied row-run by row-run with bulk copies, as they are stored swizzled.
//
// Work: items (head, q-block) from the plan's work order; a persistent CTA per SM walks
// items blockIdx.x, blockIdx.x + gridDim.x, ...  Every step is a 128 x 128 score tile S = Q K^T
// (K a key block, a centroid chunk or an entry tile) and a P V product.
//
// Inclusion-probability mode (AB-Attention abstract: sampled blocks "reweighted by inverse
// inclusion probability"): with p.incl, an item's steps are its selected blocks only (one fully
// masked step if it has none), and block j's logits carry the bias -log2 pi_j, i.e. the weight
// 1 / pi_j in both sums of the softmax; no cluster columns.
//
// Roles (384 threads):
//   warps 0-3, 4-7  two softmax warpgroups X = 0, 1 (barriers they arrive on count warps: lane 0
//              arrives after a warp barrier); warpgroup X takes the steps g with g & 1 = X of
//              every item, so the two overlap each other and the tensor core.  Thread t of a
//              warpgroup owns query row t = TMEM lane t.  It reads S into registers (S is then
//              free for S(g + 1)), takes the running max of the other warpgroup's latest step and
//              lets it grow lazily (only by more than 2^8), writes P as bf16 into its own P_X and
//              keeps its share of the row sum.  The two share one accumulator O: whichever raises
//              the max rescales O, once the previous product has landed.  At the end of an item
//              they exchange (max, sum) per row and each normalises and stores half of O's columns;
//   warp 8     producer: loads Q, key tiles / centroid chunks / entry centroid rows (3-stage ring,
//              so that a key tile loads while the two before it are read) and the softmax bias rows (4-stage ring, so a slot always serves the
//              same warpgroup);
//   warp 9     MMA issuer of S(g) = Q K^T (and TMEM allocation): at an item's start it copies the
//              query tile into tensor memory (tcgen05.cp), so S reads only the key tile from shared
//              memory; S(g) goes into the one score buffer once softmax(g - 1) has read it;
//   warp 10    producer of value tiles / cluster means / entry means (2-stage ring); a warp of its
//              own, since divergent lanes of one warp waiting on different barriers hold each other up;
//   warp 11    MMA issuer of O += P(g) V(g), a thread of its own: each issuer waits on its own
//              barriers while the other's products run, so the tensor core is fed from two queues.
// TMEM columns: S [0,128), O [128,256), P_0 [256,320), P_1 [320,384), Q_0 [384,448), Q_1 [448,512).
//
// Every mbarrier is waited at every phase, in order, by each role that waits on it (a parity
// wait is only meaningful within one phase); the host-side protocol model in the tests replays
// this schedule.
#include "da_common.cuh"
#include "da_internal.h"
#include "tma_host.h"

namespace da {

namespace {

constexpr int kD = 128;
constexpr int kBM = 128;                 // query rows per item
constexpr int kBN = 128;                 // keys per block / clusters per chunk
constexpr int kQStages = 1;             // query tiles (freed once the item's last S is computed)
constexpr int kKStages = 3;             // key / centroid tiles (freed as soon as S is computed)
constexpr int kVStages = 2;             // value / mean tiles (freed after P V)
constexpr int kBStages = 4;             // bias rows of the softmax (even: a slot serves one warpgroup)
constexpr int kTile = kBN * kD * 2;      // 32 KB bf16 tile
constexpr int kPanel = kBN * 128;        // one 64-column panel (128 rows x 128 B)
constexpr float kRescaleLog2 = 8.0f;     // lazy rescale threshold (factor 256)
constexpr int kEntSlots = 512;           // selected slots whose entry counts are prefetched
constexpr int kThreads = 384;           // three warpgroups; warp 11 idle
constexpr int kWarpProducer = 8;
constexpr int kWarpMMA = 9;
constexpr int kWarpProducerV = 10;
constexpr int kWarpPV = 11;
// Register split (setmaxnreg): the launch holds 384 x 168 registers; the softmax warpgroups grow,
// the producer / MMA warpgroup shrinks.
constexpr int kRegSoftmax = 232, kRegIssue = 40;
static_assert(128 * (2 * kRegSoftmax + kRegIssue) <= kThreads * 168, "register split above the launch");
static_assert(kBStages % 2 == 0, "a bias slot must always serve the same softmax warpgroup");
static_assert(kEntRows == kBN && kEntPanel == (size_t)kPanel, "entry tiles are read as key / value tiles");
// TMEM columns: the score buffer, the output accumulator, the two bf16 probability tiles and the
// two bf16 query tiles (the A operand of S = Q K^T, by item parity)
constexpr uint32_t kColS = 0, kColO = 128, kColP = 256, kColQ = 384;

struct __align__(8) Bars {
  uint64_t q_full[kQStages], q_empty[kQStages];   // query tile of item n in buffer n % kQStages
  uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  uint64_t b_full[kBStages], b_empty[kBStages];
  uint64_t s_full[2];                    // S(g) computed into S_{g & 1}
  uint64_t s_free[2];                    // softmax has read S_{g & 1} into registers
  uint64_t p_ready[2];                   // P(g) written into P_{g & 1}
  uint64_t p_free[2];                    // P(g) V(g) done: P_{g & 1} reusable, O holds step g
  uint64_t m_pub[2];                     // warpgroup X published its running max of step g
  uint64_t o_free, drain[2];
  // (max, sum) published at the end of an item: [item parity][warpgroup].  One barrier per item
  // parity: a warpgroup without steps in an item could otherwise complete a barrier twice before
  // the other warpgroup's parity wait on it runs.
  uint64_t xch_full[2][2];
  uint32_t tmem_base;
  int abort;
  int bflag[kBStages];                   // bit 0: the bias row is all zero (a full key block);
                                         // bit 1: an entry tile (its weights leave the sum)
  float mrow[2][kBM];                    // [warpgroup][row]: running max of its latest step
  float2 xch[2][2][kBM];                 // [item parity][warpgroup][row] = (max, sum)
  // entries of the current item's selected blocks, by slot, copied with cp.async by each producer
  // during its exact steps (one array per producer: the two run independently)
  int e8[2][kEntSlots];
};

constexpr size_t kSmemBytes = 1024 + (kQStages + kKStages + kVStages) * kTile /*Q,K,V*/ +
                              kBStages * kBN * sizeof(float) /*bias*/ + sizeof(Bars);
static_assert(kSmemBytes <= 232448, "shared memory above the 227 KB per-block limit");

struct Params {
  const int32_t* kv_idx;
  const int32_t* kv_cnt;
  const int32_t* schedule;
  int max_sel;
  const int32_t* seg_n;                  // entries per key block (from the Reassign Cache)
  const int32_t* ent_rows;               // [items] entry rows an item streams (entry_rows_kernel)
  const uint8_t* ent;                    // entry tiles, kEntTileBytes per (head, key block)
  const float* cbias;                    // [BH][cpad] log2 n_c
  __nv_bfloat16* O;
  float* lse;
  int* status;
  const float* incl;                     // [items][max_sel] inclusion probabilities, or NULL
  int N, C, nB, n_items, nchunk, cpad;
  float scale_log2;
};

// One arrival per warp: the lanes' earlier shared-memory and tensor-memory accesses are ordered
// before lane 0's arrive by the warp barrier (barrier counts are in warps, not threads, so that an
// arrival is one shared-memory atomic instead of 32).
__device__ __forceinline__ void warp_arrive(uint64_t* bar, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Rows of key block j's entry tile that an item streams: its entries, padded to a multiple of 8.
__device__ __forceinline__ int ent_rows_of(const int32_t* seg_n, int nB, int bh, int j) {
  const int e = __ldg(seg_n + (size_t)bh * nB + j);
  return (min(max(e, 0), kBN) + 7) & ~7;
}

// Item geometry shared by every role.
struct Item {
  int bh, i, q0, qlen, nsel, erows, T;
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
  it.erows = p.incl ? 0 : max(0, p.ent_rows[item]);
  it.T = p.incl ? max(cnt, 1) : cnt + p.nchunk + (it.erows + kBN - 1) / kBN;
  it.row = p.kv_idx + (size_t)item * p.max_sel;
  return it;
}

// Key block of exact step s; an out-of-range index becomes a fully masked block 0.
__device__ __forceinline__ int block_of(const Params& p, const Item& it, int s, bool* valid) {
  const int j = s < it.nsel ? it.row[s] : -1;
  *valid = (j >= 0 && j < p.nB);
  return *valid ? j : 0;
}

// Entry rows of selected slot s: its block's entry count was copied into e8s[s] by cp.async during
// the slot's exact step (slots beyond kEntSlots, or invalid blocks, are looked up here).
__device__ __forceinline__ int ent_rows_at(const Params& p, const Item& it, const int* e8s, int s) {
  bool valid;
  const int j = block_of(p, it, s, &valid);
  if (!valid) return 0;
  if (s < kEntSlots) return (min(max(e8s[s], 0), kBN) + 7) & ~7;
  return ent_rows_of(p.seg_n, p.nB, it.bh, j);
}

// Start the asynchronous copy of selected slot s's entry count into e8s[s] (exact step s).
__device__ __forceinline__ void ent_prefetch(const Params& p, const Item& it, int* e8s, int s, int j, bool valid) {
  if (s >= kEntSlots || !valid || p.incl) return;
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(e8s + s)),
               "l"(reinterpret_cast<uint64_t>(p.seg_n + (size_t)it.bh * p.nB + j))
               : "memory");
}

// One entry tile of `rows` rows: walks the item's selected blocks from the cursor (slot cs,
// source row cr of that block's entry tile) and calls emit(dst_row, block, src_row, nrows) for
// each run of rows, until the tile holds `rows` rows or the list ends.  Runs are multiples of 8
// rows, so each lands on the 1024-byte swizzle period it was stored for.
template <class F>
__device__ __forceinline__ void ent_tile_walk(const Params& p, const Item& it, const int* e8s, int rows, int& cs,
                                              int& cr, F&& emit) {
  int r0 = 0;
  while (r0 < rows && cs < it.nsel) {
    const int e8 = ent_rows_at(p, it, e8s, cs);
    const int take = min(e8 - cr, rows - r0);
    if (take > 0) {
      bool valid;
      emit(r0, block_of(p, it, cs, &valid), cr, take);
      r0 += take;
      cr += take;
    }
    if (cr >= e8) {
      ++cs;
      cr = 0;
    }
  }
}

// Orders later uses of r after a tcgen05.wait::ld already issued (emits no instruction).
__device__ __forceinline__ void reg_fence32(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

// Columns [0, 64) of the O row at o_col, times inv, stored as bf16 to out (warp-collective; once
// per item, so kept out of line).
__device__ __forceinline__ void store_row_half(uint32_t o_col, __nv_bfloat16* out, float inv, bool live) {
#pragma unroll 1
  for (int q = 0; q < 2; ++q) {
    uint32_t ra[32];
    tmem_ld32(o_col + 32 * q, ra);
    tmem_wait_ld();
    if (live) {
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(ra[8 * v + 0]) * inv, __uint_as_float(ra[8 * v + 1]) * inv);
        w.y = pack_bf16x2(__uint_as_float(ra[8 * v + 2]) * inv, __uint_as_float(ra[8 * v + 3]) * inv);
        w.z = pack_bf16x2(__uint_as_float(ra[8 * v + 4]) * inv, __uint_as_float(ra[8 * v + 5]) * inv);
        w.w = pack_bf16x2(__uint_as_float(ra[8 * v + 6]) * inv, __uint_as_float(ra[8 * v + 7]) * inv);
        *reinterpret_cast<uint4*>(out + q * 32 + v * 8) = w;
      }
    }
  }
}

// O row *= alpha in tensor memory (warp-collective; rare).
__device__ __forceinline__ void rescale_row(uint32_t o_row, float alpha) {
#pragma unroll 1
  for (int q = 0; q < 4; ++q) {
    uint32_t rr[32];
    tmem_ld32(o_row + q * 32, rr);
    tmem_wait_ld();
#pragma unroll
    for (int v = 0; v < 32; ++v) rr[v] = __float_as_uint(__uint_as_float(rr[v]) * alpha);
    tmem_st32(o_row + q * 32, rr);
  }
}

// Softmax of one S row held in registers (128 columns as raw fp32 bits).  A column's logit in
// log2 units is y_c = x_c * s*log2(e) + bias_c.  On a full key block the bias row is zero and
// the row max is taken on the raw scores (the scale is positive); otherwise y is formed in
// place first.  Returns the row max of y.
__device__ __forceinline__ float row_logits_max(uint32_t (&x)[4][32], const float* bias, bool plain, float sl2) {
  if (!plain) {
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int v = 0; v < 32; v += 4) {
        const float4 bb = *reinterpret_cast<const float4*>(bias + 32 * q + v);
        const uint64_t y0 = f2_fma(f2_pack(__uint_as_float(x[q][v]), __uint_as_float(x[q][v + 1])), sl2x2, f2_pack(bb.x, bb.y));
        const uint64_t y1 = f2_fma(f2_pack(__uint_as_float(x[q][v + 2]), __uint_as_float(x[q][v + 3])), sl2x2, f2_pack(bb.z, bb.w));
        float a, c, d, e;
        f2_unpack(y0, a, c);
        f2_unpack(y1, d, e);
        x[q][v] = __float_as_uint(a);
        x[q][v + 1] = __float_as_uint(c);
        x[q][v + 2] = __float_as_uint(d);
        x[q][v + 3] = __float_as_uint(e);
      }
  }
  float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int v = 0; v < 32; v += 8) {
      m0 = fmax3(m0, __uint_as_float(x[q][v]), __uint_as_float(x[q][v + 1]));
      m1 = fmax3(m1, __uint_as_float(x[q][v + 2]), __uint_as_float(x[q][v + 3]));
      m2 = fmax3(m2, __uint_as_float(x[q][v + 4]), __uint_as_float(x[q][v + 5]));
      m3 = fmax3(m3, __uint_as_float(x[q][v + 6]), __uint_as_float(x[q][v + 7]));
    }
  const float mr = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
  return plain ? mr * sl2 : mr;
}

// p = 2^(x * coef - mu) for the 32 columns of chunk q: packed to bf16 pairs in pk, summed (fp32
// pairs) into rsum.  coef is s*log2(e) on a full key block and 1 when x already holds y.
__device__ __forceinline__ void chunk_exp(const uint32_t (&x)[32], uint64_t coef, uint64_t negmu, uint32_t (&pk)[16],
                                          uint64_t& rsum) {
  uint64_t s0 = 0, s1 = 0;                // two accumulators: shorter dependency chains
#pragma unroll
  for (int v = 0; v < 16; ++v) {
    const uint64_t y = f2_fma(f2_pack(__uint_as_float(x[2 * v]), __uint_as_float(x[2 * v + 1])), coef, negmu);
    float a, c;
    f2_unpack(y, a, c);
    const float pa = ex2(a), pc = ex2(c);
    if (v & 1) s1 = f2_add(s1, f2_pack(pa, pc));
    else s0 = f2_add(s0, f2_pack(pa, pc));
    pk[v] = pack_bf16x2(pa, pc);
  }
  rsum = f2_add(rsum, f2_add(s0, s1));
}

// pk (bf16 pairs) *= f, in place.
__device__ __forceinline__ void scale_bf16x2(uint32_t (&pk)[16], float f) {
#pragma unroll
  for (int v = 0; v < 16; ++v) {
    const float lo = __uint_as_float(pk[v] << 16), hi = __uint_as_float(pk[v] & 0xFFFF0000u);
    pk[v] = pack_bf16x2(lo * f, hi * f);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
attention_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_c,
                    const __grid_constant__ CUtensorMap tm_m, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = base;                             // kQStages query tiles
  uint8_t* sK = sQ + kQStages * kTile;            // kKStages tiles
  uint8_t* sV = sK + kKStages * kTile;            // kVStages tiles
  float* sBias = reinterpret_cast<float*>(sV + kVStages * kTile);   // [kBStages][kBN]
  Bars* bars = reinterpret_cast<Bars*>(sBias + kBStages * kBN);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_free[b], 4);
      mbar_init(&bars->p_ready[b], 4);
      mbar_init(&bars->p_free[b], 1);
      mbar_init(&bars->m_pub[b], 4);
      mbar_init(&bars->xch_full[b][0], 4);
      mbar_init(&bars->xch_full[b][1], 4);
    }
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
    }
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&bars->b_full[s], 1);
      mbar_init(&bars->b_empty[s], 4);
    }
    mbar_init(&bars->o_free, 8);
    mbar_init(&bars->drain[0], 1);
    mbar_init(&bars->drain[1], 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  // Zero the key and value rings once: the rows past the end of an item's last entry tile keep
  // whatever an earlier step left there (their bias is -inf, so P is 0 there), which must be finite.
  for (int i = tid; i < (kKStages + kVStages) * kTile / 16; i += kThreads)
    reinterpret_cast<uint4*>(sK)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_async_smem();
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

  // the whole third warpgroup gives registers up at one instruction (setmaxnreg is warpgroup-wide)
  if (warp >= 8) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegIssue));

  if (warp == kWarpProducer) {
    // ------------------------------------------------------------------ producer (keys)
    // query tiles (double buffered), key / centroid / entry tiles and the softmax bias rows
    if (lane == 0) {
      tma_prefetch(&tm_q);
      tma_prefetch(&tm_k);
      tma_prefetch(&tm_c);
      uint32_t g = 0;
      int n = 0;                         // items walked = query tiles loaded
      for (int k = blockIdx.x; k < p.n_items && !*abort; k += gridDim.x) {
        const Item it = item_at(p, k);
        int cs = 0, cr = 0;                // entry cursor: selected slot, source row
        const int qs = n % kQStages;
        if (!mbar_wait(&bars->q_empty[qs], ((n / kQStages) & 1) ^ 1, abort, status)) break;
        mbar_expect_tx(&bars->q_full[qs], kTile);
        tma_load_3d(sQ + qs * kTile, &tm_q, &bars->q_full[qs], 0, it.q0, it.bh);
        tma_load_3d(sQ + qs * kTile + kPanel, &tm_q, &bars->q_full[qs], 64, it.q0, it.bh);
        ++n;
        bool ok = true;
        for (int s = 0; s < it.T; ++s, ++g) {
          const int ks = g % kKStages, bs = g % kBStages;
          if (!mbar_wait(&bars->k_empty[ks], ((g / kKStages) & 1) ^ 1, abort, status)) { ok = false; break; }
          uint8_t* dk = sK + ks * kTile;
          if (s < it.nsel || p.incl) {
            bool valid;
            const int j = block_of(p, it, s, &valid);
            mbar_expect_tx(&bars->k_full[ks], kTile);
            tma_load_3d(dk, &tm_k, &bars->k_full[ks], 0, j * kBN, it.bh);
            tma_load_3d(dk + kPanel, &tm_k, &bars->k_full[ks], 64, j * kBN, it.bh);
            ent_prefetch(p, it, bars->e8[0], s, j, valid);
            // bias row of a key block: 0 for its keys, -inf past the end of a short last block
            // (generic stores, published to the softmax by the arrive on b_full)
            if (!mbar_wait(&bars->b_empty[bs], ((g / kBStages) & 1) ^ 1, abort, status)) { ok = false; break; }
            int ncol = valid ? min(kBN, p.N - j * kBN) : 0;
            float w = 0.f;                 // log2 weight of the block's columns
            if (p.incl && ncol > 0) {
              const float pi = p.incl[(size_t)(it.bh * p.nB + it.i) * p.max_sel + s];
              if (pi > 0.f) w = -__log2f(pi);
              else ncol = 0;               // a block that is never included: left out
            }
            bars->bflag[bs] = (ncol == kBN && !p.incl) ? 1 : 0;
            float4* bb = reinterpret_cast<float4*>(sBias + bs * kBN);
#pragma unroll 4
            for (int c4 = 0; c4 < kBN / 4; ++c4) {
              const int c = 4 * c4;
              bb[c4] = make_float4(c < ncol ? w : -INFINITY, c + 1 < ncol ? w : -INFINITY,
                                   c + 2 < ncol ? w : -INFINITY, c + 3 < ncol ? w : -INFINITY);
            }
            mbar_arrive(&bars->b_full[bs]);
          } else if (s < it.nsel + p.nchunk) {
            // cluster chunk: centroid rows, bias log2 n_c
            const int c = s - it.nsel;
            mbar_expect_tx(&bars->k_full[ks], kTile);
            tma_load_3d(dk, &tm_c, &bars->k_full[ks], 0, c * kBN, it.bh);
            tma_load_3d(dk + kPanel, &tm_c, &bars->k_full[ks], 64, c * kBN, it.bh);
            if (!mbar_wait(&bars->b_empty[bs], ((g / kBStages) & 1) ^ 1, abort, status)) { ok = false; break; }
            bars->bflag[bs] = 0;
            mbar_expect_tx(&bars->b_full[bs], kBN * 4);
            bulk_load(sBias + bs * kBN, p.cbias + (size_t)it.bh * p.cpad + c * kBN, kBN * 4, &bars->b_full[bs]);
          } else {
            // entry tile: centroid rows and bias log2 n_e of the selected blocks' entries; the rows
            // past the item's last entry are masked (-inf, generic stores published by the arrive)
            const int t = s - it.nsel - p.nchunk;
            const int rows = min(kBN, it.erows - t * kBN);
            if (!mbar_wait(&bars->b_empty[bs], ((g / kBStages) & 1) ^ 1, abort, status)) { ok = false; break; }
            bars->bflag[bs] = 2;
            float* bb = sBias + bs * kBN;
            for (int c = rows; c < kBN; ++c) bb[c] = -INFINITY;
            mbar_expect_tx(&bars->k_full[ks], rows * 256);
            mbar_expect_tx(&bars->b_full[bs], rows * 4);
            if (t == 0) asm volatile("cp.async.wait_all;" ::: "memory");   // counts prefetched at the exact steps
            ent_tile_walk(p, it, bars->e8[0], rows, cs, cr, [&](int r0, int j, int sr, int nr) {
              const uint8_t* src = p.ent + ((size_t)it.bh * p.nB + j) * kEntTileBytes;
              bulk_load(dk + r0 * 128, src + sr * 128, nr * 128, &bars->k_full[ks]);
              bulk_load(dk + kPanel + r0 * 128, src + kEntPanel + sr * 128, nr * 128, &bars->k_full[ks]);
              bulk_load(bb + r0, src + kEntBiasOff + sr * 4, nr * 4, &bars->b_full[bs]);
            });
          }
        }
        if (!ok) break;
      }
      // no copy may still be in flight when the CTA leaves (this matters only after an abort:
      // otherwise the consumers have waited for every load)
      for (int nd = n >= kQStages ? n - kQStages : 0; nd < n; ++nd)
        mbar_wait_drain(&bars->q_full[nd % kQStages], (nd / kQStages) & 1);
      for (uint32_t gd = g >= kKStages ? g - kKStages : 0; gd < g; ++gd)
        mbar_wait_drain(&bars->k_full[gd % kKStages], (gd / kKStages) & 1);
      for (uint32_t gd = g >= kBStages ? g - kBStages : 0; gd < g; ++gd)
        mbar_wait_drain(&bars->b_full[gd % kBStages], (gd / kBStages) & 1);
    }
  } else if (warp == kWarpProducerV) {
    // ------------------------------------------------------------------ producer (values)
    if (lane == 0) {
      tma_prefetch(&tm_v);
      tma_prefetch(&tm_m);
      uint32_t g = 0;
      for (int k = blockIdx.x; k < p.n_items && !*abort; k += gridDim.x) {
        const Item it = item_at(p, k);
        int cs = 0, cr = 0;                // entry cursor: selected slot, source row
        bool ok = true;
        for (int s = 0; s < it.T; ++s, ++g) {
          const int vs = g % kVStages;
          if (!mbar_wait(&bars->v_empty[vs], ((g / kVStages) & 1) ^ 1, abort, status)) { ok = false; break; }
          uint8_t* dv = sV + vs * kTile;
          if (s < it.nsel || p.incl) {
            bool valid;
            const int j = block_of(p, it, s, &valid);
            mbar_expect_tx(&bars->v_full[vs], kTile);
            tma_load_3d(dv, &tm_v, &bars->v_full[vs], 0, j * kBN, it.bh);
            tma_load_3d(dv + kPanel, &tm_v, &bars->v_full[vs], 64, j * kBN, it.bh);
            ent_prefetch(p, it, bars->e8[1], s, j, valid);
          } else if (s < it.nsel + p.nchunk) {
            // cluster chunk: the head-wide means S_c / n_c (rows past C read as zero)
            const int c = s - it.nsel;
            mbar_expect_tx(&bars->v_full[vs], kTile);
            tma_load_3d(dv, &tm_m, &bars->v_full[vs], 0, c * kBN, it.bh);
            tma_load_3d(dv + kPanel, &tm_m, &bars->v_full[vs], 64, c * kBN, it.bh);
          } else {
            // entry tile: the negated entry means, the same runs as the producer of keys
            const int t = s - it.nsel - p.nchunk;
            const int rows = min(kBN, it.erows - t * kBN);
            mbar_expect_tx(&bars->v_full[vs], rows * 256);
            if (t == 0) asm volatile("cp.async.wait_all;" ::: "memory");   // counts prefetched at the exact steps
            ent_tile_walk(p, it, bars->e8[1], rows, cs, cr, [&](int r0, int j, int sr, int nr) {
              const uint8_t* src = p.ent + ((size_t)it.bh * p.nB + j) * kEntTileBytes + kEntVOff;
              bulk_load(dv + r0 * 128, src + sr * 128, nr * 128, &bars->v_full[vs]);
              bulk_load(dv + kPanel + r0 * 128, src + kEntPanel + sr * 128, nr * 128, &bars->v_full[vs]);
            });
          }
        }
        if (!ok) break;
      }
      for (uint32_t gd = g >= kVStages ? g - kVStages : 0; gd < g; ++gd)
        mbar_wait_drain(&bars->v_full[gd % kVStages], (gd / kVStages) & 1);
    }
  } else if (warp == kWarpMMA) {
    // ------------------------------------------------------------------ MMA issuer of S = Q K^T
    // The item's query tile is copied into tensor memory first, so that S reads only the key tile
    // from shared memory; S(g) goes into the score buffer as soon as softmax(g - 1) has read it into
    // registers.  Products of this thread and of the P V issuer (warp 11) share the tensor core; each
    // thread's commits track its own products (and its copies, which run in order with them).
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16(kBM, kBN, 0, 0);   // Q, K both K-major
      uint32_t g = 0;
      int n = 0;
      bool ok = true;
      for (int k = blockIdx.x; k < p.n_items && ok; k += gridDim.x, ++n) {
        const int T = item_at(p, k).T;
        const int qs = n % kQStages;
        const uint32_t qb = smem_u32(sQ + qs * kTile);
        const uint32_t qt = tmem + kColQ + (n & 1) * (kD / 2);    // this item's query tile
        for (int s = 0; s < T; ++s, ++g) {
          if (s == 0) {
            // the query tile into tensor memory (in order with this thread's products; the copy of
            // item n + 2 into the same columns follows item n's last S)
            if (!mbar_wait(&bars->q_full[qs], (n / kQStages) & 1, abort, status)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk)
              tmem_cp_128x256b(qt + kk * 8, sdesc_sw128(qb + (kk >> 2) * kPanel + (kk & 3) * 32, 16, 1024));
            umma_commit(&bars->q_empty[qs]);
          }
          // the one score buffer is free once softmax(g - 1) has read it
          if (g >= 1 && !mbar_wait(&bars->s_free[(g - 1) & 1], ((g - 1) >> 1) & 1, abort, status)) { ok = false; break; }
          const int ks = g % kKStages;
          if (!mbar_wait(&bars->k_full[ks], (g / kKStages) & 1, abort, status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kb = smem_u32(sK + ks * kTile);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kPanel + (kk & 3) * 32;
            umma_ts(tmem + kColS, qt + kk * 8, sdesc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0);
          }
          umma_commit(&bars->s_full[g & 1]);
          umma_commit(&bars->k_empty[ks]);
        }
      }
      umma_commit(&bars->drain[0]);
      mbar_wait_drain(&bars->drain[0], 0);
    }
  } else if (warp == kWarpPV) {
    // ------------------------------------------------------------------ MMA issuer of O += P V
    if (lane == 0) {
      const uint32_t idesc_pv = idesc_bf16(kBM, kD, 0, 1);    // P from TMEM, V MN-major
      uint32_t g = 0;
      int n = 0;
      bool ok = true;
      for (int k = blockIdx.x; k < p.n_items && ok; k += gridDim.x, ++n) {
        const int T = item_at(p, k).T;
        for (int s = 0; s < T; ++s, ++g) {
          const int vs = g % kVStages;
          if (!mbar_wait(&bars->p_ready[g & 1], (g >> 1) & 1, abort, status)) { ok = false; break; }
          if (!mbar_wait(&bars->v_full[vs], (g / kVStages) & 1, abort, status)) { ok = false; break; }
          if (s == 0 && !mbar_wait(&bars->o_free, (n & 1) ^ 1, abort, status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t vb = smem_u32(sV + vs * kTile);
          const uint32_t pt = tmem + kColP + (g & 1) * (kBN / 2);   // P(g): bf16 pairs, 64 columns
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            // V rows (keys) 16 kk .. 16 kk + 15: two 8-row groups of 1024 B; the first product of
            // an item overwrites O
            umma_ts(tmem + kColO, pt + kk * 8, sdesc_sw128(vb + kk * 2048, kPanel, 1024), idesc_pv,
                    (s > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars->v_empty[vs]);
          umma_commit(&bars->p_free[g & 1]);
        }
      }
      umma_commit(&bars->drain[1]);
      mbar_wait_drain(&bars->drain[1], 0);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax (warps 0-7)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegSoftmax));
    const int X = warp >> 2;                                  // warpgroup: steps g with g & 1 == X
    const int r = tid & 127;                                  // query row = TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t o_row = lane_addr + kColO;
    const uint32_t p_own = lane_addr + kColP + X * (kBN / 2);   // P_X
    uint32_t g0 = 0;                                          // first step of the item
    int n = 0;
    // (no abort test in the loop condition: a warp leaves as a whole, on its __all_sync'd waits)
    for (int k = blockIdx.x; k < p.n_items; k += gridDim.x, ++n) {
      const Item it = item_at(p, k);
      // m_at, l: this warpgroup's share of the row sum, expressed at the running max m_at
      float m_at = -INFINITY, l = 0.f;
      float m_seen = -INFINITY;                               // the running max of this warpgroup's last step
      bool ok = true;
      for (int s = (int)((X - g0) & 1u); s < it.T; s += 2) {
        const uint32_t g = g0 + s;
        const int bs = g % kBStages;
        bool w_ok = mbar_wait(&bars->b_full[bs], (g / kBStages) & 1, abort, status);
        w_ok = w_ok && mbar_wait(&bars->s_full[X], (g >> 1) & 1, abort, status);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        tc_fence_after();
        // The S row is loaded from TMEM once (128 registers); S_X is then free for S(g + 2).
        // Column c's logit is y_c = x_c * s*log2(e) + bias_c, the bias row in shared memory:
        // log2 n_c on a cluster chunk, log2 n_e on an entry tile, 0 on a key block (-inf past the
        // end of a short last block or of the entries).
        const uint32_t sbase = lane_addr + kColS;
        const float* bt = sBias + bs * kBN;
        const int flag = bars->bflag[bs];
        const bool plain = (flag & 1) && p.scale_log2 > 0.f;
        uint32_t x[4][32];
        tmem_ld32(sbase, x[0]);
        tmem_ld32(sbase + 32, x[1]);
        tmem_ld32(sbase + 64, x[2]);
        tmem_ld32(sbase + 96, x[3]);
        tmem_wait_ld_into(x[0]);
        reg_fence32(x[1]);
        reg_fence32(x[2]);
        reg_fence32(x[3]);
        tc_fence_before();
        warp_arrive(&bars->s_free[X], lane);
        const float mx = row_logits_max(x, bt, plain, p.scale_log2);
        // The running max is shared by the two warpgroups (one accumulator O) and moves only when a
        // row's max grows by more than 2^8 (lazy rescaling); an item starts from -inf.  The
        // exponentials are taken with the max this warpgroup saw at its previous step, before
        // waiting for the other warpgroup's latest one, so that the two warpgroups' exponentials do
        // not run in lockstep; a row whose max turns out different rescales its P and sum.
        const bool grow_g = mx > m_seen + kRescaleLog2 || (m_seen == -INFINITY && mx > -INFINITY);
        const float m_guess = grow_g ? mx : m_seen;
        uint64_t rsum = 0;
        uint32_t pk[4][16];
        {
          const float mu = (m_guess == -INFINITY) ? 0.f : m_guess;
          const uint64_t negmu = f2_pack(-mu, -mu);
          const uint64_t coef = plain ? f2_pack(p.scale_log2, p.scale_log2) : f2_pack(1.f, 1.f);
#pragma unroll
          for (int q = 0; q < 4; ++q) chunk_exp(x[q], coef, negmu, pk[q], rsum);
        }
        // the other warpgroup's running max of step g - 1 (every phase of m_pub is waited, in order)
        float mprev = -INFINITY;
        if (g >= 1) {
          const bool m_ok = mbar_wait(&bars->m_pub[X ^ 1], ((g - 1) >> 1) & 1, abort, status);
          if (!__all_sync(0xffffffffu, m_ok)) { ok = false; break; }
          const float mo = bars->mrow[X ^ 1][r];
          if (s > 0) mprev = mo;
        }
        const bool grow = mx > mprev + kRescaleLog2 || (mprev == -INFINITY && mx > -INFINITY);
        const float m_new = grow ? mx : mprev;
        bars->mrow[X][r] = m_new;
        warp_arrive(&bars->m_pub[X], lane);
        m_seen = m_new;
        float rs_lo, rs_hi;
        f2_unpack(rsum, rs_lo, rs_hi);
        float rs = rs_lo + rs_hi;
        if (m_new != m_guess && m_guess > -INFINITY) {
          // P <= 2^8 either way: m_new and m_guess both lie within 2^8 above the row's max
          const float f = ex2(m_guess - m_new);
#pragma unroll
          for (int q = 0; q < 4; ++q) scale_bf16x2(pk[q], f);
          rs *= f;
        }
        // P_X is free once P V(g - 2) is done (every phase of p_free[X] is waited, in order)
        if (g >= 2) {
          const bool f_ok = mbar_wait(&bars->p_free[X], ((g - 2) >> 1) & 1, abort, status);
          if (!__all_sync(0xffffffffu, f_ok)) { ok = false; break; }
          tc_fence_after();
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_st16(p_own + q * 16, pk[q]);
        warp_arrive(&bars->b_empty[bs], lane);    // the warp has read the bias row
        // A row whose max moved rescales O, which must first hold every product up to step g - 1.
        // Only a warp that rescales waits for P V(g - 1): P V(g - 2) is known done here (p_free[X]
        // above) and P V(g + 1) cannot start before this step's P is ready, so the other
        // warpgroup's p_free is within one phase of the awaited one whenever it is waited.
        const bool need_o = grow && s > 0 && mprev > -INFINITY;
        if (__any_sync(0xffffffffu, need_o)) {
          const bool d_ok = mbar_wait(&bars->p_free[X ^ 1], ((g - 1) >> 1) & 1, abort, status);
          if (!__all_sync(0xffffffffu, d_ok)) { ok = false; break; }
          tc_fence_after();
          rescale_row(o_row, need_o ? ex2(mprev - m_new) : 1.f);
        }
        if (m_new != m_at) {                      // the running max only grows
          if (m_at > -INFINITY) l *= ex2(m_at - m_new);
          m_at = m_new;
        }
        l += (flag & 2) ? -rs : rs;               // entry tiles take their weight out again
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(&bars->p_ready[X], lane);
      }
      if (!ok) break;
      // epilogue: once the item's last product has landed, exchange (max, sum) per row with the
      // other warpgroup; warpgroup X normalises and stores columns [64X, 64X + 64) of
      // O / (l_0 2^(m_0 - M) + l_1 2^(m_1 - M)), O being expressed at M, the larger of the two.
      // (P V(gl - 1) first: after it, P V(gl)'s barrier is within one phase of the awaited one)
      const uint32_t gl = g0 + it.T - 1;
      bool e_ok = gl < 1 || mbar_wait(&bars->p_free[(gl - 1) & 1], ((gl - 1) >> 1) & 1, abort, status);
      e_ok = e_ok && mbar_wait(&bars->p_free[gl & 1], (gl >> 1) & 1, abort, status);
      bars->xch[n & 1][X][r] = make_float2(m_at, l);
      warp_arrive(&bars->xch_full[n & 1][X], lane);
      e_ok = e_ok && mbar_wait(&bars->xch_full[n & 1][X ^ 1], (n >> 1) & 1, abort, status);
      if (!__all_sync(0xffffffffu, e_ok)) break;
      tc_fence_after();
      const float2 e0 = bars->xch[n & 1][0][r], e1 = bars->xch[n & 1][1][r];
      const float M = fmaxf(e0.x, e1.x);
      const float f0 = e0.x > -INFINITY ? ex2(e0.x - M) : 0.f;
      const float f1 = e1.x > -INFINITY ? ex2(e1.x - M) : 0.f;
      const float L = e0.y * f0 + e1.y * f1;
      const float inv = L > 0.f ? 1.f / L : 0.f;
      const bool live = r < it.qlen;
      store_row_half(o_row + 64 * X, p.O + ((size_t)it.bh * p.N + it.q0 + r) * kD + 64 * X, inv, live);
      if (X == 0 && live && p.lse) p.lse[(size_t)it.bh * p.N + it.q0 + r] = (M + __log2f(L)) * 0.69314718055994531f;
      tc_fence_before();
      warp_arrive(&bars->o_free, lane);
      g0 += it.T;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Entry rows each item streams (the sum over its valid selected blocks of ent_rows_of), so that
// every role knows an item's step count without walking its list.  A warp per item.
__global__ void __launch_bounds__(256) entry_rows_kernel(const int32_t* __restrict__ kv_idx,
                                                         const int32_t* __restrict__ kv_cnt, int max_sel,
                                                         const int32_t* __restrict__ seg_n, int nB, int n_items,
                                                         int32_t* __restrict__ out) {
  const int item = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (item >= n_items) return;
  int cnt = kv_cnt[item];
  if (cnt < 0 || cnt > max_sel) cnt = 0;
  const int bh = item / nB;
  const int32_t* row = kv_idx + (size_t)item * max_sel;
  int sum = 0;
  for (int s = lane; s < cnt; s += 32) {
    const int j = row[s];
    if (j >= 0 && j < nB) sum += ent_rows_of(seg_n, nB, bh, j);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) out[item] = sum;
}

}  // namespace

bool attention_tc_supported(const Dims& g) { return g.bf16 && g.d == kD && g.block == kBN; }

cudaError_t launch_attention_tc(const Dims& g, const void* Q, const void* K, const void* V,
                                const int32_t* kv_idx, const int32_t* kv_cnt, int max_sel,
                                const int32_t* schedule, const void* cent, const StatsPtrs& st, float scale,
                                void* O, float* lse, int* status, int32_t* ent_rows, const float* incl,
                                cudaStream_t s) {
  CUtensorMap tq, tk, tv, tc, tm;
  const unsigned long long BH = (unsigned long long)g.B * g.H;
  const CompLayout L = comp_layout(g);
  // without compensation tiles (the inclusion-probability mode) K stands in for the cluster means
  const void* cmean = (!incl && st.comp) ? static_cast<const void*>(st.comp + L.cmean) : K;
  const unsigned long long mean_rows = (!incl && st.comp) ? (unsigned long long)g.C : (unsigned long long)g.N;
  if (!incl && !st.comp) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_3d(&tq, Q, kD, g.N, BH, 64, kBM) || !make_tmap_bf16_3d(&tk, K, kD, g.N, BH, 64, kBN) ||
      !make_tmap_bf16_3d(&tv, V, kD, g.N, BH, 64, kBN) || !make_tmap_bf16_3d(&tc, cent, kD, g.C, BH, 64, kBN) ||
      !make_tmap_bf16_3d(&tm, cmean, kD, mean_rows, BH, 64, kBN))
    return cudaErrorInvalidValue;
  Params p;
  p.kv_idx = kv_idx;
  p.kv_cnt = kv_cnt;
  p.schedule = schedule;
  p.max_sel = max_sel;
  p.seg_n = st.seg_n;
  p.ent_rows = ent_rows;
  p.ent = st.comp ? st.comp + L.ent : nullptr;
  p.cbias = st.comp ? reinterpret_cast<const float*>(st.comp + L.cbias) : nullptr;
  p.O = (__nv_bfloat16*)O;
  p.lse = lse;
  p.status = status;
  p.incl = incl;
  p.N = g.N;
  p.C = g.C;
  p.nB = g.nB;
  p.n_items = (int)(BH * g.nB);
  p.nchunk = (g.C + kBN - 1) / kBN;
  p.cpad = L.cpad;
  p.scale_log2 = scale * 1.4426950408889634f;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaError_t e = cudaFuncSetAttribute(attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  if (!incl) {
    entry_rows_kernel<<<(p.n_items + 7) / 8, 256, 0, s>>>(kv_idx, kv_cnt, max_sel, st.seg_n, g.nB, p.n_items,
                                                          ent_rows);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int grid = min(sms, p.n_items);
  attention_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, tc, tm, p);
  return cudaGetLastError();
}

}  // namespace da
