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
// The compensation chunks (vbar^U rows in bf16 and log2 n^U per cluster) of every item are
// written beforehand by comp_build.cu; here they are loaded like value blocks.
//
// Inclusion-probability mode (AB-Attention abstract: sampled blocks "reweighted by inverse
// inclusion probability"): with p.incl, an item's steps are its selected blocks only (one fully
// masked step if it has none), and block j's logits carry the bias -log2 pi_j, i.e. the weight
// 1 / pi_j in both sums of the softmax; no cluster columns.
//
// Variance-corrected mode (kSpread; ESTRA abstract, second-order correction of the cluster
// logits): a cluster column's logit gains s^2/2 sum_t q_t^2 D_{c,t}, D_c the second moment of the
// cluster's keys about its representative.  The correction is a second contraction into the same
// score tile: S = Q cbar^T + Q2 Dh^T, with Q2 = q o q (bf16, written into shared memory from the
// query tile by the softmax warpgroups at the start of each item) and Dh = (s/2) D (bf16, from the
// host side).  A chunk step therefore takes two key-ring tiles (the centroid chunk, then the Dh
// chunk), so the key ring counts tiles, not steps; the query tile Q2 takes the place of one
// value-ring slot (two slots in this mode), and the key and value tiles land on barriers of their
// own.
//
// Roles (384 threads):
//   warps 0-3, 4-7  two softmax warpgroups X = 0, 1; warpgroup X takes the steps g with g & 1 = X
//              of every item, so the two overlap each other and the tensor core.  Thread t of a
//              warpgroup owns query row t = TMEM lane t.  Both warpgroups exponentiate against one
//              reference max per row and item, the row max of the item's first step (handed to
//              the other warpgroup through shared memory), so their products add into one
//              accumulator O and no rescaling is ever needed; P is written back to TMEM as bf16.
//              At the end of the item the two exchange their row sums and each normalises and
//              stores half of the columns of O;
//   warp 8     producer: loads Q, key tiles / centroid chunks (2-stage ring) and the softmax bias
//              rows (4-stage ring, so a slot always serves the same warpgroup);
//   warp 9     score issuer: allocates TMEM, issues tcgen05.mma S(g) = Q K^T into S_(g mod 3) as
//              soon as its key tile has landed and P(g-3) V(g-3) has finished reading the buffer;
//   warp 10    producer of value tiles / compensation chunks (3-stage ring); a warp of its own,
//              since divergent lanes of one warp waiting on different barriers hold each other up;
//   warp 11    product issuer: O += P(g) V(g) once P(g) is written and V(g) has landed.  Two
//              issuing threads keep the tensor core fed: one thread's waits on the softmax no
//              longer hold the other's products back (issuing blocks while the tensor core's queue
//              is full).
// Outside the variance-corrected mode a tile lands on the barrier its consumer waits on anyway,
// since every barrier operation costs a few hundred cycles here: the value tile of step g on
// p_ready[g mod 3] (beside the softmax's arrivals) and the key tile of step g on pv_done[g mod 3]
// (beside the commit of P(g-3) V(g-3)); the rings' slot rules put both in step g's phase.
// TMEM columns: S_0 [0,128), S_1 [128,256), S_2 [256,384), O [384,512).  Step g's scores go to
// S_(g mod 3): the tensor core computes S(g+1) and S(g+2) while the softmax of step g runs, and
// S(g+3) waits for P(g) V(g) to complete (pv_done), since the two issuers' products are not ordered
// with respect to each other.
//
// Range: P = 2^(y - m_ref) with m_ref the row max of the item's first step.  Later steps may
// exceed it; a row whose logits exceed m_ref by more than 2^96 (in log2 units) in some step is
// reported as DA_ERR_RANGE, since its sums could overflow fp32.
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
constexpr int kKStages = 2;             // key / centroid tiles (freed as soon as S is computed)
constexpr int kVStages = 3;             // value / vbar^U tiles (freed after P V)
constexpr int kBStages = 4;             // bias rows of the softmax (even: a slot serves one warpgroup)
constexpr int kTile = kBN * kD * 2;      // 32 KB bf16 tile
constexpr int kPanel = kBN * 128;        // one 64-column panel (128 rows x 128 B)
constexpr int kSBufs = 3;                // score buffers in TMEM (and one accumulator O)
constexpr float kRangeLog2 = 96.0f;      // largest step max above the reference max (log2 units)
constexpr int kThreads = 384;           // three warpgroups; warp 11 idle
constexpr int kWarpProducer = 8;
constexpr int kWarpMMA = 9;             // score issuer (and TMEM owner)
constexpr int kWarpProducerV = 10;
constexpr int kWarpPV = 11;              // product issuer
// Register split (setmaxnreg): the launch holds 384 x 168 registers; the softmax warpgroups grow,
// the producer / MMA warpgroup shrinks.
constexpr int kRegSoftmax = 232, kRegIssue = 40;
static_assert(128 * (2 * kRegSoftmax + kRegIssue) <= kThreads * 168, "register split above the launch");
static_assert(kBStages % 2 == 0, "a bias slot must always serve the same softmax warpgroup");
static_assert(kVStages == kSBufs, "a value tile lands on the P-ready barrier of its score buffer");
constexpr int kChunkBytes = kTile + kBN * 4;   // compensation chunk: vbar^U rows, then log2 n^U

struct __align__(8) Bars {
  uint64_t q_full, q_empty, q2_full;
  uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  uint64_t b_full[kBStages], b_empty[kBStages];
  // s_full[g mod 6]: S(g) computed (g mod 6 fixes the buffer and the warpgroup, so each barrier
  // is waited by one warpgroup at every phase); p_ready[g mod 3]: P(g) written
  uint64_t s_full[2 * kSBufs], p_ready[kSBufs];
  uint64_t pv_done[kSBufs];              // P(g) V(g) complete: S_(g mod 3) may take S(g + 3)
  uint64_t o_full, o_free, drain, drain_pv;
  // reference max published by the item's first step: [item parity]
  uint64_t mref_full[2];
  // (reference max, sum) published: [item parity][warpgroup].  One barrier per item parity: a
  // warpgroup without steps in an item could otherwise complete a barrier twice before the other
  // warpgroup's parity wait on it runs.
  uint64_t xch_full[2][2];
  uint32_t tmem_base;
  int abort;
  int bflag[kBStages];                   // 1: the slot's bias row is all zero (a full key block)
  float2 xch[2][2][kBM];                 // [item parity][warpgroup][row] = (reference max, sum)
  float mref[2][kBM];                    // [item parity][row]
};

// (the variance-corrected mode holds Q2 in place of one value-ring slot: the same size)
constexpr size_t kSmemBytes = 1024 + kTile /*Q*/ + (kKStages + kVStages) * kTile /*K,V*/ +
                              kBStages * kBN * sizeof(float) /*bias*/ + sizeof(Bars);
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
  const uint8_t* comp;                   // [items][nchunk] compensation chunks of kChunkBytes
  const float* incl;                     // [items][max_sel] inclusion probabilities, or NULL
  int N, C, nB, n_items, nchunk;
  float scale_log2;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// q o q for a pair of bf16 values: each square rounded once to bf16.
__device__ __forceinline__ uint32_t square_bf16x2(uint32_t w) {
  __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w);
  h = __hmul2(h, h);
  return *reinterpret_cast<const uint32_t*>(&h);
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
  it.T = p.incl ? max(cnt, 1) : cnt + p.nchunk;
  it.row = p.kv_idx + (size_t)item * p.max_sel;
  return it;
}

// Key block of exact step s; an out-of-range index becomes a fully masked block 0.
__device__ __forceinline__ int block_of(const Params& p, const Item& it, int s, bool* valid) {
  const int j = s < it.nsel ? it.row[s] : -1;
  *valid = (j >= 0 && j < p.nB);
  return *valid ? j : 0;
}

__device__ __forceinline__ const uint8_t* comp_chunk(const Params& p, const Item& it, int c) {
  return p.comp + ((size_t)(it.bh * p.nB + it.i) * p.nchunk + c) * kChunkBytes;
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

// kSpread: the variance-corrected mode (tm_d maps Dh = (s/2) D, [B*H][C][d] bf16); otherwise tm_d
// is unused.
template <bool kSpread>
__global__ void __launch_bounds__(kThreads, 1)
attention_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_c,
                    const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_d,
                    const Params p) {
  constexpr int kVSt = kSpread ? kVStages - 1 : kVStages;   // value-ring slots
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = base;
  uint8_t* sQ2 = sQ + kTile;                      // variance-corrected mode only
  uint8_t* sK = sQ + (kSpread ? 2 : 1) * kTile;   // kKStages tiles
  uint8_t* sV = sK + kKStages * kTile;            // kVSt tiles
  float* sBias = reinterpret_cast<float*>(sV + kVSt * kTile);   // [kBStages][kBN]
  Bars* bars = reinterpret_cast<Bars*>(sBias + kBStages * kBN);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->q2_full, 256);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < kVSt; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&bars->b_full[s], 1);
      mbar_init(&bars->b_empty[s], 128);
    }
    for (int b = 0; b < 2 * kSBufs; ++b) mbar_init(&bars->s_full[b], 1);
    for (int b = 0; b < kSBufs; ++b) {
      // outside the variance-corrected mode the value tile of step g lands on p_ready[g mod 3]
      // too: the value producer's arrival (with its bytes) joins the softmax warpgroup's 128
      mbar_init(&bars->p_ready[b], kSpread ? 128 : 129);
      // outside the variance-corrected mode the key tile of step g lands on pv_done[g mod 3] too
      // (the commit of P(g-3) V(g-3) and the key producer's arrival with the tile's bytes); the
      // first phase of each stands for a product before the first step
      mbar_init(&bars->pv_done[b], kSpread ? 1 : 2);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->mref_full[b], 128);
      mbar_init(&bars->xch_full[b][0], 128);
      mbar_init(&bars->xch_full[b][1], 128);
    }
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->o_free, 256);
    mbar_init(&bars->drain, 1);
    if (!kSpread)
      for (int b = 0; b < kSBufs; ++b) mbar_arrive(&bars->pv_done[b]);
    mbar_init(&bars->drain_pv, 1);
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

  // the whole third warpgroup gives registers up at one instruction (setmaxnreg is warpgroup-wide)
  if (warp >= 8) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegIssue));

  if (warp == kWarpProducer) {
    // ------------------------------------------------------------------ producer (keys)
    // query tiles, key / centroid tiles and the softmax bias rows
    if (lane == 0) {
      tma_prefetch(&tm_q);
      tma_prefetch(&tm_k);
      tma_prefetch(&tm_c);
      if (kSpread) tma_prefetch(&tm_d);
      uint32_t g = 0;
      uint32_t kt = 0;                   // key-ring tiles loaded (one per step; two per chunk step
                                         // in the variance-corrected mode)
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
          if (!kSpread) kt = g;          // one tile per step
          const int ks = kt % kKStages, bs = g % kBStages;
          if (!mbar_wait(&bars->k_empty[ks], ((kt / kKStages) & 1) ^ 1, abort, status)) { ok = false; break; }
          uint8_t* dk = sK + ks * kTile;
          ++kt;
          // Outside the variance-corrected mode the tile lands on pv_done[g mod 3]: a key slot is free
          // only once S(g-2) has completed, so P(g-6) V(g-6) has (S(g-3) waited for it) and that
          // barrier is in step g's phase; the score issuer then waits on one barrier for both.
          uint64_t* klanded = kSpread ? &bars->k_full[ks] : &bars->pv_done[g % kSBufs];
          if (s < it.nsel || p.incl) {
            bool valid;
            const int j = block_of(p, it, s, &valid);
            mbar_expect_tx(klanded, kTile);
            tma_load_3d(dk, &tm_k, klanded, 0, j * kBN, it.bh);
            tma_load_3d(dk + kPanel, &tm_k, klanded, 64, j * kBN, it.bh);
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
            const bool full = ncol == kBN && !p.incl && p.scale_log2 > 0.f;
            bars->bflag[bs] = full ? 1 : 0;
            if (!full) {
              // (a full block's row would be all zero: the softmax does not read it)
              float4* bb = reinterpret_cast<float4*>(sBias + bs * kBN);
#pragma unroll 4
              for (int c4 = 0; c4 < kBN / 4; ++c4) {
                const int c = 4 * c4;
                bb[c4] = make_float4(c < ncol ? w : -INFINITY, c + 1 < ncol ? w : -INFINITY,
                                     c + 2 < ncol ? w : -INFINITY, c + 3 < ncol ? w : -INFINITY);
              }
            }
            mbar_arrive(&bars->b_full[bs]);
          } else {
            const int c = s - it.nsel;
            mbar_expect_tx(klanded, kTile);
            tma_load_3d(dk, &tm_c, klanded, 0, c * kBN, it.bh);
            tma_load_3d(dk + kPanel, &tm_c, klanded, 64, c * kBN, it.bh);
            if (kSpread) {
              // the chunk's rows of Dh, into the next key-ring slot
              const int kd = kt % kKStages;
              if (!mbar_wait(&bars->k_empty[kd], ((kt / kKStages) & 1) ^ 1, abort, status)) { ok = false; break; }
              uint8_t* dd = sK + kd * kTile;
              ++kt;
              mbar_expect_tx(&bars->k_full[kd], kTile);
              tma_load_3d(dd, &tm_d, &bars->k_full[kd], 0, c * kBN, it.bh);
              tma_load_3d(dd + kPanel, &tm_d, &bars->k_full[kd], 64, c * kBN, it.bh);
            }
            if (!mbar_wait(&bars->b_empty[bs], ((g / kBStages) & 1) ^ 1, abort, status)) { ok = false; break; }
            bars->bflag[bs] = 0;
            mbar_expect_tx(&bars->b_full[bs], kBN * 4);
            bulk_load(sBias + bs * kBN, comp_chunk(p, it, c) + kTile, kBN * 4, &bars->b_full[bs]);
          }
        }
        if (!ok) break;
      }
      // no copy may still be in flight when the CTA leaves (this matters only after an abort:
      // otherwise the consumers have waited for every load)
      if (nq > 0) mbar_wait_drain(&bars->q_full, (nq - 1) & 1);
      for (uint32_t gd = kt >= kKStages ? kt - kKStages : 0; gd < kt; ++gd)
        mbar_wait_drain(kSpread ? &bars->k_full[gd % kKStages] : &bars->pv_done[gd % kSBufs],
                        kSpread ? (gd / kKStages) & 1 : (gd / kSBufs) & 1);
      for (uint32_t gd = g >= kBStages ? g - kBStages : 0; gd < g; ++gd)
        mbar_wait_drain(&bars->b_full[gd % kBStages], (gd / kBStages) & 1);
    }
  } else if (warp == kWarpProducerV) {
    // ------------------------------------------------------------------ producer (values)
    if (lane == 0) {
      tma_prefetch(&tm_v);
      tma_prefetch(&tm_p);
      uint32_t g = 0;
      int n = 0;
      for (int k = blockIdx.x; k < p.n_items && !*abort; k += gridDim.x, ++n) {
        const Item it = item_at(p, k);
        bool ok = true;
        for (int s = 0; s < it.T; ++s, ++g) {
          const int vs = g % kVSt;
          if (!mbar_wait(&bars->v_empty[vs], ((g / kVSt) & 1) ^ 1, abort, status)) { ok = false; break; }
          uint8_t* dv = sV + vs * kTile;
          // Outside the variance-corrected mode the tile lands on p_ready[g mod 3] (the ring and the
          // score buffers have the same three slots, and the slot is free only once P(g-3) V(g-3)
          // has completed, so that barrier is in step g's phase), and the product issuer waits on
          // one barrier for both P(g) and V(g).
          uint64_t* landed = kSpread ? &bars->v_full[vs] : &bars->p_ready[g % kSBufs];
          if (s < it.nsel || p.incl) {
            bool valid;
            const int j = block_of(p, it, s, &valid);
            mbar_expect_tx(landed, kTile);
            tma_load_3d(dv, &tm_v, landed, 0, j * kBN, it.bh);
            tma_load_3d(dv + kPanel, &tm_v, landed, 64, j * kBN, it.bh);
          } else {
            const int z = (it.bh * p.nB + it.i) * p.nchunk + (s - it.nsel);
            mbar_expect_tx(landed, kTile);
            tma_load_3d(dv, &tm_p, landed, 0, 0, z);
            tma_load_3d(dv + kPanel, &tm_p, landed, 64, 0, z);
          }
        }
        if (!ok) break;
      }
      for (uint32_t gd = g >= kVSt ? g - kVSt : 0; gd < g; ++gd)
        mbar_wait_drain(kSpread ? &bars->v_full[gd % kVSt] : &bars->p_ready[gd % kSBufs],
                        (gd / kVSt) & 1);
    }
  } else if (warp == kWarpMMA) {
    // ------------------------------------------------------------------ score issuer
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16(kBM, kBN, 0, 0);   // Q, K both K-major
      const uint32_t q0 = smem_u32(sQ);
      uint32_t g = 0;
      uint32_t kt = 0;                   // key-ring tiles consumed
      int n = 0;
      bool ok = true;
      for (int k = blockIdx.x; k < p.n_items && ok; k += gridDim.x, ++n) {
        const Item it = item_at(p, k);
        if (!mbar_wait(&bars->q_full, n & 1, abort, status)) break;
        for (int s = 0; s < it.T; ++s, ++g) {
          // S_(g mod 3) last held S(g - 3): its product must have read P(g - 3); every phase of
          // pv_done[g mod 3] is waited, in order
          // (outside the variance-corrected mode the same barrier also says that the key tile of
          // step g has landed; its first phase stands for a product before the first step)
          if (!kSpread) {
            if (!mbar_wait(&bars->pv_done[g % kSBufs], (g / kSBufs) & 1, abort, status)) { ok = false; break; }
          } else if (g >= (uint32_t)kSBufs &&
                     !mbar_wait(&bars->pv_done[g % kSBufs], ((g / kSBufs) & 1) ^ 1, abort, status)) {
            ok = false;
            break;
          }
          const bool two = kSpread && !p.incl && s >= it.nsel;
          const uint32_t t0 = kSpread ? kt : g;   // one tile per step outside the corrected mode
          if (kSpread && !mbar_wait(&bars->k_full[t0 % kKStages], (t0 / kKStages) & 1, abort, status)) {
            ok = false;
            break;
          }
          if (two) {
            const uint32_t t1 = t0 + 1;
            if (!mbar_wait(&bars->k_full[t1 % kKStages], (t1 / kKStages) & 1, abort, status)) { ok = false; break; }
            if (s == it.nsel && !mbar_wait(&bars->q2_full, n & 1, abort, status)) { ok = false; break; }
          }
          tc_fence_after();
          const uint32_t kb = smem_u32(sK + (t0 % kKStages) * kTile);
          const uint32_t d = tmem + (g % kSBufs) * kBN;
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const uint32_t off = (ks >> 2) * kPanel + (ks & 3) * 32;
            umma_ss(d, sdesc_sw128(q0 + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024), idesc_qk, ks > 0);
          }
          if (two) {
            // + Q2 Dh^T: the correction of the cluster logits, into the same accumulator
            const uint32_t q2 = smem_u32(sQ2);
            const uint32_t db = smem_u32(sK + ((t0 + 1) % kKStages) * kTile);
#pragma unroll 1
            for (int ks = 0; ks < kD / 16; ++ks) {
              const uint32_t off = (ks >> 2) * kPanel + (ks & 3) * 32;
              umma_ss(d, sdesc_sw128(q2 + off, 16, 1024), sdesc_sw128(db + off, 16, 1024), idesc_qk, 1u);
            }
          }
          umma_commit(&bars->s_full[g % (2 * kSBufs)]);
          umma_commit(&bars->k_empty[t0 % kKStages]);
          if (two) umma_commit(&bars->k_empty[(t0 + 1) % kKStages]);
          if (s == it.T - 1) umma_commit(&bars->q_empty);   // the item's last read of Q (and Q2)
          if (kSpread) kt = t0 + (two ? 2u : 1u);
        }
      }
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0);
    }
  } else if (warp == kWarpPV) {
    // ------------------------------------------------------------------ product issuer
    if (lane == 0) {
      const uint32_t idesc_pv = idesc_bf16(kBM, kD, 0, 1);    // P from TMEM, V MN-major
      const uint32_t ot = tmem + kSBufs * kBN;                // O
      uint32_t g = 0;
      int n = 0;
      bool ok = true;
      for (int k = blockIdx.x; k < p.n_items && ok; k += gridDim.x, ++n) {
        const Item it = item_at(p, k);
        for (int s = 0; s < it.T; ++s, ++g) {
          const int vs = g % kVSt;
          if (!mbar_wait(&bars->p_ready[g % kSBufs], (g / kSBufs) & 1, abort, status)) { ok = false; break; }
          if (kSpread && !mbar_wait(&bars->v_full[vs], (g / kVSt) & 1, abort, status)) { ok = false; break; }
          if (s == 0 && !mbar_wait(&bars->o_free, (n & 1) ^ 1, abort, status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t vb = smem_u32(sV + vs * kTile);
          const uint32_t pt = tmem + (g % kSBufs) * kBN;  // P: bf16 pairs in the S buffer's first 64 columns
#pragma unroll
          for (int ks = 0; ks < kBN / 16; ++ks) {
            // V rows (keys) 16*ks .. 16*ks+15: two 8-row groups of 1024 B; the item's first product
            // overwrites O
            umma_ts(ot, pt + ks * 8, sdesc_sw128(vb + ks * 2048, kPanel, 1024), idesc_pv,
                    (s > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(&bars->v_empty[vs]);
          umma_commit(&bars->pv_done[g % kSBufs]);
          if (s == it.T - 1) umma_commit(&bars->o_full);
        }
      }
      umma_commit(&bars->drain_pv);
      mbar_wait_drain(&bars->drain_pv, 0);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax (warps 0-7)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegSoftmax));
    const int X = warp >> 2;                                  // warpgroup: steps g with g & 1 == X
    const int r = tid & 127;                                  // query row = TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    uint32_t g0 = 0;                                          // first step of the item
    int n = 0;
    // (no abort test in the loop condition: a warp leaves as a whole, on its __all_sync'd waits)
    for (int k = blockIdx.x; k < p.n_items; k += gridDim.x, ++n) {
      const Item it = item_at(p, k);
      float mref = -INFINITY, l = 0.f;                       // -inf: no step of this warpgroup yet
      bool ok = true;
      if (kSpread) {
        // Q2 = q o q of this item in the query tile's swizzled layout (the square is elementwise, so
        // the 128-byte swizzle carries over), written by both warpgroups once the tile has landed and
        // published to the tensor core by a proxy fence and an arrival on q2_full.  The score
        // issuer waits for it at the item's first chunk step; the next query tile loads only after
        // the item's last score tile, the last reader of Q2, has completed.
        const bool q_ok = mbar_wait(&bars->q_full, n & 1, abort, status);
        if (!__all_sync(0xffffffffu, q_ok)) break;
        const uint4* src = reinterpret_cast<const uint4*>(sQ);
        uint4* dst = reinterpret_cast<uint4*>(sQ2);
#pragma unroll 1
        for (int i = tid; i < kTile / 16; i += 256) {
          uint4 v = src[i];
          v.x = square_bf16x2(v.x);
          v.y = square_bf16x2(v.y);
          v.z = square_bf16x2(v.z);
          v.w = square_bf16x2(v.w);
          dst[i] = v;
        }
        fence_async_smem();
        mbar_arrive(&bars->q2_full);
      }
      for (int s = (int)((X - g0) & 1u); s < it.T; s += 2) {
        const uint32_t g = g0 + s;
        // every phase of this warpgroup's b_full slots and s_full barriers is waited, in order
        const int bs = g % kBStages;
        bool w_ok = mbar_wait(&bars->b_full[bs], (g / kBStages) & 1, abort, status);
        w_ok = w_ok && mbar_wait(&bars->s_full[g % (2 * kSBufs)], (g / (2 * kSBufs)) & 1, abort, status);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        tc_fence_after();
        // The S row is loaded from TMEM once (128 registers): the row max, then p = 2^(y - m_ref),
        // the row sum and the bf16 P written back over S.  Column c's logit is y_c = x_c *
        // s*log2(e) + bias_c, the bias row in shared memory: log2 n^U_c on a compensation step, 0
        // on a key block (-inf past the end of a short last block).
        const uint32_t sbase = lane_addr + (g % kSBufs) * kBN;
        const float* bt = sBias + bs * kBN;
        const bool plain = bars->bflag[bs] != 0 && p.scale_log2 > 0.f;
        uint32_t x[4][32];
        tmem_ld32(sbase, x[0]);
        tmem_ld32(sbase + 32, x[1]);
        tmem_ld32(sbase + 64, x[2]);
        tmem_ld32(sbase + 96, x[3]);
        tmem_wait_ld_into(x[0]);
        reg_fence32(x[1]);
        reg_fence32(x[2]);
        reg_fence32(x[3]);
        const float mx = row_logits_max(x, bt, plain, p.scale_log2);
        if (s == 0) {
          // the item's first step sets the row's reference max for both warpgroups
          mref = mx > -INFINITY ? mx : 0.f;
          bars->mref[n & 1][r] = mref;
          mbar_arrive(&bars->mref_full[n & 1]);
        } else if (s == 1) {
          // this warpgroup's first step of the item: the other one published the reference
          const bool m_ok = mbar_wait(&bars->mref_full[n & 1], (n >> 1) & 1, abort, status);
          if (!__all_sync(0xffffffffu, m_ok)) { ok = false; break; }
          mref = bars->mref[n & 1][r];
        }
        if (mx > mref + kRangeLog2) set_status(status, DA_ERR_RANGE);
        uint64_t rsum = 0;
        {
          const uint64_t negmu = f2_pack(-mref, -mref);
          const uint64_t coef = plain ? f2_pack(p.scale_log2, p.scale_log2) : f2_pack(1.f, 1.f);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t pk[16];
            chunk_exp(x[q], coef, negmu, pk, rsum);
            tmem_st16(sbase + q * 16, pk);
          }
        }
        mbar_arrive(&bars->b_empty[bs]);          // this thread has read the bias row
        float rs_lo, rs_hi;
        f2_unpack(rsum, rs_lo, rs_hi);
        l += rs_lo + rs_hi;
        tmem_wait_st();
        tc_fence_before();
#ifdef DA_FAULT_INJECT
        // Test build only (libda_fault.so): the second softmax warpgroup of CTA 0 withholds its
        // P-ready arrival at step 5, a plain software arrival (no copy or product is left in
        // flight).  The MMA issuer's bounded wait for it gives up, records DA_ERR_TIMEOUT and makes
        // every role of the CTA leave; the producers drain their copies first.
        const bool withhold = blockIdx.x == 0 && g == 5;
#else
        constexpr bool withhold = false;
#endif
        if (!withhold) mbar_arrive(&bars->p_ready[g % kSBufs]);
      }
      if (!ok) break;
      // epilogue: once the item's last product has landed in O, exchange (reference max, sum) per
      // row with the other warpgroup; warpgroup X normalises and stores columns [64X, 64X + 64) of
      // O / (l_0 + l_1).  Both sums are taken against the same reference; a warpgroup without a
      // step in the item (a one-step item) publishes (-inf, 0).
      bool e_ok = mbar_wait(&bars->o_full, n & 1, abort, status);
      bars->xch[n & 1][X][r] = make_float2(mref, l);
      mbar_arrive(&bars->xch_full[n & 1][X]);
      e_ok = e_ok && mbar_wait(&bars->xch_full[n & 1][X ^ 1], (n >> 1) & 1, abort, status);
      if (!__all_sync(0xffffffffu, e_ok)) break;
      tc_fence_after();
      const float2 e0 = bars->xch[n & 1][0][r], e1 = bars->xch[n & 1][1][r];
      const float M = fmaxf(e0.x, e1.x);
      const float L = e0.y + e1.y;
      const float inv = L > 0.f ? 1.f / L : 0.f;
      const bool live = r < it.qlen;
      __nv_bfloat16* op = p.O + ((size_t)it.bh * p.N + it.q0 + r) * kD + 64 * X;
#pragma unroll 1
      for (int q = 0; q < 2; ++q) {
        uint32_t ra[32];
        tmem_ld32(lane_addr + kSBufs * kBN + 64 * X + 32 * q, ra);
        tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(ra[8 * v + 0]) * inv, __uint_as_float(ra[8 * v + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(ra[8 * v + 2]) * inv, __uint_as_float(ra[8 * v + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(ra[8 * v + 4]) * inv, __uint_as_float(ra[8 * v + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(ra[8 * v + 6]) * inv, __uint_as_float(ra[8 * v + 7]) * inv);
            *reinterpret_cast<uint4*>(op + q * 32 + v * 8) = w;
          }
        }
      }
      if (X == 0 && live && p.lse) p.lse[(size_t)it.bh * p.N + it.q0 + r] = (M + __log2f(L)) * 0.69314718055994531f;
      tc_fence_before();
      mbar_arrive(&bars->o_free);
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

}  // namespace

bool attention_tc_supported(const Dims& g) { return g.bf16 && g.d == kD && g.block == kBN; }

size_t attention_tc_scratch_bytes(const Dims& g) {
  if (!attention_tc_supported(g)) return 0;
  return (size_t)g.B * g.H * g.nB * ((g.C + kBN - 1) / kBN) * kChunkBytes;
}

cudaError_t launch_attention_tc(const Dims& g, const void* Q, const void* K, const void* V,
                                const int32_t* kv_idx, const int32_t* kv_cnt, int max_sel,
                                const int32_t* schedule, const void* cent, const StatsPtrs& st, float scale,
                                void* O, float* lse, int* status, void* comp, const float* incl,
                                const void* spread_half, cudaStream_t s) {
  if (spread_half && incl) return cudaErrorInvalidValue;   // the two modes do not combine
  CUtensorMap tq, tk, tv, tc, tp, td;
  const unsigned long long BH = (unsigned long long)g.B * g.H;
  const int nchunk = (g.C + kBN - 1) / kBN;
  if (!make_tmap_bf16_3d(&tq, Q, kD, g.N, BH, 64, kBM) || !make_tmap_bf16_3d(&tk, K, kD, g.N, BH, 64, kBN) ||
      !make_tmap_bf16_3d(&tv, V, kD, g.N, BH, 64, kBN) || !make_tmap_bf16_3d(&tc, cent, kD, g.C, BH, 64, kBN) ||
      !make_tmap_bf16_tiles(&tp, comp, kD, kBN, BH * g.nB * nchunk, kChunkBytes, kBN))
    return cudaErrorInvalidValue;
  td = tc;                                                   // unused unless spread_half is given
  if (spread_half && !make_tmap_bf16_3d(&td, spread_half, kD, g.C, BH, 64, kBN)) return cudaErrorInvalidValue;
  Params p;
  p.kv_idx = kv_idx;
  p.kv_cnt = kv_cnt;
  p.schedule = schedule;
  p.max_sel = max_sel;
  p.st = st;
  p.O = (__nv_bfloat16*)O;
  p.lse = lse;
  p.status = status;
  p.comp = static_cast<const uint8_t*>(comp);
  p.incl = incl;
  p.N = g.N;
  p.C = g.C;
  p.nB = g.nB;
  p.n_items = (int)(BH * g.nB);
  p.nchunk = nchunk;
  p.scale_log2 = scale * 1.4426950408889634f;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  auto kernel = spread_half ? attention_tc_kernel<true> : attention_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = min(sms, p.n_items);
  kernel<<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, tc, tp, td, p);
  return cudaGetLastError();
}

}  // namespace da
