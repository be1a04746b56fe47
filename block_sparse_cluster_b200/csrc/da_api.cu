// C ABI of libda.so: argument checks, workspace layout and kernel launches.
// Every check happens before the first launch, so a call that returns an error launched nothing.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include "da.h"
#include "da_internal.h"

using namespace da;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace da {

da_status check_dims(const da_dims* dims, Dims* g) {
  if (!dims) return DA_ERR_INVALID_ARG;
  if (dims->B <= 0 || dims->H <= 0 || dims->N <= 0 || dims->d <= 0 || dims->C <= 0 || dims->block <= 0)
    return DA_ERR_INVALID_ARG;
  if (dims->dtype != DA_BF16 && dims->dtype != DA_F32) return DA_ERR_DTYPE;
  if (dims->d != 64 && dims->d != 128) return DA_ERR_UNSUPPORTED;
  if (dims->block != 64 && dims->block != 128) return DA_ERR_UNSUPPORTED;
  if (dims->C % 32 != 0 || dims->C > 1024) return DA_ERR_UNSUPPORTED;
  g->B = dims->B;
  g->H = dims->H;
  g->N = dims->N;
  g->d = dims->d;
  g->C = dims->C;
  g->block = dims->block;
  g->nB = (dims->N + dims->block - 1) / dims->block;
  g->bf16 = dims->dtype == DA_BF16;
  const long long BH = (long long)dims->B * dims->H;
  // work items and block-row indices are int32 on the device
  if (BH * g->nB >= (1LL << 31) || BH * dims->N >= (1LL << 31)) return DA_ERR_SHAPE;
  // a head's lookup rows (seg_idx, blk_hist: nB x C) are indexed in 32 bits
  if ((long long)g->nB * dims->C >= (1LL << 31)) return DA_ERR_SHAPE;
  // the tensor-core path addresses block entries (block row x block + entry) in 32 bits
  if (g->bf16 && BH * g->nB * g->block >= (1LL << 32)) return DA_ERR_SHAPE;
  return DA_OK;
}

da_status check_stats(const da_cluster_stats* st, StatsPtrs* p) {
  if (!st) return DA_ERR_INVALID_ARG;
  if (!st->assign || !st->blk_hist || !st->seg_idx || !st->seg_n || !st->seg_c || !st->seg_cnt ||
      !st->seg_vsum || !st->n_tot || !st->S_tot)
    return DA_ERR_INVALID_ARG;
  if (!aligned16(st->assign) || !aligned16(st->blk_hist) || !aligned16(st->seg_idx) || !aligned16(st->seg_n) ||
      !aligned16(st->seg_c) || !aligned16(st->seg_cnt) || !aligned16(st->seg_vsum) || !aligned16(st->n_tot) ||
      !aligned16(st->S_tot))
    return DA_ERR_ALIGNMENT;
  *p = StatsPtrs{st->assign, st->blk_hist, st->seg_idx, st->seg_n, st->seg_c,
                 st->seg_cnt, st->seg_vsum, st->n_tot, st->S_tot};
  return DA_OK;
}

}  // namespace da

namespace {

// An NVTX range around the host side of a call (argument checks and launches), named after the
// call, so that a profiler's timeline groups each call's kernels; header-only NVTX costs next to
// nothing without a profiler attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

da_status check_ws(const Dims& g, void* ws, size_t ws_bytes) {
  if (!ws) return DA_ERR_INVALID_ARG;
  if (!aligned16(ws)) return DA_ERR_ALIGNMENT;
  if (ws_bytes < ws_layout(g).total) return DA_ERR_WORKSPACE;
  return DA_OK;
}

da_status check_mask(const Dims& g, const da_block_mask* mask) {
  if (!mask || !mask->kv_idx || !mask->kv_cnt) return DA_ERR_INVALID_ARG;
  if (mask->max_sel < 1) return DA_ERR_SHAPE;
  if ((long long)g.B * g.H * g.nB * mask->max_sel >= (1LL << 40)) return DA_ERR_SHAPE;
  if (!aligned16(mask->kv_idx) || !aligned16(mask->kv_cnt)) return DA_ERR_ALIGNMENT;
  if (mask->schedule && !aligned16(mask->schedule)) return DA_ERR_ALIGNMENT;
  return DA_OK;
}

da_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DA_OK : DA_ERR_CUDA; }

}  // namespace

extern "C" {

int da_version(void) { return 103; }

size_t da_workspace_bytes(const da_dims* dims) {
  Dims g;
  if (check_dims(dims, &g) != DA_OK) return 0;
  return ws_layout(g).total;
}

size_t da_schedule_bytes(const da_dims* dims) {
  Dims g;
  if (check_dims(dims, &g) != DA_OK) return 0;
  return (size_t)g.B * g.H * g.nB * sizeof(int32_t);
}

da_status da_reassign(const da_dims* dims, const void* K, const void* V, const void* centroids,
                      const da_cluster_stats* out, void* ws, size_t ws_bytes, da_stream stream) {
  NvtxRange nvtx("da_reassign");
  Dims g;
  da_status st = check_dims(dims, &g);
  if (st != DA_OK) return st;
  if (!K || !V || !centroids) return DA_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(V) || !aligned16(centroids)) return DA_ERR_ALIGNMENT;
  StatsPtrs sp;
  if ((st = check_stats(out, &sp)) != DA_OK) return st;
  if ((st = check_ws(g, ws, ws_bytes)) != DA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(g);
  int* status = reinterpret_cast<int*>(static_cast<char*>(ws) + L.status);
  float* norms = reinterpret_cast<float*>(static_cast<char*>(ws) + L.norms);
  cudaError_t e;
  if (reassign_tc_supported(g)) {
    e = launch_centroid_norms(g, centroids, norms, s);
    if (e == cudaSuccess) e = launch_reassign_tc(g, K, V, centroids, norms, sp, status, s);
  } else {
    e = g.bf16 ? launch_assign_simt_bf16(g, K, centroids, sp.assign, s)
               : launch_assign_simt_f32(g, K, centroids, sp.assign, s);
    if (e == cudaSuccess) e = launch_block_stats(g, V, sp, s);
  }
  if (e == cudaSuccess) e = launch_totals(g, sp, s);
  return cuda_status(e);
}

da_status da_mask_prepare(const da_dims* dims, const da_block_mask* mask, int32_t* schedule,
                          size_t schedule_bytes, void* ws, size_t ws_bytes, da_stream stream) {
  NvtxRange nvtx("da_mask_prepare");
  Dims g;
  da_status st = check_dims(dims, &g);
  if (st != DA_OK) return st;
  if ((st = check_mask(g, mask)) != DA_OK) return st;
  if (!schedule) return DA_ERR_INVALID_ARG;
  if (!aligned16(schedule)) return DA_ERR_ALIGNMENT;
  if (schedule_bytes < (size_t)g.B * g.H * g.nB * sizeof(int32_t)) return DA_ERR_WORKSPACE;
  if ((st = check_ws(g, ws, ws_bytes)) != DA_OK) return st;
  const WsLayout L = ws_layout(g);
  int* status = reinterpret_cast<int*>(static_cast<char*>(ws) + L.status);
  return cuda_status(launch_schedule(g, mask->kv_idx, mask->kv_cnt, mask->max_sel, schedule, status,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

// Validation shared by da_compensation, da_attention_prebuilt and da_attention.
static da_status attention_common(const da_dims* dims, const da_block_mask* mask, const da_cluster_stats* stats,
                                  void* ws, size_t ws_bytes, Dims* g, StatsPtrs* sp) {
  da_status st = check_dims(dims, g);
  if (st != DA_OK) return st;
  if ((st = check_mask(*g, mask)) != DA_OK) return st;
  if ((st = check_stats(stats, sp)) != DA_OK) return st;
  return check_ws(*g, ws, ws_bytes);
}

static da_status check_attention_ptrs(const void* Q, const void* K, const void* V, const void* centroids,
                                      const void* O, const float* lse) {
  if (!Q || !K || !V || !centroids || !O) return DA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(centroids) || !aligned16(O) ||
      (lse && !aligned16(lse)))
    return DA_ERR_ALIGNMENT;
  return DA_OK;
}

static cudaError_t compensation_launch(const Dims& g, const da_block_mask* mask, const StatsPtrs& sp, void* ws,
                                       cudaStream_t s) {
  if (!attention_tc_supported(g)) return cudaSuccess;   // the CUDA-core path compensates in-kernel
  const WsLayout L = ws_layout(g);
  return launch_comp_build(g, mask->kv_idx, mask->kv_cnt, mask->max_sel, sp, static_cast<char*>(ws) + L.comp, s);
}

static da_status attention_launch(const Dims& g, const void* Q, const void* K, const void* V,
                                  const da_block_mask* mask, const void* centroids, const StatsPtrs& sp, float scale,
                                  void* O, float* lse, void* ws, cudaStream_t s) {
  const da_status pst = check_attention_ptrs(Q, K, V, centroids, O, lse);
  if (pst != DA_OK) return pst;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)g.d);
  const WsLayout L = ws_layout(g);
  int* status = reinterpret_cast<int*>(static_cast<char*>(ws) + L.status);
  const int32_t* sched = mask->schedule;
  cudaError_t e = cudaSuccess;
  if (!sched) {
    int32_t* own = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + L.sched);
    e = launch_schedule(g, mask->kv_idx, mask->kv_cnt, mask->max_sel, own, status, s);
    sched = own;
  }
  if (e == cudaSuccess) {
    if (attention_tc_supported(g))
      e = launch_attention_tc(g, Q, K, V, mask->kv_idx, mask->kv_cnt, mask->max_sel, sched, centroids, sp, scale, O,
                              lse, status, static_cast<char*>(ws) + L.comp, nullptr, nullptr, s);
    else
      e = (g.bf16 ? launch_attention_simt_bf16 : launch_attention_simt_f32)(
          g, Q, K, V, mask->kv_idx, mask->kv_cnt, mask->max_sel, sched, centroids, sp, nullptr, scale, O, lse, status,
          s);
  }
  return cuda_status(e);
}

da_status da_compensation(const da_dims* dims, const da_block_mask* mask, const da_cluster_stats* stats, void* ws,
                          size_t ws_bytes, da_stream stream) {
  NvtxRange nvtx("da_compensation");
  Dims g;
  StatsPtrs sp;
  da_status st = attention_common(dims, mask, stats, ws, ws_bytes, &g, &sp);
  if (st != DA_OK) return st;
  return cuda_status(compensation_launch(g, mask, sp, ws, reinterpret_cast<cudaStream_t>(stream)));
}

da_status da_attention_prebuilt(const da_dims* dims, const void* Q, const void* K, const void* V,
                                const da_block_mask* mask, const void* centroids, const da_cluster_stats* stats,
                                float scale, void* O, float* lse, void* ws, size_t ws_bytes, da_stream stream) {
  NvtxRange nvtx("da_attention_prebuilt");
  Dims g;
  StatsPtrs sp;
  da_status st = attention_common(dims, mask, stats, ws, ws_bytes, &g, &sp);
  if (st != DA_OK) return st;
  return attention_launch(g, Q, K, V, mask, centroids, sp, scale, O, lse, ws, reinterpret_cast<cudaStream_t>(stream));
}

da_status da_attention(const da_dims* dims, const void* Q, const void* K, const void* V,
                       const da_block_mask* mask, const void* centroids, const da_cluster_stats* stats,
                       float scale, void* O, float* lse, void* ws, size_t ws_bytes, da_stream stream) {
  NvtxRange nvtx("da_attention");
  Dims g;
  StatsPtrs sp;
  da_status st = attention_common(dims, mask, stats, ws, ws_bytes, &g, &sp);
  if (st != DA_OK) return st;
  if ((st = check_attention_ptrs(Q, K, V, centroids, O, lse)) != DA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e = compensation_launch(g, mask, sp, ws, s);
  if (e != cudaSuccess) return cuda_status(e);
  return attention_launch(g, Q, K, V, mask, centroids, sp, scale, O, lse, ws, s);
}

da_status da_centroid_update(const da_dims* dims, const da_cluster_stats* stats, void* centroids,
                             da_stream stream) {
  NvtxRange nvtx("da_centroid_update");
  Dims g;
  da_status st = check_dims(dims, &g);
  if (st != DA_OK) return st;
  if (!centroids) return DA_ERR_INVALID_ARG;
  if (!aligned16(centroids)) return DA_ERR_ALIGNMENT;
  StatsPtrs sp;
  if ((st = check_stats(stats, &sp)) != DA_OK) return st;
  return cuda_status(launch_centroid_update(g, sp, centroids, reinterpret_cast<cudaStream_t>(stream)));
}

da_status da_cluster_spread(const da_dims* dims, const void* K, const void* centroids, const da_cluster_stats* stats,
                            float* spread, da_stream stream) {
  NvtxRange nvtx("da_cluster_spread");
  Dims g;
  da_status st = check_dims(dims, &g);
  if (st != DA_OK) return st;
  if (!K || !centroids || !spread) return DA_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(centroids) || !aligned16(spread)) return DA_ERR_ALIGNMENT;
  StatsPtrs sp;
  if ((st = check_stats(stats, &sp)) != DA_OK) return st;
  return cuda_status(launch_cluster_spread(g, K, centroids, sp, spread, reinterpret_cast<cudaStream_t>(stream)));
}

da_status da_attention_spread(const da_dims* dims, const void* Q, const void* K, const void* V,
                              const da_block_mask* mask, const void* centroids, const da_cluster_stats* stats,
                              const float* spread, float scale, void* O, float* lse, void* ws, size_t ws_bytes,
                              da_stream stream) {
  NvtxRange nvtx("da_attention_spread");
  Dims g;
  StatsPtrs sp;
  da_status st = attention_common(dims, mask, stats, ws, ws_bytes, &g, &sp);
  if (st != DA_OK) return st;
  if ((st = check_attention_ptrs(Q, K, V, centroids, O, lse)) != DA_OK) return st;
  if (!spread) return DA_ERR_INVALID_ARG;
  if (!aligned16(spread)) return DA_ERR_ALIGNMENT;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)g.d);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(g);
  int* status = reinterpret_cast<int*>(static_cast<char*>(ws) + L.status);
  const int32_t* sched = mask->schedule;
  cudaError_t e = cudaSuccess;
  if (!sched) {
    int32_t* own = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + L.sched);
    e = launch_schedule(g, mask->kv_idx, mask->kv_cnt, mask->max_sel, own, status, s);
    sched = own;
  }
  if (e == cudaSuccess && attention_tc_supported(g)) {
    // tensor cores: the compensation pre-pass, Dh = (s/2) D in bf16, then the fused kernel in its
    // variance-corrected mode
    void* dh = static_cast<char*>(ws) + L.spread;
    e = launch_comp_build(g, mask->kv_idx, mask->kv_cnt, mask->max_sel, sp, static_cast<char*>(ws) + L.comp, s);
    if (e == cudaSuccess) e = launch_spread_half(g, spread, scale, dh, s);
    if (e == cudaSuccess)
      e = launch_attention_tc(g, Q, K, V, mask->kv_idx, mask->kv_cnt, mask->max_sel, sched, centroids, sp, scale, O,
                              lse, status, static_cast<char*>(ws) + L.comp, nullptr, dh, s);
  } else if (e == cudaSuccess) {
    e = (g.bf16 ? launch_attention_simt_bf16 : launch_attention_simt_f32)(
        g, Q, K, V, mask->kv_idx, mask->kv_cnt, mask->max_sel, sched, centroids, sp, spread, scale, O, lse, status,
        s);
  }
  return cuda_status(e);
}

da_status da_attention_sip(const da_dims* dims, const void* Q, const void* K, const void* V,
                           const da_block_mask* mask, const float* incl, float scale, void* O, float* lse, void* ws,
                           size_t ws_bytes, da_stream stream) {
  NvtxRange nvtx("da_attention_sip");
  Dims g;
  da_status st = check_dims(dims, &g);
  if (st != DA_OK) return st;
  if (!attention_tc_supported(g)) return DA_ERR_UNSUPPORTED;
  if ((st = check_mask(g, mask)) != DA_OK) return st;
  if ((st = check_ws(g, ws, ws_bytes)) != DA_OK) return st;
  if ((st = check_attention_ptrs(Q, K, V, K, O, lse)) != DA_OK) return st;
  if (!incl) return DA_ERR_INVALID_ARG;
  if (!aligned16(incl)) return DA_ERR_ALIGNMENT;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)g.d);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(g);
  int* status = reinterpret_cast<int*>(static_cast<char*>(ws) + L.status);
  const int32_t* sched = mask->schedule;
  cudaError_t e = cudaSuccess;
  if (!sched) {
    int32_t* own = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + L.sched);
    e = launch_schedule(g, mask->kv_idx, mask->kv_cnt, mask->max_sel, own, status, s);
    sched = own;
  }
  // no cluster steps: the centroid map is never read (K stands in for it), nor are the statistics
  if (e == cudaSuccess)
    e = launch_attention_tc(g, Q, K, V, mask->kv_idx, mask->kv_cnt, mask->max_sel, sched, K, StatsPtrs{}, scale, O,
                            lse, status, static_cast<char*>(ws) + L.comp, incl, nullptr, s);
  return cuda_status(e);
}

da_status da_device_status(void* ws, da_stream stream) {
  if (!ws) return DA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int word = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DA_ERR_CUDA;
  if (cudaMemcpyAsync(&word, ws, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return DA_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess) return DA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DA_ERR_CUDA;
  switch (word) {
    case 0: return DA_OK;
    case DA_ERR_TIMEOUT: return DA_ERR_TIMEOUT;
    case DA_ERR_DEVICE_INDEX: return DA_ERR_DEVICE_INDEX;
    case DA_ERR_RANGE: return DA_ERR_RANGE;
    default: return DA_ERR_CUDA;
  }
}

const char* da_status_string(da_status s) {
  switch (s) {
    case DA_OK: return "ok";
    case DA_ERR_INVALID_ARG: return "invalid argument (NULL pointer or non-positive size)";
    case DA_ERR_SHAPE: return "inconsistent or too large shape";
    case DA_ERR_DTYPE: return "unknown dtype";
    case DA_ERR_ALIGNMENT: return "tensor base pointer not 16-byte aligned";
    case DA_ERR_UNSUPPORTED: return "sizes not supported by this library (d, block or C)";
    case DA_ERR_CUDA: return "CUDA runtime or driver call failed";
    case DA_ERR_TIMEOUT: return "a bounded device wait gave up";
    case DA_ERR_DEVICE_INDEX: return "malformed block plan seen on the device";
    case DA_ERR_WORKSPACE: return "workspace or schedule buffer too small";
    case DA_ERR_RANGE: return "logits beyond the attention kernel's range (a later step's max far above the first's)";
  }
  return "unknown status";
}

}  // extern "C"
