// Internal launch interface between the C ABI (da_api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "da.h"

namespace da {

struct StatsPtrs {
  int32_t* assign;
  int32_t* blk_hist;
  uint8_t* seg_idx;
  int32_t* seg_n;
  int32_t* seg_c;
  int32_t* seg_cnt;
  float* seg_vsum;
  int32_t* n_tot;
  float* S_tot;
};

struct Dims {
  int B, H, N, d, C, block, nB;
  bool bf16;
};

// Argument checks shared by every entry point (da_api.cu).  check_dims fills g from dims and
// enforces every size limit of include/da.h; check_stats validates the output pointers.
da_status check_dims(const da_dims* dims, Dims* g);
da_status check_stats(const da_cluster_stats* st, StatsPtrs* p);

// Workspace layout (byte offsets), shared by every call.
struct WsLayout {
  size_t status, norms, sched, comp, spread, total;
};
WsLayout ws_layout(const Dims& g);

// stats.cu
cudaError_t launch_centroid_norms(const Dims& g, const void* cent, float* norms, cudaStream_t s);
cudaError_t launch_block_stats(const Dims& g, const void* V, const StatsPtrs& st, cudaStream_t s);
cudaError_t launch_totals(const Dims& g, const StatsPtrs& st, cudaStream_t s);
cudaError_t launch_centroid_update(const Dims& g, const StatsPtrs& st, void* cent, cudaStream_t s);
cudaError_t launch_cluster_spread(const Dims& g, const void* K, const void* cent, const StatsPtrs& st, float* spread,
                                  cudaStream_t s);
cudaError_t launch_schedule(const Dims& g, const int32_t* kv_idx, const int32_t* kv_cnt, int max_sel,
                            int32_t* schedule, int* status, cudaStream_t s);
// Dh = (scale / 2) D in bf16, the second operand of the variance-corrected cluster logits on the
// tensor cores ([B*H][C][d], from the fp32 second moments D).
cudaError_t launch_spread_half(const Dims& g, const float* spread, float scale, void* out, cudaStream_t s);

// reassign_tc.cu
bool reassign_tc_supported(const Dims& g);
cudaError_t launch_reassign_tc(const Dims& g, const void* K, const void* V, const void* cent, const float* norms,
                               const StatsPtrs& st, int* status, cudaStream_t s);

// attention_tc.cu
bool attention_tc_supported(const Dims& g);
size_t attention_tc_scratch_bytes(const Dims& g);   // compensation chunks of every item
cudaError_t launch_attention_tc(const Dims& g, const void* Q, const void* K, const void* V,
                                const int32_t* kv_idx, const int32_t* kv_cnt, int max_sel,
                                const int32_t* schedule, const void* cent, const StatsPtrs& st, float scale,
                                void* O, float* lse, int* status, void* comp, const float* incl,
                                const void* spread_half, cudaStream_t s);

// comp_build.cu
cudaError_t launch_comp_build(const Dims& g, const int32_t* kv_idx, const int32_t* kv_cnt, int max_sel,
                              const StatsPtrs& st, void* out, cudaStream_t s);

// simt_f32.cu / simt_bf16.cu
#define DA_SIMT_DECL(SUFFIX)                                                                                 \
  cudaError_t launch_assign_simt_##SUFFIX(const Dims& g, const void* K, const void* cent, int32_t* assign,    \
                                          cudaStream_t s);                                                    \
  cudaError_t launch_attention_simt_##SUFFIX(const Dims& g, const void* Q, const void* K, const void* V,      \
                                             const int32_t* kv_idx, const int32_t* kv_cnt, int max_sel,       \
                                             const int32_t* schedule, const void* cent, const StatsPtrs& st,  \
                                             const float* spread, float scale, void* O, float* lse,           \
                                             int* status, cudaStream_t s);
DA_SIMT_DECL(f32)
DA_SIMT_DECL(bf16)
#undef DA_SIMT_DECL

}  // namespace da
