// Internal launch interface between the C ABI (da_api.cu, noalloc.cu) and the kernel files.
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
  uint8_t* comp;       // compensation tiles of the tensor-core path, or NULL
};

struct Dims {
  int B, H, N, d, C, block, nB;
  bool bf16;
};

// Argument checks shared by every entry point (da_api.cu).  check_dims fills g from dims and
// enforces every size limit of include/da.h; check_stats validates the output pointers for g.
da_status check_dims(const da_dims* dims, Dims* g);
da_status check_stats(const Dims& g, const da_cluster_stats* st, StatsPtrs* p);

// Workspace layout (byte offsets), shared by every call.
struct WsLayout {
  size_t status, norms, sched, ent_rows, total;
};
WsLayout ws_layout(const Dims& g);

// Compensation tiles (byte offsets inside da_cluster_stats.comp_tiles; layout in include/da.h).
// An entry tile's operand rows come in groups of 8: group a holds the 64-column panel 0 of its
// 8 rows (1024 B) and then panel 1 (1024 B), each 128-byte row with 16-byte chunk k stored at
// k XOR (row mod 8).  A run of whole groups is thus one contiguous range for both panels.
constexpr int kEntRows = 128;                           // rows of one block's entry tile (= block)
constexpr size_t kEntGroup = 2048;                       // 8 rows x 2 panels x 128 B
constexpr size_t kEntVOff = 16 * kEntGroup;              // -S_e / n_e rows (after the 32 KB of centroid rows)
constexpr size_t kEntBiasOff = 2 * kEntVOff;             // log2 n_e per row (fp32)
__host__ __device__ constexpr size_t ent_byte(int row, int panel, int chunk) {
  return (size_t)(row >> 3) * kEntGroup + (size_t)panel * 1024 + (size_t)(row & 7) * 128 + (size_t)((chunk ^ (row & 7)) << 4);
}
constexpr size_t kEntTileBytes = kEntBiasOff + kEntRows * sizeof(float);   // 66048
struct CompLayout {
  size_t ent, cmean, cbias, total;
  int cpad;                                              // C rounded up to 128 (bias row length)
};
bool comp_tiles_used(const Dims& g);                     // the tensor-core path
CompLayout comp_layout(const Dims& g);                   // total 0 when not used

// stats.cu
cudaError_t launch_centroid_norms(const Dims& g, const void* cent, float* norms, cudaStream_t s);
cudaError_t launch_block_stats(const Dims& g, const void* V, const StatsPtrs& st, cudaStream_t s);
cudaError_t launch_totals(const Dims& g, const StatsPtrs& st, cudaStream_t s);
cudaError_t launch_centroid_update(const Dims& g, const StatsPtrs& st, void* cent, cudaStream_t s);
cudaError_t launch_cluster_spread(const Dims& g, const void* K, const void* cent, const StatsPtrs& st, float* spread,
                                  cudaStream_t s);
cudaError_t launch_schedule(const Dims& g, const int32_t* kv_idx, const int32_t* kv_cnt, int max_sel,
                            int32_t* schedule, int* status, cudaStream_t s);

// reassign_tc.cu
bool reassign_tc_supported(const Dims& g);
cudaError_t launch_reassign_tc(const Dims& g, const void* K, const void* V, const void* cent, const float* norms,
                               const StatsPtrs& st, int* status, cudaStream_t s);

// attention_tc.cu
bool attention_tc_supported(const Dims& g);
// ent_rows: [B*H*nB] int32 workspace for the per-item entry row counts (written, then read, by
// this call); stats unused (a zero StatsPtrs) in the inclusion-probability mode.
cudaError_t launch_attention_tc(const Dims& g, const void* Q, const void* K, const void* V,
                                const int32_t* kv_idx, const int32_t* kv_cnt, int max_sel,
                                const int32_t* schedule, const void* cent, const StatsPtrs& st, float scale,
                                void* O, float* lse, int* status, int32_t* ent_rows, const float* incl,
                                cudaStream_t s);

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
