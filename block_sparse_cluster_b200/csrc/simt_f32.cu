// fp32 instantiations of the CUDA-core reassignment and attention kernels.
#include "simt_kernels.cuh"

namespace da {

using T = float;
#include "simt_launch.inc"

cudaError_t launch_assign_simt_f32(const Dims& g, const void* K, const void* cent, int32_t* assign, cudaStream_t s) {
  return launch_assign_simt_t(g, K, cent, assign, s);
}

cudaError_t launch_attention_simt_f32(const Dims& g, const void* Q, const void* K, const void* V,
                                      const int32_t* kv_idx, const int32_t* kv_cnt, int max_sel,
                                      const int32_t* schedule, const void* cent, const StatsPtrs& st,
                                      const float* spread, float scale, void* O, float* lse, int* status,
                                      cudaStream_t s) {
  return launch_attention_simt_t(g, Q, K, V, kv_idx, kv_cnt, max_sel, schedule, cent, st, spread, scale, O, lse,
                                 status, s);
}

}  // namespace da
