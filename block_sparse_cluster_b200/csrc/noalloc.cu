// da_reassign_noalloc: Reassign Cache for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) when they run the step: a
// runtime whose memory plan is fixed once at start-up and forbids later device allocations, a
// host application that hands every byte of device memory to its own pool, or code on a path
// where an allocation would implicitly synchronise the device.  da_reassign needs a small
// caller-provided workspace for its scratch (the centroid norms and the device status word); this
// variant keeps that scratch in a file-scope __device__ array instead, so the caller passes only
// inputs and outputs.
//
// The array is a static allocation of the library image: every GPU that loads libda.so holds it
// until the process exits.  It is shared by every call on a device and keeps the last call's
// contents; the status word is cleared at the start of each call, the norms are rewritten in
// full.  Calls whose kernels overlap on the GPU (for instance on two streams) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "da.h"
#include "da_internal.h"

// Largest B*H*C the built-in scratch holds (one fp32 norm per centroid); 1 MiB of norms.
constexpr size_t kNoAllocMaxNorms = size_t(1) << 18;
constexpr size_t kStatusFloats = 64;   // 256 bytes ahead of the norms hold the status word

// The scratch: a file-scope device array of a fixed size (about 1 MiB).
static __device__ __align__(256) float g_noalloc_scratch[kStatusFloats + kNoAllocMaxNorms];

namespace {

// Device address of g_noalloc_scratch per device.  In host code the symbol's name is a host-side
// stand-in, not a device address: the address comes from cudaGetSymbolAddress, taken once per
// device with that device current (the first call on a device does it).
constexpr int kMaxDevices = 64;
std::mutex g_lock;
float* g_addr[kMaxDevices] = {};

cudaError_t scratch_address(int dev, float** out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> guard(g_lock);
  if (!g_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = static_cast<float*>(p);
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" DA_API da_status da_reassign_noalloc(const da_dims* dims, const void* K, const void* V,
                                                const void* centroids, const da_cluster_stats* out,
                                                da_stream stream) {
  using namespace da;
  if (!dims || !K || !V || !centroids || !out) return DA_ERR_INVALID_ARG;
  if (dims->B <= 0 || dims->H <= 0 || dims->N <= 0 || dims->d <= 0 || dims->C <= 0 || dims->block <= 0)
    return DA_ERR_INVALID_ARG;
  if (dims->dtype != DA_BF16 && dims->dtype != DA_F32) return DA_ERR_DTYPE;
  if (dims->d != 64 && dims->d != 128) return DA_ERR_UNSUPPORTED;
  if (dims->block != 64 && dims->block != 128) return DA_ERR_UNSUPPORTED;
  if (dims->C % 32 != 0 || dims->C > 1024) return DA_ERR_UNSUPPORTED;
  Dims g{dims->B, dims->H, dims->N, dims->d, dims->C, dims->block, (dims->N + dims->block - 1) / dims->block,
         dims->dtype == DA_BF16};
  const long long BH = (long long)g.B * g.H;
  if (BH * g.nB >= (1LL << 31) || BH * g.N >= (1LL << 31)) return DA_ERR_SHAPE;
  if ((size_t)BH * g.C > kNoAllocMaxNorms) return DA_ERR_WORKSPACE;   // beyond the built-in scratch
  const void* ptrs[] = {K, V, centroids, out->assign, out->blk_hist, out->seg_idx, out->seg_n, out->seg_c,
                        out->seg_cnt, out->seg_vsum, out->n_tot, out->S_tot};
  for (const void* q : ptrs) {
    if (!q) return DA_ERR_INVALID_ARG;
    if (!aligned16(q)) return DA_ERR_ALIGNMENT;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DA_ERR_CUDA;
  float* scratch = nullptr;
  if (scratch_address(dev, &scratch) != cudaSuccess) return DA_ERR_CUDA;
  int* status = reinterpret_cast<int*>(scratch);
  float* norms = scratch + kStatusFloats;
  const StatsPtrs sp{out->assign, out->blk_hist, out->seg_idx, out->seg_n, out->seg_c,
                     out->seg_cnt, out->seg_vsum, out->n_tot, out->S_tot};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), s);
  if (e == cudaSuccess) {
    if (reassign_tc_supported(g)) {
      e = launch_centroid_norms(g, centroids, norms, s);
      if (e == cudaSuccess) e = launch_reassign_tc(g, K, V, centroids, norms, sp, status, s);
    } else {
      e = g.bf16 ? launch_assign_simt_bf16(g, K, centroids, sp.assign, s)
                 : launch_assign_simt_f32(g, K, centroids, sp.assign, s);
      if (e == cudaSuccess) e = launch_block_stats(g, V, sp, s);
    }
  }
  if (e == cudaSuccess) e = launch_totals(g, sp, s);
  return e == cudaSuccess ? DA_OK : DA_ERR_CUDA;
}
