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
#include <nvtx3/nvToolsExt.h>

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

static da_status reassign_noalloc(const da_dims* dims, const void* K, const void* V, const void* centroids,
                                  const da_cluster_stats* out, da_stream stream);

extern "C" DA_API da_status da_reassign_noalloc(const da_dims* dims, const void* K, const void* V,
                                                const void* centroids, const da_cluster_stats* out,
                                                da_stream stream) {
  using namespace da;
  nvtxRangePushA("da_reassign_noalloc");
  const da_status st = reassign_noalloc(dims, K, V, centroids, out, stream);
  nvtxRangePop();
  return st;
}

static da_status reassign_noalloc(const da_dims* dims, const void* K, const void* V, const void* centroids,
                                  const da_cluster_stats* out, da_stream stream) {
  using namespace da;
  // the same argument checks as da_reassign, then the size of the built-in scratch
  Dims g;
  da_status st = check_dims(dims, &g);
  if (st != DA_OK) return st;
  if (!K || !V || !centroids) return DA_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(V) || !aligned16(centroids)) return DA_ERR_ALIGNMENT;
  StatsPtrs sp;
  if ((st = check_stats(out, &sp)) != DA_OK) return st;
  if ((size_t)g.B * g.H * g.C > kNoAllocMaxNorms) return DA_ERR_WORKSPACE;   // beyond the built-in scratch
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DA_ERR_CUDA;
  float* scratch = nullptr;
  if (scratch_address(dev, &scratch) != cudaSuccess) return DA_ERR_CUDA;
  int* status = reinterpret_cast<int*>(scratch);
  float* norms = scratch + kStatusFloats;
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
