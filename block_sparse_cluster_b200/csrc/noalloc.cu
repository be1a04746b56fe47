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

#include "da.h"
#include "da_internal.h"

// Largest B*H*C the built-in scratch holds (one fp32 norm per centroid); 1 MiB of norms.
constexpr size_t kNoAllocMaxNorms = size_t(1) << 18;
constexpr size_t kStatusFloats = 64;   // 256 bytes ahead of the norms hold the status word

// The scratch: a file-scope device array of a fixed size (about 1 MiB).
static __device__ __align__(256) float g_noalloc_scratch[kStatusFloats + kNoAllocMaxNorms];

namespace {

// Device address of g_noalloc_scratch on the current device.  In host code the symbol's name is a
// host-side stand-in, not a device address: the address comes from cudaGetSymbolAddress with the
// device current.  It is looked up on every call, not cached, so that a context that was torn down
// and made again (cudaDeviceReset) never leaves a stale address behind; after the first call on a
// device, which loads the library's module there, the lookup is a table read.
cudaError_t scratch_address(float** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  *out = static_cast<float*>(p);
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
  float* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return DA_ERR_CUDA;
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

// The status word of the built-in scratch on the current device: synchronise `stream`, read the
// word, clear it.  The same codes as da_device_status.
extern "C" DA_API da_status da_noalloc_device_status(da_stream stream) {
  float* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return DA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int word = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DA_ERR_CUDA;
  if (cudaMemcpyAsync(&word, scratch, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return DA_ERR_CUDA;
  if (cudaMemsetAsync(scratch, 0, sizeof(int), s) != cudaSuccess) return DA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DA_ERR_CUDA;
  switch (word) {
    case 0: return DA_OK;
    case DA_ERR_TIMEOUT: return DA_ERR_TIMEOUT;
    case DA_ERR_DEVICE_INDEX: return DA_ERR_DEVICE_INDEX;
    case DA_ERR_RANGE: return DA_ERR_RANGE;
    default: return DA_ERR_CUDA;
  }
}
