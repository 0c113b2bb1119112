// instagen_cluster_static: the k-means + permutation call with its scratch in
// a fixed device array owned by the library, for callers that must not
// allocate device memory (see include/instagen.h).
//
// The scratch is the centroid operand of the distance GEMM ([BH, C_pad, 2d]
// bf16), the norm rows ([BH, C_pad, 32] bf16), the update's piece map, partial sums and
// its arrival counters, the same layout instagen_cluster carves from a
// caller-provided workspace.  Every element the kernels read from it is first
// written by the same call (the init kernel writes every operand row, padding
// included, and zeroes the counters), so nothing has to be cleared between
// calls; stale contents of an earlier call are never read.
#include "instagen.h"
#include "internal.cuh"

#include <cuda_runtime.h>

#include <mutex>

namespace {

// File-scope device array: every GPU that loads the library holds these
// INSTAGEN_CLUSTER_STATIC_SCRATCH_BYTES until the process exits.
static __device__ __align__(256) unsigned char g_cluster_scratch[INSTAGEN_CLUSTER_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  return fn;
}

// Device address of g_cluster_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress with that device current.  It is looked up on the
// first call on a device and again whenever the device's current context
// differs from the one it was looked up in (a cudaDeviceReset, or a primary
// context destroyed and created again, reloads the module at a new address).
int static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return IG_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return IG_ERR_UNSUPPORTED;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  CUcontext ctx = nullptr;
  if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return IG_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev] || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_cluster_scratch) != cudaSuccess || !p) return IG_ERR_CUDA;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_addr[dev];
  return IG_OK;
}

}  // namespace

extern "C" int instagen_cluster_static(const void* X, int32_t C, int32_t iters, const float* init,
                                       const instagen_params* p, float* centroids, int32_t* assign, int32_t* perm,
                                       int32_t* offsets, void* stream) {
  int rc = check_params(p);
  if (rc) return rc;
  if ((rc = check_clusters(C))) return rc;
  if (iters < 1 || iters > 10000) return IG_ERR_INVALID_ARG;
  if (!X || !centroids || !assign || !perm || !offsets || !aligned16(X)) return IG_ERR_INVALID_ARG;
  const size_t need = ig::kmeans_scratch_bytes(ig::kmeans_geom(p->B * p->H, p->N, p->d, C));
  if (need > (size_t)INSTAGEN_CLUSTER_STATIC_SCRATCH_BYTES) return IG_ERR_WORKSPACE;
  void* ws = nullptr;
  if ((rc = static_scratch_address(&ws))) return rc;
  return run_cluster(X, C, iters, init, p, centroids, assign, perm, offsets, ws,
                     (size_t)INSTAGEN_CLUSTER_STATIC_SCRATCH_BYTES, static_cast<cudaStream_t>(stream));
}
