// Router top-k for callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc, or any allocator, at the point where they
// route tokens: a serving engine that carved all of device memory into its own pools at start-up,
// a step replayed from a captured CUDA graph that must not allocate, or code running under a
// memory budget enforced by a framework allocator it cannot reach from C. They cannot provide the
// workspace moe_route_topk needs. moe_route_topk_noalloc computes the same routing decision with
// its scratch (the partial router logits) in a fixed device array that belongs to this library.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds its
// MOE_NOALLOC_SCRATCH_BYTES until the process exits. In host code its name is only a host-side
// stand-in, so the kernels get its device address from cudaGetSymbolAddress, taken once per
// device (with that device current) by the first call on that device.
#include <algorithm>
#include <atomic>
#include <cstring>

#include "../../include/moe.h"
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

static __device__ __align__(256) unsigned char g_route_scratch[MOE_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
// One cached address per device. Host threads that make their first call on a device at the same
// time may both look it up; they store the same value, so relaxed atomics suffice.
std::atomic<void*> g_scratch_addr[kMaxDevices] = {};

// Device address of g_route_scratch on the current device (looked up once per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  void* p = g_scratch_addr[dev].load(std::memory_order_relaxed);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    g_scratch_addr[dev].store(p, std::memory_order_relaxed);
  }
  *out = p;
  return MOE_OK;
}
}  // namespace

}  // namespace moe

using namespace moe;

extern "C" int moe_route_topk_noalloc(const moe_dims* dims, const uint16_t* hidden,
                                      const float* router_w, const float* router_bias, int32_t k,
                                      const int32_t* k_per_token, int32_t* topk_ids,
                                      float* topk_w, void* stream) {
  if (!dims) return MOE_ERR_INVALID_ARG;
  Plan p;
  int rc = plan_make(dims->T, dims->d, dims->E, dims->F, dims->k_max, dims->F_shared, &p);
  if (rc != MOE_OK) return rc;
  if (p.T == 0) return MOE_OK;
  if (!hidden || !router_w || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(hidden) | reinterpret_cast<uintptr_t>(router_w)) % 16)
    return MOE_ERR_INVALID_ARG;
  if (k_per_token ? (reinterpret_cast<uintptr_t>(k_per_token) % 4) != 0
                  : (k < 1 || k > std::min(p.E, p.k_max)))
    return MOE_ERR_INVALID_ARG;
  // Scratch: the fp64 partial logits of the CUDA-core router (the fused small-E router needs
  // none), cut into pieces of d the same way as the workspace router's CUDA-core path
  const bool fused = router_is_fused(p);
  int chunks = 0;
  const int splits = router_splits(p.T, p.d, p.E, &chunks);
  const size_t need = fused ? 0 : sizeof(double) * (size_t)splits * p.T * p.E;
  if (need > MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int major = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (major != 10) return MOE_ERR_UNSUPPORTED;
  if (fused) {
    // k_t out of range is clamped; there is no status word to report it in
    if (launch_route_fused(p, hidden, router_w, router_bias, k, k_per_token, topk_ids, topk_w,
                           nullptr, nullptr, false, nullptr, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  void* scratch = nullptr;
  rc = scratch_address(&scratch);
  if (rc != MOE_OK) return rc;
  Plan q = p;                      // always the CUDA-core logits (no tensor-core weight planes)
  q.r_splits = splits;
  q.r_chunks_per_split = chunks;
  double* part = static_cast<double*>(scratch);
  if (launch_router_logits(q, hidden, router_w, part, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_topk_quant(q, part, router_bias, k, k_per_token, topk_ids, topk_w, hidden, nullptr,
                        nullptr, true, false, nullptr, nullptr, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
