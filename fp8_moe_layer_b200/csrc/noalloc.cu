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
#include <cstring>

#include "../../include/moe.h"
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

static __device__ __align__(256) unsigned char g_route_scratch[MOE_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_route_scratch on the current device (looked up once per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
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
  // Scratch: the partial logits of the CUDA-core router (the fused small-E router needs none).
  const bool fused = router_is_fused(p);
  // the CUDA-core logits kernel's cut of d: 32x32 (token x expert) tiles, enough pieces of d for
  // about two waves of 148 SMs
  const long long rtiles = ((std::max(p.T, 1) + kRouterTile - 1) / kRouterTile) *
                           (long long)((p.E + kRouterTile - 1) / kRouterTile);
  const int nchunks = (p.d + kRouterTile - 1) / kRouterTile;
  const int want = (int)std::max(1LL, (2LL * 148 + rtiles - 1) / rtiles);
  const int cut = std::min(nchunks, want);
  const int chunks = (nchunks + cut - 1) / cut;
  const int splits = (nchunks + chunks - 1) / chunks;
  const size_t need = fused ? 0 : sizeof(float) * (size_t)splits * p.T * p.E;
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
  float* part = static_cast<float*>(scratch);
  if (launch_router_logits(q, hidden, router_w, part, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_topk_quant(q, part, router_bias, k, k_per_token, topk_ids, topk_w, hidden, nullptr,
                        nullptr, true, false, nullptr, nullptr, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
