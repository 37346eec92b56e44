// Router logits on the tensor cores for large E and T: l[t, e] = sum_d x[t, d] W[e, d].
//
// x is bf16 (exact); the fp32 router weights are split into two bf16 planes, W ~ hi + mid
// (hi = bf16(W), mid = bf16(W - hi): 16 of fp32's 24 significand bits, |W - hi - mid| <=
// 2^-18 |W|). Every product x * plane is exact in fp32, so two tcgen05.mma kind::f16
// (bf16 x bf16 -> fp32) per K-step give logits within 2^-18 sum|x W| plus the fp32 accumulation
// error of the exact ones. They only pick the candidates that the top-k kernel recomputes in
// fp64: an error far below half of its candidate window is all they need.
//
// Method: "Routage MoE entre GPU" (viite.ai): the router scores every expert from the token's
// hidden state. The top-k and the weights follow in topk_quant_kernel (route.cu).
//
// Tiles: 128 experts (MMA M, TMEM lanes) x NT tokens (MMA N, 64 or 128); K-step = 64 bf16 = one
// 128-byte swizzled row. One stage holds the two weight planes and the token tile (40 or 48 KB;
// five or four stages). 128-token tiles halve the weight bytes per MMA; they are used when they
// still give about a wave of tiles (DeepSeek-V3 T=8192: 128 tiles instead of 1.7 waves of 64).
// Persistent grid, one CTA per SM, warp 0 = TMA producer, warp 1 = MMA issuer, warp 2 = TMEM
// allocator, warps 4-7 = epilogue (fp32 logits, coalesced over experts). Bounded waits as in
// gemm.cu.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int kRtPlaneBytes = 128 * kBK;         // 128 experts x 64 bf16
constexpr int kRtPlanes = 2;                      // bf16 planes of the router weights
template <int NT>
struct RtCfg {
  static constexpr int B_BYTES = NT * kBK;                       // NT tokens x 64 bf16
  static constexpr int STAGE_BYTES = kRtPlanes * kRtPlaneBytes + B_BYTES;
  static constexpr int STAGES = NT == 64 ? 5 : 4;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 256;
};

__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// planes[p][e][d], p = 0 hi, 1 mid.
__global__ void __launch_bounds__(256) router_split_kernel(const float* __restrict__ W, int64_t n,
                                                           uint16_t* __restrict__ planes) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  for (int64_t i = blockIdx.x * 256LL + threadIdx.x; i < n; i += (int64_t)gridDim.x * 256) {
    const float w = W[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    planes[i] = __bfloat16_as_ushort(hi);
    planes[n + i] = __bfloat16_as_ushort(mid);
  }
}

template <int kRtN>
__global__ void __launch_bounds__(256, 1)
    router_mma_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                      int T, int E, int num_kb, double* __restrict__ logits, int* status) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  constexpr int kRtStageBytes = RtCfg<kRtN>::STAGE_BYTES;
  constexpr int kRtStages = RtCfg<kRtN>::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRtStages * kRtStageBytes);
  uint64_t* empty = full + kRtStages;
  uint64_t* tfull = empty + kRtStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (E + 127) / 128, n_tiles = (T + kRtN - 1) / kRtN;
  const int total = m_tiles * n_tiles;
  if (static_cast<int>(blockIdx.x) >= total) return;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRtStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    fence_mbarrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 2 * kRtN);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_map(&map_w);
      tma_prefetch_map(&map_x);
      const uint64_t pol = l2_policy_evict_last();
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const int m = tile / n_tiles, n = tile % n_tiles;   // n fastest: shared weight tile
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u)) {
            report(status, kStatusDeviceTimeout, kWhereRoute, 10);
            ok = false;
            break;
          }
          uint8_t* st = smem + stage * kRtStageBytes;
          mbar_arrive_expect_tx(&full[stage], kRtStageBytes);
          for (int p = 0; p < kRtPlanes; ++p)
            tma_load_3d(st + p * kRtPlaneBytes, &map_w, &full[stage], kb * 64, m * 128, p, pol);
          tma_load_2d(st + kRtPlanes * kRtPlaneBytes, &map_x, &full[stage], kb * 64, n * kRtN, pol);
          ++issued;
          if (++stage == kRtStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      for (int i = 0; i < min(issued, kRtStages); ++i) {
        int st = stage - 1 - i;
        uint32_t ph = phase;
        while (st < 0) {
          st += kRtStages;
          ph ^= 1u;
        }
        mbar_wait(&full[st], ph);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kRtN);
      int stage = 0, it = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++it) {
        const int ab = it & 1;
        if (!mbar_wait(&tempty[ab], ((it >> 1) & 1) ^ 1u)) {
          report(status, kStatusDeviceTimeout, kWhereRoute, 11);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + ab * kRtN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase)) {
            report(status, kStatusDeviceTimeout, kWhereRoute, 12);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t st = smem_addr(smem + stage * kRtStageBytes);
          const uint64_t bdesc = smem_desc_sw128(st + kRtPlanes * kRtPlaneBytes);
#pragma unroll
          for (int p = 0; p < kRtPlanes; ++p) {
            const uint64_t adesc = smem_desc_sw128(st + p * kRtPlaneBytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)          // K = 16 bf16 (32 bytes) per instruction
              mma_bf16(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc,
                       (kb > 0 || p > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
          if (++stage == kRtStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) mma_commit(&tfull[ab]);
      }
      mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else if (warp >= 4) {
    const int q = warp & 3;
    bool bad = false;
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      const int m = tile / n_tiles, n = tile % n_tiles;
      const int ab = it & 1;
      if (!bad) {
        const bool ok = mbar_wait(&tfull[ab], (it >> 1) & 1);
        bad = __any_sync(0xffffffffu, !ok);
        if (bad && lane == 0) report(status, kStatusDeviceTimeout, kWhereRoute, 13);
      }
      tc_fence_after_sync();
      const int e = m * 128 + 32 * q + lane;
      const uint32_t tbase = tmem_base + ab * kRtN + (static_cast<uint32_t>(32 * q) << 16);
      const int t0 = n * kRtN;
      const int nvalid = min(kRtN, T - t0);
      for (int c0 = 0; !bad && c0 < nvalid; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(tbase + c0, r);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c)
          if (c0 + c < nvalid && e < E)
            logits[(size_t)(t0 + c0 + c) * E + e] = static_cast<double>(__uint_as_float(r[c]));
      }
      tc_fence_before_sync();
      __syncwarp();
      if (!bad && lane == 0) mbar_arrive(&tempty[ab]);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, 2 * kRtN);
  }
}

int router_mma_tokens(int T, int E) {
  return ((E + 127) / 128) * ((T + 127) / 128) >= 100 ? 128 : 64;
}

template <int NT>
static cudaError_t launch_router_mma_t(const Plan& p, const CUtensorMap& map_w,
                                       const CUtensorMap& map_x, double* logits, int* status,
                                       cudaStream_t s) {
  static bool attr_done[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 64 && !attr_done[dev]) {
    err = cudaFuncSetAttribute(router_mma_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               RtCfg<NT>::SMEM);
    if (err != cudaSuccess) return err;
    attr_done[dev] = true;
  }
  const int tiles = ((p.E + 127) / 128) * ((p.T + NT - 1) / NT);
  const int grid = std::min(tiles, num_sms());
  launch_pdl(router_mma_kernel<NT>, dim3(grid), dim3(256), RtCfg<NT>::SMEM, s, map_w, map_x, p.T,
             p.E, (p.d + 63) / 64, logits, status);
  return cudaGetLastError();
}

cudaError_t launch_router_mma(const Plan& p, const float* router_w, uint16_t* planes,
                              const CUtensorMap& map_w, const CUtensorMap& map_x, double* logits,
                              int* status, cudaStream_t s) {
  const int64_t n = (int64_t)p.E * p.d;
  const int split_blocks = (int)std::min<int64_t>((n + 255) / 256, 4LL * num_sms());
  launch_pdl(router_split_kernel, dim3(split_blocks), dim3(256), 0, s, router_w, n, planes);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  return router_mma_tokens(p.T, p.E) == 128
             ? launch_router_mma_t<128>(p, map_w, map_x, logits, status, s)
             : launch_router_mma_t<64>(p, map_w, map_x, logits, status, s);
}

}  // namespace moe
