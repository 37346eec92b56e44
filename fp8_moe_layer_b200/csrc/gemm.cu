// Grouped W8A8 FP8 GEMMs of the expert FFN on the 5th-generation tensor cores (tcgen05):
// TMA loads of e4m3 tiles into 128-byte-swizzled shared memory, tcgen05.mma kind::f8f6f4 with
// fp32 accumulators in tensor memory (TMEM), and fused epilogues read back with tcgen05.ld.
//
//   gate/up GEMM: h = x_scale[r] * w13_scale[e, j] * sum_d xq[r, d] w13[e, j, d];
//                 epilogue act = silu(h_gate) * h_up, stored fp32, per-row max |act| (atomicMax)
//   down GEMM:    o = s2[r] * w2_scale[e, i] * sum_f aq[r, f] w2[e, i, f]  (optionally split K)
//
// Method: the megakernel page (seventnews.com), W8A8 paragraph and section "Comment fonctionne le
// megakernel" (expert compute on 8-bit weights and activations, intermediates kept on chip).
//
// Shape of the work: "swap-AB". The MMA's M = 128 rows come from the WEIGHTS (output channels of
// one expert) and its N = BN columns from the routed TOKEN rows of that expert, so a decode
// batch with a handful of tokens per expert still fills the 128-row tensor-core tile and every
// weight byte is streamed from HBM once. A gate/up tile holds 64 gate rows and the matching 64
// up rows (two TMA boxes), so SwiGLU is computed inside one CTA.
//
// Persistent kernel, one CTA per SM, static round-robin over tiles (group, m-tile, K-split,
// n-tile) with n fastest so CTAs working on the same weight tile at the same time share it in L2.
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer, warp 2 = TMEM allocator, warps 4-7 =
// epilogue (warp w reads TMEM lanes 32*(w%4) .. +31). Two TMEM accumulator buffers let the
// epilogue of one tile overlap the main loop of the next. Every wait is bounded (about 1 s); on
// expiry the kernel records MOE_ERR_DEVICE_TIMEOUT, drains its in-flight copies and MMAs, frees
// TMEM and returns.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

template <int BN, bool GATEUP>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int A_BYTES = BM * kBK;
  static constexpr int B_BYTES = BN * kBK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int XCHG_LD = 33;                       // padded row of the exchange buffer
  static constexpr int XCHG_BYTES = GATEUP ? 128 * XCHG_LD * 4 : 0;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_MAX = 232448;                  // 227 KB per block
  static constexpr int STAGES_FIT = (SMEM_MAX - 1024 - XCHG_BYTES - BAR_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + XCHG_BYTES + BAR_BYTES;
  static constexpr int TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;   // two accumulator buffers
  static constexpr int CW = BN < 32 ? BN : 32;                 // epilogue column chunk
  static_assert(STAGES >= 3, "pipeline too shallow");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M=128");
};

// tile -> (group g, m-tile, K-split s, n-tile). Group g covers tiles
// [MS * prefix[g], MS * prefix[g+1]) with MS = m_tiles * splits; inside it n runs fastest.
__device__ __forceinline__ void decode_tile(const GemmArgs& a, int tile, int& g, int& m, int& n,
                                            int& s) {
  const int ms = a.m_tiles * a.splits;
  const int v = tile / ms;
  int lo = 0, hi = a.G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.tile_prefix[mid] <= v) lo = mid;
    else hi = mid - 1;
  }
  g = lo;
  const int local = tile - ms * a.tile_prefix[g];
  const int nt = a.tile_prefix[g + 1] - a.tile_prefix[g];
  n = local % nt;
  const int rest = local / nt;
  s = rest % a.splits;
  m = rest / a.splits;
}

template <int BN, bool GATEUP>
__global__ void __launch_bounds__(256, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                        const __grid_constant__ CUtensorMap map_a_shared,
                        const __grid_constant__ CUtensorMap map_b, const GemmArgs args) {
  using C = GemmCfg<BN, GATEUP>;
  constexpr int kWhere = GATEUP ? kWhereGemm1 : kWhereGemm2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = smem;
  float* xchg = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::XCHG_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total_tiles = args.m_tiles * args.splits * args.tile_prefix[args.G];
  if (static_cast<int>(blockIdx.x) >= total_tiles) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    fence_mbarrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_map(&map_a);
      tma_prefetch_map(&map_a_shared);
      tma_prefetch_map(&map_b);
      const uint64_t pol_w = l2_policy_evict_first();   // weights: streamed once
      const uint64_t pol_x = l2_policy_evict_last();    // activations: reused by every m-tile
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        int g, m, n, s;
        decode_tile(args, tile, g, m, n, s);
        const int row0 = args.group_offsets[g] + n * BN;
        const int kb0 = s * args.kb_per_split;
        const int kb1 = min(args.num_kb, kb0 + args.kb_per_split);
        const bool sh = g >= args.E_routed;
        const CUtensorMap* ma = sh ? &map_a_shared : &map_a;
        const int ga = sh ? 0 : g;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u)) {
            report(args.status, kStatusDeviceTimeout, kWhere, 1);
            ok = false;
            break;
          }
          uint8_t* sa = stages + stage * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          if (GATEUP) {
            tma_load_4d(sa, ma, &full[stage], kb * kBK, m * 64, 0, ga, pol_w);
            tma_load_4d(sa + C::A_BYTES / 2, ma, &full[stage], kb * kBK, m * 64, 1, ga, pol_w);
          } else {
            tma_load_3d(sa, ma, &full[stage], kb * kBK, m * 128, ga, pol_w);
          }
          tma_load_2d(sa + C::A_BYTES, &map_b, &full[stage], kb * kBK, row0, pol_x);
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: the most recent load of every stage must have landed before the CTA exits.
      const int outstanding = min(issued, C::STAGES);
      for (int i = 0; i < outstanding; ++i) {
        int st = stage - 1 - i;
        uint32_t ph = phase;
        while (st < 0) {
          st += C::STAGES;
          ph ^= 1u;
        }
        mbar_wait(&full[st], ph);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (one thread)
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3_f32(128, BN);
      int stage = 0, it = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++it) {
        int g, m, n, s;
        decode_tile(args, tile, g, m, n, s);
        const int kb0 = s * args.kb_per_split;
        const int kb1 = min(args.num_kb, kb0 + args.kb_per_split);
        const int ab = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait(&tempty[ab], aph ^ 1u)) {
          report(args.status, kStatusDeviceTimeout, kWhere, 2);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + ab * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase)) {
            report(args.status, kStatusDeviceTimeout, kWhere, 3);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sa = smem_addr(stages + stage * C::STAGE_BYTES);
          const uint64_t adesc = smem_desc_sw128(sa);
          const uint64_t bdesc = smem_desc_sw128(sa + C::A_BYTES);
#pragma unroll
          for (int kk = 0; kk < kBK / 32; ++kk)   // K = 32 e4m3 (32 bytes) per instruction
            mma_e4m3(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc,
                     (kb > kb0 || kk > 0) ? 1u : 0u);
          mma_commit(&empty[stage]);               // frees the stage when these MMAs finish
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) mma_commit(&tfull[ab]);            // accumulator ready for the epilogue
      }
      mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue (4 warps)
    // After a timeout a warp keeps walking the tile list and joins every named barrier (so the
    // other epilogue warps never wait on it) but touches neither TMEM nor global memory.
    const int q = warp & 3;
    const int tid_e = threadIdx.x - 128;
    bool bad = false;
    int it = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++it) {
      int g, m, n, s;
      decode_tile(args, tile, g, m, n, s);
      const int ab = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      if (!bad) {
        const bool ok = mbar_wait(&tfull[ab], aph);
        bad = __any_sync(0xffffffffu, !ok);         // warp-uniform: TMEM loads are .sync.aligned
        if (bad && lane == 0) report(args.status, kStatusDeviceTimeout, kWhere, 4);
      }
      tc_fence_after_sync();
      const int row0 = args.group_offsets[g] + n * BN;
      const int nvalid = min(BN, args.group_offsets[g + 1] - row0);
      const bool sh = g >= args.E_routed;
      const float* wsc = sh ? args.w_scale_shared : args.w_scale + (size_t)g * args.w_scale_ld;
      const uint32_t tbase = tmem_base + ab * BN + (static_cast<uint32_t>(32 * q) << 16);
      if constexpr (GATEUP) {
        constexpr int CW = C::CW;
        const int jj = 32 * (q & 1) + lane;           // row inside the 64-row half
        const int half = q >> 1;                       // 0: gate rows, 1: up rows
        const int frow = m * 64 + jj;
        const float wsv = frow < args.M_valid ? wsc[half * args.M_valid + frow] : 0.f;
        const int j = tid_e & 63;                      // compute mapping: fixed row j per thread
        const int f = m * 64 + j;
        for (int c0 = 0; c0 < nvalid; c0 += CW) {
          if (!bad) {
            uint32_t r[CW];
            tmem_ld16(tbase + c0, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
            if constexpr (CW == 32)
              tmem_ld16(tbase + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
            tmem_wait_ld();
            float* xr = xchg + (32 * q + lane) * C::XCHG_LD;
#pragma unroll
            for (int c = 0; c < CW; ++c) xr[c] = __uint_as_float(r[c]) * wsv;
          }
          named_bar_sync(1, 128);
          if (!bad) {
#pragma unroll 4
            for (int ii = 0; ii < CW / 2; ++ii) {
              const int c = (tid_e >> 6) + 2 * ii;      // warp-uniform column
              const int nn = c0 + c;
              float act = 0.f;
              if (nn < nvalid && f < args.M_valid) {
                const float rs = args.row_scale[row0 + nn];
                const float gv = xchg[j * C::XCHG_LD + c] * rs;
                const float uv = xchg[(64 + j) * C::XCHG_LD + c] * rs;
                act = gv / (1.f + expf(-gv)) * uv;
                args.out[(size_t)(row0 + nn) * args.out_ld + f] = act;
              }
              float a = fabsf(act);
#pragma unroll
              for (int off = 16; off > 0; off >>= 1)
                a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
              if (lane == 0 && nn < nvalid)
                atomicMax(&args.row_amax[row0 + nn], __float_as_uint(a));
            }
          }
          named_bar_sync(1, 128);
        }
      } else {
        const int i = m * 128 + 32 * q + lane;         // output channel
        const float wsv = i < args.M_valid ? wsc[i] : 0.f;
        float* outp = args.out + (size_t)s * args.out_split_stride;
        for (int c0 = 0; !bad && c0 < nvalid; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(tbase + c0, r);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int nn = c0 + c;
            if (nn < nvalid && i < args.M_valid)
              outp[(size_t)(row0 + nn) * args.out_ld + i] =
                  __uint_as_float(r[c]) * args.row_scale[row0 + nn] * wsv;
          }
        }
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
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

namespace {
template <int BN, bool GATEUP>
cudaError_t launch_gemm_t(const CUtensorMap& a, const CUtensorMap& ash, const CUtensorMap& b,
                          const GemmArgs& args, cudaStream_t s) {
  using C = GemmCfg<BN, GATEUP>;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 64 && !attr_done[dev]) {
    err = cudaFuncSetAttribute(grouped_gemm_kernel<BN, GATEUP>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (err != cudaSuccess) return err;
    attr_done[dev] = true;
  }
  grouped_gemm_kernel<BN, GATEUP><<<num_sms(), 256, C::SMEM, s>>>(a, ash, b, args);
  return cudaGetLastError();
}

template <bool GATEUP>
cudaError_t launch_by_bn(int BN, const CUtensorMap& a, const CUtensorMap& ash,
                         const CUtensorMap& b, const GemmArgs& args, cudaStream_t s) {
  switch (BN) {
    case 16: return launch_gemm_t<16, GATEUP>(a, ash, b, args, s);
    case 32: return launch_gemm_t<32, GATEUP>(a, ash, b, args, s);
    case 64: return launch_gemm_t<64, GATEUP>(a, ash, b, args, s);
    case 128: return launch_gemm_t<128, GATEUP>(a, ash, b, args, s);
    case 256: return launch_gemm_t<256, GATEUP>(a, ash, b, args, s);
    default: return cudaErrorInvalidValue;
  }
}
}  // namespace

cudaError_t launch_gemm_gateup(const Plan& p, const CUtensorMap& w13, const CUtensorMap& w13s,
                               const CUtensorMap& acts, const GemmArgs& a, cudaStream_t s) {
  return launch_by_bn<true>(p.BN, w13, w13s, acts, a, s);
}

cudaError_t launch_gemm_down(const Plan& p, const CUtensorMap& w2, const CUtensorMap& w2s,
                             const CUtensorMap& acts, const GemmArgs& a, cudaStream_t s) {
  return launch_by_bn<false>(p.BN, w2, w2s, acts, a, s);
}

}  // namespace moe
