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
// one expert) and its N columns from the routed TOKEN rows of that expert, so a decode batch with
// a handful of tokens per expert still fills the 128-row tensor-core tile and every weight byte
// is streamed from HBM once. A tile loads and multiplies only its valid token rows (N = rows
// rounded up to 16, chosen per tile at run time). A gate/up tile holds 64 gate rows and the
// matching 64 up rows (two TMA boxes), so SwiGLU is computed inside one CTA.
//
// Pipeline: a ring of shared-memory stages, each holding one K-block of weights (16 KB) and of the
// tile's token rows; as many stages as fit in 227 KB. Persistent kernel, one CTA per SM, static
// round-robin over tiles (group, m-tile, K-split, n-tile) with n fastest so CTAs working on the
// same weight tile at the same time share it in L2.
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer, warp 2 = TMEM allocator, warps 4-7 =
// epilogue (warp w reads TMEM lanes 32*(w%4) .. +31). Two TMEM accumulator buffers let the
// epilogue of one tile overlap the main loop of the next. Every wait is bounded (about 1 s); on
// expiry the kernel records MOE_ERR_DEVICE_TIMEOUT, drains its in-flight copies and MMAs, frees
// TMEM and returns.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

#ifdef MOE_ROLE_COUNTERS
// Role-counter build only: cycles each warp role of each CTA spent waiting, per GEMM mode
// ([mode][cta][counter]): 0 producer waiting for a free stage, 1 MMA issuer waiting for a free
// accumulator, 2 MMA issuer waiting for a stage's data, 3 K blocks issued, 4 epilogue waiting for
// an accumulator, 5 cycles from set-up to the end, 6 tiles.
constexpr int kRoleMaxCtas = 256;
__device__ unsigned long long g_role_cycles[3][kRoleMaxCtas][8];
#define MOE_ROLE_T0(v) const unsigned long long v = clock64()
#define MOE_ROLE_ADD(mode, i, val) \
  do { if (blockIdx.x < kRoleMaxCtas) g_role_cycles[mode][blockIdx.x][i] += (val); } while (0)
#else
#define MOE_ROLE_T0(v)
#define MOE_ROLE_ADD(mode, i, val)
#endif

template <int BN, int MODE, bool PAIR, int SLABS = 1>
struct GemmCfg {
  static constexpr int BM = 128;                           // weight rows of one slab
  static constexpr int BROWS = PAIR ? BN / 2 : BN;         // token rows held by one CTA
  static constexpr int ROUND = PAIR ? 32 : 16;             // MMA N granule (halves of 16 rows)
  static constexpr int SLAB_BYTES = BM * kBK;
  static constexpr int A_BYTES = SLABS * SLAB_BYTES;       // weight rows held by one CTA
  static constexpr int B_BYTES = BROWS * kBK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int XCHG_LD = 33;                       // padded row of the exchange buffer
  // SwiGLU: gate/up exchange; down GEMM with prefill tiles: per-warp transpose for 16-byte stores
  static constexpr bool DOWN_T = MODE == kModeDown && BN >= 128;
  static constexpr int XCHG_BYTES = (MODE == kModeSwiGLU || DOWN_T) ? 128 * XCHG_LD * 4 : 0;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_MAX = 232448;                  // 227 KB per block
  // group offsets and tile prefix of up to kMaxExperts + 1 groups, cached in shared memory
  static constexpr int TABLE_BYTES = 2 * (kMaxExperts + 2) * 4;
  static constexpr int STAGES_FIT =
      (SMEM_MAX - 1024 - XCHG_BYTES - BAR_BYTES - TABLE_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + XCHG_BYTES + BAR_BYTES + TABLE_BYTES;
  // TMEM: two halves, each holding one tile's accumulators (double buffering). One slab: a half
  // is BN columns. Two slabs: a half is 256 columns; a tile of <= 128 valid token columns keeps
  // both slabs' accumulators in one half (slab j at column 128 j), a wider tile takes both
  // halves (slab j in the j-th half it takes). The allocation is a power of two >= 32 columns.
  static constexpr int HALF_COLS = SLABS == 1 ? BN : 256;
  static constexpr int TMEM_COLS = 2 * HALF_COLS <= 32 ? 32 : 2 * HALF_COLS <= 64 ? 64
                                   : 2 * HALF_COLS <= 128 ? 128 : 2 * HALF_COLS <= 256 ? 256
                                   : 512;
  static constexpr int CW = BN < 32 ? BN : 32;                 // epilogue column chunk
  static_assert(STAGES >= 3 || SLABS == 2, "pipeline too shallow");
  static_assert(STAGES >= 4 || SLABS == 1, "pipeline too shallow");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M=128");
  static_assert(BN % CW == 0, "epilogue chunks");
  static_assert(!PAIR || (BN >= 64 && MODE != kModeGateUpPartial), "pair tiles: prefill shapes");
  static_assert(SLABS == 1 || (PAIR && MODE == kModeSwiGLU), "two slabs: prefill gate/up pairs");
};

// Which TMEM half (and column offset) holds each slab's accumulator of a CTA's tiles, in the
// order the CTA processes them; the MMA issuer and the epilogue keep one each and step it
// identically. cnt[h] counts the tiles that have used half h so far (its barrier phase).
template <int SLABS, int HALF_COLS>
struct AccSeq {
  uint32_t cnt[2] = {0u, 0u};
  int next = 0;
  // For a tile with `ncols` MMA columns: the halves it takes (h[0], and h[1] if two) and the
  // column of slab j's accumulator.
  __device__ __forceinline__ int take(int ncols, int (&h)[2], uint32_t (&ph)[2],
                                      uint32_t (&col)[SLABS]) {
    int nh = 1;
    h[0] = next;
    h[1] = next ^ 1;
    if (SLABS == 2 && ncols > 128) nh = 2;
    ph[0] = cnt[h[0]] & 1u;
    ph[1] = cnt[h[1]] & 1u;
#pragma unroll
    for (int j = 0; j < SLABS; ++j)
      col[j] = nh == 2 ? static_cast<uint32_t>(h[j] * HALF_COLS)
                       : static_cast<uint32_t>(h[0] * HALF_COLS + j * 128);
    return nh;
  }
  __device__ __forceinline__ void advance(int nh) {
    ++cnt[next];
    if (nh == 2) ++cnt[next ^ 1];
    else next ^= 1;
  }
};

// The tile list, read from shared-memory copies of the group offsets and the tile prefix (a tile
// boundary then costs a few shared-memory loads instead of a chain of global ones).
struct TileTable {
  const int* off;   // [G+1] first routed row of each group
  const int* tp;    // [G+1] prefix over groups of the token tiles
  int G, ms, splits;
};

// tile -> (group g, m-tile, K-split s, n-tile). Group g covers tiles [ms * tp[g], ms * tp[g+1])
// with ms = m_tiles * splits; inside it n runs fastest.
__device__ __forceinline__ void decode_tile(const TileTable& tt, int tile, int& g, int& m, int& n,
                                            int& s) {
  const int v = tile / tt.ms;
  int lo = 0, hi = tt.G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tt.tp[mid] <= v) lo = mid;
    else hi = mid - 1;
  }
  g = lo;
  const int local = tile - tt.ms * tt.tp[g];
  const int nt = tt.tp[g + 1] - tt.tp[g];
  n = local % nt;
  const int rest = local / nt;
  s = rest % tt.splits;
  m = rest / tt.splits;
}

// Valid token rows of the tile starting at row0 of group g, rounded up to a multiple of ROUND.
template <int BN, int ROUND>
__device__ __forceinline__ int tile_rows_rounded(const TileTable& tt, int g, int row0) {
  const int rows = min(BN, tt.off[g + 1] - row0);
  return (rows + ROUND - 1) / ROUND * ROUND;
}


template <int BN, int MODE, bool PAIR, int SLABS>
__global__ void __launch_bounds__(256, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                        const __grid_constant__ CUtensorMap map_a_shared,
                        const __grid_constant__ CUtensorMap map_b64,
                        const __grid_constant__ CUtensorMap map_b16,
                        const __grid_constant__ CUtensorMap map_out, const GemmArgs args) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  using C = GemmCfg<BN, MODE, PAIR, SLABS>;
  using Seq = AccSeq<SLABS, C::HALF_COLS>;
  constexpr bool kGateUp = MODE != kModeDown;     // A slab = 64 gate rows + the 64 up rows
  constexpr int kWhere = kGateUp ? kWhereGemm1 : kWhereGemm2;
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
  // A pair (2-CTA cluster) works on one tile of 256 x SLABS weight rows: CTA rank r holds the
  // SLABS weight m-tiles from (2 mu + r) SLABS on, and half of the token rows; the even CTA
  // issues the MMAs. Both CTAs of a pair see the same tile sequence, so they leave (or stay)
  // together.
  const uint32_t crank = PAIR ? cluster_rank() : 0u;
  const bool leader = crank == 0;
  const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int nunits = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  constexpr int kMPerUnit = (PAIR ? 2 : 1) * SLABS;
  const int m_units = (args.m_tiles + kMPerUnit - 1) / kMPerUnit;
  const int total_tiles = m_units * args.splits * args.tile_prefix[args.G];
  if (unit >= total_tiles) return;
  int* s_off = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + C::BAR_BYTES);
  int* s_tp = s_off + (kMaxExperts + 2);
  for (int i = threadIdx.x; i <= args.G; i += blockDim.x) {
    s_off[i] = args.group_offsets[i];
    s_tp[i] = args.tile_prefix[i];
  }
  const TileTable tt{s_off, s_tp, args.G, m_units * args.splits, args.splits};

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], PAIR ? 8 : 4);     // the epilogue warps of both CTAs of a pair
    }
    mbar_init(drain, 1);
    fence_mbarrier_init();
  }
  if (warp == 2) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before_sync();
  if constexpr (PAIR) cluster_sync_all();    // both CTAs' barriers initialised before any remote use
  else __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  MOE_ROLE_T0(t_setup);
  // shared::cluster addresses of the even CTA's barriers (pair loads, commits and arrivals)
  const uint32_t full_l = PAIR ? cluster_addr(full, 0) : 0u;
  const uint32_t tempty_l = PAIR ? cluster_addr(tempty, 0) : 0u;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_map(&map_a);
      tma_prefetch_map(&map_a_shared);
      tma_prefetch_map(&map_b64);
      tma_prefetch_map(&map_b16);
      const uint64_t pol_w = l2_policy_evict_first();   // weights: streamed once
      const uint64_t pol_x = l2_policy_evict_last();    // activations: reused by every m-tile
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = unit; ok && tile < total_tiles; tile += nunits) {
        int g, mu, n, s;
        decode_tile(tt, tile, g, mu, n, s);
        const int mc = (PAIR ? 2 * mu + static_cast<int>(crank) : mu) * SLABS;  // first m-tile
        const int row0 = tt.off[g] + n * BN;
        const int rowsN = tile_rows_rounded<BN, C::ROUND>(tt, g, row0);   // the MMA's N
        const int myrows = PAIR ? rowsN / 2 : rowsN;       // token rows this CTA loads
        const int myrow0 = row0 + static_cast<int>(crank) * myrows;
        // bytes that complete the (even CTA's) full barrier: both CTAs' loads for a pair
        const uint32_t stage_bytes = (PAIR ? 2 : 1) * C::A_BYTES + rowsN * kBK;
        const int kb0 = s * args.kb_per_split;
        const int kb1 = min(args.num_kb, kb0 + args.kb_per_split);
        const bool sh = g >= args.E_routed;
        const CUtensorMap* ma = sh ? &map_a_shared : &map_a;
        const int ga = sh ? 0 : g;
        for (int kb = kb0; kb < kb1; ++kb) {
          MOE_ROLE_T0(tq0);
          const bool got = PAIR ? mbar_wait_cluster(&empty[stage], phase ^ 1u)
                                : mbar_wait(&empty[stage], phase ^ 1u);
          MOE_ROLE_ADD(MODE, 0, clock64() - tq0);
          if (!got) {
            report(args.status, kStatusDeviceTimeout, kWhere, 1);
            ok = false;
            break;
          }
          uint8_t* sa = stages + stage * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          if (leader) mbar_arrive_expect_tx(&full[stage], stage_bytes);
          if constexpr (PAIR) {
            const uint32_t fb = full_l + 8u * stage;
#pragma unroll
            for (int j = 0; j < SLABS; ++j) {
              uint8_t* sj = sa + j * C::SLAB_BYTES;
              if (kGateUp) {
                tma_load_4d_pair(sj, ma, fb, kb * kBK, (mc + j) * 64, 0, ga, pol_w);
                tma_load_4d_pair(sj + C::SLAB_BYTES / 2, ma, fb, kb * kBK, (mc + j) * 64, 1, ga,
                                 pol_w);
              } else {
                tma_load_3d_pair(sj, ma, fb, kb * kBK, (mc + j) * 128, ga, pol_w);
              }
            }
            int r = 0;
            for (; r + 64 <= myrows; r += 64)
              tma_load_2d_pair(sb + r * kBK, &map_b64, fb, kb * kBK, myrow0 + r, pol_x);
            for (; r < myrows; r += 16)
              tma_load_2d_pair(sb + r * kBK, &map_b16, fb, kb * kBK, myrow0 + r, pol_x);
          } else {
            if (kGateUp) {
              tma_load_4d(sa, ma, &full[stage], kb * kBK, mc * 64, 0, ga, pol_w);
              tma_load_4d(sa + C::SLAB_BYTES / 2, ma, &full[stage], kb * kBK, mc * 64, 1, ga, pol_w);
            } else {
              tma_load_3d(sa, ma, &full[stage], kb * kBK, mc * 128, ga, pol_w);
            }
            // only the tile's valid token rows: 64-row boxes, then 16-row boxes
            int r = 0;
            if constexpr (BN >= 64)
              for (; r + 64 <= myrows; r += 64)
                tma_load_2d(sb + r * kBK, &map_b64, &full[stage], kb * kBK, myrow0 + r, pol_x);
            for (; r < myrows; r += 16)
              tma_load_2d(sb + r * kBK, &map_b16, &full[stage], kb * kBK, myrow0 + r, pol_x);
          }
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: the most recent load of every stage must have landed before the CTA exits. (In
      // a pair the even CTA's full barriers count both CTAs' bytes; the odd CTA relies on the
      // final cluster barrier, which the even CTA reaches only after this drain.)
      const int outstanding = leader ? min(issued, C::STAGES) : 0;
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
    // ------------------------------------------------------------ MMA issuer (one thread; in a
    // pair the even CTA's, for both CTAs)
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      Seq seq;
      const uint32_t empty_l = PAIR ? cluster_addr(empty, 0) : 0u;
      const uint32_t empty_p = PAIR ? cluster_addr(empty, 1) : 0u;
      const uint32_t tfull_l = PAIR ? cluster_addr(tfull, 0) : 0u;
      const uint32_t tfull_p = PAIR ? cluster_addr(tfull, 1) : 0u;
      for (int tile = unit; ok && tile < total_tiles; tile += nunits) {
        int g, mu, n, s;
        decode_tile(tt, tile, g, mu, n, s);
        const int kb0 = s * args.kb_per_split;
        const int kb1 = min(args.num_kb, kb0 + args.kb_per_split);
        // MMA N = the tile's valid rows rounded up (M = 128 takes N = 16 .. 256 by 16; the pair's
        // M = 256 the same, here by 32 so that each CTA's half is whole 16-row boxes)
        const int ncols = tile_rows_rounded<BN, C::ROUND>(tt, g, tt.off[g] + n * BN);
        const uint32_t idesc = idesc_e4m3_f32(PAIR ? 256 : 128, ncols);
        int h[2];
        uint32_t ph[2], col[SLABS];
        const int nh = seq.take(ncols, h, ph, col);
        for (int i = 0; ok && i < nh; ++i) {
          MOE_ROLE_T0(tq0);
          const bool freed = PAIR ? mbar_wait_cluster(&tempty[h[i]], ph[i] ^ 1u)
                                  : mbar_wait(&tempty[h[i]], ph[i] ^ 1u);
          MOE_ROLE_ADD(MODE, 1, clock64() - tq0);
          if (!freed) {
            report(args.status, kStatusDeviceTimeout, kWhere, 2);
            ok = false;
          }
        }
        if (!ok) break;
        tc_fence_after_sync();
        for (int kb = kb0; kb < kb1; ++kb) {
          MOE_ROLE_T0(tf0);
          const bool landed = mbar_wait(&full[stage], phase);
          MOE_ROLE_ADD(MODE, 2, clock64() - tf0);
          MOE_ROLE_ADD(MODE, 3, 1ull);
          if (!landed) {
            report(args.status, kStatusDeviceTimeout, kWhere, 3);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sa = smem_addr(stages + stage * C::STAGE_BYTES);
          const uint64_t bdesc = smem_desc_sw128(sa + C::A_BYTES);
#pragma unroll
          for (int j = 0; j < SLABS; ++j) {
            const uint64_t adesc = smem_desc_sw128(sa + j * C::SLAB_BYTES);
            const uint32_t d_tmem = tmem_base + col[j];
#pragma unroll
            for (int kk = 0; kk < kBK / 32; ++kk) {  // K = 32 e4m3 (32 bytes) per instruction
              if constexpr (PAIR)
                mma_e4m3_pair(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc,
                              (kb > kb0 || kk > 0) ? 1u : 0u);
              else
                mma_e4m3(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc,
                         (kb > kb0 || kk > 0) ? 1u : 0u);
            }
          }
          // frees the stage (in both CTAs of a pair) when these MMAs finish
          if constexpr (PAIR) {
            mma_commit_pair(empty_l + 8u * stage);
            mma_commit_pair(empty_p + 8u * stage);
          } else {
            mma_commit(&empty[stage]);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        bool signal = ok;
#ifdef MOE_WAIT_TEST
        if (args.withhold && tile == unit) signal = false;   // the epilogue's wait will expire
#endif
        if (signal) {                              // accumulators ready for the epilogue(s)
          for (int i = 0; i < nh; ++i) {
            if constexpr (PAIR) {
              mma_commit_pair(tfull_l + 8u * h[i]);
              mma_commit_pair(tfull_p + 8u * h[i]);
            } else {
              mma_commit(&tfull[h[i]]);
            }
          }
        }
        seq.advance(nh);
      }
      if constexpr (PAIR) mma_commit_pair(cluster_addr(drain, 0));
      else mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue (4 warps)
    // After a timeout a warp keeps walking the tile list and joins every named barrier (so the
    // other epilogue warps never wait on it) but touches neither TMEM nor global memory.
    const int q = warp & 3;
    bool bad = false;
    Seq seq;
    for (int tile = unit; tile < total_tiles; tile += nunits) {
      int g, mu, n, s;
      decode_tile(tt, tile, g, mu, n, s);
      const int mc = (PAIR ? 2 * mu + static_cast<int>(crank) : mu) * SLABS;
      const int row0 = tt.off[g] + n * BN;
      const int nvalid = min(BN, tt.off[g + 1] - row0);
      int h[2];
      uint32_t ph[2], col[SLABS];
      const int nh = seq.take(tile_rows_rounded<BN, C::ROUND>(tt, g, row0), h, ph, col);
      // this lane's row scales (token column CW u + lane of every column chunk u), loaded before
      // the accumulator wait so that their latency hides behind it
      constexpr int kRsRegs = BN / C::CW;
      float rs[kRsRegs];
#pragma unroll
      for (int u = 0; u < kRsRegs; ++u) {
        const int c = u * C::CW + lane;
        rs[u] = (c < nvalid && (C::CW == 32 || lane < C::CW)) ? args.row_scale[row0 + c] : 0.f;
      }
      const bool sh = g >= args.E_routed;
      const float* wsc = sh ? args.w_scale_shared : args.w_scale + (size_t)g * args.w_scale_ld;
#pragma unroll 1
      for (int j = 0; j < SLABS; ++j) {
        const int m = mc + j;
        const int hi = nh == 2 ? j : 0;            // the half holding slab j
        // output channel of this lane: the weight row of TMEM lane 32 q + lane
        int ch;
        bool valid;
        float wsv;
        if constexpr (MODE == kModeDown) {
          ch = m * 128 + 32 * q + lane;                      // down: output channel i
          valid = ch < args.M_valid;
          wsv = valid ? wsc[ch] : 0.f;
        } else {
          const int frow = m * 64 + 32 * (q & 1) + lane;    // gate (q < 2) / up (q >= 2) row
          valid = frow < args.M_valid;
          ch = (q >> 1) * args.M_valid + frow;               // its column of [gate | up]
          wsv = valid ? wsc[ch] : 0.f;
        }
        if (!bad && (j == 0 || nh == 2)) {
          MOE_ROLE_T0(te0);
          const bool ok = PAIR ? mbar_wait_cluster(&tfull[h[hi]], ph[hi])
                               : mbar_wait(&tfull[h[hi]], ph[hi]);
          if (warp == 4 && lane == 0) MOE_ROLE_ADD(MODE, 4, clock64() - te0);
          bad = __any_sync(0xffffffffu, !ok);       // warp-uniform: TMEM loads are .sync.aligned
          if (bad && lane == 0) report(args.status, kStatusDeviceTimeout, kWhere, 5);
        }
        tc_fence_after_sync();
        const uint32_t tbase = tmem_base + col[j] + (static_cast<uint32_t>(32 * q) << 16);
        if constexpr (MODE == kModeSwiGLU) {
          // TMEM lane 32q+i holds gate row (q<2) or up row (q>=2) 32*(q&1)+i of this 64-row half
          // pair. Step 1: every warp parks its rows (scaled by the weight scale) in smem.
          // Step 2: thread (q, lane) takes token column `lane` and the 16 features 16q .. 16q+15:
          // SwiGLU, one 64-byte store, and the in-thread max |act| for the row amax.
          constexpr int CW = C::CW;
          const int f0 = m * 64 + 16 * q;                // this thread's first feature
          for (int c0 = 0, jj = 0; c0 < nvalid; c0 += CW, ++jj) {
            float rsv = 0.f;
#pragma unroll
            for (int u = 0; u < kRsRegs; ++u)
              if (u == jj) rsv = rs[u];
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
            const int nn = c0 + lane;
            if (!bad && lane < CW && nn < nvalid && f0 < args.M_valid) {
              const float rsc = rsv;
              float act[16];
              float amax = 0.f;
#pragma unroll
              for (int k2 = 0; k2 < 16; ++k2) {
                const int jf = 16 * q + k2;
                const float gv = xchg[jf * C::XCHG_LD + lane] * rsc;
                const float uv = xchg[(64 + jf) * C::XCHG_LD + lane] * rsc;
                act[k2] = silu(gv) * uv;
                amax = fmaxf(amax, fabsf(act[k2]));
              }
              float4* dst = reinterpret_cast<float4*>(args.out + (size_t)(row0 + nn) * args.out_ld + f0);
#pragma unroll
              for (int v = 0; v < 4; ++v)
                dst[v] = make_float4(act[4 * v], act[4 * v + 1], act[4 * v + 2], act[4 * v + 3]);
              atomicMax(&args.row_amax[row0 + nn], __float_as_uint(amax));
            }
            named_bar_sync(1, 128);
          }
        } else {
          // Down GEMM (output channel i = TMEM lane) or K-split gate/up (gate column frow of
          // [0, F), up column F + frow). Lane l holds the row scales of token columns
          // c0 + l of every 32-column chunk (one coalesced load per chunk, issued above before
          // the accumulator wait); a shuffle hands column c's scale to the whole warp.
          constexpr int CW = C::CW;
          float* outp = args.out + (size_t)s * args.out_split_stride + (size_t)row0 * args.out_ld + ch;
          const int split_rows = (int)(args.out_split_stride / (size_t)args.out_ld);   // map rows
#pragma unroll 1
          for (int jj = 0; !bad && jj * CW < nvalid; ++jj) {
            const int c0 = jj * CW;
            uint32_t r[CW];
            tmem_ld16(tbase + c0, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
            if constexpr (CW == 32)
              tmem_ld16(tbase + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
            float rsv = 0.f;
#pragma unroll
            for (int u = 0; u < kRsRegs; ++u)
              if (u == jj) rsv = rs[u];
            tmem_wait_ld();
            const int ncol = min(CW, nvalid - c0);
            float* dst = outp + (size_t)c0 * args.out_ld;
            float v[CW];
#pragma unroll
            for (int c = 0; c < CW; ++c)
              v[c] = __uint_as_float(r[c]) * __shfl_sync(0xffffffffu, rsv, c) * wsv;
            if constexpr (C::DOWN_T) {
              // Through this warp's dense 32 x 32 fp32 block of shared memory (row = token): a
              // full chunk leaves by one TMA tensor store, a ragged one by 16-byte stores of its
              // valid rows. (In this kernel the count of global store instructions, not the
              // bytes, set the epilogue's pace; the TMA store takes them off the SM's load/store
              // path.)
              float* tr = xchg + 32 * q * 32;
              if (lane == 0) bulk_wait_read_all();       // the previous store has read the block
              __syncwarp();
#pragma unroll
              for (int c = 0; c < CW; ++c) tr[c * 32 + lane] = v[c];
              const int chq = m * 128 + 32 * q;
              if (ncol == CW) {
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && chq < args.M_valid) {
                  tma_store_2d(&map_out, tr, chq, s * split_rows + row0 + c0);
                  bulk_commit();
                }
              } else {
                __syncwarp();
                const int cc = 4 * (lane & 7);
                float* base = args.out + (size_t)s * args.out_split_stride +
                              (size_t)(row0 + c0) * args.out_ld + chq + cc;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  const int c = 4 * i + (lane >> 3);
                  if (c < ncol && chq + cc < args.M_valid)
                    *reinterpret_cast<float4*>(base + (size_t)c * args.out_ld) =
                        *reinterpret_cast<const float4*>(tr + c * 32 + cc);
                }
                __syncwarp();
              }
            } else if (valid) {
#pragma unroll
              for (int c = 0; c < CW; ++c)
                if (c < ncol) dst[(size_t)c * args.out_ld] = v[c];
            }
          }
        }
        if (j == SLABS - 1 || nh == 2) {            // this half's accumulators are read
          tc_fence_before_sync();
          __syncwarp();
          if (!bad && lane == 0) {
            if constexpr (PAIR) mbar_arrive_cluster(tempty_l + 8u * h[hi]);   // the even CTA's barrier
            else mbar_arrive(&tempty[h[hi]]);
          }
        }
      }
      seq.advance(nh);
    }
    if constexpr (C::DOWN_T) {
      if (lane == 0) bulk_wait_all();              // this warp's TMA stores have completed
    }
  }

  if (warp == 4 && lane == 0) {
    MOE_ROLE_ADD(MODE, 5, clock64() - t_setup);
    MOE_ROLE_ADD(MODE, 6, (unsigned long long)((total_tiles - unit + nunits - 1) / nunits));
  }
  tc_fence_before_sync();
  if constexpr (PAIR) cluster_sync_all();   // no CTA leaves while its pair still uses its memory
  else __syncthreads();
  if (warp == 2) {
    tc_fence_after_sync();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

namespace {
template <int BN, int MODE, bool PAIR, int SLABS = 1>
cudaError_t launch_gemm_t(const CUtensorMap& a, const CUtensorMap& ash, const CUtensorMap& b64,
                          const CUtensorMap& b16, const CUtensorMap& out, const GemmArgs& args,
                          cudaStream_t s) {
  using C = GemmCfg<BN, MODE, PAIR, SLABS>;
  static int grid_cache[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev >= 64) return cudaErrorInvalidDevice;
  if (!grid_cache[dev]) {
    err = cudaFuncSetAttribute(grouped_gemm_kernel<BN, MODE, PAIR, SLABS>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (err != cudaSuccess) return err;
    int grid = num_sms();
    if (PAIR) {
      // persistent pairs: as many 2-CTA clusters as can be resident at once
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(num_sms());
      cfg.blockDim = dim3(256);
      cfg.dynamicSmemBytes = C::SMEM;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      err = cudaOccupancyMaxActiveClusters(&clusters, grouped_gemm_kernel<BN, MODE, PAIR, SLABS>, &cfg);
      if (err != cudaSuccess) return err;
      if (clusters < 1) return cudaErrorInvalidConfiguration;
      grid = 2 * std::min(clusters, num_sms() / 2);
    }
    grid_cache[dev] = grid;
  }
  launch_pdl_cluster(grouped_gemm_kernel<BN, MODE, PAIR, SLABS>, dim3(grid_cache[dev]), dim3(256), C::SMEM,
                     PAIR ? 2 : 1, s, a, ash, b64, b16, out, args);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_by_bn(int BN, bool pair, int slabs, const CUtensorMap& a, const CUtensorMap& ash,
                         const CUtensorMap& b64, const CUtensorMap& b16, const CUtensorMap& out,
                         const GemmArgs& args, cudaStream_t s) {
  if constexpr (MODE == kModeSwiGLU) {
    if (pair && slabs == 2) {
      switch (BN) {
        case 128: return launch_gemm_t<128, MODE, true, 2>(a, ash, b64, b16, out, args, s);
        case 192: return launch_gemm_t<192, MODE, true, 2>(a, ash, b64, b16, out, args, s);
        case 256: return launch_gemm_t<256, MODE, true, 2>(a, ash, b64, b16, out, args, s);
        default: return cudaErrorInvalidValue;
      }
    }
  }
  switch (BN) {
    case 16: return launch_gemm_t<16, MODE, false>(a, ash, b64, b16, out, args, s);
    case 32: return launch_gemm_t<32, MODE, false>(a, ash, b64, b16, out, args, s);
    case 64: return launch_gemm_t<64, MODE, false>(a, ash, b64, b16, out, args, s);
    default:
      if constexpr (MODE == kModeGateUpPartial) return cudaErrorInvalidValue;  // decode tiles only
      else {
        if (pair) {
          switch (BN) {
            case 128: return launch_gemm_t<128, MODE, true>(a, ash, b64, b16, out, args, s);
            case 192: return launch_gemm_t<192, MODE, true>(a, ash, b64, b16, out, args, s);
            case 256: return launch_gemm_t<256, MODE, true>(a, ash, b64, b16, out, args, s);
            default: return cudaErrorInvalidValue;
          }
        }
        switch (BN) {
          case 128: return launch_gemm_t<128, MODE, false>(a, ash, b64, b16, out, args, s);
          case 192: return launch_gemm_t<192, MODE, false>(a, ash, b64, b16, out, args, s);
          case 256: return launch_gemm_t<256, MODE, false>(a, ash, b64, b16, out, args, s);
          default: return cudaErrorInvalidValue;
        }
      }
  }
}
}  // namespace

cudaError_t launch_gemm_gateup(const Plan& p, const CUtensorMap& w13, const CUtensorMap& w13s,
                               const CUtensorMap& acts64, const CUtensorMap& acts16,
                               const GemmArgs& a, bool partial, cudaStream_t s) {
  // (the output map is used by the down GEMM only; the weight map stands in)
  if (partial)
    return launch_by_bn<kModeGateUpPartial>(p.BN, false, 1, w13, w13s, acts64, acts16, w13, a, s);
  return launch_by_bn<kModeSwiGLU>(p.BN, p.pair1, p.slabs1, w13, w13s, acts64, acts16, w13, a, s);
}

cudaError_t launch_gemm_down(const Plan& p, const CUtensorMap& w2, const CUtensorMap& w2s,
                             const CUtensorMap& acts64, const CUtensorMap& acts16,
                             const CUtensorMap& out, const GemmArgs& a, cudaStream_t s) {
  return launch_by_bn<kModeDown>(p.BN, p.pair2, 1, w2, w2s, acts64, acts16, out, a, s);
}

}  // namespace moe

#ifdef MOE_ROLE_COUNTERS
extern "C" int moe_role_counters_read(uint64_t* out) {
  return cudaMemcpyFromSymbol(out, moe::g_role_cycles, sizeof(moe::g_role_cycles)) == cudaSuccess
             ? 0 : -4;
}
extern "C" int moe_role_counters_reset(void) {
  static unsigned long long zero[3 * moe::kRoleMaxCtas * 8] = {};
  return cudaMemcpyToSymbol(moe::g_role_cycles, zero, sizeof(zero)) == cudaSuccess ? 0 : -4;
}
#endif
