// C ABI of the FP8 MoE layer (declared in include/moe.h): argument validation, the launch plan
// (tile sizes, split counts, workspace carve-up), TMA tensor-map encoding and the kernel
// sequence of each entry point. Host code only; the kernels live in route.cu, permute.cu,
// gemm.cu and combine.cu.
#include <algorithm>
#include <cstring>

#include "../../include/moe.h"
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

#ifdef MOE_WAIT_TEST
int g_withhold_gemm_commit = 0;
#endif

int num_sms() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return kPlanSMs;
  if (dev < 64 && cache[dev]) return cache[dev];
  int n = kPlanSMs;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev < 64) cache[dev] = n;
  return n;
}

// K-split count of a grouped GEMM: the s (each split >= 4 K blocks) that minimises the estimated
// HBM time -- ceil(tiles * s / units) waves of tiles that each read w_tile / s weight bytes and
// write out_tile output bytes (plus a fixed per-tile cost), and the read-back of the s partial
// sums by the kernel that reduces them.
static int choose_splits(int64_t base_tiles, int num_kb, int units, double w_tile,
                         double out_tile) {
  constexpr double kTileOverheadBytes = 32e3;
  const int max_s = std::max(1, std::min(32, num_kb / 4));
  int best = 1;
  double best_cost = 0.0;
  for (int s = 1; s <= max_s; ++s) {
    const double waves = (double)ceil_div(base_tiles * s, units);
    const double cost = waves * (w_tile / s + out_tile + kTileOverheadBytes) +
                        (double)base_tiles * s * out_tile / units;
    if (s == 1 || cost < best_cost * (1.0 - 1e-9)) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

int router_splits(int T, int d, int E, int* chunks_per_split) {
  const int64_t rtiles = ceil_div(std::max(T, 1), kRtTok) * ceil_div(E, kRtExp);
  const int nchunks = (int)ceil_div(d, kRtK);
  // about two waves of tiles, but at most 8192 partial logits per token for the top-k kernel
  // to add up
  const int64_t waves2 = std::max<int64_t>(1, ceil_div(2 * kPlanSMs, rtiles));
  const int64_t cap = std::max<int64_t>(1, 8192 / E);
  const int rs = (int)std::min<int64_t>(nchunks, std::min(waves2, cap));
  *chunks_per_split = (int)ceil_div(nchunks, rs);
  return (int)ceil_div(nchunks, *chunks_per_split);
}

int plan_make(int T, int d, int E, int F, int k_max, int Fs, Plan* p, int k_est) {
  if (T < 0 || d < 16 || d % 16 || F < 16 || F % 16 || E < 1 || k_max < 1) return MOE_ERR_INVALID_ARG;
  if (E > kMaxExperts || k_max > kMaxK) return MOE_ERR_UNSUPPORTED;
  if (Fs < 0) return MOE_ERR_INVALID_ARG;
  if (Fs != 0 && Fs != F) return MOE_ERR_UNSUPPORTED;
  if ((int64_t)T * (k_max + 1) >= (1LL << 30) || (int64_t)d * F >= (1LL << 31)) return MOE_ERR_UNSUPPORTED;
  std::memset(p, 0, sizeof(*p));
  p->T = T; p->d = d; p->E = E; p->F = F; p->k_max = k_max; p->Fs = Fs;
  p->shared = Fs > 0;
  p->G = E + (p->shared ? 1 : 0);
  const int64_t routed = (int64_t)T * k_max;
  p->Rcap = routed + (p->shared ? T : 0);
  p->Rpad = std::max<int64_t>(256, ceil_div(p->Rcap, 256) * 256);

  // token tile: the smallest of {16, 32, 64, 128, 192, 256} >= 1.25 x the mean rows of an active
  // expert. A tile only loads and multiplies its valid rows, so a tile larger than the group
  // costs shared memory (fewer pipeline stages), not traffic. The tiles are planned for k_est
  // experts per token (the fixed k, or an estimate of the mean k_t of an elastic batch); the
  // buffers for k_max.
  const int64_t routed_est = (int64_t)T * std::max(1, std::min(k_est > 0 ? k_est : k_max, k_max));
  const int64_t active = std::max<int64_t>(1, std::min<int64_t>(E, routed_est));
  const double mean_rows = double(routed_est) / double(active);
  static const int kTiles[] = {16, 32, 64, 128, 192, 256};
  int BN = 256;
  for (int t : kTiles)
    if (t >= 1.25 * mean_rows) { BN = t; break; }
#ifdef MOE_FORCE_BN
  BN = MOE_FORCE_BN;
#endif
  p->BN = BN;
  // Prefill-sized token tiles run on SM pairs: the pair's M = 256 MMA shares one token tile
  // between two SMs (each loads half of it), so a token row crosses L2 -> shared memory once per
  // 256 weight rows instead of once per 128. That pays when the tiles are full (BN >= 192, i.e.
  // >= ~100 rows per active expert) and, for the down GEMM, when K = F is long enough (>= 16 K
  // blocks) for the main loop rather than the epilogue to set the pace.
  p->pair1 = BN >= 192;
  p->pair2 = BN >= 192 && ceil_div(F, kBK) >= 16;
#ifdef MOE_FORCE_PAIR
  p->pair1 = p->pair2 = MOE_FORCE_PAIR;
#endif
  // Weight slabs per gate/up CTA. Two slabs (two TMEM accumulators against one token tile: a
  // quarter fewer L2 -> shared-memory bytes per MMA) measured slower on B200 than one -- DeepSeek
  // T=8192 gate/up 2802 vs 2659 us, Mixtral T=512 layer 352 vs 317 us: only four pipeline stages
  // fit, and tiles wider than 128 tokens lose the accumulator double buffering -- so one.
  p->slabs1 = 1;
#ifdef MOE_FORCE_SLABS
  p->slabs1 = p->pair1 ? MOE_FORCE_SLABS : 1;
#endif

  // router: 64 x 64 tiles; split d so that the grid covers about two waves (the tensor-core
  // router writes whole logits)
  if (router_uses_mma(E, T, d)) {
    p->r_splits = 1;
    p->r_chunks_per_split = (int)ceil_div(d, kRtK);
  } else {
    p->r_splits = router_splits(T, d, E, &p->r_chunks_per_split);
  }

  p->g1_kb = (int)ceil_div(d, kBK);
  p->g1_m_tiles = (int)ceil_div(F, 64);
  // gate/up: split K (partial sums + a row kernel for SwiGLU) when the tiles would leave the last
  // wave of SMs mostly idle; only for decode-sized token tiles
  p->g1_splits = 1;
  p->g1_kb_per_split = p->g1_kb;
  p->g2_kb = (int)ceil_div(F, kBK);
  p->g2_m_tiles = (int)ceil_div(d, 128);
  const int64_t est_ntiles = std::max<int64_t>(active, ceil_div(routed_est, BN)) +
                             (p->shared ? ceil_div(T, BN) : 0);
  const double tile_rows = std::min<double>(BN, mean_rows);
  if (BN <= 64) {   // gate/up partials: 64 gate + 64 up fp32 columns per routed row
    const int s1 = choose_splits(est_ntiles * p->g1_m_tiles, p->g1_kb, kPlanSMs, 128.0 * d,
                                 tile_rows * 128 * 4);
    p->g1_kb_per_split = (int)ceil_div(p->g1_kb, s1);
    p->g1_splits = (int)ceil_div(p->g1_kb, p->g1_kb_per_split);
  }
  const int m_rows2 = p->pair2 ? 256 : 128;      // weight rows of one down-GEMM work unit
  int s2 = choose_splits(est_ntiles * ceil_div(p->g2_m_tiles, m_rows2 / 128), p->g2_kb,
                         p->pair2 ? kPlanSMs / 2 : kPlanSMs, (double)m_rows2 * F,
                         tile_rows * m_rows2 * 4);
  p->g2_kb_per_split = (int)ceil_div(p->g2_kb, s2);
  p->g2_splits = (int)ceil_div(p->g2_kb, p->g2_kb_per_split);   // every split non-empty

  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off = align256(off + std::max<size_t>(bytes, 1)); return o; };
  p->off_status = take(256);
  p->off_part = take(sizeof(double) * (size_t)p->r_splits * T * E);
  p->off_ids = take(sizeof(int32_t) * (size_t)routed);
  p->off_w = take(sizeof(float) * (size_t)routed);
  p->off_offsets = take(sizeof(int32_t) * (size_t)(E + 2));
  p->off_tiles = take(sizeof(int32_t) * (size_t)(p->G + 2));
  p->off_perm = take(sizeof(int32_t) * (size_t)p->Rpad);
  p->off_inv = take(sizeof(int32_t) * (size_t)routed);
  p->off_pscr = take(sizeof(int32_t) * 2 * (size_t)permute_blocks(*p) * E);
  p->off_xq = take((size_t)T * d);
  p->off_xs = take(sizeof(float) * (size_t)T);
  p->off_xqp = take((size_t)p->Rpad * d);
  p->off_xsp = take(sizeof(float) * (size_t)p->Rpad);
  p->off_amax = take(sizeof(uint32_t) * (size_t)p->Rpad);
  p->off_act = take(sizeof(float) * (size_t)p->Rpad * F);
  p->off_aq = take((size_t)p->Rpad * F);
  p->off_s2 = take(sizeof(float) * (size_t)p->Rpad);
  p->off_o = take(sizeof(float) * (size_t)p->g2_splits * p->Rpad * d);
  p->off_planes = take(router_uses_mma(E, T, d) ? 2 * sizeof(uint16_t) * (size_t)E * d : 0);
  p->off_hpart = take(p->g1_splits > 1 ? sizeof(float) * p->g1_splits * (size_t)p->Rcap * 2 * F : 0);
  p->bytes = off;
  return MOE_OK;
}

// ---------------------------------------------------------------- TMA tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 128-byte swizzle, zero fill outside the tensor. dims/strides in elements/bytes, innermost
// first; strides[i] is the byte stride of dimension i+1.
static bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides, const uint32_t* box,
                     CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_UINT8,
                     CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) gs[i] = strides[i];
  }
  return fn(m, dtype, rank, const_cast<void*>(base), gd, gs, bx, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 down-GEMM output [rows][d] (all K-split partials stacked): box 32 channels x 32 rows,
// no swizzle, for the epilogue's TMA stores.
static bool map_out(CUtensorMap* m, const float* o, int64_t rows, int d) {
  const uint64_t dims[2] = {(uint64_t)d, (uint64_t)std::max<int64_t>(rows, 1)};
  const uint64_t str[1] = {(uint64_t)d * 4};
  const uint32_t box[2] = {32, 32};
  return make_map(m, o, 2, dims, str, box, CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
}

// bf16 router weight planes [2][E][d]: box 64 (K) x 128 experts of one plane.
static bool map_router_planes(CUtensorMap* m, const uint16_t* planes, int E, int d) {
  const uint64_t dims[3] = {(uint64_t)d, (uint64_t)E, 2};
  const uint64_t str[2] = {(uint64_t)d * 2, (uint64_t)E * d * 2};
  const uint32_t box[3] = {64, 128, 1};
  return make_map(m, planes, 3, dims, str, box, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}
// bf16 hidden states [T][d]: box 64 (K) x `tokens` tokens.
static bool map_hidden(CUtensorMap* m, const uint16_t* hidden, int T, int d, int tokens) {
  const uint64_t dims[2] = {(uint64_t)d, (uint64_t)T};
  const uint64_t str[1] = {(uint64_t)d * 2};
  const uint32_t box[2] = {64, (uint32_t)tokens};
  return make_map(m, hidden, 2, dims, str, box, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

// W13 [experts, 2F, d] viewed as [experts][2][F][d]: box 128 (K) x 64 rows of one half. (One box
// over both halves, and 128-row token boxes, measured slower: Mixtral T=512 416 vs 338 us.)
static bool map_w13(CUtensorMap* m, const uint8_t* w, int experts, int F, int d) {
  const uint64_t dims[4] = {(uint64_t)d, (uint64_t)F, 2, (uint64_t)experts};
  const uint64_t str[3] = {(uint64_t)d, (uint64_t)F * d, 2ull * F * d};
  const uint32_t box[4] = {(uint32_t)kBK, 64, 1, 1};
  return make_map(m, w, 4, dims, str, box);
}
// W2 [experts, d, F]: box 128 (K) x 128 rows.
static bool map_w2(CUtensorMap* m, const uint8_t* w, int experts, int d, int F) {
  const uint64_t dims[3] = {(uint64_t)F, (uint64_t)d, (uint64_t)experts};
  const uint64_t str[2] = {(uint64_t)F, (uint64_t)d * F};
  const uint32_t box[3] = {(uint32_t)kBK, 128, 1};
  return make_map(m, w, 3, dims, str, box);
}
// Row-major activations [rows, K]: box 128 (K) x BN rows.
static bool map_rows(CUtensorMap* m, const uint8_t* a, int64_t rows, int K, int BN) {
  const uint64_t dims[2] = {(uint64_t)K, (uint64_t)rows};
  const uint64_t str[1] = {(uint64_t)K};
  const uint32_t box[2] = {(uint32_t)kBK, (uint32_t)BN};
  return make_map(m, a, 2, dims, str, box);
}

// ---------------------------------------------------------------- helpers
static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static int check_device() {
  static int ok_cache[64] = {};   // 0 unknown, 1 ok, 2 bad
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 64 && ok_cache[dev]) return ok_cache[dev] == 1 ? MOE_OK : MOE_ERR_UNSUPPORTED;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int rc = major == 10 ? MOE_OK : MOE_ERR_UNSUPPORTED;
  if (dev < 64) ok_cache[dev] = rc == MOE_OK ? 1 : 2;
  return rc;
}

struct Ws {
  int* status;
  double* part;
  float *w, *xs, *xsp, *act, *s2, *o, *hpart;
  uint16_t* planes;
  int32_t *ids, *offsets, *tiles, *perm, *inv, *pscr;
  uint8_t *xq, *xqp, *aq;
  uint32_t* amax;
};

static Ws carve(const Plan& p, void* ws) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  Ws w;
  w.status = reinterpret_cast<int*>(b + p.off_status);
  w.part = reinterpret_cast<double*>(b + p.off_part);
  w.ids = reinterpret_cast<int32_t*>(b + p.off_ids);
  w.w = reinterpret_cast<float*>(b + p.off_w);
  w.offsets = reinterpret_cast<int32_t*>(b + p.off_offsets);
  w.tiles = reinterpret_cast<int32_t*>(b + p.off_tiles);
  w.perm = reinterpret_cast<int32_t*>(b + p.off_perm);
  w.inv = reinterpret_cast<int32_t*>(b + p.off_inv);
  w.pscr = reinterpret_cast<int32_t*>(b + p.off_pscr);
  w.xq = b + p.off_xq;
  w.xs = reinterpret_cast<float*>(b + p.off_xs);
  w.xqp = b + p.off_xqp;
  w.xsp = reinterpret_cast<float*>(b + p.off_xsp);
  w.amax = reinterpret_cast<uint32_t*>(b + p.off_amax);
  w.act = reinterpret_cast<float*>(b + p.off_act);
  w.aq = b + p.off_aq;
  w.s2 = reinterpret_cast<float*>(b + p.off_s2);
  w.o = reinterpret_cast<float*>(b + p.off_o);
  w.planes = reinterpret_cast<uint16_t*>(b + p.off_planes);
  w.hpart = reinterpret_cast<float*>(b + p.off_hpart);
  return w;
}

static int check_ws(const Plan& p, const void* ws, size_t ws_bytes) {
  if (!ws || ws_bytes < p.bytes || !aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

static int check_k(const Plan& p, int k, const int32_t* k_per_token) {
  if (k_per_token) return aligned(k_per_token, 4) ? MOE_OK : MOE_ERR_INVALID_ARG;
  return (k >= 1 && k <= std::min(p.E, p.k_max)) ? MOE_OK : MOE_ERR_INVALID_ARG;
}

#define MOE_TRY(expr)                         \
  do {                                        \
    const int rc_ = (expr);                   \
    if (rc_ != MOE_OK) return rc_;            \
  } while (0)
#define MOE_CUDA(expr)                        \
  do {                                        \
    if ((expr) != cudaSuccess) return MOE_ERR_CUDA; \
  } while (0)

// Router logits into w.part for the non-fused paths (tensor cores or CUDA cores).
static int run_router_logits(const Plan& p, const Ws& w, const uint16_t* hidden,
                             const float* router_w, cudaStream_t s) {
  if (router_uses_mma(p)) {
    CUtensorMap mw, mx;
    if (!map_router_planes(&mw, w.planes, p.E, p.d) ||
        !map_hidden(&mx, hidden, p.T, p.d, router_mma_tokens(p.T, p.E)))
      return MOE_ERR_UNSUPPORTED;
    MOE_CUDA(launch_router_mma(p, router_w, w.planes, mw, mx, w.part, w.status, s));
    return MOE_OK;
  }
  MOE_CUDA(launch_router_logits(p, hidden, router_w, w.part, s));
  return MOE_OK;
}

// Grouped FFN: gate/up GEMM + SwiGLU, requantisation, down GEMM into `o` (split partials
// `split_stride` apart).
// Grouped FFN core shared by moe_forward and moe_grouped_ffn_fp8 (`gathered`: the grouping
// kernel already laid the token rows out).
static int run_ffn(const Plan& p, const Ws& w, const uint8_t* w13, const float* w13_scale,
                   const uint8_t* w2, const float* w2_scale, const uint8_t* w13s,
                   const float* w13s_scale, const uint8_t* w2s, const float* w2s_scale,
                   float* o, size_t split_stride, int64_t o_rows, void* const* ev,
                   cudaStream_t s, bool gathered = false) {
  CUtensorMap m13, m13s, mx64, mx16, m2, m2s, maq64, maq16;
  if (!map_w13(&m13, w13, p.E, p.F, p.d) || !map_w2(&m2, w2, p.E, p.d, p.F) ||
      !map_rows(&mx64, w.xqp, p.Rpad, p.d, 64) || !map_rows(&mx16, w.xqp, p.Rpad, p.d, 16) ||
      !map_rows(&maq64, w.aq, p.Rpad, p.F, 64) || !map_rows(&maq16, w.aq, p.Rpad, p.F, 16))
    return MOE_ERR_UNSUPPORTED;
  m13s = m13;
  m2s = m2;
  if (p.shared) {
    if (!map_w13(&m13s, w13s, 1, p.F, p.d) || !map_w2(&m2s, w2s, 1, p.d, p.F))
      return MOE_ERR_UNSUPPORTED;
  }
  auto record = [&](int i) {
    if (ev && ev[i]) cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s);
  };
  const int32_t* total_rows = w.offsets + p.G;     // offsets[G] = routed (+ shared) rows

  record(3);
  if (!gathered)   // (else the grouping kernel already laid the rows out)
    MOE_CUDA(launch_gather(p, w.xq, w.xs, w.perm, total_rows, w.xqp, w.xsp, w.amax, w.status, s));

  GemmArgs g1{};
  g1.group_offsets = w.offsets;
  g1.tile_prefix = w.tiles;
  g1.G = p.G;
  g1.E_routed = p.E;
  g1.m_tiles = p.g1_m_tiles;
  g1.splits = 1;
  g1.kb_per_split = p.g1_kb;
  g1.num_kb = p.g1_kb;
  g1.M_valid = p.F;
  g1.row_scale = w.xsp;
  g1.w_scale = w13_scale;
  g1.w_scale_shared = w13s_scale;
  g1.w_scale_ld = 2 * p.F;
  g1.out = w.act;
  g1.out_ld = p.F;
  g1.out_split_stride = 0;
  g1.row_amax = w.amax;
  g1.status = w.status;
#ifdef MOE_WAIT_TEST
  g1.withhold = g_withhold_gemm_commit;
#endif
  const bool split1 = p.g1_splits > 1;
  if (split1) {
    g1.splits = p.g1_splits;
    g1.kb_per_split = p.g1_kb_per_split;
    g1.out = w.hpart;
    g1.out_ld = 2 * p.F;
    g1.out_split_stride = (size_t)p.Rcap * 2 * p.F;
    g1.row_amax = nullptr;
  }
  record(4);
  MOE_CUDA(launch_gemm_gateup(p, m13, m13s, mx64, mx16, g1, split1, s));

  record(5);
  if (split1) {
    MOE_CUDA(launch_swiglu_requant(p, w.hpart, p.g1_splits, g1.out_split_stride, total_rows, w.aq,
                                   w.s2, s));
  } else {
    MOE_CUDA(launch_requant(p, w.act, w.amax, total_rows, w.aq, w.s2, s));
  }

  GemmArgs g2 = g1;
  g2.m_tiles = p.g2_m_tiles;
  g2.splits = p.g2_splits;
  g2.kb_per_split = p.g2_kb_per_split;
  g2.num_kb = p.g2_kb;
  g2.M_valid = p.d;
  g2.row_scale = w.s2;
  g2.w_scale = w2_scale;
  g2.w_scale_shared = w2s_scale;
  g2.w_scale_ld = p.d;
  g2.out = o;
  g2.out_ld = p.d;
  g2.out_split_stride = split_stride;
  g2.row_amax = nullptr;
#ifdef MOE_WAIT_TEST
  g2.withhold = 0;
#endif
  // the down GEMM's TMA stores: o as [splits x split rows][d] fp32 (a caller's unsplit buffer
  // has exactly o_rows rows)
  CUtensorMap mo;
  const int64_t out_rows = p.g2_splits == 1 ? o_rows
                                            : (int64_t)p.g2_splits * (int64_t)(split_stride / p.d);
  if (!map_out(&mo, o, out_rows, p.d)) return MOE_ERR_UNSUPPORTED;
  record(6);
  MOE_CUDA(launch_gemm_down(p, m2, m2s, maq64, maq16, mo, g2, s));
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_bytes(const moe_dims* dims) {
  if (!dims) return 0;
  // the largest need over the tile plans moe_forward may use (fixed k = 1 .. k_max, or the
  // elastic estimate k_max / 2)
  size_t need = 0;
  for (int k = 1; k <= std::max(1, dims->k_max); ++k) {
    Plan p;
    if (plan_make(dims->T, dims->d, dims->E, dims->F, dims->k_max, dims->F_shared, &p, k) != MOE_OK)
      return 0;
    need = std::max(need, p.bytes);
  }
  return need;
}

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument (shape, null or misaligned pointer, k)";
    case MOE_ERR_UNSUPPORTED: return "unsupported device or size";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "CUDA runtime or launch error";
    case MOE_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel expired";
    case MOE_ERR_DEVICE_CHECK: return "routing data out of range (expert id, k_t or offsets)";
    default: return "unknown status";
  }
}

uint64_t moe_kernel_launch_count(void) {
  return static_cast<uint64_t>(launch_counter().load(std::memory_order_relaxed));
}

#ifdef MOE_WAIT_TEST
void moe_test_withhold_gemm_commit(int on) { g_withhold_gemm_commit = on ? 1 : 0; }
#endif

int moe_clear_status(void* ws, void* stream) {
  if (!ws) return MOE_ERR_WORKSPACE;
  return cudaMemsetAsync(ws, 0, 16, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK
                                                                                       : MOE_ERR_CUDA;
}

int moe_device_status(const void* ws, void* stream, int32_t* out_status) {
  if (!ws || !out_status) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  *out_status = v;
  return MOE_OK;
}

int moe_route_topk(const moe_dims* dims, const uint16_t* hidden, const float* router_w,
                   const float* router_bias, int32_t k, const int32_t* k_per_token,
                   int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes, void* stream) {
  if (!dims) return MOE_ERR_INVALID_ARG;
  Plan p;
  MOE_TRY(plan_make(dims->T, dims->d, dims->E, dims->F, dims->k_max, dims->F_shared, &p));
  if (p.T == 0) return MOE_OK;
  if (!hidden || !router_w || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(router_w, 16)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_k(p, k, k_per_token));
  MOE_TRY(check_ws(p, ws, ws_bytes));
  MOE_TRY(check_device());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Ws w = carve(p, ws);
  if (router_is_fused(p)) {
    MOE_CUDA(launch_route_fused(p, hidden, router_w, router_bias, k, k_per_token, topk_ids, topk_w,
                                nullptr, nullptr, false, w.status, s));
    return MOE_OK;
  }
  if (router_uses_gemv(p)) {
    MOE_CUDA(cudaMemsetAsync(w.status + 3, 0, sizeof(int), s));   // the last-block counter
    MOE_CUDA(launch_route_gemv(p, hidden, router_w, router_bias, k, k_per_token, w.part, topk_ids,
                               topk_w, nullptr, nullptr, false, w.status, DecodeGrouping{}, s));
    return MOE_OK;
  }
  MOE_TRY(run_router_logits(p, w, hidden, router_w, s));
  MOE_CUDA(launch_topk_quant(p, w.part, router_bias, k, k_per_token, topk_ids, topk_w, hidden,
                             nullptr, nullptr, true, false,
                             router_uses_mma(p) ? router_w : nullptr, w.status, s));
  return MOE_OK;
}

int moe_permute(const moe_dims* dims, const int32_t* topk_ids, int32_t k,
                const int32_t* k_per_token, int32_t* expert_offsets, int32_t* perm_token,
                int32_t* inv_row, void* ws, size_t ws_bytes, void* stream) {
  if (!dims) return MOE_ERR_INVALID_ARG;
  Plan p;
  MOE_TRY(plan_make(dims->T, dims->d, dims->E, dims->F, dims->k_max, dims->F_shared, &p));
  if (p.T == 0) return MOE_OK;
  if (!topk_ids || !expert_offsets || !perm_token || !inv_row) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_k(p, k, k_per_token));
  MOE_TRY(check_ws(p, ws, ws_bytes));
  MOE_TRY(check_device());
  Ws w = carve(p, ws);
  Plan q = p;                 // routed experts only
  q.shared = false;
  q.G = p.E;
  MOE_CUDA(launch_permute(q, topk_ids, k, k_per_token, expert_offsets, perm_token, inv_row,
                          w.tiles, w.pscr, w.status, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

int moe_grouped_ffn_fp8(const moe_dims* dims, const uint16_t* hidden, const uint8_t* w13,
                        const float* w13_scale, const uint8_t* w2, const float* w2_scale,
                        const int32_t* expert_offsets, const int32_t* perm_token,
                        float* expert_out, float* act_scale_out, void* ws, size_t ws_bytes,
                        void* stream) {
  if (!dims) return MOE_ERR_INVALID_ARG;
  Plan p;
  MOE_TRY(plan_make(dims->T, dims->d, dims->E, dims->F, dims->k_max, dims->F_shared, &p));
  if (p.T == 0) return MOE_OK;
  if (!hidden || !w13 || !w13_scale || !w2 || !w2_scale || !expert_offsets || !perm_token ||
      !expert_out)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(w13, 16) || !aligned(w2, 16) || !aligned(expert_out, 16))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(p, ws, ws_bytes));
  MOE_TRY(check_device());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Ws w = carve(p, ws);
  Plan q = p;
  q.shared = false;
  q.G = p.E;
  q.Rcap = (int64_t)p.T * p.k_max;
  MOE_CUDA(launch_topk_quant(q, nullptr, nullptr, 1, nullptr, nullptr, nullptr, hidden, w.xq,
                             w.xs, false, true, nullptr, w.status, s));
  if (act_scale_out)
    MOE_CUDA(cudaMemcpyAsync(act_scale_out, w.xs, sizeof(float) * p.T, cudaMemcpyDeviceToDevice, s));
  MOE_CUDA(launch_tile_prefix(q, expert_offsets, w.tiles, w.status, s));
  // the grouped FFN reads offsets/perm from the workspace copies: keep one layout for both paths
  MOE_CUDA(cudaMemcpyAsync(w.offsets, expert_offsets, sizeof(int32_t) * (p.E + 1),
                           cudaMemcpyDeviceToDevice, s));
  MOE_CUDA(cudaMemcpyAsync(w.perm, perm_token, sizeof(int32_t) * q.Rcap, cudaMemcpyDeviceToDevice, s));
  const bool direct = p.g2_splits == 1;
  MOE_TRY(run_ffn(q, w, w13, w13_scale, w2, w2_scale, nullptr, nullptr, nullptr, nullptr,
                  direct ? expert_out : w.o, (size_t)p.Rpad * p.d, q.Rcap, nullptr, s));
  if (!direct)
    MOE_CUDA(launch_reduce_splits(q, w.o, p.g2_splits, (size_t)p.Rpad * p.d, w.offsets + p.E,
                                  expert_out, s));
  return MOE_OK;
}

int moe_combine(const moe_dims* dims, const float* expert_out, const float* topk_w,
                const int32_t* inv_row, const float* shared_out, uint16_t* y, float* y_f32,
                void* stream) {
  if (!dims) return MOE_ERR_INVALID_ARG;
  Plan p;
  MOE_TRY(plan_make(dims->T, dims->d, dims->E, dims->F, dims->k_max, dims->F_shared, &p));
  if (p.T == 0) return MOE_OK;
  if (!expert_out || !topk_w || !inv_row || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned(expert_out, 16) || !aligned(y, 16) || (shared_out && !aligned(shared_out, 16)) ||
      (y_f32 && !aligned(y_f32, 16)))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_device());
  Plan q = p;
  q.Rcap = (int64_t)p.T * p.k_max;
  MOE_CUDA(launch_combine(q, expert_out, 1, 0, topk_w, inv_row, shared_out, nullptr, 1, y, y_f32,
                          static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

int moe_forward(const moe_dims* dims, const uint16_t* hidden, const float* router_w,
                const float* router_bias, int32_t k, const int32_t* k_per_token,
                const uint8_t* w13, const float* w13_scale, const uint8_t* w2,
                const float* w2_scale, const uint8_t* w13_shared, const float* w13s_scale,
                const uint8_t* w2_shared, const float* w2s_scale, uint16_t* y, void* ws,
                size_t ws_bytes, void* stream, const moe_debug_out* dbg) {
  if (!dims) return MOE_ERR_INVALID_ARG;
  Plan p;
  // tiles planned for the fixed k, or for k_max / 2 experts per token of an elastic batch
  const int k_est = k_per_token ? std::max(1, dims->k_max / 2) : k;
  MOE_TRY(plan_make(dims->T, dims->d, dims->E, dims->F, dims->k_max, dims->F_shared, &p, k_est));
  if (p.T == 0) return MOE_OK;
  if (!hidden || !router_w || !w13 || !w13_scale || !w2 || !w2_scale || !y) return MOE_ERR_INVALID_ARG;
  if (p.shared && (!w13_shared || !w13s_scale || !w2_shared || !w2s_scale)) return MOE_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(router_w, 16) || !aligned(w13, 16) || !aligned(w2, 16) ||
      !aligned(y, 16) || (p.shared && (!aligned(w13_shared, 16) || !aligned(w2_shared, 16))))
    return MOE_ERR_INVALID_ARG;
  if (dbg && dbg->y_f32 && !aligned(dbg->y_f32, 16)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_k(p, k, k_per_token));
  MOE_TRY(check_ws(p, ws, ws_bytes));
  MOE_TRY(check_device());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Ws w = carve(p, ws);
  void* const* ev = dbg ? dbg->stage_events : nullptr;
  auto record = [&](int i) {
    if (ev && ev[i]) cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s);
  };

  MOE_CUDA(cudaMemsetAsync(w.status, 0, 16, s));
  record(0);
  if (router_is_fused(p)) {
    // one kernel for stages 0 and 1 (stage 1's events bracket nothing)
    MOE_CUDA(launch_route_fused(p, hidden, router_w, router_bias, k, k_per_token, w.ids, w.w, w.xq,
                                w.xs, true, w.status, s));
    record(1);
  } else if (router_uses_gemv(p)) {
    // decode batch: logits, top-k, quantisation and the grouping in one kernel (the events of
    // stages 1 and 2 bracket nothing)
    const DecodeGrouping grp{w.offsets, w.perm, w.inv, w.tiles, w.amax, p.BN, p.shared ? 1 : 0,
                             w.xqp, w.xsp};
    MOE_CUDA(launch_route_gemv(p, hidden, router_w, router_bias, k, k_per_token, w.part, w.ids,
                               w.w, w.xq, w.xs, true, w.status, grp, s));
    record(1);
  } else {
    MOE_TRY(run_router_logits(p, w, hidden, router_w, s));
    record(1);
    MOE_CUDA(launch_topk_quant(p, w.part, router_bias, k, k_per_token, w.ids, w.w, hidden, w.xq,
                               w.xs, true, true, router_uses_mma(p) ? router_w : nullptr,
                               w.status, s));
  }
  record(2);
  // grouping and row gather: by the decode router itself (T <= 8), in one kernel
  // (T * k_max <= 8192), or the grouping kernels followed by the gather kernel
  bool gathered = false;
  if (router_uses_gemv(p)) {
    gathered = true;                 // the decode router also gathered the rows
  } else if (!permute_gather_fused(p)) {
    MOE_CUDA(launch_permute(p, w.ids, k, k_per_token, w.offsets, w.perm, w.inv, w.tiles, w.pscr,
                            w.status, s));
  } else {
    MOE_CUDA(launch_permute_gather(p, w.ids, k, k_per_token, w.offsets, w.perm, w.inv, w.tiles,
                                   w.xq, w.xs, w.xqp, w.xsp, w.amax, w.status, s));
    gathered = true;
  }
  const size_t split_stride = (size_t)p.Rpad * p.d;
  MOE_TRY(run_ffn(p, w, w13, w13_scale, w2, w2_scale, w13_shared, w13s_scale, w2_shared,
                  w2s_scale, w.o, split_stride, p.Rcap, ev, s, gathered));
  record(7);
  MOE_CUDA(launch_combine(p, w.o, p.g2_splits, split_stride, w.w, w.inv,
                          p.shared ? w.o : nullptr, p.shared ? w.offsets + p.E : nullptr,
                          p.g2_splits, y, dbg ? dbg->y_f32 : nullptr, s));
  record(8);
  if (dbg) {
    const size_t kk = (size_t)p.T * p.k_max;
    if (dbg->topk_ids) MOE_CUDA(cudaMemcpyAsync(dbg->topk_ids, w.ids, 4 * kk, cudaMemcpyDeviceToDevice, s));
    if (dbg->topk_w) MOE_CUDA(cudaMemcpyAsync(dbg->topk_w, w.w, 4 * kk, cudaMemcpyDeviceToDevice, s));
    if (dbg->expert_offsets)
      MOE_CUDA(cudaMemcpyAsync(dbg->expert_offsets, w.offsets, 4 * (size_t)(p.E + 1), cudaMemcpyDeviceToDevice, s));
    if (dbg->perm_token) MOE_CUDA(cudaMemcpyAsync(dbg->perm_token, w.perm, 4 * kk, cudaMemcpyDeviceToDevice, s));
    if (dbg->inv_row) MOE_CUDA(cudaMemcpyAsync(dbg->inv_row, w.inv, 4 * kk, cudaMemcpyDeviceToDevice, s));
  }
  return MOE_OK;
}

int moe_ep_dispatch(const moe_dims* dims, int32_t n_ranks, const uint16_t* hidden,
                    const int32_t* topk_ids, const float* topk_w, int32_t k,
                    const int32_t* k_per_token, uint16_t* send_hidden, int32_t* send_ids,
                    float* send_w, int32_t* send_counts, int32_t* slot_of, float* slot_w,
                    void* ws, size_t ws_bytes, void* stream) {
  if (!dims) return MOE_ERR_INVALID_ARG;
  Plan p;
  MOE_TRY(plan_make(dims->T, dims->d, dims->E, dims->F, dims->k_max, dims->F_shared, &p));
  if (n_ranks < 1 || n_ranks > 32 || p.E % n_ranks != 0) return MOE_ERR_INVALID_ARG;
  if (!send_counts) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (p.T == 0) {
    MOE_TRY(check_device());
    MOE_CUDA(cudaMemsetAsync(send_counts, 0, sizeof(int32_t) * n_ranks, s));
    return MOE_OK;
  }
  if (!hidden || !topk_ids || !topk_w || !send_hidden || !send_ids || !send_w || !slot_of ||
      !slot_w)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(send_hidden, 16)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_k(p, k, k_per_token));
  MOE_TRY(check_ws(p, ws, ws_bytes));
  MOE_TRY(check_device());
  Ws w = carve(p, ws);
  MOE_CUDA(launch_ep_dispatch(p, n_ranks, hidden, topk_ids, topk_w, k, k_per_token, send_hidden,
                              send_ids, send_w, send_counts, slot_of, slot_w, w.status, s));
  return MOE_OK;
}

}  // extern "C"
