// Internal launch plan and kernel launchers of the FP8 MoE layer (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

constexpr int kBK = 128;            // bytes (= e4m3 elements) of K per pipeline stage
// CUDA-core router logits tile: 64 tokens x 64 experts, d in chunks of 16
constexpr int kRtTok = 64, kRtExp = 64, kRtK = 16;
constexpr int kMaxExperts = 1024;
constexpr int kMaxK = 32;

// Everything the host decides for one (dims) configuration: tile sizes, split counts and the
// carve-up of the workspace. Offsets are bytes from the workspace base, 256-byte aligned.
struct Plan {
  int T, d, E, F, k_max, Fs;
  bool shared;
  int G;             // GEMM groups: E routed experts (+1 shared expert)
  int64_t Rcap;      // routed-row capacity: T*k_max (+T shared rows)
  int64_t Rpad;      // rows allocated for row-indexed buffers (>= Rcap, >= 256)
  int BN;            // token tile of the grouped GEMMs (max MMA N; a tile uses its valid rows)
  bool pair1, pair2; // gate/up, down GEMM on 2-CTA pairs (M = 256 tcgen05 MMA)
  int slabs1;        // weight slabs of 128 rows per CTA in the gate/up GEMM (2: pairs only)
  int r_splits, r_chunks_per_split;           // router: split of d into 32-wide chunks
  int g1_kb, g1_m_tiles;                      // gate/up GEMM: K blocks (d/128), 64-row tiles
  int g1_splits, g1_kb_per_split;             // gate/up K split (decode); 1 = SwiGLU epilogue
  int g2_kb, g2_m_tiles, g2_splits, g2_kb_per_split;  // down GEMM
  size_t off_status, off_part, off_ids, off_w, off_offsets, off_tiles, off_perm, off_inv, off_pscr;
  size_t off_xq, off_xs, off_xqp, off_xsp, off_amax, off_act, off_aq, off_s2, off_o, off_planes;
  size_t off_hpart;
  size_t bytes;
};

// Grouped GEMM variants: gate/up with the SwiGLU epilogue (act + row max), down projection, and
// gate/up split over K (scaled partial sums; SwiGLU and the requantisation follow in a row kernel).
constexpr int kModeSwiGLU = 0;
constexpr int kModeDown = 1;
constexpr int kModeGateUpPartial = 2;

// Arguments of one grouped GEMM launch (tile decode + epilogue).
struct GemmArgs {
  const int32_t* group_offsets;  // [G+1] first routed row of each group
  const int32_t* tile_prefix;    // [G+1] prefix sum over groups of ceil(rows / BN)
  int G, E_routed;               // groups >= E_routed use the shared-expert weights
  int m_tiles, splits, kb_per_split, num_kb;
  int M_valid;                   // valid weight rows: F (gate/up halves) or d (down)
  const float* row_scale;        // [Rpad] activation scale of each routed row
  const float* w_scale;          // [E, w_scale_ld] per-output-channel weight scales
  const float* w_scale_shared;   // [w_scale_ld] shared expert (or null)
  int w_scale_ld;                // 2F (gate/up) or d (down)
  float* out;                    // gate/up: act [Rpad, F]; down: o [splits][Rpad, d]
  int out_ld;
  size_t out_split_stride;       // elements between split partials
  uint32_t* row_amax;            // gate/up: [Rpad] |act| max as fp32 bits
  int* status;
#ifdef MOE_WAIT_TEST
  int withhold;                  // wait-test build: skip the first tile's accumulator signal
#endif
};

#ifdef MOE_WAIT_TEST
// Wait-test build only: when set, every CTA of the next gate/up GEMMs withholds the "accumulator
// ready" signal of its first tile, so that the epilogue's bounded wait expires.
extern int g_withhold_gemm_commit;
#endif

// Planning assumes the B200's 148 SMs so that moe_workspace_bytes stays a pure host function;
// persistent grids use the real SM count of the current device.
constexpr int kPlanSMs = 148;

// The CUDA-core router logits kernel's cut of d: 32-token x 32-expert tiles and enough pieces of
// d (each `*chunks_per_split` 32-wide chunks) for about two waves of kPlanSMs; returns the number
// of pieces (the splits of the partial logits).
int router_splits(int T, int d, int E, int* chunks_per_split);

// k_est: experts per token the GEMM tiles are planned for (0 = k_max); buffers are for k_max.
int plan_make(int T, int d, int E, int F, int k_max, int Fs, Plan* p, int k_est = 0);

// Router logits are fp64 (part [splits][T][E] doubles): see route.cu.
cudaError_t launch_router_logits(const Plan& p, const uint16_t* hidden, const float* router_w,
                                 double* part, cudaStream_t s);
cudaError_t launch_topk_quant(const Plan& p, const double* part, const float* bias, int k,
                              const int32_t* k_per_token, int32_t* ids, float* w,
                              const uint16_t* hidden, uint8_t* xq, float* xs, bool do_route,
                              bool do_quant, const float* refine_w, int* status, cudaStream_t s);
// Router paths. E <= 32: one fused kernel (logits, top-k, weights, quantisation). E > 32 and
// T >= 64: tensor-core logits (bf16 split of the fp32 weights) + topk_quant. Otherwise: CUDA-core
// logits + topk_quant.
// (the fused router holds a token's row in registers: d <= 8192)
inline bool router_is_fused(int E, int d) { return E <= 32 && d <= 8192; }
// Router logits on the tensor cores (two bf16 planes + exact refinement of the candidates) once
// the fp32 CUDA-core work 2·T·E·d is large: measured on B200, the exact CUDA-core router is faster
// up to T·E·d ~ 2.4e8 (Qwen3 T=64, DeepSeek T=128, MoE-Prism T=64) and the tensor-core one from
// ~1.1e9 (Qwen3 T=4096, MoE-Prism T=2048, DeepSeek T=8192); the switch sits at 2^29.
inline bool router_uses_mma(int E, int T, int d) {
  return E > 32 && (long long)T * E * d >= (1LL << 29);
}
inline bool router_is_fused(const Plan& p) { return router_is_fused(p.E, p.d); }
inline bool router_uses_mma(const Plan& p) { return router_uses_mma(p.E, p.T, p.d); }
// decode batches (T <= 8) with E > 32: the one-kernel GEMV router (logits [T][E] in the
// workspace's partial-logit buffer, the status word's counter for the last block)
inline bool router_uses_gemv(int E, int T, int d) {
  return E > 32 && T >= 1 && T <= 8 && !router_uses_mma(E, T, d);
}
inline bool router_uses_gemv(const Plan& p) { return router_uses_gemv(p.E, p.T, p.d); }
// Grouping done by the decode router's last block (null offsets: routing only). Same outputs as
// launch_permute (offsets [E+2], perm, inv, tiles [E+2] with the shared expert's group when
// has_shared), and amax zeroed for every routed / shared row.
struct DecodeGrouping {
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv;
  int32_t* tiles;
  uint32_t* amax;
  int BN, has_shared;
  uint8_t* xqp;     // gathered FP8 rows [rows][d] (with the quantisation), or null
  float* xsp;       // their scales [rows]
};
cudaError_t launch_route_gemv(const Plan& p, const uint16_t* hidden, const float* router_w,
                              const float* bias, int k, const int32_t* k_per_token,
                              double* logits, int32_t* ids, float* w, uint8_t* xq, float* xs,
                              bool do_quant, int* status, const DecodeGrouping& grp,
                              cudaStream_t s);
// Tokens per tile of the tensor-core router (64 or 128): the box height of map_x.
int router_mma_tokens(int T, int E);
// planes: 2 * E * d bf16 (workspace); map_w over planes [2][E][d], map_x over hidden [T][d]
cudaError_t launch_router_mma(const Plan& p, const float* router_w, uint16_t* planes,
                              const CUtensorMap& map_w, const CUtensorMap& map_x, double* logits,
                              int* status, cudaStream_t s);
cudaError_t launch_route_fused(const Plan& p, const uint16_t* hidden, const float* router_w,
                               const float* bias, int k, const int32_t* k_per_token,
                               int32_t* ids, float* w, uint8_t* xq, float* xs, bool do_quant,
                               int* status, cudaStream_t s);
// scratch: 2 * permute_blocks(p) * E int32 (per-block counts and bases; unused for one block)
int permute_blocks(const Plan& p);
// grouping + row gather in one kernel (when the grouping fits one block, T * k_max <= 8192)
bool permute_gather_fused(const Plan& p);
cudaError_t launch_permute_gather(const Plan& p, const int32_t* ids, int k,
                                  const int32_t* k_per_token, int32_t* offsets, int32_t* perm,
                                  int32_t* inv, int32_t* tiles, const uint8_t* xq, const float* xs,
                                  uint8_t* xqp, float* xsp, uint32_t* amax, int* status,
                                  cudaStream_t s);
cudaError_t launch_permute(const Plan& p, const int32_t* ids, int k, const int32_t* k_per_token,
                           int32_t* offsets, int32_t* perm, int32_t* inv, int32_t* tiles,
                           int32_t* scratch, int* status, cudaStream_t s);
cudaError_t launch_tile_prefix(const Plan& p, const int32_t* offsets, int32_t* tiles, int* status,
                               cudaStream_t s);
cudaError_t launch_gather(const Plan& p, const uint8_t* xq, const float* xs, const int32_t* perm,
                          const int32_t* total_rows, uint8_t* xqp, float* xsp, uint32_t* amax,
                          int* status, cudaStream_t s);
// acts64 / acts16: the routed-row activations with 64-row and 16-row TMA boxes
cudaError_t launch_gemm_gateup(const Plan& p, const CUtensorMap& w13, const CUtensorMap& w13s,
                               const CUtensorMap& acts64, const CUtensorMap& acts16,
                               const GemmArgs& a, bool partial, cudaStream_t s);
// K-split gate/up: h[s][r][2F] partials -> act = silu(gate) * up, row amax, FP8 codes and scales
cudaError_t launch_swiglu_requant(const Plan& p, const float* h, int splits, size_t split_stride,
                                  const int32_t* total_rows, uint8_t* aq, float* s2,
                                  cudaStream_t s);
cudaError_t launch_gemm_down(const Plan& p, const CUtensorMap& w2, const CUtensorMap& w2s,
                             const CUtensorMap& acts64, const CUtensorMap& acts16,
                             const CUtensorMap& out, const GemmArgs& a, cudaStream_t s);
cudaError_t launch_requant(const Plan& p, const float* act, const uint32_t* amax,
                           const int32_t* total_rows, uint8_t* aq, float* s2, cudaStream_t s);
cudaError_t launch_combine(const Plan& p, const float* o, int splits, size_t split_stride,
                           const float* topk_w, const int32_t* inv_row, const float* shared_src,
                           const int32_t* shared_row0, int shared_splits, uint16_t* y,
                           float* y_f32, cudaStream_t s);
cudaError_t launch_reduce_splits(const Plan& p, const float* o, int splits, size_t split_stride,
                                 const int32_t* total_rows, float* out, cudaStream_t s);

// Expert-parallel dispatch over n_ranks contiguous expert blocks: plan (send rows in (rank,
// token) order, local ids and weights, per-rank counts, the combine map) and the row gather.
__host__ __device__ inline int ep_local_k(int E, int k_max, int n_ranks) {
  const int el = E / n_ranks;
  return k_max < el ? k_max : el;
}
cudaError_t launch_ep_dispatch(const Plan& p, int n_ranks, const uint16_t* hidden,
                               const int32_t* ids, const float* topk_w, int k,
                               const int32_t* k_per_token, uint16_t* send_hidden,
                               int32_t* send_ids, float* send_w, int32_t* send_counts,
                               int32_t* slot_of, float* slot_w, int* status, cudaStream_t s);

int num_sms();

}  // namespace moe
