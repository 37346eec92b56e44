// Router of the MoE layer: logits, softmax / top-k with renormalised weights, and the token's
// dynamic FP8 e4m3 quantisation (scale = amax / 448). Four kernels, by shape:
//   route_block_kernel   E <= 32: one block per token does all of it;
//   route_gemv_kernel    decode batches (T <= 8, E > 32): a warp per expert, and the last block
//                        to finish selects and quantises;
//   router_logits_kernel fp32 CUDA-core logits (deterministic split over the hidden dimension),
//   + topk_quant_kernel  then per token a warp-level top-k and the quantisation;
//   topk_quant_kernel    also after the tensor-core logits (router_mma.cu), refining the
//                        candidates' logits exactly before the selection.
//
// Method: "Routage MoE entre GPU" (viite.ai) -- the router scores all experts from the hidden
// state, keeps the top-k and emits one routing weight per selection; the megakernel page
// (seventnews.com), W8A8 paragraph -- 8-bit FP8 activations.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

// part[s][t][e] = sum over the d-chunks of split s of x[t, d] * W[e, d], fp32, d ascending,
// one partial sum per 32-wide chunk (blocked summation keeps the rounding error near fp64).
// Block: 256 threads computing a 32-token x 32-expert tile; thread (ty, tx) owns tokens
// 4*ty .. 4*ty+3 of expert tx.
__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t* __restrict__ x,
                                                            const float* __restrict__ W, int T,
                                                            int d, int E, int chunks_per_split,
                                                            float* __restrict__ part) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  __shared__ float xs[kRouterTile][kRouterTile + 1];
  __shared__ float ws[kRouterTile][kRouterTile + 1];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int t0 = blockIdx.x * kRouterTile, e0 = blockIdx.y * kRouterTile;
  const int split = blockIdx.z;
  const int nchunks = (d + kRouterTile - 1) / kRouterTile;
  const int c_begin = split * chunks_per_split;
  const int c_end = min(nchunks, c_begin + chunks_per_split);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int c = c_begin; c < c_end; ++c) {
    const int dbase = c * kRouterTile;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty + 8 * i;            // row of the tile this thread loads
      const int dd = dbase + tx;
      const int t = t0 + r, e = e0 + r;
      xs[r][tx] = (t < T && dd < d) ? bf16_bits_to_float(x[(size_t)t * d + dd]) : 0.f;
      ws[r][tx] = (e < E && dd < d) ? W[(size_t)e * d + dd] : 0.f;
    }
    __syncthreads();
    // blocked summation: each 32-wide chunk is summed on its own, then added to the total
    float chunk[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int kk = 0; kk < kRouterTile; ++kk) {
      const float w = ws[tx][kk];
#pragma unroll
      for (int i = 0; i < 4; ++i) chunk[i] = fmaf(xs[4 * ty + i][kk], w, chunk[i]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] += chunk[i];
    __syncthreads();
  }
  const int e = e0 + tx;
  if (e < E) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = t0 + 4 * ty + i;
      if (t < T) part[((size_t)split * T + t) * E + e] = acc[i];
    }
  }
}

// One block (128 threads) per token.
//  route: l[e] = sum_s part[s][t][e] + bias[e]; k_t largest (descending, exact ties to the lower
//         expert id); w_j = exp(l_j - l_max) / sum_sel exp(l_sel - l_max), which equals the
//         softmax over all E renormalised over the selection.
//  quant: s_t = amax|x[t,:]| / 448 (IEEE fp32 division; 1 if amax = 0);
//         xq = e4m3_rne_satfinite(x / s_t) (IEEE fp32 division).
//  refine (refine_w != null, for the tensor-core logits): the approximate logits only pick the
//         candidates -- every expert within kRefineWindow of the approximate k_t-th largest, which
//         contains the exact top-k_t while the approximation error stays below half the window --
//         and each candidate's logit is recomputed exactly (fp32, one warp per candidate, fixed
//         order) before the selection and the weights.
constexpr float kRefineWindow = 1e-2f;
constexpr int kMaxCandidates = 256;

__global__ void __launch_bounds__(128) topk_quant_kernel(
    const float* __restrict__ part, int splits, const float* __restrict__ bias, int T, int E,
    int k, const int32_t* __restrict__ k_per_token, int k_max, int32_t* __restrict__ ids,
    float* __restrict__ wout, const uint16_t* __restrict__ x, int d, uint8_t* __restrict__ xq,
    float* __restrict__ xs, int do_route, int do_quant, const float* __restrict__ refine_w,
    int* status) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  __shared__ float lg[kMaxExperts];
  __shared__ float red[4];
  const int t = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (do_route) {
    for (int e = tid; e < E; e += 128) {
      // split partials in fixed order: eight independent accumulators keep eight loads in
      // flight (a decode batch splits d finely, and these loads are the kernel's latency)
      float a8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      int s = 0;
      for (; s + 8 <= splits; s += 8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) a8[u] += part[((size_t)(s + u) * T + t) * E + e];
      }
      for (int u = 0; s < splits; ++s, ++u) a8[u] += part[((size_t)s * T + t) * E + e];
      float v = ((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]));
      if (bias) v += bias[e];
      lg[e] = v;
    }
    __syncthreads();
    int kt = k_per_token ? k_per_token[t] : k;
    const int kcap = min(E, k_max);
    if (kt < 1 || kt > kcap) {
      if (tid == 0) report(status, kStatusDeviceCheck, kWhereRoute, t);
      kt = max(1, min(kt, kcap));
    }
    __shared__ int cand[kMaxCandidates];
    __shared__ int ncand;
    bool by_cand = false;          // exact selection over the refined candidates only
    if (refine_w) {
      __shared__ float vk_s;
      if (warp == 0) {
        // approximate k_t-th largest logit
        uint32_t taken = 0;
        float bv = -INFINITY;
        for (int j = 0; j < kt; ++j) {
          bv = -INFINITY;
          int be = 0x7FFFFFFF;
          for (int i = 0, e = lane; e < E; ++i, e += 32) {
            const float v = lg[e];
            if (!((taken >> i) & 1u) && (v > bv || (v == bv && e < be))) {
              bv = v;
              be = e;
            }
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (ov > bv || (ov == bv && oe < be)) {
              bv = ov;
              be = oe;
            }
          }
          if ((be & 31) == lane) taken |= 1u << (be >> 5);
        }
        if (lane == 0) {
          vk_s = bv;
          ncand = 0;
        }
      }
      __syncthreads();
      const float floor_v = vk_s - kRefineWindow;
      for (int e = tid; e < E; e += 128) {
        if (lg[e] >= floor_v) {
          const int c = atomicAdd(&ncand, 1);
          if (c < kMaxCandidates) cand[c] = e;
        } else {
          lg[e] = -INFINITY;                            // out of the selection
        }
      }
      __syncthreads();
      const bool all = ncand > kMaxCandidates;          // pathological: recompute every expert
      const int nc = all ? E : ncand;
      const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * d);
      const int nv = d / 8;
      for (int c = warp; c < nc; c += 4) {
        const int e = all ? c : cand[c];
        const float4* wr = reinterpret_cast<const float4*>(refine_w + (size_t)e * d);
        float acc = 0.f;
#pragma unroll 8
        for (int i = lane; i < nv; i += 32) {
          const uint4 v = xr[i];
          const float4 a = __ldg(wr + 2 * i), b = __ldg(wr + 2 * i + 1);
          float c8 = __uint_as_float(v.x << 16) * a.x;
          c8 = fmaf(__uint_as_float(v.x & 0xFFFF0000u), a.y, c8);
          c8 = fmaf(__uint_as_float(v.y << 16), a.z, c8);
          c8 = fmaf(__uint_as_float(v.y & 0xFFFF0000u), a.w, c8);
          c8 = fmaf(__uint_as_float(v.z << 16), b.x, c8);
          c8 = fmaf(__uint_as_float(v.z & 0xFFFF0000u), b.y, c8);
          c8 = fmaf(__uint_as_float(v.w << 16), b.z, c8);
          c8 = fmaf(__uint_as_float(v.w & 0xFFFF0000u), b.w, c8);
          acc += c8;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) lg[e] = acc + (bias ? bias[e] : 0.f);
      }
      __syncthreads();
      by_cand = !all;
    }
    if (warp == 0) {
      // bit i of `taken`: scan slot lane + 32 i already selected (slot = expert, or candidate
      // index when the refined candidates are scanned; the others hold -inf then)
      uint32_t taken = 0;
      float sel_v = 0.f;             // lane j keeps the j-th selected logit
      int sel_e = -1;
      const int n_scan = by_cand ? ncand : E;
      for (int j = 0; j < kt; ++j) {
        float bv = -INFINITY;
        int be = 0x7FFFFFFF;
        for (int i = 0, c = lane; c < n_scan; ++i, c += 32) {
          const int e = by_cand ? cand[c] : c;
          const float v = lg[e];
          if (!((taken >> i) & 1u) && (v > bv || (v == bv && e < be))) {
            bv = v;
            be = e;
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
          const int oe = __shfl_xor_sync(0xffffffffu, be, off);
          if (ov > bv || (ov == bv && oe < be)) {
            bv = ov;
            be = oe;
          }
        }
        if (by_cand) {
          for (int i = 0, c = lane; c < n_scan; ++i, c += 32)
            if (cand[c] == be) taken |= 1u << i;
        } else if ((be & 31) == lane) {
          taken |= 1u << (be >> 5);
        }
        if (lane == j) {
          sel_v = bv;
          sel_e = be;
        }
      }
      const float lmax = __shfl_sync(0xffffffffu, sel_v, 0);
      const float z = lane < kt ? expf(sel_v - lmax) : 0.f;
      float zs = z;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, off);
      if (lane < k_max) {
        ids[(size_t)t * k_max + lane] = lane < kt ? sel_e : -1;
        wout[(size_t)t * k_max + lane] = lane < kt ? z / zs : 0.f;
      }
    }
  }

  if (do_quant) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * d);
    const int nv = d / 8;
    float amax = 0.f;
    for (int i = tid; i < nv; i += 128) {
      const uint4 v = xr[i];
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        amax = fmaxf(amax, fabsf(__uint_as_float(w4[q] << 16)));
        amax = fmaxf(amax, fabsf(__uint_as_float(w4[q] & 0xFFFF0000u)));
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    if (tid == 0) xs[t] = sc;
    uint2* out = reinterpret_cast<uint2*>(xq + (size_t)t * d);
    for (int i = tid; i < nv; i += 128) {
      const uint4 v = xr[i];
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      uint32_t packed[2];
#pragma unroll
      for (int q = 0; q < 4; q += 2) {
        const float a0 = __fdiv_rn(__uint_as_float(w4[q] << 16), sc);
        const float a1 = __fdiv_rn(__uint_as_float(w4[q] & 0xFFFF0000u), sc);
        const float a2 = __fdiv_rn(__uint_as_float(w4[q + 1] << 16), sc);
        const float a3 = __fdiv_rn(__uint_as_float(w4[q + 1] & 0xFFFF0000u), sc);
        packed[q / 2] = static_cast<uint32_t>(e4m3x2(a0, a1)) |
                        (static_cast<uint32_t>(e4m3x2(a2, a3)) << 16);
      }
      out[i] = make_uint2(packed[0], packed[1]);
    }
  }
}

// Decode router (T <= 8 tokens, E > 32): one warp per expert computes that expert's logit for
// every token (lane-strided chunks of 8 along d, fp32, then a butterfly; all loads in flight),
// writes it to `logits` [T][E], and the last block to finish (a counter in the status word,
// status[3]) selects the top-k, the weights and the FP8 quantisation of every token, then resets
// the counter. One kernel instead of the tiled logits kernel (one global round trip per 32-wide
// chunk of d) plus a separate top-k kernel.
constexpr int kGemvMaxT = 8;

template <int TT>
__global__ void __launch_bounds__(256) route_gemv_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ W, const float* __restrict__ bias,
    int T, int d, int E, int k, const int32_t* __restrict__ k_per_token, int k_max,
    float* __restrict__ logits, int32_t* __restrict__ ids, float* __restrict__ wout,
    uint8_t* __restrict__ xq, float* __restrict__ xs, int do_quant, int* status) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  __shared__ int s_last;
  __shared__ float lg[kGemvMaxT][kMaxExperts];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int e = blockIdx.x * 8 + warp;
  const int nv = d / 8;
  if (e < E) {
    float acc[TT];
#pragma unroll
    for (int j = 0; j < TT; ++j) acc[j] = 0.f;
    const float4* wr = reinterpret_cast<const float4*>(W + (size_t)e * d);
#pragma unroll 4
    for (int i = lane; i < nv; i += 32) {
      const float4 a = __ldg(wr + 2 * i), b = __ldg(wr + 2 * i + 1);
#pragma unroll
      for (int j = 0; j < TT; ++j) {
        if (j < T) {
          const uint4 v = reinterpret_cast<const uint4*>(x + (size_t)j * d)[i];
          float c8 = __uint_as_float(v.x << 16) * a.x;
          c8 = fmaf(__uint_as_float(v.x & 0xFFFF0000u), a.y, c8);
          c8 = fmaf(__uint_as_float(v.y << 16), a.z, c8);
          c8 = fmaf(__uint_as_float(v.y & 0xFFFF0000u), a.w, c8);
          c8 = fmaf(__uint_as_float(v.z << 16), b.x, c8);
          c8 = fmaf(__uint_as_float(v.z & 0xFFFF0000u), b.y, c8);
          c8 = fmaf(__uint_as_float(v.w << 16), b.z, c8);
          c8 = fmaf(__uint_as_float(v.w & 0xFFFF0000u), b.w, c8);
          acc[j] += c8;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < TT; ++j) {
      if (j < T) {
        float v = acc[j];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) logits[(size_t)j * E + e] = v + (bias ? bias[e] : 0.f);
      }
    }
  }
  // the last block to arrive sees every block's logits
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&status[3], 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (warp < T) {
    const int t = warp;
    float* my = lg[warp];
    for (int ee = lane; ee < E; ee += 32) my[ee] = __ldcg(logits + (size_t)t * E + ee);
    __syncwarp();
    int kt = k_per_token ? k_per_token[t] : k;
    const int kcap = min(E, k_max);
    if (kt < 1 || kt > kcap) {
      if (lane == 0) report(status, kStatusDeviceCheck, kWhereRoute, t);
      kt = max(1, min(kt, kcap));
    }
    uint32_t taken = 0;            // bit i: expert lane + 32*i already selected
    float sel_v = 0.f;             // lane j keeps the j-th selected logit
    int sel_e = -1;
    for (int j = 0; j < kt; ++j) {
      float bv = -INFINITY;
      int be = 0x7FFFFFFF;
      for (int i = 0, ee = lane; ee < E; ++i, ee += 32) {
        const float v = my[ee];
        if (!((taken >> i) & 1u) && (v > bv || (v == bv && ee < be))) {
          bv = v;
          be = ee;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oe = __shfl_xor_sync(0xffffffffu, be, off);
        if (ov > bv || (ov == bv && oe < be)) {
          bv = ov;
          be = oe;
        }
      }
      if ((be & 31) == lane) taken |= 1u << (be >> 5);
      if (lane == j) {
        sel_v = bv;
        sel_e = be;
      }
    }
    const float lmax = __shfl_sync(0xffffffffu, sel_v, 0);
    const float z = lane < kt ? expf(sel_v - lmax) : 0.f;
    float zs = z;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, off);
    if (lane < k_max) {
      ids[(size_t)t * k_max + lane] = lane < kt ? sel_e : -1;
      wout[(size_t)t * k_max + lane] = lane < kt ? z / zs : 0.f;
    }
  }
  if (do_quant) {
    // the FP8 quantisation of each token by the whole block
    __shared__ float red[8];
    for (int t = 0; t < T; ++t) {
      const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * d);
      float amax = 0.f;
      for (int i = tid; i < nv; i += 256) {
        const uint4 v = xr[i];
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          amax = fmaxf(amax, fabsf(__uint_as_float(w4[q] << 16)));
          amax = fmaxf(amax, fabsf(__uint_as_float(w4[q] & 0xFFFF0000u)));
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      if (lane == 0) red[warp] = amax;
      __syncthreads();
      float am = red[0];
#pragma unroll
      for (int w = 1; w < 8; ++w) am = fmaxf(am, red[w]);
      __syncthreads();                                   // red[] is reused by the next token
      const float sc = am > 0.f ? __fdiv_rn(am, 448.f) : 1.f;
      if (tid == 0) xs[t] = sc;
      uint2* out = reinterpret_cast<uint2*>(xq + (size_t)t * d);
      for (int i = tid; i < nv; i += 256) {
        const uint4 v = xr[i];
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
        uint32_t packed[2];
#pragma unroll
        for (int q = 0; q < 4; q += 2) {
          const float a0 = __fdiv_rn(__uint_as_float(w4[q] << 16), sc);
          const float a1 = __fdiv_rn(__uint_as_float(w4[q] & 0xFFFF0000u), sc);
          const float a2 = __fdiv_rn(__uint_as_float(w4[q + 1] << 16), sc);
          const float a3 = __fdiv_rn(__uint_as_float(w4[q + 1] & 0xFFFF0000u), sc);
          packed[q / 2] = static_cast<uint32_t>(e4m3x2(a0, a1)) |
                          (static_cast<uint32_t>(e4m3x2(a2, a3)) << 16);
        }
        out[i] = make_uint2(packed[0], packed[1]);
      }
    }
  }
  if (tid == 0) status[3] = 0;             // the counter is ready for the next launch
}

// Small-E router (E <= 32), one 256-thread block per token, fully fused: logits, top-k, weights
// and the token's FP8 quantisation. Thread i accumulates x[t, 8c..8c+7] . W[e, 8c..8c+7] for the
// chunks c = i, i + 256, ... (fp32), a butterfly inside each warp and a fixed-order sum over the
// 8 warps complete each logit (deterministic), and lane e of warp 0 owns expert e's logit for the
// selection. The row amax comes from the same pass and the chunks stay in registers for the
// quantisation.
template <int EP>   // experts rounded up: 8, 16 or 32
__global__ void __launch_bounds__(256) route_block_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ W, const float* __restrict__ bias,
    int T, int d, int E, int k, const int32_t* __restrict__ k_per_token, int k_max,
    int32_t* __restrict__ ids, float* __restrict__ wout, uint8_t* __restrict__ xq,
    float* __restrict__ xs, int do_quant, int* status) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  constexpr int kChunks = 4;                      // d <= 256 * 8 * kChunks = 8192
  __shared__ float part[8][EP];
  __shared__ float red[8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t = blockIdx.x;
  const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  const int nv = d / 8;
  float acc[EP];
#pragma unroll
  for (int e = 0; e < EP; ++e) acc[e] = 0.f;
  uint4 xv[kChunks];
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    const int i = tid + 256 * c;
    if (i < nv) {
      xv[c] = xr[i];
      const uint32_t w4[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
      float xf[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        xf[2 * q] = __uint_as_float(w4[q] << 16);
        xf[2 * q + 1] = __uint_as_float(w4[q] & 0xFFFF0000u);
        amax = fmaxf(amax, fmaxf(fabsf(xf[2 * q]), fabsf(xf[2 * q + 1])));
      }
#pragma unroll
      for (int e = 0; e < EP; ++e) {
        if (e < E) {
          const float4* wr = reinterpret_cast<const float4*>(W + (size_t)e * d) + 2 * i;
          const float4 a = __ldg(wr), b = __ldg(wr + 1);
          float v = xf[0] * a.x;
          v = fmaf(xf[1], a.y, v);
          v = fmaf(xf[2], a.z, v);
          v = fmaf(xf[3], a.w, v);
          v = fmaf(xf[4], b.x, v);
          v = fmaf(xf[5], b.y, v);
          v = fmaf(xf[6], b.z, v);
          v = fmaf(xf[7], b.w, v);
          acc[e] += v;
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EP; ++e) {
    float v = acc[e];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) part[warp][e] = v;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if (lane == 0) red[warp] = amax;
  __syncthreads();

  if (warp == 0) {
    float logit = -INFINITY;
    if (lane < E) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) v += part[w][lane < EP ? lane : 0];
      logit = v + (bias ? bias[lane] : 0.f);
    }
    // top-k over the lanes (lane e holds expert e), exact ties to the lower id
    int kt = k_per_token ? k_per_token[t] : k;
    const int kcap = min(E, k_max);
    if (kt < 1 || kt > kcap) {
      if (lane == 0) report(status, kStatusDeviceCheck, kWhereRoute, t);
      kt = max(1, min(kt, kcap));
    }
    bool taken = lane >= E;
    float sel_v = 0.f;
    int sel_e = -1;
    for (int j = 0; j < kt; ++j) {
      float bv = taken ? -INFINITY : logit;
      int be = taken ? 0x7FFFFFFF : lane;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oe = __shfl_xor_sync(0xffffffffu, be, off);
        if (ov > bv || (ov == bv && oe < be)) {
          bv = ov;
          be = oe;
        }
      }
      if (be == lane) taken = true;
      if (lane == j) {
        sel_v = bv;
        sel_e = be;
      }
    }
    const float lmax = __shfl_sync(0xffffffffu, sel_v, 0);
    const float z = lane < kt ? expf(sel_v - lmax) : 0.f;
    float zs = z;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, off);
    if (lane < k_max) {
      ids[(size_t)t * k_max + lane] = lane < kt ? sel_e : -1;
      wout[(size_t)t * k_max + lane] = lane < kt ? z / zs : 0.f;
    }
  }
  if (!do_quant) return;
  float am = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) am = fmaxf(am, red[w]);
  const float sc = am > 0.f ? __fdiv_rn(am, 448.f) : 1.f;
  if (tid == 0) xs[t] = sc;
  uint2* out = reinterpret_cast<uint2*>(xq + (size_t)t * d);
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    const int i = tid + 256 * c;
    if (i < nv) {
      const uint32_t w4[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
      uint32_t packed[2];
#pragma unroll
      for (int q = 0; q < 4; q += 2) {
        const float a0 = __fdiv_rn(__uint_as_float(w4[q] << 16), sc);
        const float a1 = __fdiv_rn(__uint_as_float(w4[q] & 0xFFFF0000u), sc);
        const float a2 = __fdiv_rn(__uint_as_float(w4[q + 1] << 16), sc);
        const float a3 = __fdiv_rn(__uint_as_float(w4[q + 1] & 0xFFFF0000u), sc);
        packed[q / 2] = static_cast<uint32_t>(e4m3x2(a0, a1)) |
                        (static_cast<uint32_t>(e4m3x2(a2, a3)) << 16);
      }
      out[i] = make_uint2(packed[0], packed[1]);
    }
  }
}

cudaError_t launch_route_fused(const Plan& p, const uint16_t* hidden, const float* router_w,
                               const float* bias, int k, const int32_t* k_per_token,
                               int32_t* ids, float* w, uint8_t* xq, float* xs, bool do_quant,
                               int* status, cudaStream_t s) {
  const int q = do_quant ? 1 : 0;
  if (p.E <= 8)
    launch_pdl(route_block_kernel<8>, dim3(p.T), dim3(256), 0, s, hidden, router_w, bias, p.T,
               p.d, p.E, k, k_per_token, p.k_max, ids, w, xq, xs, q, status);
  else if (p.E <= 16)
    launch_pdl(route_block_kernel<16>, dim3(p.T), dim3(256), 0, s, hidden, router_w, bias, p.T,
               p.d, p.E, k, k_per_token, p.k_max, ids, w, xq, xs, q, status);
  else
    launch_pdl(route_block_kernel<32>, dim3(p.T), dim3(256), 0, s, hidden, router_w, bias, p.T,
               p.d, p.E, k, k_per_token, p.k_max, ids, w, xq, xs, q, status);
  return cudaGetLastError();
}

cudaError_t launch_route_gemv(const Plan& p, const uint16_t* hidden, const float* router_w,
                              const float* bias, int k, const int32_t* k_per_token, float* logits,
                              int32_t* ids, float* w, uint8_t* xq, float* xs, bool do_quant,
                              int* status, cudaStream_t s) {
  const dim3 grid((p.E + 7) / 8);
  const int q = do_quant ? 1 : 0;
  if (p.T <= 1)
    launch_pdl(route_gemv_kernel<1>, grid, dim3(256), 0, s, hidden, router_w, bias, p.T, p.d, p.E,
               k, k_per_token, p.k_max, logits, ids, w, xq, xs, q, status);
  else if (p.T <= 2)
    launch_pdl(route_gemv_kernel<2>, grid, dim3(256), 0, s, hidden, router_w, bias, p.T, p.d, p.E,
               k, k_per_token, p.k_max, logits, ids, w, xq, xs, q, status);
  else if (p.T <= 4)
    launch_pdl(route_gemv_kernel<4>, grid, dim3(256), 0, s, hidden, router_w, bias, p.T, p.d, p.E,
               k, k_per_token, p.k_max, logits, ids, w, xq, xs, q, status);
  else
    launch_pdl(route_gemv_kernel<8>, grid, dim3(256), 0, s, hidden, router_w, bias, p.T, p.d, p.E,
               k, k_per_token, p.k_max, logits, ids, w, xq, xs, q, status);
  return cudaGetLastError();
}

cudaError_t launch_router_logits(const Plan& p, const uint16_t* hidden, const float* router_w,
                                 float* part, cudaStream_t s) {
  dim3 grid((p.T + kRouterTile - 1) / kRouterTile, (p.E + kRouterTile - 1) / kRouterTile,
            p.r_splits);
  launch_pdl(router_logits_kernel, dim3(grid), dim3(256), 0, s, hidden, router_w, p.T, p.d, p.E,
                                            p.r_chunks_per_split, part);
  return cudaGetLastError();
}

cudaError_t launch_topk_quant(const Plan& p, const float* part, const float* bias, int k,
                              const int32_t* k_per_token, int32_t* ids, float* w,
                              const uint16_t* hidden, uint8_t* xq, float* xs, bool do_route,
                              bool do_quant, const float* refine_w, int* status, cudaStream_t s) {
  launch_pdl(topk_quant_kernel, dim3(p.T), dim3(128), 0, s, part, p.r_splits, bias, p.T, p.E, k, k_per_token,
                                        p.k_max, ids, w, hidden, p.d, xq, xs, do_route ? 1 : 0,
                                        do_quant ? 1 : 0, refine_w, status);
  return cudaGetLastError();
}

}  // namespace moe
