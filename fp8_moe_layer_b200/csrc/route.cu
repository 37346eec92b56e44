// Router of the MoE layer: logits, softmax / top-k with renormalised weights, and the token's
// dynamic FP8 e4m3 quantisation (scale = amax / 448). Four kernels, by shape:
//   route_block_kernel   E <= 32: one block per token does all of it;
//   route_gemv_kernel    decode batches (T <= 8, E > 32): a warp per expert, and the last block
//                        to finish selects, quantises, and (in moe_forward) groups and gathers;
//   router_logits_kernel fp64 CUDA-core logits (64 x 64 register-blocked tiles, deterministic
//   + topk_quant_kernel  split over the hidden dimension), then per token the top-k (a warp
//                        selection, or a block sort for k_t > 8) and the quantisation;
//   topk_quant_kernel    also after the tensor-core logits (router_mma.cu), refining the
//                        candidates' logits exactly before the selection.
//
// Method: "Routage MoE entre GPU" (viite.ai) -- the router scores all experts from the hidden
// state, keeps the top-k and emits one routing weight per selection; the megakernel page
// (seventnews.com), W8A8 paragraph -- 8-bit FP8 activations.
//
// Precision of the routing decision: a bf16 hidden value times an fp32 router weight is exact in
// fp64 (8 + 24 significand bits), so every logit that decides a selection is summed in fp64. The
// selection and the slot order then agree with an fp64 evaluation of the same dot products except
// where two logits lie within the fp64 summation error (~1e-12 at d = 7168) of each other. The
// tensor-core logits (router_mma.cu) are only a filter: the experts they leave in play are
// recomputed in fp64 before the selection. The weights exp(l_j - l_max) / sum are computed in fp64
// and rounded once to fp32.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

// Warp-wide selection of the kt largest of n values, descending, exact ties to the lower id:
// candidate slot c (c = lane, lane + 32, ...; n <= 1024) has value val(c) and id idf(c). Lane j < kt
// receives the j-th selected (value, id).
template <typename ValFn, typename IdFn>
__device__ __forceinline__ void warp_select_desc(int n, int kt, ValFn val, IdFn idf, double& sel_v,
                                                 int& sel_e) {
  const int lane = threadIdx.x & 31;
  uint32_t taken = 0;            // bit i: slot lane + 32 i already selected
  sel_v = 0.0;
  sel_e = -1;
  for (int j = 0; j < kt; ++j) {
    double bv = -INFINITY;
    int be = 0x7FFFFFFF, bslot = -1;
    for (int i = 0, c = lane; c < n; ++i, c += 32) {
      const double v = val(c);
      const int e = idf(c);
      if (!((taken >> i) & 1u) && (v > bv || (v == bv && e < be))) {
        bv = v;
        be = e;
        bslot = c;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      const int os = __shfl_xor_sync(0xffffffffu, bslot, off);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
        bslot = os;
      }
    }
    if (bslot >= 0 && (bslot & 31) == lane) taken |= 1u << (bslot >> 5);
    if (lane == j) {
      sel_v = bv;
      sel_e = be;
    }
  }
}

// Block-wide descending sort of n <= kMaxExperts (value, id) pairs (equal values: lower id
// first, the order warp_select_desc produces) into sv / si, bitonic over the next power of two
// (padding: -inf, id INT_MAX). For selections with a large k_t, where the warp selection's k_t
// dependent rounds are the kernel's critical path. Every thread of the block calls it.
template <typename ValFn, typename IdFn>
__device__ void block_sort_desc(int n, ValFn val, IdFn idf, double* sv, int* si) {
  int np = 1;
  while (np < n) np <<= 1;
  for (int i = threadIdx.x; i < np; i += blockDim.x) {
    sv[i] = i < n ? val(i) : -INFINITY;
    si[i] = i < n ? idf(i) : 0x7FFFFFFF;
  }
  __syncthreads();
  for (int k = 2; k <= np; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < np; i += blockDim.x) {
        const int q = i ^ j;
        if (q > i) {
          const double a = sv[i], b = sv[q];
          const int ia = si[i], ib = si[q];
          const bool a_first = a > b || (a == b && ia < ib);
          if (a_first != ((i & k) == 0)) {
            sv[i] = b;
            sv[q] = a;
            si[i] = ib;
            si[q] = ia;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Renormalised weights of the selection held by lanes j < kt (sel_v descending): fp64
// exp(l_j - l_max) / sum, rounded once to fp32; ids and weights of slots >= kt are -1 and 0.
__device__ __forceinline__ void warp_store_selection(double sel_v, int sel_e, int kt, int k_max,
                                                     int32_t* ids, float* wout) {
  const int lane = threadIdx.x & 31;
  const double lmax = __shfl_sync(0xffffffffu, sel_v, 0);
  const double z = lane < kt ? exp(sel_v - lmax) : 0.0;
  double zs = z;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, off);
  if (lane < k_max) {
    ids[lane] = lane < kt ? sel_e : -1;
    wout[lane] = lane < kt ? static_cast<float>(z / zs) : 0.f;
  }
}

// fp64 dot product of 8 bf16 values (packed in v) with 8 fp32 weights (a, b): each product is exact.
__device__ __forceinline__ double dot8_f64(const uint4 v, const float4 a, const float4 b) {
  double c = static_cast<double>(__uint_as_float(v.x << 16)) * a.x;
  c = fma(static_cast<double>(__uint_as_float(v.x & 0xFFFF0000u)), static_cast<double>(a.y), c);
  c = fma(static_cast<double>(__uint_as_float(v.y << 16)), static_cast<double>(a.z), c);
  c = fma(static_cast<double>(__uint_as_float(v.y & 0xFFFF0000u)), static_cast<double>(a.w), c);
  c = fma(static_cast<double>(__uint_as_float(v.z << 16)), static_cast<double>(b.x), c);
  c = fma(static_cast<double>(__uint_as_float(v.z & 0xFFFF0000u)), static_cast<double>(b.y), c);
  c = fma(static_cast<double>(__uint_as_float(v.w << 16)), static_cast<double>(b.z), c);
  c = fma(static_cast<double>(__uint_as_float(v.w & 0xFFFF0000u)), static_cast<double>(b.w), c);
  return c;
}

// Eight bf16 values (one 16-byte load) as fp64 (exact), in order.
__device__ __forceinline__ void bf16x8_to_f64(const uint4 v, double (&o)[8]) {
  const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    o[2 * q] = static_cast<double>(__uint_as_float(w4[q] << 16));
    o[2 * q + 1] = static_cast<double>(__uint_as_float(w4[q] & 0xFFFF0000u));
  }
}
// sum_j x[j] * w[j] for eight fp64 token values and eight fp32 weights, in the order of dot8_f64.
__device__ __forceinline__ double dot8_xw(const double (&x)[8], const float4 a, const float4 b) {
  double c = x[0] * static_cast<double>(a.x);
  c = fma(x[1], static_cast<double>(a.y), c);
  c = fma(x[2], static_cast<double>(a.z), c);
  c = fma(x[3], static_cast<double>(a.w), c);
  c = fma(x[4], static_cast<double>(b.x), c);
  c = fma(x[5], static_cast<double>(b.y), c);
  c = fma(x[6], static_cast<double>(b.z), c);
  c = fma(x[7], static_cast<double>(b.w), c);
  return c;
}

// part[s][t][e] = sum over the d-chunks of split s of x[t, d] * W[e, d], fp64, d ascending.
// Block: 256 threads computing a 64-token x 64-expert tile; thread (ty, tx) = (tid / 16,
// tid % 16) owns tokens ty + 16 i and experts tx + 16 j (i, j < 4). d goes by chunks of 16: the
// next chunk's inputs are loaded into registers while the current one is multiplied from shared
// memory, where both tiles sit as fp64 (exact conversions, once per element and block), K-major
// and double-buffered. Per chunk step a thread reads 4 token and 4 weight values for 16 fma.
__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t* __restrict__ x,
                                                            const float* __restrict__ W, int T,
                                                            int d, int E, int chunks_per_split,
                                                            double* __restrict__ part) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  __shared__ __align__(16) double xs[2][kRtK][kRtTok];
  __shared__ __align__(16) double ws[2][kRtK][kRtExp];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int t0 = blockIdx.x * kRtTok, e0 = blockIdx.y * kRtExp;
  const int split = blockIdx.z;
  const int nchunks = d / kRtK;
  const int c_begin = split * chunks_per_split;
  const int c_end = min(nchunks, c_begin + chunks_per_split);
  // loader: row lr (token / expert of the tile) and 4 consecutive d of the chunk
  const int lr = tid >> 2, lk = 4 * (tid & 3);
  const bool tok_ok = t0 + lr < T, exp_ok = e0 + lr < E;
  const uint16_t* xrow = x + (size_t)(tok_ok ? t0 + lr : 0) * d + lk;
  const float* wrow = W + (size_t)(exp_ok ? e0 + lr : 0) * d + lk;
  uint2 xv = make_uint2(0u, 0u);
  float4 wv = make_float4(0.f, 0.f, 0.f, 0.f);
  auto fetch = [&](int c) {
    if (tok_ok) xv = *reinterpret_cast<const uint2*>(xrow + (size_t)c * kRtK);
    if (exp_ok) wv = *reinterpret_cast<const float4*>(wrow + (size_t)c * kRtK);
  };
  auto park = [&](int buf) {
    xs[buf][lk + 0][lr] = static_cast<double>(__uint_as_float(xv.x << 16));
    xs[buf][lk + 1][lr] = static_cast<double>(__uint_as_float(xv.x & 0xFFFF0000u));
    xs[buf][lk + 2][lr] = static_cast<double>(__uint_as_float(xv.y << 16));
    xs[buf][lk + 3][lr] = static_cast<double>(__uint_as_float(xv.y & 0xFFFF0000u));
    ws[buf][lk + 0][lr] = static_cast<double>(wv.x);
    ws[buf][lk + 1][lr] = static_cast<double>(wv.y);
    ws[buf][lk + 2][lr] = static_cast<double>(wv.z);
    ws[buf][lk + 3][lr] = static_cast<double>(wv.w);
  };
  double acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
  if (c_begin < c_end) {
    fetch(c_begin);
    park(0);
    __syncthreads();
    for (int c = c_begin; c < c_end; ++c) {
      const int buf = (c - c_begin) & 1;
      if (c + 1 < c_end) fetch(c + 1);
#pragma unroll
      for (int kk = 0; kk < kRtK; ++kk) {
        double xa[4], wb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) xa[i] = xs[buf][kk][ty + 16 * i];
#pragma unroll
        for (int j = 0; j < 4; ++j) wb[j] = ws[buf][kk][tx + 16 * j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fma(xa[i], wb[j], acc[i][j]);
      }
      if (c + 1 < c_end) park(buf ^ 1);
      __syncthreads();
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty + 16 * i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx + 16 * j;
      if (e < E) part[((size_t)split * T + t) * E + e] = acc[i][j];
    }
  }
}

// One block (128 threads) per token.
//  route: l[e] = sum_s part[s][t][e] + bias[e] (fp64, splits in fixed order); the k_t largest
//         (descending, exact ties to the lower expert id) and their renormalised weights
//         exp(l_j - l_max) / sum_sel exp(l_sel - l_max), which equal the softmax over all E
//         renormalised over the selection.
//  quant: s_t = amax|x[t,:]| / 448 (IEEE fp32 division; 1 if amax = 0);
//         xq = e4m3_rne_satfinite(x / s_t) (IEEE fp32 division).
//  refine (refine_w != null, for the tensor-core logits): the approximate logits only pick the
//         candidates -- every expert within kRefineWindow of the approximate k_t-th largest, which
//         contains the exact top-k_t while the approximation error stays below half the window --
//         and each candidate's logit is recomputed in fp64 before the selection and the weights
//         (a warp takes two candidates, so each token value is converted once for both).
constexpr double kRefineWindow = 1e-2;
constexpr int kMaxCandidates = 256;

__global__ void __launch_bounds__(128) topk_quant_kernel(
    const double* __restrict__ part, int splits, const float* __restrict__ bias, int T, int E,
    int k, const int32_t* __restrict__ k_per_token, int k_max, int32_t* __restrict__ ids,
    float* __restrict__ wout, const uint16_t* __restrict__ x, int d, uint8_t* __restrict__ xq,
    float* __restrict__ xs, int do_route, int do_quant, const float* __restrict__ refine_w,
    int* status) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  __shared__ double lg[kMaxExperts];
  __shared__ float red[4];
  __shared__ int cand[kMaxCandidates];
  __shared__ double sort_v[kMaxExperts];
  __shared__ int sort_i[kMaxExperts];
  __shared__ int ncand;
  __shared__ double vk_s;
  const int t = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (do_route) {
    for (int e = tid; e < E; e += 128) {
      // split partials in fixed order: eight independent accumulators keep eight loads in
      // flight (a decode batch splits d finely, and these loads are the kernel's latency)
      double a8[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
      int s = 0;
      for (; s + 8 <= splits; s += 8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) a8[u] += part[((size_t)(s + u) * T + t) * E + e];
      }
      for (int u = 0; s < splits; ++s, ++u) a8[u] += part[((size_t)s * T + t) * E + e];
      double v = ((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]));
      if (bias) v += static_cast<double>(bias[e]);
      lg[e] = v;
    }
    __syncthreads();
    int kt = k_per_token ? k_per_token[t] : k;
    const int kcap = min(E, k_max);
    if (kt < 1 || kt > kcap) {
      if (tid == 0) report(status, kStatusDeviceCheck, kWhereRoute, t);
      kt = max(1, min(kt, kcap));
    }
    bool by_cand = false;          // exact selection over the refined candidates only
    // large k_t: a block-wide sort instead of k_t rounds of the warp selection
    const bool sort_all = kt > 8 && E > 64;
    if (refine_w) {
      if (sort_all) {
        block_sort_desc(E, [&](int c) { return lg[c]; }, [](int c) { return c; }, sort_v, sort_i);
        if (tid == 0) {
          vk_s = sort_v[kt - 1];                                   // approximate k_t-th largest
          ncand = 0;
        }
      } else if (warp == 0) {
        double sv;
        int se;
        warp_select_desc(E, kt, [&](int c) { return lg[c]; }, [](int c) { return c; }, sv, se);
        const double vk = __shfl_sync(0xffffffffu, sv, kt - 1);   // approximate k_t-th largest
        if (lane == 0) {
          vk_s = vk;
          ncand = 0;
        }
      }
      __syncthreads();
      const double floor_v = vk_s - kRefineWindow;
      for (int e = tid; e < E; e += 128) {
        if (lg[e] >= floor_v) {
          const int c = atomicAdd(&ncand, 1);
          if (c < kMaxCandidates) cand[c] = e;
        }
      }
      __syncthreads();
      const bool all = ncand > kMaxCandidates;          // pathological: recompute every expert
      const int nc = all ? E : ncand;
      const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * d);
      const int nv = d / 8;
      for (int c0 = 2 * warp; c0 < nc; c0 += 8) {
        const bool two = c0 + 1 < nc;
        const int e0 = all ? c0 : cand[c0];
        const int e1 = two ? (all ? c0 + 1 : cand[c0 + 1]) : e0;
        const float4* w0 = reinterpret_cast<const float4*>(refine_w + (size_t)e0 * d);
        const float4* w1 = reinterpret_cast<const float4*>(refine_w + (size_t)e1 * d);
        double acc0 = 0.0, acc1 = 0.0;
#pragma unroll 2
        for (int i = lane; i < nv; i += 32) {
          double xv[8];
          bf16x8_to_f64(xr[i], xv);
          acc0 += dot8_xw(xv, __ldg(w0 + 2 * i), __ldg(w0 + 2 * i + 1));
          if (two) acc1 += dot8_xw(xv, __ldg(w1 + 2 * i), __ldg(w1 + 2 * i + 1));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          acc0 += __shfl_xor_sync(0xffffffffu, acc0, off);
          acc1 += __shfl_xor_sync(0xffffffffu, acc1, off);
        }
        if (lane == 0) {
          lg[e0] = acc0 + (bias ? static_cast<double>(bias[e0]) : 0.0);
          if (two) lg[e1] = acc1 + (bias ? static_cast<double>(bias[e1]) : 0.0);
        }
      }
      __syncthreads();
      by_cand = !all;
    }
    const int nsel = by_cand ? ncand : E;
    if (kt > 8 && nsel > 64) {
      if (by_cand)
        block_sort_desc(ncand, [&](int c) { return lg[cand[c]]; }, [&](int c) { return cand[c]; },
                        sort_v, sort_i);
      else
        block_sort_desc(E, [&](int c) { return lg[c]; }, [](int c) { return c; }, sort_v, sort_i);
      if (warp == 0) {
        const double sv = lane < kt ? sort_v[lane] : 0.0;
        const int se = lane < kt ? sort_i[lane] : -1;
        warp_store_selection(sv, se, kt, k_max, ids + (size_t)t * k_max, wout + (size_t)t * k_max);
      }
    } else if (warp == 0) {
      double sv;
      int se;
      if (by_cand)
        warp_select_desc(ncand, kt, [&](int c) { return lg[cand[c]]; },
                         [&](int c) { return cand[c]; }, sv, se);
      else
        warp_select_desc(E, kt, [&](int c) { return lg[c]; }, [](int c) { return c; }, sv, se);
      warp_store_selection(sv, se, kt, k_max, ids + (size_t)t * k_max, wout + (size_t)t * k_max);
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

// Decode router (T <= 8 tokens, E > 32): one warp per expert computes that expert's fp64 logit
// for every token (lane-strided chunks of 8 along d, then a butterfly; all loads in flight),
// writes it to `logits` [T][E], and the last block to finish (a counter in the status word,
// status[3]) selects the top-k and the weights of every token, groups the routed pairs by expert
// (when given a DecodeGrouping), quantises every token to FP8 -- writing the codes to the token
// rows and straight to the token's routed rows of the gathered copy -- then resets the counter.
// One kernel instead of the logits, top-k, grouping and gather kernels. Dynamic shared memory:
// T * E doubles (the last block's copy of the logits, reused by the grouping).
constexpr int kGemvMaxT = 8;

// Exclusive prefix sum over the 256 threads of a block (tmp: 9 ints of shared memory); returns
// this thread's exclusive prefix and the block total in `total`.
__device__ __forceinline__ int block_exscan256(int v, int* tmp, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) tmp[warp] = incl;
  __syncthreads();
  if (threadIdx.x == 0) {
    int s = 0;
    for (int w = 0; w < 8; ++w) {
      const int c = tmp[w];
      tmp[w] = s;
      s += c;
    }
    tmp[8] = s;
  }
  __syncthreads();
  const int r = tmp[warp] + incl - v;
  total = tmp[8];
  __syncthreads();
  return r;
}

template <int TT>
__global__ void __launch_bounds__(256) route_gemv_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ W, const float* __restrict__ bias,
    int T, int d, int E, int k, const int32_t* __restrict__ k_per_token, int k_max,
    double* __restrict__ logits, int32_t* __restrict__ ids, float* __restrict__ wout,
    uint8_t* __restrict__ xq, float* __restrict__ xs, int do_quant, int* status,
    const DecodeGrouping grp) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  __shared__ int s_last;
  extern __shared__ double lgd[];                 // [T][E], used by the last block only
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int e = blockIdx.x * 8 + warp;
  const int nv = d / 8;
  if (e < E) {
    double acc[TT];
#pragma unroll
    for (int j = 0; j < TT; ++j) acc[j] = 0.0;
    const float4* wr = reinterpret_cast<const float4*>(W + (size_t)e * d);
#pragma unroll 4
    for (int i = lane; i < nv; i += 32) {
      const float4 a = __ldg(wr + 2 * i), b = __ldg(wr + 2 * i + 1);
#pragma unroll
      for (int j = 0; j < TT; ++j)
        if (j < T) acc[j] += dot8_f64(reinterpret_cast<const uint4*>(x + (size_t)j * d)[i], a, b);
    }
#pragma unroll
    for (int j = 0; j < TT; ++j) {
      if (j < T) {
        double v = acc[j];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) logits[(size_t)j * E + e] = v + (bias ? static_cast<double>(bias[e]) : 0.0);
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
  // the selection, kept in shared memory for the grouping and the gather (-1: unused slot)
  __shared__ int s_ids[kGemvMaxT * kMaxK];
  __shared__ int s_inv[kGemvMaxT * kMaxK];
  __shared__ int s_kt[kGemvMaxT];
  __shared__ int s_R;
  if (warp < T) {
    const int t = warp;
    double* my = lgd + (size_t)t * E;
    for (int ee = lane; ee < E; ee += 32) my[ee] = __ldcg(logits + (size_t)t * E + ee);
    __syncwarp();
    int kt = k_per_token ? k_per_token[t] : k;
    const int kcap = min(E, k_max);
    if (kt < 1 || kt > kcap) {
      if (lane == 0) report(status, kStatusDeviceCheck, kWhereRoute, t);
      kt = max(1, min(kt, kcap));
    }
    double sv;
    int se;
    warp_select_desc(E, kt, [&](int c) { return my[c]; }, [](int c) { return c; }, sv, se);
    warp_store_selection(sv, se, kt, k_max, ids + (size_t)t * k_max, wout + (size_t)t * k_max);
    if (lane < k_max) s_ids[t * k_max + lane] = lane < kt ? se : -1;
    if (lane == 0) s_kt[t] = kt;
  }
  __syncthreads();                                     // the selection of every token
  if (grp.offsets) {
    // The grouping of the (at most 8 x 32) routed pairs, by this block: expert counts, their
    // exclusive prefix (offsets), each pair's row = offset + its rank among the earlier pairs of
    // the same expert (token-major order: stable), and the GEMM tile prefix. Same result as the
    // grouping kernels (permute.cu); it also zeroes the rows' SwiGLU maxima.
    __shared__ int tmp[9];
    int* cnt = reinterpret_cast<int*>(lgd);            // [E] (the logit copies are done with)
    int* off = cnt + E;                                // [E]
    for (int e = tid; e < E; e += 256) cnt[e] = 0;
    __syncthreads();
    const int npairs = T * k_max;                      // <= 8 * 32 = 256 = blockDim
    int my_e = -1;
    if (tid < npairs) {
      const int e = s_ids[tid];
      if (e >= 0 && e < E) {
        my_e = e;
        atomicAdd(&cnt[e], 1);
      }
    }
    __syncthreads();
    const int per = (E + 255) / 256;
    const int e_lo = min(E, tid * per), e_hi = min(E, e_lo + per);
    int seg = 0, seg_tiles = 0;
    for (int e = e_lo; e < e_hi; ++e) {
      seg += cnt[e];
      seg_tiles += (cnt[e] + grp.BN - 1) / grp.BN;
    }
    int R = 0, total_tiles = 0;
    int base = block_exscan256(seg, tmp, R);
    int tbase = block_exscan256(seg_tiles, tmp, total_tiles);
    for (int e = e_lo; e < e_hi; ++e) {
      off[e] = base;
      grp.offsets[e] = base;
      grp.tiles[e] = tbase;
      base += cnt[e];
      tbase += (cnt[e] + grp.BN - 1) / grp.BN;
    }
    __syncthreads();
    if (tid < npairs) {
      int row = -1;
      if (my_e >= 0) {
        int rank = 0;
        for (int i = 0; i < tid; ++i) rank += s_ids[i] == my_e ? 1 : 0;
        row = off[my_e] + rank;
        grp.perm[row] = tid / k_max;
        grp.amax[row] = 0u;
      }
      grp.inv[tid] = row;
      s_inv[tid] = row;
    }
    if (tid == 0) {
      s_R = R;
      grp.offsets[E] = R;
      grp.tiles[E] = total_tiles;
      if (grp.has_shared) {
        grp.offsets[E + 1] = R + T;
        grp.tiles[E + 1] = total_tiles + (T + grp.BN - 1) / grp.BN;
      }
    }
    if (grp.has_shared && tid < T) {
      grp.perm[R + tid] = tid;
      grp.amax[R + tid] = 0u;
    }
    __syncthreads();                                   // s_inv, s_R
  }
  if (do_quant) {
    // The FP8 quantisation of each token by the whole block: the row maxima of all tokens in one
    // pass (every token's loads in flight), then the codes, written to the token's row of xq
    // and, with the grouping, straight to its routed rows (and shared-expert row) of the
    // gathered copy, with their scales.
    __shared__ float s_am[8][kGemvMaxT];
    float am[TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) am[t] = 0.f;
    for (int i = tid; i < nv; i += 256) {
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        if (t < T) {
          const uint4 v = reinterpret_cast<const uint4*>(x + (size_t)t * d)[i];
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            am[t] = fmaxf(am[t], fabsf(__uint_as_float(w4[q] << 16)));
            am[t] = fmaxf(am[t], fabsf(__uint_as_float(w4[q] & 0xFFFF0000u)));
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < TT; ++t) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        am[t] = fmaxf(am[t], __shfl_xor_sync(0xffffffffu, am[t], off));
      if (lane == 0 && t < T) s_am[warp][t] = am[t];
    }
    __syncthreads();
    const bool gather = grp.offsets && grp.xqp;
    for (int t = 0; t < T; ++t) {
      float amx = s_am[0][t];
#pragma unroll
      for (int w = 1; w < 8; ++w) amx = fmaxf(amx, s_am[w][t]);
      const float sc = amx > 0.f ? __fdiv_rn(amx, 448.f) : 1.f;
      const int kt = s_kt[t];
      if (tid == 0) {
        xs[t] = sc;
        if (gather) {
          for (int j = 0; j < kt; ++j) {
            const int r = s_inv[t * k_max + j];
            if (r >= 0) grp.xsp[r] = sc;
          }
          if (grp.has_shared) grp.xsp[s_R + t] = sc;
        }
      }
      const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * d);
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
        const uint2 pk = make_uint2(packed[0], packed[1]);
        reinterpret_cast<uint2*>(xq + (size_t)t * d)[i] = pk;
        if (gather) {
          for (int j = 0; j < kt; ++j) {
            const int r = s_inv[t * k_max + j];
            if (r >= 0) reinterpret_cast<uint2*>(grp.xqp + (size_t)r * d)[i] = pk;
          }
          if (grp.has_shared) reinterpret_cast<uint2*>(grp.xqp + (size_t)(s_R + t) * d)[i] = pk;
        }
      }
    }
  }
  if (tid == 0) status[3] = 0;             // the counter is ready for the next launch
}

// Small-E router (E <= 32), one 256-thread block per token, fully fused: logits, top-k, weights
// and the token's FP8 quantisation. Thread i accumulates x[t, 8c..8c+7] . W[e, 8c..8c+7] for the
// chunks c = i, i + 256, ... in fp64, a butterfly inside each warp and a fixed-order sum over the
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
  __shared__ double part[8][EP];
  __shared__ float red[8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t = blockIdx.x;
  const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  const int nv = d / 8;
  double acc[EP];
#pragma unroll
  for (int e = 0; e < EP; ++e) acc[e] = 0.0;
  uint4 xv[kChunks];
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    const int i = tid + 256 * c;
    if (i < nv) {
      xv[c] = xr[i];
      const uint32_t w4[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
        amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w4[q] << 16)),
                                 fabsf(__uint_as_float(w4[q] & 0xFFFF0000u))));
#pragma unroll
      for (int e = 0; e < EP; ++e) {
        if (e < E) {
          const float4* wr = reinterpret_cast<const float4*>(W + (size_t)e * d) + 2 * i;
          acc[e] += dot8_f64(xv[c], __ldg(wr), __ldg(wr + 1));
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EP; ++e) {
    double v = acc[e];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) part[warp][e] = v;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if (lane == 0) red[warp] = amax;
  __syncthreads();

  if (warp == 0) {
    double logit = -INFINITY;
    if (lane < E) {
      double v = 0.0;
#pragma unroll
      for (int w = 0; w < 8; ++w) v += part[w][lane < EP ? lane : 0];
      logit = v + (bias ? static_cast<double>(bias[lane]) : 0.0);
    }
    // top-k over the lanes (lane e holds expert e), exact ties to the lower id
    int kt = k_per_token ? k_per_token[t] : k;
    const int kcap = min(E, k_max);
    if (kt < 1 || kt > kcap) {
      if (lane == 0) report(status, kStatusDeviceCheck, kWhereRoute, t);
      kt = max(1, min(kt, kcap));
    }
    double sv;
    int se;
    warp_select_desc(E, kt, [&](int) { return logit; }, [](int c) { return c; }, sv, se);
    warp_store_selection(sv, se, kt, k_max, ids + (size_t)t * k_max, wout + (size_t)t * k_max);
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

// Sets a kernel's dynamic shared-memory limit once per device (the first launch there).
template <typename K>
static cudaError_t allow_dynamic_smem(K kernel, int bytes, bool (&done)[64]) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev >= 64) return cudaErrorInvalidDevice;
  if (!done[dev]) {
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (err != cudaSuccess) return err;
    done[dev] = true;
  }
  return cudaSuccess;
}

template <int TT>
static cudaError_t launch_gemv_t(const Plan& p, const uint16_t* hidden, const float* router_w,
                                 const float* bias, int k, const int32_t* k_per_token,
                                 double* logits, int32_t* ids, float* w, uint8_t* xq, float* xs,
                                 int q, int* status, const DecodeGrouping& grp, cudaStream_t s) {
  static bool done[64] = {};
  cudaError_t err = allow_dynamic_smem(route_gemv_kernel<TT>, kGemvMaxT * kMaxExperts * 8, done);
  if (err != cudaSuccess) return err;
  // the logit copies of the last block; the grouping reuses it for two ints per expert
  const size_t smem = std::max(sizeof(double) * (size_t)p.T * p.E, sizeof(int) * 2 * (size_t)p.E);
  launch_pdl(route_gemv_kernel<TT>, dim3((p.E + 7) / 8), dim3(256), smem, s, hidden, router_w,
             bias, p.T, p.d, p.E, k, k_per_token, p.k_max, logits, ids, w, xq, xs, q, status, grp);
  return cudaGetLastError();
}

cudaError_t launch_route_gemv(const Plan& p, const uint16_t* hidden, const float* router_w,
                              const float* bias, int k, const int32_t* k_per_token,
                              double* logits, int32_t* ids, float* w, uint8_t* xq, float* xs,
                              bool do_quant, int* status, const DecodeGrouping& grp,
                              cudaStream_t s) {
  const int q = do_quant ? 1 : 0;
  if (p.T <= 1)
    return launch_gemv_t<1>(p, hidden, router_w, bias, k, k_per_token, logits, ids, w, xq, xs, q,
                            status, grp, s);
  if (p.T <= 2)
    return launch_gemv_t<2>(p, hidden, router_w, bias, k, k_per_token, logits, ids, w, xq, xs, q,
                            status, grp, s);
  if (p.T <= 4)
    return launch_gemv_t<4>(p, hidden, router_w, bias, k, k_per_token, logits, ids, w, xq, xs, q,
                            status, grp, s);
  return launch_gemv_t<8>(p, hidden, router_w, bias, k, k_per_token, logits, ids, w, xq, xs, q,
                          status, grp, s);
}

cudaError_t launch_router_logits(const Plan& p, const uint16_t* hidden, const float* router_w,
                                 double* part, cudaStream_t s) {
  dim3 grid((p.T + kRtTok - 1) / kRtTok, (p.E + kRtExp - 1) / kRtExp, p.r_splits);
  launch_pdl(router_logits_kernel, dim3(grid), dim3(256), 0, s, hidden, router_w, p.T, p.d, p.E,
                                            p.r_chunks_per_split, part);
  return cudaGetLastError();
}

cudaError_t launch_topk_quant(const Plan& p, const double* part, const float* bias, int k,
                              const int32_t* k_per_token, int32_t* ids, float* w,
                              const uint16_t* hidden, uint8_t* xq, float* xs, bool do_route,
                              bool do_quant, const float* refine_w, int* status, cudaStream_t s) {
  launch_pdl(topk_quant_kernel, dim3(p.T), dim3(128), 0, s, part, p.r_splits, bias, p.T, p.E, k,
             k_per_token, p.k_max, ids, w, hidden, p.d, xq, xs, do_route ? 1 : 0,
             do_quant ? 1 : 0, refine_w, status);
  return cudaGetLastError();
}

}  // namespace moe
