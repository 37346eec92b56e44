// Router of the MoE layer: logits on CUDA cores (fp32 FMA, deterministic split over the hidden
// dimension), then per token a warp-level softmax / top-k with renormalised weights, fused with
// the token's dynamic FP8 e4m3 quantisation (scale = amax / 448).
//
// Method: "Routage MoE entre GPU" (viite.ai) -- the router scores all experts from the hidden
// state, keeps the top-k and emits one routing weight per selection; the megakernel page
// (seventnews.com), W8A8 paragraph -- 8-bit FP8 activations.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

// part[s][t][e] = sum over the d-chunks of split s of x[t, d] * W[e, d], fp32, d ascending.
// Block: 256 threads computing a 32-token x 32-expert tile; thread (ty, tx) owns tokens
// 4*ty .. 4*ty+3 of expert tx.
__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t* __restrict__ x,
                                                            const float* __restrict__ W, int T,
                                                            int d, int E, int chunks_per_split,
                                                            float* __restrict__ part) {
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
#pragma unroll 8
    for (int kk = 0; kk < kRouterTile; ++kk) {
      const float w = ws[tx][kk];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = fmaf(xs[4 * ty + i][kk], w, acc[i]);
    }
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
__global__ void __launch_bounds__(128) topk_quant_kernel(
    const float* __restrict__ part, int splits, const float* __restrict__ bias, int T, int E,
    int k, const int32_t* __restrict__ k_per_token, int k_max, int32_t* __restrict__ ids,
    float* __restrict__ wout, const uint16_t* __restrict__ x, int d, uint8_t* __restrict__ xq,
    float* __restrict__ xs, int do_route, int do_quant, int* status) {
  __shared__ float lg[kMaxExperts];
  __shared__ float red[4];
  const int t = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (do_route) {
    for (int e = tid; e < E; e += 128) {
      float v = 0.f;
      for (int s = 0; s < splits; ++s) v += part[((size_t)s * T + t) * E + e];
      if (bias) v += bias[e];
      lg[e] = v;
    }
    __syncthreads();
    if (warp == 0) {
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

cudaError_t launch_router_logits(const Plan& p, const uint16_t* hidden, const float* router_w,
                                 float* part, cudaStream_t s) {
  dim3 grid((p.T + kRouterTile - 1) / kRouterTile, (p.E + kRouterTile - 1) / kRouterTile,
            p.r_splits);
  router_logits_kernel<<<grid, 256, 0, s>>>(hidden, router_w, p.T, p.d, p.E,
                                            p.r_chunks_per_split, part);
  return cudaGetLastError();
}

cudaError_t launch_topk_quant(const Plan& p, const float* part, const float* bias, int k,
                              const int32_t* k_per_token, int32_t* ids, float* w,
                              const uint16_t* hidden, uint8_t* xq, float* xs, bool do_route,
                              bool do_quant, int* status, cudaStream_t s) {
  topk_quant_kernel<<<p.T, 128, 0, s>>>(part, p.r_splits, bias, p.T, p.E, k, k_per_token,
                                        p.k_max, ids, w, hidden, p.d, xq, xs, do_route ? 1 : 0,
                                        do_quant ? 1 : 0, status);
  return cudaGetLastError();
}

}  // namespace moe
