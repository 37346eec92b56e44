// Row-wise kernels between and after the grouped GEMMs: the FP8 requantisation of the SwiGLU
// intermediate (per routed row, over all F), the routing-weighted combine that restores token
// order, and the reduction of K-split partials for the split entry point. All are HBM-bound:
// 128-bit loads/stores, one block (or warp) per row, grids sized in multiples of the SM count.
//
// Method: megakernel page (seventnews.com), W8A8 paragraph -- FP8 activations, here also for the
// expert intermediate; "Routage MoE entre GPU" (viite.ai) -- outputs weighted by their routing
// weights, summed, and put back in the original token order.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

// s2[r] = amax[r] / 448 (IEEE fp32; 1 if 0); aq[r, f] = e4m3_rne_satfinite(act[r, f] / s2[r]).
// The row max is already complete (from the gate/up epilogue), so every 16-element chunk of every
// row is independent: thread (x, y) of a (chunks x rows) block takes chunk blockIdx.y * blockDim.x
// + x of rows blockIdx.x * blockDim.y + y, stepping by gridDim.x * blockDim.y (short rows fill the
// block with several rows); four 16-byte loads in flight per thread and one 16-byte store, no
// thread divides its index.
__global__ void __launch_bounds__(256) requant_kernel(const float* __restrict__ act,
                                                      const uint32_t* __restrict__ amax,
                                                      const int32_t* __restrict__ total_rows,
                                                      int64_t rcap, int F,
                                                      uint8_t* __restrict__ aq,
                                                      float* __restrict__ s2) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  const int R = (int)min((int64_t)max(*total_rows, 0), rcap);
  const int n16 = F / 16;
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  if (c >= n16) return;
#pragma unroll 2
  for (int r = blockIdx.x * blockDim.y + threadIdx.y; r < R; r += gridDim.x * blockDim.y) {
    const float am = __uint_as_float(amax[r]);
    const float sc = am > 0.f ? __fdiv_rn(am, 448.f) : 1.f;
    if (c == 0) s2[r] = sc;
    const float4* src = reinterpret_cast<const float4*>(act + (size_t)r * F) + 4 * c;
    const float4 v[4] = {src[0], src[1], src[2], src[3]};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      o[q] = static_cast<uint32_t>(e4m3x2(__fdiv_rn(v[q].x, sc), __fdiv_rn(v[q].y, sc))) |
             (static_cast<uint32_t>(e4m3x2(__fdiv_rn(v[q].z, sc), __fdiv_rn(v[q].w, sc))) << 16);
    reinterpret_cast<uint4*>(aq + (size_t)r * F)[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// K-split gate/up: per routed row, gate[f] = sum_s h[s][r][f], up[f] = sum_s h[s][r][F + f]
// (split order fixed), act = silu(gate) * up, s2 = amax|act| / 448 (IEEE fp32; 1 if 0),
// aq = e4m3(act / s2). One block (up to 1024 threads) per row; act is recomputed in the second
// pass instead of stored.
__global__ void __launch_bounds__(1024) swiglu_requant_kernel(
    const float* __restrict__ h, int splits, size_t split_stride,
    const int32_t* __restrict__ total_rows, int64_t rcap, int F, uint8_t* __restrict__ aq,
    float* __restrict__ s2) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  __shared__ float red[32];
  const int R = (int)min((int64_t)max(*total_rows, 0), rcap);
  const int nv = F / 4;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int r = blockIdx.x; r < R; r += gridDim.x) {
    auto act4 = [&](int i) {
      const float4* g4 = reinterpret_cast<const float4*>(h + (size_t)r * 2 * F);
      const float4* u4 = reinterpret_cast<const float4*>(h + (size_t)r * 2 * F + F);
      float4 g = g4[i], u = u4[i];
      for (int sp = 1; sp < splits; ++sp) {
        const float4 gs = reinterpret_cast<const float4*>(h + sp * split_stride + (size_t)r * 2 * F)[i];
        const float4 us = reinterpret_cast<const float4*>(h + sp * split_stride + (size_t)r * 2 * F + F)[i];
        g.x += gs.x; g.y += gs.y; g.z += gs.z; g.w += gs.w;
        u.x += us.x; u.y += us.y; u.z += us.z; u.w += us.w;
      }
      return make_float4(silu(g.x) * u.x, silu(g.y) * u.y, silu(g.z) * u.z, silu(g.w) * u.w);
    };
    float amax = 0.f;
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
      const float4 a = act4(i);
      amax = fmaxf(fmaxf(amax, fmaxf(fabsf(a.x), fabsf(a.y))), fmaxf(fabsf(a.z), fabsf(a.w)));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    float am = red[0];
    for (int w = 1; w < nwarps; ++w) am = fmaxf(am, red[w]);
    const float sc = am > 0.f ? __fdiv_rn(am, 448.f) : 1.f;
    if (threadIdx.x == 0) s2[r] = sc;
    uint32_t* dst = reinterpret_cast<uint32_t*>(aq + (size_t)r * F);
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
      const float4 v = act4(i);
      dst[i] = static_cast<uint32_t>(e4m3x2(__fdiv_rn(v.x, sc), __fdiv_rn(v.y, sc))) |
               (static_cast<uint32_t>(e4m3x2(__fdiv_rn(v.z, sc), __fdiv_rn(v.w, sc))) << 16);
    }
    __syncthreads();                                   // red[] is reused by the next row
  }
}

// Eight consecutive fp32 values of row r (K-split partials summed in split order).
__device__ __forceinline__ void load8_rows(const float* o, int splits, size_t split_stride,
                                           int64_t r, int d, int i, float (&v)[8]) {
  const float4* p = reinterpret_cast<const float4*>(o + (size_t)r * d) + 2 * i;
  float4 a = p[0], b = p[1];
  for (int s = 1; s < splits; ++s) {
    const float4* q = reinterpret_cast<const float4*>(o + s * split_stride + (size_t)r * d) + 2 * i;
    const float4 c = q[0], e = q[1];
    a.x += c.x; a.y += c.y; a.z += c.z; a.w += c.w;
    b.x += e.x; b.y += e.y; b.z += e.z; b.w += e.w;
  }
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
// y[t, :] = bf16_rne( sum_j w[t, j] * (sum_s o[s][inv[t, j], :]) + sum_s shared[s][row0 + t, :] )
// Slots with inv < 0 are skipped; fp32, slot order and split order fixed (deterministic). A
// thread takes 8 channels: two 16-byte loads per expert row, one 16-byte bf16 store.
__global__ void __launch_bounds__(256) combine_kernel(
    const float* __restrict__ o, int splits, size_t split_stride, const float* __restrict__ topk_w,
    const int32_t* __restrict__ inv_row, int k_max, int64_t rcap,
    const float* __restrict__ shared_src, const int32_t* __restrict__ shared_row0,
    int shared_splits, size_t shared_split_stride, int T, int d, uint16_t* __restrict__ y,
    float* __restrict__ y_f32, int* status) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  __shared__ int rows[kMaxK];
  __shared__ float wts[kMaxK];
  const int nv = d / 8;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();
    if (threadIdx.x < k_max) {
      int r = inv_row[(size_t)t * k_max + threadIdx.x];
      if (r >= rcap) {
        report(status, kStatusDeviceCheck, kWhereCombine, t);
        r = -1;
      }
      rows[threadIdx.x] = r;
      wts[threadIdx.x] = topk_w[(size_t)t * k_max + threadIdx.x];
    }
    __syncthreads();
    const int64_t srow = shared_src ? (int64_t)(shared_row0 ? *shared_row0 : 0) + t : -1;
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int j = 0; j < k_max; ++j) {
        const int r = rows[j];
        if (r < 0) continue;
        float v[8];
        load8_rows(o, splits, split_stride, r, d, i, v);
        const float w = wts[j];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = fmaf(w, v[c], acc[c]);
      }
      if (srow >= 0) {
        float v[8];
        load8_rows(shared_src, shared_splits, shared_split_stride, srow, d, i, v);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] += v[c];
      }
      uint32_t pk[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        pk[q] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * q]))) |
                (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * q + 1])))
                 << 16);
      reinterpret_cast<uint4*>(y + (size_t)t * d)[i] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      if (y_f32) {
        float4* yf = reinterpret_cast<float4*>(y_f32 + (size_t)t * d) + 2 * i;
        yf[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        yf[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      }
    }
  }
}

// out[r, :] = sum_s o[s][r, :] for r < R (split entry point with a K-split down GEMM).
__global__ void __launch_bounds__(256) reduce_splits_kernel(const float* __restrict__ o, int splits,
                                                            size_t split_stride,
                                                            const int32_t* __restrict__ total_rows,
                                                            int64_t rcap, int d,
                                                            float* __restrict__ out) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  const int R = (int)min((int64_t)max(*total_rows, 0), rcap);
  const int nv = d / 4;
  for (int r = blockIdx.x; r < R; r += gridDim.x) {
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
      float4 v = reinterpret_cast<const float4*>(o + (size_t)r * d)[i];
      for (int s = 1; s < splits; ++s) {
        const float4 u = reinterpret_cast<const float4*>(o + s * split_stride + (size_t)r * d)[i];
        v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
      }
      reinterpret_cast<float4*>(out + (size_t)r * d)[i] = v;
    }
  }
}

static int row_grid(int64_t rows) {
  return (int)std::min<int64_t>(std::max<int64_t>(rows, 1), 8LL * num_sms());
}

cudaError_t launch_requant(const Plan& p, const float* act, const uint32_t* amax,
                           const int32_t* total_rows, uint8_t* aq, float* s2, cudaStream_t s) {
  const int n16 = p.F / 16;
  const int bx = std::min(256, n16);                 // chunks of a row per block
  const int by = std::max(1, 256 / bx);              // rows per block
  const int gy = (n16 + bx - 1) / bx;
  const int64_t row_blocks = (p.Rcap + by - 1) / by;
  const int gx = (int)std::min<int64_t>(std::max<int64_t>(row_blocks, 1),
                                        std::max<int64_t>(16LL * num_sms() / gy, 1));
  launch_pdl(requant_kernel, dim3(gx, gy), dim3(bx, by), 0, s, act, amax, total_rows, p.Rcap,
             p.F, aq, s2);
  return cudaGetLastError();
}

cudaError_t launch_swiglu_requant(const Plan& p, const float* h, int splits, size_t split_stride,
                                  const int32_t* total_rows, uint8_t* aq, float* s2,
                                  cudaStream_t s) {
  // few long rows at decode: up to 1024 threads per row (one float4 of F per thread)
  const int threads = std::min(1024, std::max(128, ((p.F / 4 + 31) / 32) * 32));
  launch_pdl(swiglu_requant_kernel, dim3(row_grid(p.Rcap)), dim3(threads), 0, s, h, splits,
             split_stride, total_rows, p.Rcap, p.F, aq, s2);
  return cudaGetLastError();
}

cudaError_t launch_combine(const Plan& p, const float* o, int splits, size_t split_stride,
                           const float* topk_w, const int32_t* inv_row, const float* shared_src,
                           const int32_t* shared_row0, int shared_splits, uint16_t* y,
                           float* y_f32, cudaStream_t s) {
  // status pointer: the combine of the split entry point has no workspace; pass none
  launch_pdl(combine_kernel, dim3(row_grid(p.T)), dim3(256), 0, s, o, splits,
             split_stride, topk_w, inv_row, p.k_max, p.Rcap, shared_src, shared_row0,
             shared_splits, split_stride, p.T, p.d, y, y_f32, nullptr);
  return cudaGetLastError();
}

cudaError_t launch_reduce_splits(const Plan& p, const float* o, int splits, size_t split_stride,
                                 const int32_t* total_rows, float* out, cudaStream_t s) {
  launch_pdl(reduce_splits_kernel, dim3(row_grid(p.Rcap)), dim3(256), 0, s, o, splits, split_stride, total_rows,
                                                        p.Rcap, p.d, out);
  return cudaGetLastError();
}

}  // namespace moe
