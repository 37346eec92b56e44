// Grouping of the routed (token, slot) pairs by expert: per-warp histograms, an exclusive prefix
// sum over experts, and a stable scatter so routed rows are ordered by (expert, token). Then the
// gather that lays the quantised token rows out in that order for the grouped GEMMs. (The GEMM
// could fetch the rows through the permutation with four-row tile::gather4 TMA loads instead;
// measured on B200 that is slower at every batch size -- the 32 gather4 loads per pipeline stage
// of a 256-token tile make the gate/up GEMM TMA-issue-bound, 7650 vs 2659 us at DeepSeek T=8192,
// and decode layers lose 0.4-230 us -- so the rows are gathered.)
//
// Method: "Routage MoE entre GPU" (viite.ai) -- only the selected experts process a token; the
// tokens are dispatched to their experts and their order restored at the combine.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int kPermThreads = 1024;
constexpr int kPermWarps = kPermThreads / 32;

// Exclusive scan of one int per thread over a 1024-thread block; returns the block total too.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int ws = warp_sums[lane];
    int wincl = ws;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, wincl, off);
      if (lane >= off) wincl += o;
    }
    warp_sums[lane] = wincl - ws;          // exclusive prefix of warp totals
    if (lane == 31) warp_sums[32] = wincl;
  }
  __syncthreads();
  total = warp_sums[32];
  const int r = warp_sums[warp] + incl - v;
  __syncthreads();
  return r;
}

// One block computes the whole grouping. Warp w owns tokens [w*chunk, (w+1)*chunk) and walks its
// (token, slot) pairs in token-major order, 32 at a time. Lanes holding the same expert find each
// other with __match_any_sync; a lane's rank among them plus the warp's running cursor for that
// expert gives its row, so rows inside an expert are in ascending token order. `write` selects
// the block that stores offsets / perm / inv / tiles (and reports bad ids); `s_perm`, when given,
// receives perm[] in shared memory. Returns the routed row count R.
__device__ int permute_block_body(const int32_t* __restrict__ ids, int T, int k_max, int k,
                                  const int32_t* __restrict__ k_per_token, int E, int has_shared,
                                  int BN, int32_t* __restrict__ offsets,
                                  int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                  int32_t* __restrict__ tiles, int* status, int* hist,
                                  int* warp_sums, int* s_perm, bool write) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kPermWarps * E; i += kPermThreads) hist[i] = 0;
  __syncthreads();

  const int chunk = (T + kPermWarps - 1) / kPermWarps;
  const int t_begin = min(T, warp * chunk), t_end = min(T, t_begin + chunk);
  const long long i_begin = (long long)t_begin * k_max, i_end = (long long)t_end * k_max;
  int* my_hist = hist + warp * E;

  // pass 1: per-warp counts
  for (long long base = i_begin; base < i_end; base += 32) {
    const long long idx = base + lane;
    if (idx < i_end) {
      const int t = (int)(idx / k_max), j = (int)(idx % k_max);
      const int kt = k_per_token ? k_per_token[t] : k;
      if (j < kt) {
        const int e = ids[idx];
        if (e >= 0 && e < E) atomicAdd(&my_hist[e], 1);
        else if (write && e != -1) report(status, kStatusDeviceCheck, kWherePermute, t);
      }
    }
  }
  __syncthreads();

  // pass 2: expert totals, exclusive scan -> offsets, per-warp cursors, GEMM tile prefix
  int total_rows = 0, total_tiles = 0;
  {
    const int e = threadIdx.x;                 // E <= 1024 = blockDim
    int cnt = 0;
    if (e < E)
      for (int w = 0; w < kPermWarps; ++w) cnt += hist[w * E + e];
    const int off = block_exclusive_scan(cnt, warp_sums, total_rows);
    if (e < E) {
      if (write) offsets[e] = off;
      int run = off;
      for (int w = 0; w < kPermWarps; ++w) {
        const int c = hist[w * E + e];
        hist[w * E + e] = run;
        run += c;
      }
    }
    const int nt = e < E ? (cnt + BN - 1) / BN : 0;
    const int toff = block_exclusive_scan(nt, warp_sums, total_tiles);
    if (write && e < E) tiles[e] = toff;
    if (write && threadIdx.x == 0) {
      offsets[E] = total_rows;
      if (has_shared) {
        offsets[E + 1] = total_rows + T;
        tiles[E] = total_tiles;
        tiles[E + 1] = total_tiles + (T + BN - 1) / BN;
      } else {
        tiles[E] = total_tiles;
      }
    }
  }
  __syncthreads();

  // pass 3: stable scatter
  for (long long base = i_begin; base < i_end; base += 32) {
    const long long idx = base + lane;
    bool valid = false;
    int t = 0, e = -1;
    if (idx < i_end) {
      t = (int)(idx / k_max);
      const int j = (int)(idx % k_max);
      const int kt = k_per_token ? k_per_token[t] : k;
      if (j < kt) {
        e = ids[idx];
        valid = e >= 0 && e < E;
      }
      if (!valid && write) inv[idx] = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : E + lane);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int cursor = valid ? my_hist[e] : 0;
    __syncwarp();
    if (valid) {
      const int r = cursor + rank;
      if (write) {
        perm[r] = t;
        inv[idx] = r;
      }
      if (s_perm) s_perm[r] = t;
      if (rank == 0) my_hist[e] = cursor + __popc(peers);
    }
    __syncwarp();
  }
  if (has_shared)
    for (int t = threadIdx.x; t < T; t += kPermThreads) {
      if (write) perm[total_rows + t] = t;
      if (s_perm) s_perm[total_rows + t] = t;
    }
  return total_rows;
}

__global__ void __launch_bounds__(kPermThreads) permute_kernel(
    const int32_t* __restrict__ ids, int T, int k_max, int k, const int32_t* __restrict__ k_per_token,
    int E, int has_shared, int BN, int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
    int32_t* __restrict__ inv, int32_t* __restrict__ tiles, int* status) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  extern __shared__ int hist[];                  // [kPermWarps][E]
  __shared__ int warp_sums[33];
  permute_block_body(ids, T, k_max, k, k_per_token, E, has_shared, BN, offsets, perm, inv, tiles,
                     status, hist, warp_sums, nullptr, true);
}

// Grouping and row gather in one kernel, for batches whose grouping fits one block (T * k_max <=
// 8192): every block computes the (small) grouping itself into shared memory -- so no block
// waits for another -- block 0 also stores it, and each block then copies its share of the
// quantised token rows into grouped order (one warp per row): xqp[r, :] = xq[perm[r], :],
// xsp[r] = xs[perm[r]], amax[r] = 0. Saves the separate gather launch and its dependency wait.
__global__ void __launch_bounds__(kPermThreads) permute_gather_kernel(
    const int32_t* __restrict__ ids, int T, int k_max, int k, const int32_t* __restrict__ k_per_token,
    int E, int has_shared, int BN, int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
    int32_t* __restrict__ inv, int32_t* __restrict__ tiles, const uint8_t* __restrict__ xq,
    const float* __restrict__ xs, int d, uint8_t* __restrict__ xqp, float* __restrict__ xsp,
    uint32_t* __restrict__ amax, int* status) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  extern __shared__ int smem_i[];                // hist [kPermWarps][E], then perm [rows]
  __shared__ int warp_sums[33];
  int* hist = smem_i;
  int* s_perm = smem_i + kPermWarps * E;
  const int R = permute_block_body(ids, T, k_max, k, k_per_token, E, has_shared, BN, offsets, perm,
                                   inv, tiles, status, hist, warp_sums, s_perm, blockIdx.x == 0);
  __syncthreads();
  const int rows = R + (has_shared ? T : 0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nv = d / 16;
  for (int r = blockIdx.x * kPermWarps + warp; r < rows; r += gridDim.x * kPermWarps) {
    const int t = s_perm[r];
    const uint4* src = reinterpret_cast<const uint4*>(xq + (size_t)t * d);
    uint4* dst = reinterpret_cast<uint4*>(xqp + (size_t)r * d);
#pragma unroll 4
    for (int i = lane; i < nv; i += 32) dst[i] = src[i];
    if (lane == 0) {
      xsp[r] = xs[t];
      amax[r] = 0u;
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Multi-block grouping for large T * k_max. Block b owns tokens [b*chunk, (b+1)*chunk) and its
// warps own contiguous sub-ranges, so (block, warp, batch, lane) order is token order:
//   count:   per-block expert counts -> bcount[b][e]
//   scan:    offsets, per-block bases bbase[b][e] = offsets[e] + sum_{b'<b} bcount[b'][e],
//            GEMM tile prefix (one block)
//   scatter: per-warp cursors = bbase[b][e] + counts of the block's earlier warps, then the same
//            stable __match_any_sync ranking as the single-block kernel.
constexpr int kPermBlkThreads = 256;
constexpr int kPermBlkWarps = kPermBlkThreads / 32;

__device__ __forceinline__ void warp_range(int T, int k_max, int blocks, long long& i_begin,
                                           long long& i_end) {
  const int bchunk = (T + blocks - 1) / blocks;
  const int bt0 = min(T, (int)blockIdx.x * bchunk), bt1 = min(T, bt0 + bchunk);
  const int wchunk = (bt1 - bt0 + kPermBlkWarps - 1) / kPermBlkWarps;
  const int warp = threadIdx.x >> 5;
  const int t0 = min(bt1, bt0 + warp * wchunk), t1 = min(bt1, t0 + wchunk);
  i_begin = (long long)t0 * k_max;
  i_end = (long long)t1 * k_max;
}

// shared-memory per-warp counts of this block's (token, slot) pairs
__device__ __forceinline__ void block_warp_counts(const int32_t* ids, int T, int k_max, int k,
                                                  const int32_t* k_per_token, int E, int blocks,
                                                  int* whist, int* status, bool flag) {
  for (int i = threadIdx.x; i < kPermBlkWarps * E; i += kPermBlkThreads) whist[i] = 0;
  __syncthreads();
  long long i_begin, i_end;
  warp_range(T, k_max, blocks, i_begin, i_end);
  int* my = whist + (threadIdx.x >> 5) * E;
  const int lane = threadIdx.x & 31;
  for (long long base = i_begin; base < i_end; base += 32) {
    const long long idx = base + lane;
    if (idx < i_end) {
      const int t = (int)(idx / k_max), j = (int)(idx % k_max);
      const int kt = k_per_token ? k_per_token[t] : k;
      if (j < kt) {
        const int e = ids[idx];
        if (e >= 0 && e < E) atomicAdd(&my[e], 1);
        else if (flag && e != -1) report(status, kStatusDeviceCheck, kWherePermute, t);
      }
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kPermBlkThreads) permute_count_kernel(
    const int32_t* __restrict__ ids, int T, int k_max, int k, const int32_t* __restrict__ k_per_token,
    int E, int32_t* __restrict__ bcount, int* status) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  extern __shared__ int whist[];
  block_warp_counts(ids, T, k_max, k, k_per_token, E, gridDim.x, whist, status, true);
  for (int e = threadIdx.x; e < E; e += kPermBlkThreads) {
    int c = 0;
    for (int w = 0; w < kPermBlkWarps; ++w) c += whist[w * E + e];
    bcount[(size_t)blockIdx.x * E + e] = c;
  }
}

__global__ void __launch_bounds__(kPermThreads) permute_scan_kernel(
    const int32_t* __restrict__ bcount, int blocks, int T, int E, int has_shared, int BN,
    int32_t* __restrict__ bbase, int32_t* __restrict__ offsets, int32_t* __restrict__ tiles) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  __shared__ int warp_sums[33];
  const int e = threadIdx.x;                 // E <= 1024 = blockDim
  int cnt = 0;
  if (e < E)
    for (int b = 0; b < blocks; ++b) cnt += bcount[(size_t)b * E + e];
  int total_rows = 0, total_tiles = 0;
  const int off = block_exclusive_scan(cnt, warp_sums, total_rows);
  if (e < E) {
    offsets[e] = off;
    int run = off;
    for (int b = 0; b < blocks; ++b) {
      bbase[(size_t)b * E + e] = run;
      run += bcount[(size_t)b * E + e];
    }
  }
  const int nt = e < E ? (cnt + BN - 1) / BN : 0;
  const int toff = block_exclusive_scan(nt, warp_sums, total_tiles);
  if (e < E) tiles[e] = toff;
  if (threadIdx.x == 0) {
    offsets[E] = total_rows;
    tiles[E] = total_tiles;
    if (has_shared) {
      offsets[E + 1] = total_rows + T;
      tiles[E + 1] = total_tiles + (T + BN - 1) / BN;
    }
  }
}

__global__ void __launch_bounds__(kPermBlkThreads) permute_scatter_kernel(
    const int32_t* __restrict__ ids, int T, int k_max, int k, const int32_t* __restrict__ k_per_token,
    int E, int has_shared, const int32_t* __restrict__ bbase, const int32_t* __restrict__ offsets,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  extern __shared__ int whist[];
  block_warp_counts(ids, T, k_max, k, k_per_token, E, gridDim.x, whist, nullptr, false);
  // per-warp cursors: the block's base plus the counts of its earlier warps
  for (int e = threadIdx.x; e < E; e += kPermBlkThreads) {
    int run = bbase[(size_t)blockIdx.x * E + e];
    for (int w = 0; w < kPermBlkWarps; ++w) {
      const int c = whist[w * E + e];
      whist[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  long long i_begin, i_end;
  warp_range(T, k_max, gridDim.x, i_begin, i_end);
  int* my = whist + (threadIdx.x >> 5) * E;
  const int lane = threadIdx.x & 31;
  for (long long base = i_begin; base < i_end; base += 32) {
    const long long idx = base + lane;
    bool valid = false;
    int t = 0, e = -1;
    if (idx < i_end) {
      t = (int)(idx / k_max);
      const int j = (int)(idx % k_max);
      const int kt = k_per_token ? k_per_token[t] : k;
      if (j < kt) {
        e = ids[idx];
        valid = e >= 0 && e < E;
      }
      if (!valid) inv[idx] = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : E + lane);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int cursor = valid ? my[e] : 0;
    __syncwarp();
    if (valid) {
      const int r = cursor + rank;
      perm[r] = t;
      inv[idx] = r;
      if (rank == 0) my[e] = cursor + __popc(peers);
    }
    __syncwarp();
  }
  if (has_shared) {
    const int R = offsets[E];
    for (int t = blockIdx.x * kPermBlkThreads + threadIdx.x; t < T; t += gridDim.x * kPermBlkThreads)
      perm[R + t] = t;
  }
}

// For caller-provided offsets (split entry point): validate and build the GEMM tile prefix.
__global__ void __launch_bounds__(kPermThreads) tile_prefix_kernel(
    const int32_t* __restrict__ offsets, int E, int64_t rcap, int BN, int32_t* __restrict__ tiles,
    int* status) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  __shared__ int warp_sums[33];
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  const int e = threadIdx.x;
  int nt = 0;
  if (e < E) {
    const int a = offsets[e], b = offsets[e + 1];
    if (a < 0 || b < a || b > rcap) bad = 1;
    else nt = (b - a + BN - 1) / BN;
  }
  int total = 0;
  const int toff = block_exclusive_scan(nt, warp_sums, total);
  __syncthreads();
  if (bad) {
    // inconsistent offsets: publish an empty tile list so no GEMM work is done
    if (e <= E) tiles[e] = 0;
    if (threadIdx.x == 0) report(status, kStatusDeviceCheck, kWhereTilePrefix, 0);
    return;
  }
  if (e < E) tiles[e] = toff;
  if (threadIdx.x == 0) tiles[E] = total;
}

// One warp per routed row: xqp[r, :] = xq[perm[r], :], xsp[r] = xs[perm[r]], amax[r] = 0.
// A token index outside [0, T) (caller-provided permutation) gives a zero row and flags
// MOE_ERR_DEVICE_CHECK.
__global__ void __launch_bounds__(256) gather_rows_kernel(
    const uint8_t* __restrict__ xq, const float* __restrict__ xs, const int32_t* __restrict__ perm,
    const int32_t* __restrict__ total_rows, int64_t rcap, int T, int d, uint8_t* __restrict__ xqp,
    float* __restrict__ xsp, uint32_t* __restrict__ amax, int* status) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  const int R = (int)min((int64_t)max(*total_rows, 0), rcap);
  const int lane = threadIdx.x & 31;
  const int nv = d / 16;
  for (int r = blockIdx.x * 8 + (threadIdx.x >> 5); r < R; r += gridDim.x * 8) {
    const int t = perm[r];
    const bool ok = t >= 0 && t < T;
    uint4* dst = reinterpret_cast<uint4*>(xqp + (size_t)r * d);
    if (ok) {
      const uint4* src = reinterpret_cast<const uint4*>(xq + (size_t)t * d);
#pragma unroll 4
      for (int i = lane; i < nv; i += 32) dst[i] = src[i];
    } else {
      for (int i = lane; i < nv; i += 32) dst[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (lane == 0) {
      xsp[r] = ok ? xs[t] : 0.f;
      amax[r] = 0u;
      if (!ok) report(status, kStatusDeviceCheck, kWhereGather, r);
    }
  }
}

// Blocks of the multi-block grouping: about 1024 (token, slot) pairs each, at most 4 per SM.
int permute_blocks(const Plan& p) {
  const long long slots = (long long)p.T * p.k_max;
  if (slots <= 8192) return 1;
  return (int)std::min<long long>((slots + 1023) / 1024, 4LL * 148);
}

cudaError_t launch_permute(const Plan& p, const int32_t* ids, int k, const int32_t* k_per_token,
                           int32_t* offsets, int32_t* perm, int32_t* inv, int32_t* tiles,
                           int32_t* scratch, int* status, cudaStream_t s) {
  const int blocks = permute_blocks(p);
  if (blocks == 1) {
    const size_t smem = sizeof(int) * kPermWarps * p.E;
    static bool attr_set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    if (dev < 64 && !attr_set[dev]) {
      cudaError_t e = cudaFuncSetAttribute(permute_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kPermWarps * kMaxExperts * (int)sizeof(int));
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
    launch_pdl(permute_kernel, dim3(1), dim3(kPermThreads), smem, s, ids, p.T, p.k_max, k, k_per_token, p.E,
                                                 p.shared ? 1 : 0, p.BN, offsets, perm, inv, tiles,
                                                 status);
    return cudaGetLastError();
  }
  int32_t* bcount = scratch;
  int32_t* bbase = scratch + (size_t)blocks * p.E;
  const size_t smem = sizeof(int) * kPermBlkWarps * p.E;   // <= 32 KB
  launch_pdl(permute_count_kernel, dim3(blocks), dim3(kPermBlkThreads), smem, s, ids, p.T, p.k_max, k, k_per_token,
                                                             p.E, bcount, status);
  launch_pdl(permute_scan_kernel, dim3(1), dim3(kPermThreads), 0, s, bcount, blocks, p.T, p.E, p.shared ? 1 : 0, p.BN,
                                                 bbase, offsets, tiles);
  launch_pdl(permute_scatter_kernel, dim3(blocks), dim3(kPermBlkThreads), smem, s, ids, p.T, p.k_max, k, k_per_token,
                                                               p.E, p.shared ? 1 : 0, bbase,
                                                               offsets, perm, inv);
  return cudaGetLastError();
}

bool permute_gather_fused(const Plan& p) { return permute_blocks(p) == 1; }

cudaError_t launch_permute_gather(const Plan& p, const int32_t* ids, int k,
                                  const int32_t* k_per_token, int32_t* offsets, int32_t* perm,
                                  int32_t* inv, int32_t* tiles, const uint8_t* xq, const float* xs,
                                  uint8_t* xqp, float* xsp, uint32_t* amax, int* status,
                                  cudaStream_t s) {
  // T * k_max <= 8192 here, so rows = T * k_max (+ T) <= 16384
  const size_t smem = sizeof(int) * ((size_t)kPermWarps * p.E + (size_t)p.Rcap);
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(permute_gather_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(int) * (kPermWarps * kMaxExperts + 16384));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  // about 32 KB of rows per block (one warp per row), at most one block per SM
  const int64_t bytes = p.Rcap * (int64_t)p.d;
  const int grid = (int)std::min<int64_t>(std::max<int64_t>((bytes + 32767) / 32768, 1), num_sms());
  launch_pdl(permute_gather_kernel, dim3(grid), dim3(kPermThreads), smem, s, ids, p.T, p.k_max, k,
             k_per_token, p.E, p.shared ? 1 : 0, p.BN, offsets, perm, inv, tiles, xq, xs, p.d,
             xqp, xsp, amax, status);
  return cudaGetLastError();
}

cudaError_t launch_tile_prefix(const Plan& p, const int32_t* offsets, int32_t* tiles, int* status,
                               cudaStream_t s) {
  launch_pdl(tile_prefix_kernel, dim3(1), dim3(kPermThreads), 0, s, offsets, p.E, (int64_t)p.T * p.k_max, p.BN, tiles,
                                                status);
  return cudaGetLastError();
}

cudaError_t launch_gather(const Plan& p, const uint8_t* xq, const float* xs, const int32_t* perm,
                          const int32_t* total_rows, uint8_t* xqp, float* xsp, uint32_t* amax,
                          int* status, cudaStream_t s) {
  const int64_t blocks_needed = (p.Rcap + 7) / 8;
  const int grid = (int)std::min<int64_t>(std::max<int64_t>(blocks_needed, 1), 8LL * num_sms());
  launch_pdl(gather_rows_kernel, dim3(grid), dim3(256), 0, s, xq, xs, perm, total_rows, p.Rcap, p.T, p.d, xqp, xsp,
                                          amax, status);
  return cudaGetLastError();
}

}  // namespace moe
