// Expert-parallel dispatch: the E experts are split over n_ranks GPUs in contiguous blocks of
// E / n_ranks, and every token's hidden row is sent once to each GPU that holds at least one of
// its selected experts, together with the local ids and routing weights of those experts. The
// plan kernel (one block) lays out the send rows in (rank, token) order; the gather kernel copies
// the token rows into that order. What crosses the links is then one all-to-all of rows, and one
// of partial outputs on the way back ("Routage MoE entre GPU", the paragraphs on sending a
// token's activations to the GPUs that hold its experts and returning the results; "Semantic
// Parallelism", section 1, the all-to-all of expert parallelism).
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int kEpThreads = 1024;
constexpr int kEpWarps = kEpThreads / 32;

// Bit r set when rank r holds one of token t's selected experts (slots j < k_t; id -1 = unused
// slot). Out-of-range ids and k_t are reported when `check` is set and left out.
__device__ __forceinline__ uint32_t ep_token_ranks(const int32_t* __restrict__ ids, int t,
                                                   int k_max, int kt, int E, int E_local,
                                                   int* status, bool check) {
  uint32_t m = 0;
  for (int j = 0; j < kt; ++j) {
    const int e = ids[(size_t)t * k_max + j];
    if (e < 0) continue;
    if (e >= E) {
      if (check) report(status, kStatusDeviceCheck, kWhereDispatch, t);
      continue;
    }
    m |= 1u << (e / E_local);
  }
  return m;
}

__device__ __forceinline__ int ep_token_k(const int32_t* __restrict__ k_per_token, int k, int t,
                                          int k_max) {
  const int kt = k_per_token ? k_per_token[t] : k;
  return min(max(kt, 0), k_max);
}

// One block. Pass 1 counts the send rows of every rank; pass 2 walks the tokens in order, 1024 at
// a time, and gives (t, r) the row base[r] + (rows of rank r from earlier tokens): a ballot per
// rank inside each warp, then a scan over the 32 warps per rank. A row's local ids are the
// token's experts on rank r in slot order (e - r * E_local), then -1; its weights likewise, then 0.
__global__ void __launch_bounds__(kEpThreads) ep_plan_kernel(
    const int32_t* __restrict__ ids, const float* __restrict__ topk_w, int T, int k_max, int k,
    const int32_t* __restrict__ k_per_token, int E, int n_ranks, int kl,
    int32_t* __restrict__ send_ids, float* __restrict__ send_w, int32_t* __restrict__ send_counts,
    int32_t* __restrict__ slot_of, float* __restrict__ slot_w, int* status) {
  pdl_wait();      // predecessor kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  __shared__ int s_cnt[32], s_base[32], s_done[32];
  __shared__ int s_wrow[kEpWarps][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int E_local = E / n_ranks;
  if (threadIdx.x < 32) s_cnt[threadIdx.x] = 0;
  __syncthreads();

  // pass 1: rows per destination rank
  for (int t = threadIdx.x; t < T; t += kEpThreads) {
    const int kraw = k_per_token ? k_per_token[t] : k;
    if (kraw < 0 || kraw > k_max) report(status, kStatusDeviceCheck, kWhereDispatch, t);
    uint32_t m = ep_token_ranks(ids, t, k_max, ep_token_k(k_per_token, k, t, k_max), E, E_local,
                                status, true);
    while (m) {
      atomicAdd(&s_cnt[__ffs(m) - 1], 1);
      m &= m - 1;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int r = 0; r < n_ranks; ++r) {
      s_base[r] = run;
      s_done[r] = 0;
      send_counts[r] = s_cnt[r];
      run += s_cnt[r];
    }
  }
  __syncthreads();

  // pass 2: row of every (token, rank), in (rank, token) order
  for (int c0 = 0; c0 < T; c0 += kEpThreads) {
    const int t = c0 + threadIdx.x;
    const int kt = t < T ? ep_token_k(k_per_token, k, t, k_max) : 0;
    const uint32_t m =
        t < T ? ep_token_ranks(ids, t, k_max, kt, E, E_local, status, false) : 0u;
    for (int r = 0; r < n_ranks; ++r) {
      const uint32_t b = __ballot_sync(0xffffffffu, (m >> r) & 1u);
      if (lane == 0) s_wrow[warp][r] = __popc(b);
    }
    __syncthreads();
    if (threadIdx.x < n_ranks) {
      const int r = threadIdx.x;
      int run = s_base[r] + s_done[r];
      for (int w = 0; w < kEpWarps; ++w) {
        const int c = s_wrow[w][r];
        s_wrow[w][r] = run;
        run += c;
      }
      s_done[r] = run - s_base[r];
    }
    __syncthreads();
    for (int r = 0; r < n_ranks; ++r) {
      const bool has = (m >> r) & 1u;
      const uint32_t b = __ballot_sync(0xffffffffu, has);
      if (t >= T) continue;
      const size_t ts = (size_t)t * n_ranks + r;
      if (!has) {
        slot_of[ts] = -1;
        slot_w[ts] = 0.f;
        continue;
      }
      const int row = s_wrow[warp][r] + __popc(b & ((1u << lane) - 1u));
      slot_of[ts] = row;
      slot_w[ts] = 1.f;
      const int lo = r * E_local, hi = lo + E_local;
      int q = 0;
      for (int j = 0; j < kt; ++j) {
        const int e = ids[(size_t)t * k_max + j];
        if (e < lo || e >= hi) continue;
        if (q < kl) {
          send_ids[(size_t)row * kl + q] = e - lo;
          send_w[(size_t)row * kl + q] = topk_w[(size_t)t * k_max + j];
        } else {
          report(status, kStatusDeviceCheck, kWhereDispatch, t);   // an expert selected twice
        }
        ++q;
      }
      for (; q < kl; ++q) {
        send_ids[(size_t)row * kl + q] = -1;
        send_w[(size_t)row * kl + q] = 0.f;
      }
    }
    __syncthreads();     // s_wrow is rewritten by the next chunk
  }
}

// send_hidden[slot_of[t, r], :] = hidden[t, :] for every rank r that token t goes to: one block
// per token (grid-stride), each thread one 16-byte piece of the row, loaded once and stored to
// each destination row.
__global__ void __launch_bounds__(256) ep_gather_kernel(
    const uint16_t* __restrict__ hidden, int T, int d, int n_ranks,
    const int32_t* __restrict__ slot_of, uint16_t* __restrict__ send_hidden) {
  pdl_wait();      // the plan kernel complete, its writes visible
  pdl_trigger();   // let the next kernel launch
  __shared__ int s_slot[32];
  const int nv = d / 8;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();
    if (threadIdx.x < n_ranks) s_slot[threadIdx.x] = slot_of[(size_t)t * n_ranks + threadIdx.x];
    __syncthreads();
    const uint4* src = reinterpret_cast<const uint4*>(hidden + (size_t)t * d);
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
      const uint4 v = src[i];
      for (int r = 0; r < n_ranks; ++r) {
        const int row = s_slot[r];
        if (row >= 0) reinterpret_cast<uint4*>(send_hidden + (size_t)row * d)[i] = v;
      }
    }
  }
}

cudaError_t launch_ep_dispatch(const Plan& p, int n_ranks, const uint16_t* hidden,
                               const int32_t* ids, const float* topk_w, int k,
                               const int32_t* k_per_token, uint16_t* send_hidden,
                               int32_t* send_ids, float* send_w, int32_t* send_counts,
                               int32_t* slot_of, float* slot_w, int* status, cudaStream_t s) {
  const int kl = ep_local_k(p.E, p.k_max, n_ranks);
  launch_pdl(ep_plan_kernel, dim3(1), dim3(kEpThreads), 0, s, ids, topk_w, p.T, p.k_max, k,
             k_per_token, p.E, n_ranks, kl, send_ids, send_w, send_counts, slot_of, slot_w,
             status);
  const int grid = (int)std::min<int64_t>(std::max(p.T, 1), 8LL * num_sms());
  launch_pdl(ep_gather_kernel, dim3(grid), dim3(256), 0, s, hidden, p.T, p.d, n_ranks, slot_of,
             send_hidden);
  return cudaGetLastError();
}

}  // namespace moe
