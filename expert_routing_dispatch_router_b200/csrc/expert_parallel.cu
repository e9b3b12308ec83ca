// Expert parallelism across G ranks: the exchange of token rows between the
// rank that routed a token and the rank that owns the expert.
//
// Ascend LongCat-2.0 deployment article (10100.com): the decode instance
// shards the experts over 128 cards ("Decode节点：EP128超大专家并行", DP128 + EP128
// in "多场景模型分层切分优化"), with Dispatch/Combine operators that support
// zero-computation experts ("底层定制算子深度优化").
//
// Rank r owns the routed experts [lo_r, hi_r), an even split of the N routed
// ids (the first N % G ranks take one more). Zero experts belong to no rank:
// their slots never leave the token's rank, and its combine adds the identity
// term. Every rank first dispatches locally (moe_dispatch: rows in (expert,
// token) order, per-expert counts and offsets); the counts and offsets of all
// ranks are then gathered on every rank (G x E and G x (N + 1) integers).
// From them each rank knows, without another exchange, where each of its rows
// lands in the owner's receive buffer, which is expert-major: (expert, source
// rank, source order). So:
//  - ep_plan_kernel (one block): for this rank, the first destination row of
//    each expert's block in its owner's buffer, and this rank's own receive
//    offsets (the expert FFN's offsets over its experts);
//  - ep_dispatch_kernel: each routed row x[row_token[j]] is copied straight
//    into the owner's buffer (a peer's memory on one node: plain stores);
//  - ep_return_kernel: each expert output row of this rank's buffer is copied
//    back into its source rank's y_perm, at the row the source's dispatch gave
//    it, so the source combines as on one GPU.
// No row is sent to a rank that does not own its expert, and no rank waits on
// another inside a kernel: ordering between ranks is the caller's (a barrier
// or a collective between the calls).
#include "moe_internal.cuh"

namespace moe {
namespace {

// Owner rank of routed expert e under the even split of N ids over G ranks.
__device__ __forceinline__ int ep_owner(int e, int N, int G) {
  const int base = N / G, extra = N % G;
  const int big = extra * (base + 1);  // ids held by the ranks with one more
  return e < big ? e / (base + 1) : extra + (e - big) / base;
}
__host__ __device__ __forceinline__ int ep_lo(int r, int N, int G) {
  const int base = N / G, extra = N % G;
  return r * base + (r < extra ? r : extra);
}

// Largest j in [0, n) with v[j] <= x (v ascending, v[0] <= x).
__device__ __forceinline__ int last_le(const int32_t* v, int n, int64_t x) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (v[mid] <= x)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(1024)
    ep_plan_kernel(const int32_t* __restrict__ counts_all, int G, int E, int N, int rank,
                   int32_t* __restrict__ dest_row, int32_t* __restrict__ recv_offsets) {
  __shared__ int32_t prefix[kMaxExperts + 1];  // over experts of all sources' rows
  __shared__ int32_t warp_sums[32];
  griddep_wait();
  griddep_launch_dependents();
  const int e = threadIdx.x;
  int32_t total = 0, before = 0;  // rows of expert e from all sources / sources < rank
  if (e < N)
    for (int s = 0; s < G; ++s) {
      const int32_t c = counts_all[(int64_t)s * E + e];
      total += c;
      if (s < rank) before += c;
    }
  // block exclusive scan of total over e
  const int lane = e & 31, wid = e >> 5;
  int32_t incl = total;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int32_t o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_sums[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int32_t v = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t o = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += o;
    }
    warp_sums[lane] = v;
  }
  __syncthreads();
  const int32_t excl = (wid > 0 ? warp_sums[wid - 1] : 0) + incl - total;
  if (e < N) prefix[e] = excl;
  if (e == 0) prefix[N] = warp_sums[31];
  __syncthreads();
  if (e < N) {
    const int lo = ep_lo(ep_owner(e, N, G), N, G);
    dest_row[e] = prefix[e] - prefix[lo] + before;
  }
  const int my_lo = ep_lo(rank, N, G), my_n = ep_lo(rank + 1, N, G) - my_lo;
  for (int j = e; j <= my_n; j += blockDim.x) recv_offsets[j] = prefix[my_lo + j] - prefix[my_lo];
}

// One warp per routed row of this rank: x[row_token[j]] -> the owner's buffer.
__global__ void __launch_bounds__(256)
    ep_dispatch_kernel(const uint8_t* __restrict__ x, const int32_t* __restrict__ offsets,
                       const int32_t* __restrict__ row_token,
                       const int32_t* __restrict__ dest_row, uint8_t* const* __restrict__ recv,
                       int N, int G, int64_t row_bytes) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t R = offsets[N];
  const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t j = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); j < R;
       j += nw) {
    const int e = last_le(offsets, N, j);
    const int64_t dst = (int64_t)dest_row[e] + (j - offsets[e]);
    const uint4* src = reinterpret_cast<const uint4*>(x + (int64_t)row_token[j] * row_bytes);
    uint4* out = reinterpret_cast<uint4*>(recv[ep_owner(e, N, G)] + dst * row_bytes);
    for (int64_t v = lane; v < row_bytes / 16; v += 32) out[v] = src[v];
  }
}

// One warp per row i of this rank's receive buffer: y_recv[i] -> its source.
__global__ void __launch_bounds__(256)
    ep_return_kernel(const uint8_t* __restrict__ y_recv,
                     const int32_t* __restrict__ recv_offsets, int n_local, int my_lo,
                     const int32_t* __restrict__ counts_all,
                     const int32_t* __restrict__ offsets_all, uint8_t* const* __restrict__ home,
                     int N, int E, int G, int64_t row_bytes) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t rows = recv_offsets[n_local];
  const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < rows;
       i += nw) {
    const int j = last_le(recv_offsets, n_local, i);  // local expert
    const int e = my_lo + j;
    int64_t within = i - recv_offsets[j];
    int s = 0;  // source rank: blocks of expert e arrive in source order
    for (; s < G - 1; ++s) {
      const int32_t c = counts_all[(int64_t)s * E + e];
      if (within < c) break;
      within -= c;
    }
    const int64_t dst = (int64_t)offsets_all[(int64_t)s * (N + 1) + e] + within;
    const uint4* src = reinterpret_cast<const uint4*>(y_recv + i * row_bytes);
    uint4* out = reinterpret_cast<uint4*>(home[s] + dst * row_bytes);
    for (int64_t v = lane; v < row_bytes / 16; v += 32) out[v] = src[v];
  }
}

}  // namespace

int ep_local_experts(int rank, int N, int G) { return ep_lo(rank + 1, N, G) - ep_lo(rank, N, G); }
int ep_first_expert(int rank, int N, int G) { return ep_lo(rank, N, G); }

cudaError_t launch_ep_plan(const Shape& sh, int rank, int G, const int32_t* counts_all,
                           int32_t* dest_row, int32_t* recv_offsets, cudaStream_t st) {
  return launch_pdl(ep_plan_kernel, dim3(1), dim3(1024), 0, st, counts_all, G, (int)sh.E,
                    (int)sh.N, rank, dest_row, recv_offsets);
}

cudaError_t launch_ep_dispatch(const Shape& sh, int G, const void* x, const int32_t* offsets,
                               const int32_t* row_token, const int32_t* dest_row,
                               void* const* recv, cudaStream_t st) {
  const int64_t row_bytes = sh.d * sh.es;
  const unsigned blocks = (unsigned)(4 * num_sms());
  return launch_pdl(ep_dispatch_kernel, dim3(blocks), dim3(256), 0, st,
                    static_cast<const uint8_t*>(x), offsets, row_token, dest_row,
                    reinterpret_cast<uint8_t* const*>(recv), (int)sh.N, G, row_bytes);
}

cudaError_t launch_ep_return(const Shape& sh, int rank, int G, const void* y_recv,
                             const int32_t* recv_offsets, const int32_t* counts_all,
                             const int32_t* offsets_all, void* const* home, cudaStream_t st) {
  const int64_t row_bytes = sh.d * sh.es;
  const unsigned blocks = (unsigned)(4 * num_sms());
  return launch_pdl(ep_return_kernel, dim3(blocks), dim3(256), 0, st,
                    static_cast<const uint8_t*>(y_recv), recv_offsets,
                    ep_local_experts(rank, (int)sh.N, G), ep_first_expert(rank, (int)sh.N, G),
                    counts_all, offsets_all, reinterpret_cast<uint8_t* const*>(home),
                    (int)sh.N, (int)sh.E, G, row_bytes);
}

}  // namespace moe
