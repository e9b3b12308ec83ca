// Dispatch: group the routing slots by expert, drop zero-expert slots from the
// compute set, and copy each routed token row into a per-expert contiguous
// buffer.
//
// Ascend LongCat-2.0 deployment article (10100.com), "底层定制算子深度优化":
// a Dispatch operator that supports zero-computation experts. The rows are
// ordered by (expert, token), a stable counting sort, so the permutation is
// the same on every run (the deterministic operators of "LongCat-2.0 Derruba
// Dois Tetos", section "A Primeira Parede").
//
// Three small kernels plus a gather, no atomics whose order matters:
//  1. dispatch_count_kernel: each block takes 256 tokens and builds, in shared
//     memory, one 256-bit mask per expert (which of its tokens chose it), then
//     writes popcount(mask) = the block's count per expert.
//  2. dispatch_scan_kernel (one block): per expert, an exclusive scan over the
//     blocks gives each block's base row inside the expert; an exclusive scan
//     over the routed experts gives offsets[]; rows past R get row_token = -1.
//  3. dispatch_scatter_kernel: rebuilds the masks; the rank of token t inside
//     (block, expert) is popcount(mask bits below t), so
//     row = offsets[e] + base[block][e] + rank, independent of thread timing.
//  4. gather_rows_kernel: x_perm[r] = x[row_token[r]], 16-byte vectors, one
//     warp per row.
// Expert ids outside [0, E) or repeated inside one token are skipped and
// recorded in the workspace error word (code 2) instead of being written.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kWords = kChunkTokens / 32;  // mask words per expert per block

__device__ __forceinline__ void record_error(int32_t* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// Builds mask[e * kWords + w] bit b = token (w*32 + b) of this block chose e.
__device__ __forceinline__ void build_masks(uint32_t* mask, const int32_t* idx,
                                            int64_t T, int k, int E,
                                            int32_t* err) {
  for (int i = threadIdx.x; i < E * kWords; i += blockDim.x) mask[i] = 0u;
  __syncthreads();
  const int64_t t = (int64_t)blockIdx.x * kChunkTokens + threadIdx.x;
  if (t < T) {
    const int w = threadIdx.x >> 5;
    const uint32_t bit = 1u << (threadIdx.x & 31);
    for (int j = 0; j < k; ++j) {
      const int e = idx[t * k + j];
      if (e < 0 || e >= E) {
        record_error(err, kErrBadExpertId);
        continue;
      }
      const uint32_t old = atomicOr(&mask[e * kWords + w], bit);
      if (old & bit) record_error(err, kErrBadExpertId);
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kChunkTokens)
    dispatch_count_kernel(const int32_t* __restrict__ idx, int64_t T, int k,
                          int E, int32_t* __restrict__ chunk_base,
                          int32_t* err) {
  extern __shared__ uint32_t mask[];
  build_masks(mask, idx, T, k, E, err);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kWords; ++w) c += __popc(mask[e * kWords + w]);
    chunk_base[(int64_t)blockIdx.x * E + e] = c;
  }
}

__global__ void __launch_bounds__(1024)
    dispatch_scan_kernel(int32_t* __restrict__ chunk_base, int64_t nchunks,
                         int E, int N, int32_t* __restrict__ counts,
                         int32_t* __restrict__ offsets,
                         int32_t* __restrict__ row_token, int64_t rows_cap) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t total_s;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = 0;
    for (int64_t c = 0; c < nchunks; ++c) {
      const int32_t v = chunk_base[c * E + e];
      chunk_base[c * E + e] = run;
      run += v;
    }
    counts[e] = run;
  }
  __syncthreads();
  // exclusive scan of counts[0..N) (N <= 1024 = blockDim.x)
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int32_t v = (threadIdx.x < N) ? counts[threadIdx.x] : 0;
  int32_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int32_t o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_sums[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int32_t s = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t o = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += o;
    }
    warp_sums[lane] = s;  // inclusive over warps
    if (lane == 31) total_s = s;
  }
  __syncthreads();
  const int32_t before = (wid > 0 ? warp_sums[wid - 1] : 0) + incl - v;
  if (threadIdx.x < N) offsets[threadIdx.x] = before;
  const int32_t R = total_s;
  if (threadIdx.x == 0) offsets[N] = R;
  for (int64_t r = R + threadIdx.x; r < rows_cap; r += blockDim.x) row_token[r] = -1;
}

__global__ void __launch_bounds__(kChunkTokens)
    dispatch_scatter_kernel(const int32_t* __restrict__ idx, int64_t T, int k,
                            int E, int N,
                            const int32_t* __restrict__ chunk_base,
                            const int32_t* __restrict__ offsets,
                            int32_t* __restrict__ row_token,
                            int32_t* __restrict__ slot_row) {
  extern __shared__ uint32_t mask[];
  build_masks(mask, idx, T, k, E, nullptr);
  const int64_t t = (int64_t)blockIdx.x * kChunkTokens + threadIdx.x;
  if (t >= T) return;
  const int w = threadIdx.x >> 5;
  const uint32_t below = (1u << (threadIdx.x & 31)) - 1u;
  for (int j = 0; j < k; ++j) {
    const int e = idx[t * k + j];
    int32_t r = -1;
    if (e >= 0 && e < N) {
      int rank = __popc(mask[e * kWords + w] & below);
      for (int w2 = 0; w2 < w; ++w2) rank += __popc(mask[e * kWords + w2]);
      r = offsets[e] + chunk_base[(int64_t)blockIdx.x * E + e] + rank;
      row_token[r] = (int32_t)t;
    }
    slot_row[t * k + j] = r;
  }
}

// x_perm[r, :] = x[row_token[r], :] for r < R; one warp per row, 16-byte vectors.
__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint4* __restrict__ x,
                       const int32_t* __restrict__ row_token,
                       const int32_t* __restrict__ offsets, int N,
                       int64_t vec_per_row, int64_t rows_cap,
                       uint4* __restrict__ x_perm) {
  const int64_t R = offsets[N];
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       r < R && r < rows_cap; r += warps) {
    const int64_t t = row_token[r];
    const uint4* src = x + t * vec_per_row;
    uint4* dst = x_perm + r * vec_per_row;
    for (int64_t v = lane; v < vec_per_row; v += 32) dst[v] = src[v];
  }
}

}  // namespace

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

cudaError_t launch_dispatch(const Shape& sh, const void* x, const int32_t* idx,
                            int32_t* chunk_base, int32_t* counts,
                            int32_t* offsets, int32_t* row_token,
                            int32_t* slot_row, void* x_perm, int32_t* err,
                            cudaStream_t st) {
  const int E = (int)sh.E, N = (int)sh.N, k = (int)sh.k;
  const size_t smem = (size_t)E * kWords * sizeof(uint32_t);
  const unsigned nch = (unsigned)sh.nchunks;
  dispatch_count_kernel<<<nch, kChunkTokens, smem, st>>>(idx, sh.T, k, E,
                                                         chunk_base, err);
  dispatch_scan_kernel<<<1, 1024, 0, st>>>(chunk_base, sh.nchunks, E, N, counts,
                                           offsets, row_token, sh.T * sh.k);
  dispatch_scatter_kernel<<<nch, kChunkTokens, smem, st>>>(
      idx, sh.T, k, E, N, chunk_base, offsets, row_token, slot_row);
  if (N > 0) {
    const int64_t vpr = sh.d * sh.es / 16;
    int64_t rows = sh.T * sh.k;
    int64_t blocks = (rows + 7) / 8;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    gather_rows_kernel<<<(unsigned)blocks, 256, 0, st>>>(
        static_cast<const uint4*>(x), row_token, offsets, N, vpr, rows,
        static_cast<uint4*>(x_perm));
  }
  return cudaGetLastError();
}

}  // namespace moe
