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
// For small batches (the masks of all T tokens fit in shared memory) one block
// does steps 1-3 in a single launch (dispatch_small_kernel); with at most
// 2048 routing slots that launch also gathers x_perm. Otherwise three small
// kernels plus the gather, no atomics whose order matters:
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
  griddep_wait();
  griddep_launch_dependents();
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
  griddep_wait();
  griddep_launch_dependents();
  // per expert, the exclusive scan over the blocks' counts; the counts of 16
  // blocks are loaded before any of them is overwritten, so a scan over many
  // blocks takes one memory round trip per 16 of them
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = 0;
    for (int64_t c0 = 0; c0 < nchunks; c0 += 16) {
      int32_t v[16];
#pragma unroll
      for (int q = 0; q < 16; ++q)
        v[q] = c0 + q < nchunks ? chunk_base[(c0 + q) * E + e] : 0;
#pragma unroll
      for (int q = 0; q < 16; ++q)
        if (c0 + q < nchunks) {
          chunk_base[(c0 + q) * E + e] = run;
          run += v[q];
        }
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
  griddep_wait();
  griddep_launch_dependents();
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

// Block-wide exclusive scan of v over threads (blockDim.x == 1024). Returns
// the sum of the values before this thread; *total gets the sum of all.
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t* warp_sums,
                                                        int32_t* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
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
    warp_sums[lane] = s;
  }
  __syncthreads();
  *total = warp_sums[31];
  return (wid > 0 ? warp_sums[wid - 1] : 0) + incl - v;
}

// Steps 1-3 in one block for a batch whose masks fit in shared memory:
// mask[e*W + w] bit b = token 32w + b chose e; pre[e*W + w] = set bits of
// expert e in words before w. rank of token t in expert e = pre + bits below t.
// With x_perm given (few routing slots), the gather is done in the same
// launch: every block of the grid repeats steps 1-3 in its own shared memory
// (the result does not depend on the block), block 0 alone writes them out,
// and each block copies the token rows of its own run of slots.
__global__ void __launch_bounds__(1024)
    dispatch_small_kernel(const int32_t* __restrict__ idx, int T, int k, int E, int N,
                          int W, int32_t* __restrict__ counts,
                          int32_t* __restrict__ offsets, int32_t* __restrict__ row_token,
                          int32_t* __restrict__ slot_row, int64_t rows_cap,
                          int32_t* err, int32_t* __restrict__ tile_start, int tile_gu,
                          int tile_dn, const uint4* __restrict__ x,
                          uint4* __restrict__ x_perm, int64_t vec_per_row) {
  extern __shared__ uint32_t sm[];
  uint32_t* mask = sm;
  int32_t* pre = reinterpret_cast<int32_t*>(sm + (size_t)E * W);
  int32_t* s_off = pre + (size_t)E * W;
  __shared__ int32_t warp_sums[32];
  const bool lead = blockIdx.x == 0;  // the block that writes the results
  if (!lead) err = nullptr;
  griddep_wait();
  griddep_launch_dependents();
  // one thread per routing slot s (token s / k): every slot's expert id is
  // one load, and a thread's first slot stays in a register for the ranks
  const int Tk = T * k;
  const int e_first = (int)threadIdx.x < Tk ? idx[threadIdx.x] : -1;
  for (int i = threadIdx.x; i < E * W; i += blockDim.x) mask[i] = 0u;
  __syncthreads();
  for (int s = threadIdx.x; s < Tk; s += blockDim.x) {
    const int e = s == (int)threadIdx.x ? e_first : idx[s];
    const int t = s / k;
    if (e < 0 || e >= E) {
      record_error(err, kErrBadExpertId);
      continue;
    }
    const uint32_t bit = 1u << (t & 31);
    const uint32_t old = atomicOr(&mask[e * W + (t >> 5)], bit);
    if (old & bit) record_error(err, kErrBadExpertId);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = 0;
    for (int w = 0; w < W; ++w) {
      pre[e * W + w] = run;
      run += __popc(mask[e * W + w]);
    }
    if (lead) counts[e] = run;
    if (e < N) s_off[e] = run;
  }
  __syncthreads();
  int32_t R = 0;
  const int32_t v = ((int)threadIdx.x < N) ? s_off[threadIdx.x] : 0;
  const int32_t before = block_exclusive_scan(v, warp_sums, &R);
  __syncthreads();
  if ((int)threadIdx.x < N) {
    s_off[threadIdx.x] = before;
    if (lead) offsets[threadIdx.x] = before;
  }
  if (lead && threadIdx.x == 0) offsets[N] = R;
  __syncthreads();
  if (x_perm) {
    // this block's slots [s0, s1), each row cut into `seg` pieces so that
    // every warp copies about one piece, four 16-byte vectors per lane in
    // flight
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int per = (Tk + (int)gridDim.x - 1) / (int)gridDim.x;
    const int s0 = (int)blockIdx.x * per, s1 = min(Tk, s0 + per);
    const int seg = per >= 32 ? 1 : 32 / per;
    const int64_t seg_len = (vec_per_row + seg - 1) / seg;
    for (int item = warp; item < (s1 - s0) * seg; item += 32) {
      const int s = s0 + item / seg;
      const int e = idx[s];
      if (e < 0 || e >= N) continue;
      const int t = s / k;
      const int w = t >> 5;
      const int r = s_off[e] + pre[e * W + w] + __popc(mask[e * W + w] & ((1u << (t & 31)) - 1u));
      const int64_t q0 = (int64_t)(item % seg) * seg_len;
      const int64_t q1 = min(vec_per_row, q0 + seg_len);
      const uint4* src = x + (int64_t)t * vec_per_row;
      uint4* dst = x_perm + (int64_t)r * vec_per_row;
      for (int64_t q = q0 + lane; q < q1; q += 4 * 32) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (q + u * 32 < q1) v[u] = src[q + u * 32];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (q + u * 32 < q1) dst[q + u * 32] = v[u];
      }
    }
  }
  if (!lead) return;
  if (tile_start) {
    // the expert GEMMs' plans: token-tile prefixes of both GEMMs (v is the
    // count of routed expert threadIdx.x, 0 past N)
    int32_t tot = 0;
    const int32_t g = block_exclusive_scan((v + tile_gu - 1) / tile_gu, warp_sums, &tot);
    if ((int)threadIdx.x < N) tile_start[threadIdx.x] = g;
    if (threadIdx.x == 0) tile_start[N] = tot;
    __syncthreads();
    const int32_t dn = block_exclusive_scan((v + tile_dn - 1) / tile_dn, warp_sums, &tot);
    if ((int)threadIdx.x < N) tile_start[N + 1 + threadIdx.x] = dn;
    if (threadIdx.x == 0) {
      tile_start[2 * N + 1] = tot;
      tile_start[2 * N + 2] = 0;  // the CTA-pair GEMMs' unit counters
      tile_start[2 * N + 3] = 0;
    }
    __syncthreads();
  }
  for (int s = threadIdx.x; s < Tk; s += blockDim.x) {
    const int e = s == (int)threadIdx.x ? e_first : idx[s];
    const int t = s / k;
    const int w = t >> 5;
    int32_t r = -1;
    if (e >= 0 && e < N) {
      r = s_off[e] + pre[e * W + w] + __popc(mask[e * W + w] & ((1u << (t & 31)) - 1u));
      row_token[r] = t;
    }
    slot_row[s] = r;
  }
  for (int64_t r = R + threadIdx.x; r < rows_cap; r += blockDim.x) row_token[r] = -1;
}

// x_perm[r, :] = x[row_token[r], :] for r < R; one warp per row, 16-byte vectors.
__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint4* __restrict__ x,
                       const int32_t* __restrict__ row_token,
                       const int32_t* __restrict__ offsets, int N,
                       int64_t vec_per_row, int64_t rows_cap,
                       uint4* __restrict__ x_perm) {
  griddep_wait();
  griddep_launch_dependents();
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

constexpr size_t kSmallDispatchSmem = 96 * 1024;

size_t dispatch_small_smem(const Shape& sh) {
  const size_t W = (size_t)((sh.T + 31) / 32);
  return (2 * (size_t)sh.E * W + (size_t)sh.N) * sizeof(uint32_t);
}

bool dispatch_small_fits(const Shape& sh) {
  return sh.T <= 4096 && dispatch_small_smem(sh) <= kSmallDispatchSmem;
}

bool dispatch_plans_tiles(const Shape& sh) { return dispatch_small_fits(sh); }

// Batches of at most this many routing slots gather x_perm inside the
// one-block dispatch's launch (one warp per slot over the grid).
constexpr int64_t kSortGatherMaxSlots = 2048;

bool dispatch_gathers_in_sort(const Shape& sh) {
  return dispatch_small_fits(sh) && sh.T * sh.k <= kSortGatherMaxSlots;
}

int dispatch_launch_count(const Shape& sh) {
  return (dispatch_small_fits(sh) ? 1 : 3) + (sh.N > 0 && !dispatch_gathers_in_sort(sh) ? 1 : 0);
}

int num_sms() {  // of the current device, cached per device
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::atomic<int>& c = cache[dev & 63];
  int n = c.load();
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        n <= 0)
      n = 148;
    c.store(n);
  }
  return n;
}

cudaError_t launch_dispatch(const Shape& sh, const void* x, const int32_t* idx,
                            int32_t* chunk_base, int32_t* counts,
                            int32_t* offsets, int32_t* row_token,
                            int32_t* slot_row, void* x_perm, int32_t* err,
                            cudaStream_t st, int32_t* tile_start, int tile_gu,
                            int tile_dn) {
  const int E = (int)sh.E, N = (int)sh.N, k = (int)sh.k;
  cudaError_t e = cudaSuccess;
  if (dispatch_small_fits(sh)) {
    const int W = (int)((sh.T + 31) / 32);
    const size_t smem = dispatch_small_smem(sh);
    static std::atomic<uint64_t> attr_set{0};
    e = raise_smem_once(attr_set, dispatch_small_kernel, (int)kSmallDispatchSmem);
    if (e != cudaSuccess) return e;
    const bool gather = N > 0 && x_perm && dispatch_gathers_in_sort(sh);
    const int64_t slots = sh.T * sh.k;
    // a few slots per block: the redundant sorts run side by side, and the
    // copies spread over as many SMs
    int64_t nb = (slots + 3) / 4;
    if (nb > num_sms()) nb = num_sms();
    const unsigned blocks = gather ? (unsigned)(nb < 1 ? 1 : nb) : 1u;
    e = launch_pdl(dispatch_small_kernel, dim3(blocks), dim3(1024), smem, st, idx, (int)sh.T,
                   k, E, N, W, counts, offsets, row_token, slot_row, sh.T * sh.k, err,
                   tile_start, tile_gu, tile_dn, static_cast<const uint4*>(x),
                   gather ? static_cast<uint4*>(x_perm) : nullptr, sh.d * sh.es / 16);
    if (e != cudaSuccess) return e;
    if (gather) return cudaGetLastError();
  } else {
    const size_t smem = (size_t)E * kWords * sizeof(uint32_t);
    const unsigned nch = (unsigned)sh.nchunks;
    e = launch_pdl(dispatch_count_kernel, dim3(nch), dim3(kChunkTokens), smem, st, idx,
                   sh.T, k, E, chunk_base, err);
    if (e != cudaSuccess) return e;
    e = launch_pdl(dispatch_scan_kernel, dim3(1), dim3(1024), 0, st, chunk_base,
                   sh.nchunks, E, N, counts, offsets, row_token, sh.T * sh.k);
    if (e != cudaSuccess) return e;
    e = launch_pdl(dispatch_scatter_kernel, dim3(nch), dim3(kChunkTokens), smem, st, idx,
                   sh.T, k, E, N, chunk_base, offsets, row_token, slot_row);
    if (e != cudaSuccess) return e;
  }
  if (N > 0 && x_perm) {  // no x_perm: the GEMM gathers the rows itself
    const int64_t vpr = sh.d * sh.es / 16;
    int64_t rows = sh.T * sh.k;
    int64_t blocks = (rows + 7) / 8;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    e = launch_pdl(gather_rows_kernel, dim3((unsigned)blocks), dim3(256), 0, st,
                   static_cast<const uint4*>(x), row_token, offsets, N, vpr, rows,
                   static_cast<uint4*>(x_perm));
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace moe
