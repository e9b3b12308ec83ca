// Router: fp32-accumulated logits GEMM, correction bias, warp-level top-k and
// gates.
//
// LongCat-2.0 model card (archdb), "Mixture of experts": one router classifier
// [E, d] scores routed and zero experts together, with a per-expert
// e_score_correction_bias; 12 experts per token. The score function and the
// renormalisation are not disclosed there; the library uses the reading that
// the bias steers selection only and that the gates are the softmax of the
// selected raw logits (they sum to 1).
//
// Three ways to the logits, all with fp32 products and sums, each followed by
// the same warp top-k (warp_select_token):
//  - T <= 256 (decode): router_small_kernel, one launch. TMA-staged router
//    rows and x, FFMA partials per contraction split, and the split sums and
//    top-k done by the last CTA of each token group.
//  - otherwise router_logits_kernel + topk_kernel: a CUDA-core GEMM split
//    over blockIdx.z, partials to the workspace, added in a fixed order by the
//    top-k kernel (bit-reproducible run to run).
//  - bf16 with T >= 512: the logits on the tensor cores from an exact
//    three-plane bf16 split of the router weights (router_split_kernel + the
//    grouped GEMM), then topk_kernel.
// The top-k is one warp per token: the E keys sit in registers, ceil(E/32)
// per lane, sorted once per lane; k+1 rounds of a warp arg-max (ties to the
// lower id) give the selection in descending key order and the margin
// between the k-th and (k+1)-th key.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <float.h>
#include <math.h>

#include <atomic>

#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int RT = 64;   // tokens per CTA
constexpr int RE = 32;   // experts per CTA
constexpr int RK = 32;   // contraction chunk
constexpr int kRouterThreads = 256;

// Register staging of one 64-token x 32-k chunk of x (converted to fp32 when
// stored to shared memory) and one 32-expert x 32-k chunk of w_r.
template <typename XT>
struct XChunk;

// bf16 x: 64 tokens x 32 k = 256 vectors of 8 elements, one per thread.
template <>
struct XChunk<__nv_bfloat16> {
  uint4 v;
  __device__ __forceinline__ void load(const __nv_bfloat16* x, int64_t T, int64_t d,
                                       int64_t t0, int64_t k0, int64_t kend) {
    const int tt = threadIdx.x >> 2;
    const int kk = (threadIdx.x & 3) * 8;
    const int64_t t = t0 + tt, k = k0 + kk;
    v = make_uint4(0, 0, 0, 0);
    if (t < T && k < kend) v = *reinterpret_cast<const uint4*>(x + t * d + k);
  }
  __device__ __forceinline__ void store(float (*xs)[RT + 4]) const {
    const int tt = threadIdx.x >> 2;
    const int kk = (threadIdx.x & 3) * 8;
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xs[kk + 2 * i][tt] = __uint_as_float(w[i] << 16);
      xs[kk + 2 * i + 1][tt] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

// f32 x: 64 tokens x 32 k = 512 vectors of 4 elements, two per thread.
template <>
struct XChunk<float> {
  float4 v[2];
  __device__ __forceinline__ void load(const float* x, int64_t T, int64_t d, int64_t t0,
                                       int64_t k0, int64_t kend) {
#pragma unroll
    for (int rep = 0; rep < 2; ++rep) {
      const int v_id = threadIdx.x + rep * kRouterThreads;
      const int64_t t = t0 + (v_id >> 3), k = k0 + (v_id & 7) * 4;
      v[rep] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t < T && k < kend) v[rep] = *reinterpret_cast<const float4*>(x + t * d + k);
    }
  }
  __device__ __forceinline__ void store(float (*xs)[RT + 4]) const {
#pragma unroll
    for (int rep = 0; rep < 2; ++rep) {
      const int v_id = threadIdx.x + rep * kRouterThreads;
      const int tt = v_id >> 3, kk = (v_id & 7) * 4;
      xs[kk + 0][tt] = v[rep].x;
      xs[kk + 1][tt] = v[rep].y;
      xs[kk + 2][tt] = v[rep].z;
      xs[kk + 3][tt] = v[rep].w;
    }
  }
};

struct WChunk {  // 32 experts x 32 k floats = 256 float4, one per thread
  float4 v;
  __device__ __forceinline__ void load(const float* w_r, int64_t E, int64_t d,
                                       int64_t e0, int64_t k0, int64_t kend) {
    const int64_t e = e0 + (threadIdx.x >> 3), k = k0 + (threadIdx.x & 7) * 4;
    v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (e < E && k < kend) v = *reinterpret_cast<const float4*>(w_r + e * d + k);
  }
  __device__ __forceinline__ void store(float (*wsm)[RE + 4]) const {
    const int ee = threadIdx.x >> 3, kk = (threadIdx.x & 7) * 4;
    wsm[kk + 0][ee] = v.x;
    wsm[kk + 1][ee] = v.y;
    wsm[kk + 2][ee] = v.z;
    wsm[kk + 3][ee] = v.w;
  }
};

// part[z][t][e] = sum over this split's k of x[t,k] * w_r[e,k]  (fp32 FFMA).
// The next chunk is loaded into registers while the current one is used.
template <typename XT>
__global__ void __launch_bounds__(kRouterThreads)
    router_logits_kernel(const XT* __restrict__ x, const float* __restrict__ w_r,
                         float* __restrict__ part, int64_t T, int64_t d,
                         int64_t E, int64_t k_per_split) {
  __shared__ __align__(16) float xs[RK][RT + 4];
  __shared__ __align__(16) float wsm[RK][RE + 4];
  griddep_wait();
  const int tid = threadIdx.x;
  const int tx = tid & 15;  // expert pair
  const int ty = tid >> 4;  // token quad
  const int64_t e0 = (int64_t)blockIdx.x * RE;
  const int64_t t0 = (int64_t)blockIdx.y * RT;
  const int64_t kbeg = (int64_t)blockIdx.z * k_per_split;
  const int64_t kend = min(d, kbeg + k_per_split);

  // Blocked summation: each 32-term chunk is summed into a fresh partial that
  // is then added to the running total, which keeps the fp32 rounding error
  // of a d-term dot product ~sqrt(32) times below a single running sum.
  float acc[4][2];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = 0.f;

  XChunk<XT> xc;
  WChunk wc;
  if (kbeg < kend) {
    xc.load(x, T, d, t0, kbeg, kend);
    wc.load(w_r, E, d, e0, kbeg, kend);
  }
  for (int64_t k0 = kbeg; k0 < kend; k0 += RK) {
    xc.store(xs);
    wc.store(wsm);
    __syncthreads();
    if (k0 + RK < kend) {
      xc.load(x, T, d, t0, k0 + RK, kend);
      wc.load(w_r, E, d, e0, k0 + RK, kend);
    }
    float part_acc[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i) part_acc[i][0] = part_acc[i][1] = 0.f;
#pragma unroll 8
    for (int kk = 0; kk < RK; ++kk) {
      const float4 xv = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
      const float2 wv = *reinterpret_cast<const float2*>(&wsm[kk][tx * 2]);
      part_acc[0][0] = fmaf(xv.x, wv.x, part_acc[0][0]);
      part_acc[0][1] = fmaf(xv.x, wv.y, part_acc[0][1]);
      part_acc[1][0] = fmaf(xv.y, wv.x, part_acc[1][0]);
      part_acc[1][1] = fmaf(xv.y, wv.y, part_acc[1][1]);
      part_acc[2][0] = fmaf(xv.z, wv.x, part_acc[2][0]);
      part_acc[2][1] = fmaf(xv.z, wv.y, part_acc[2][1]);
      part_acc[3][0] = fmaf(xv.w, wv.x, part_acc[3][0]);
      part_acc[3][1] = fmaf(xv.w, wv.y, part_acc[3][1]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[i][0] += part_acc[i][0];
      acc[i][1] += part_acc[i][1];
    }
    __syncthreads();
  }
  griddep_launch_dependents();
  float* out = part + (int64_t)blockIdx.z * T * E;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int64_t e = e0 + tx * 2 + j;
      if (e < E) out[t * E + e] = acc[i][j];
    }
  }
}

// Order-preserving map of a float to uint32 (a < b  <=>  ord(a) < ord(b) for
// non-NaN values; -inf maps to 0x007fffff, so 0 is below every key).
__device__ __forceinline__ uint32_t ord_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Correction bias of experts lane + 32 i (0 past E), loaded ahead of the
// selection so that its latency overlaps other work.
template <int PL>
__device__ __forceinline__ void load_bias(const float* __restrict__ bias, int E, int lane,
                                          float (&bv)[PL]) {
#pragma unroll
  for (int i = 0; i < PL; ++i) bv[i] = (lane + 32 * i < E) ? bias[lane + 32 * i] : 0.f;
}

__device__ __forceinline__ float ord_key_inv(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

// Sorts a lane's (key, id) pairs so that larger keys come first and, among
// equal keys, lower ids (a bitonic network; N is a power of two).
template <int N>
__device__ __forceinline__ void sort_pairs_desc(uint32_t (&o)[N], int (&id)[N]) {
#pragma unroll
  for (int size = 2; size <= N; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          const bool i_first = o[i] > o[j] || (o[i] == o[j] && id[i] < id[j]);
          const bool swap = ((i & size) == 0) ? !i_first : i_first;
          const uint32_t oi = o[i], oj = o[j];
          const int di = id[i], dj = id[j];
          o[i] = swap ? oj : oi;
          o[j] = swap ? oi : oj;
          id[i] = swap ? dj : di;
          id[j] = swap ? di : dj;
        }
      }
}

// Top-k of one token by one warp, from its logits lg[i] of experts
// lane + 32 i: keys = logits + bias, k+1 rounds of a warp arg-max (ties to the
// lower id), gates = softmax of the selected raw logits, and the near-tie flag.
// Each lane first sorts its own keys, so a round is two warp reductions over
// the lanes' heads: the largest key, then the lowest id holding it; the
// winning lane drops its head. Writes logits_out (if given), idx_out,
// gate_out and flags (if given) of t.
template <int PL>
__device__ __forceinline__ void warp_select_token(const float (&lg)[PL],
                                                  const float (&bv)[PL],
                                                  float* __restrict__ logits_out,
                                                  int32_t* __restrict__ idx_out,
                                                  float* __restrict__ gate_out,
                                                  uint8_t* __restrict__ flags, int64_t t,
                                                  int E, int k, int lane) {
  // ordered keys: a NaN key counts as -inf; 0 marks an empty slot, below the
  // key of -inf
  uint32_t o[PL];
  int id[PL];
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const int e = lane + 32 * i;
    o[i] = 0u;
    id[i] = 0x7fffffff;
    if (e < E) {
      const float kv = lg[i] + bv[i];
      o[i] = ord_key((kv != kv) ? -INFINITY : kv);
      id[i] = e;
      if (logits_out) logits_out[t * E + e] = lg[i];
    }
  }
  sort_pairs_desc<PL>(o, id);

  uint32_t kth_o = 0u, next_o = 0u;
  int my_e = 0;
  const int rounds = (k < E) ? k + 1 : k;  // never more than the E real keys
  for (int j = 0; j < rounds; ++j) {
    const uint32_t mo = __reduce_max_sync(0xffffffffu, o[0]);
    const uint32_t we = __reduce_min_sync(0xffffffffu, o[0] == mo ? (uint32_t)id[0] : 0xffffffffu);
    if (lane == (int)(we & 31u)) {
#pragma unroll
      for (int i = 0; i + 1 < PL; ++i) {
        o[i] = o[i + 1];
        id[i] = id[i + 1];
      }
      o[PL - 1] = 0u;
      id[PL - 1] = 0x7fffffff;
    }
    if (j < k) {
      if (lane == j) my_e = (int)we;
      kth_o = mo;
    } else {
      next_o = mo;
    }
  }
  // raw logit of this lane's pick, from the lane that holds it
  float my_logit = 0.f;
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const float v = __shfl_sync(0xffffffffu, lg[i], my_e & 31);
    if ((my_e >> 5) == i) my_logit = v;
  }

  // gates: softmax of the selected raw logits
  float m = (lane < k) ? my_logit : -INFINITY;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float p = (lane < k) ? expf(my_logit - m) : 0.f;
  float zsum = p;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    zsum += __shfl_xor_sync(0xffffffffu, zsum, off);
  if (lane < k) {
    idx_out[t * k + lane] = my_e;
    gate_out[t * k + lane] = p / zsum;
  }
  if (flags && lane == 0) {
    const float margin = (k < E) ? ord_key_inv(kth_o) - ord_key_inv(next_o) : INFINITY;
    flags[t] = (margin < 1e-4f) ? 1 : 0;
  }
}


template <int PL>
__global__ void __launch_bounds__(256)
    topk_kernel(const float* __restrict__ part, int n_outer, int64_t outer_stride,
                int n_inner, int64_t inner_stride, int64_t row_stride,
                const float* __restrict__ bias, float* __restrict__ logits_out,
                int32_t* __restrict__ idx_out, float* __restrict__ gate_out,
                uint8_t* __restrict__ flags, int64_t T, int E, int k) {
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  griddep_launch_dependents();
  if (t >= T) return;
  float bv[PL];
  load_bias<PL>(bias, E, lane, bv);

  // logits = partial sums added in a fixed order (outer, then inner index),
  // so results are reproducible; the loads of several partials are issued
  // together
  float lg[PL];
#pragma unroll
  for (int i = 0; i < PL; ++i) lg[i] = 0.f;
  const float* pt = part + t * row_stride + lane;
  for (int zo = 0; zo < n_outer; ++zo) {
#pragma unroll 4
    for (int zi = 0; zi < n_inner; ++zi) {
      const float* pz = pt + zo * outer_stride + zi * inner_stride;
#pragma unroll
      for (int i = 0; i < PL; ++i)
        if (lane + 32 * i < E) lg[i] += pz[32 * i];
    }
  }
  warp_select_token<PL>(lg, bv, logits_out, idx_out, gate_out, flags, t, E, k, lane);
}

template <int PL>
void launch_topk(const float* part, int n_outer, int64_t outer_stride, int n_inner,
                 int64_t inner_stride, int64_t row_stride, const float* bias,
                 float* logits, int32_t* idx, float* gate, uint8_t* flags,
                 int64_t T, int E, int k, cudaStream_t st) {
  const int warps = 8;
  const unsigned grid = (unsigned)((T + warps - 1) / warps);
  launch_pdl(topk_kernel<PL>, dim3(grid), dim3(warps * 32), 0, st, part, n_outer,
             outer_stride, n_inner, inner_stride, row_stride, bias,
             logits, idx, gate, flags, T, E, k);
}

// ------------------------------------------------------- small batches --
// Router for T <= 256 in one launch. CTA (g, et, z) takes the 8 tokens of
// group g, the 32 experts of tile et and the contraction range
// [z * ksplit, (z + 1) * ksplit). The host picks ksplit (a multiple of 32) so
// that the grid fills the SMs once where shared memory allows. One thread
// brings the CTA's router rows (a 32 x 256 box) and x rows (an 8 x 256 box)
// into shared memory by TMA, chunk by chunk, one mbarrier per chunk, so the
// arithmetic on a chunk starts as soon as that chunk has landed; rows past E
// or T and columns past d arrive as zeros. Each warp
// computes 4 experts x 8 tokens with lanes along the contraction; a warp tree
// adds the lanes, and the partial sums of the splits go to the workspace. The
// last CTA to finish a token group (a counter per group, incremented after a
// fence) adds the partials of its 8 tokens in split order and runs their
// top-k, then resets the counter to zero for the next call. No CTA waits for
// another. A chunk that has not landed within the wait limit sets the error
// word; the CTA still takes its turn on the counter, so the counters stay
// consistent.
constexpr int DG = 8;             // tokens per group
constexpr int DE = 32;            // experts per CTA (8 warps x 4)
constexpr int kSmallChunk = 256;  // contraction elements per mbarrier
constexpr int kSmallHeader = 128; // shared bytes before the first chunk
constexpr int kSmallMaxBytes = 220 * 1024;  // shared memory budget of one CTA
constexpr int kSmallMaxChunks = (kSmallHeader - 16) / 8;
constexpr uint64_t kSmallWaitNs = 2000000000ull;  // wait limit for a chunk

__device__ __forceinline__ bool wait_chunk(uint32_t bar, volatile int* abort_flag,
                                           int32_t* err) {
  if (ptx::mbar_try_wait(bar, 0)) return true;
  const uint64_t t0 = ptx::global_timer_ns();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (ptx::mbar_try_wait(bar, 0)) return true;
    if (*abort_flag) return false;
    if (ptx::global_timer_ns() - t0 > kSmallWaitNs) {
      *abort_flag = 1;
      atomicCAS(err, 0, kErrWaitTimeout);
      return false;
    }
  }
}

// 4 consecutive x values of one token from shared memory, as fp32
template <typename XT>
__device__ __forceinline__ float4 ld_x4(const XT* p);
template <>
__device__ __forceinline__ float4 ld_x4<__nv_bfloat16>(const __nv_bfloat16* p) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                     __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
}
template <>
__device__ __forceinline__ float4 ld_x4<float>(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}

template <typename XT, int PL>
__global__ void __launch_bounds__(256, 1)
    router_small_kernel(const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_x,
                        const float* __restrict__ bias, float* __restrict__ part,
                        int32_t* __restrict__ counter, int32_t* __restrict__ err,
                        float* __restrict__ logits_out, int32_t* __restrict__ idx_out,
                        float* __restrict__ gate_out, uint8_t* __restrict__ flags, int T,
                        int d, int E, int k, int ksplit) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + kSmallHeader - 8);
  int* s_last = reinterpret_cast<int*>(smem + kSmallHeader - 4);
  // chunk c: router rows [DE][256] fp32, then x rows [DG][256]
  constexpr int kWBytes = DE * kSmallChunk * 4;
  constexpr int kChunkBytes = kWBytes + DG * kSmallChunk * (int)sizeof(XT);
  uint8_t* chunks = smem + kSmallHeader;
  const int g = blockIdx.x, et = blockIdx.y, z = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = g * DG, e0 = et * DE;
  const int kbeg = z * ksplit;
  const int klen = min(d, kbeg + ksplit) - kbeg;  // > 0, a multiple of 8
  const int nch = (klen + kSmallChunk - 1) / kSmallChunk;
  const int nt = min(DG, T - t0);
  if (threadIdx.x == 0) {
    ptx::prefetch_tensormap(&tm_w);
    ptx::prefetch_tensormap(&tm_x);
    for (int c = 0; c < nch; ++c) ptx::mbar_init(ptx::smem_addr(&bars[c]), 1);
    *s_abort = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    // both are re-read by other CTAs: router rows by every token group, x by
    // every expert tile
    const uint64_t pol = ptx::policy_evict_last();
    for (int c = 0; c < nch; ++c) {
      const uint32_t bar = ptx::smem_addr(&bars[c]);
      const uint32_t dst = ptx::smem_addr(chunks + (size_t)c * kChunkBytes);
      ptx::mbar_arrive_expect_tx(bar, (uint32_t)kChunkBytes);
      ptx::tma_load_2d(&tm_w, dst, bar, kbeg + c * kSmallChunk, e0, pol);
      ptx::tma_load_2d(&tm_x, dst + kWBytes, bar, kbeg + c * kSmallChunk, t0, pol);
    }
  }
  float bv[PL];
  load_bias<PL>(bias, E, lane, bv);

  // Each accumulator adds its products in ascending k; columns of a chunk
  // past this split's end are loaded but not used.
  float acc[4][DG];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int tt = 0; tt < DG; ++tt) acc[j][tt] = 0.f;
  for (int c = 0; c < nch; ++c) {
    if (!wait_chunk(ptx::smem_addr(&bars[c]), s_abort, err)) break;
    const float* wrow = reinterpret_cast<const float*>(chunks + (size_t)c * kChunkBytes) +
                        warp * 4 * kSmallChunk;
    const XT* xrow = reinterpret_cast<const XT*>(chunks + (size_t)c * kChunkBytes + kWBytes);
    const int cl = min(kSmallChunk, klen - c * kSmallChunk);
#pragma unroll
    for (int h = 0; h < kSmallChunk / 128; ++h) {
      if (128 * h + 4 * lane < cl) {
        const int kk = 128 * h + 4 * lane;
        float4 w4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          w4[j] = *reinterpret_cast<const float4*>(wrow + j * kSmallChunk + kk);
#pragma unroll
        for (int tt = 0; tt < DG; ++tt) {
          const float4 xv = ld_x4<XT>(xrow + tt * kSmallChunk + kk);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc[j][tt] = fmaf(w4[j].x, xv.x, acc[j][tt]);
            acc[j][tt] = fmaf(w4[j].y, xv.y, acc[j][tt]);
            acc[j][tt] = fmaf(w4[j].z, xv.z, acc[j][tt]);
            acc[j][tt] = fmaf(w4[j].w, xv.w, acc[j][tt]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = e0 + warp * 4 + j;
    if (e >= E) break;
#pragma unroll
    for (int tt = 0; tt < DG; ++tt)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        acc[j][tt] += __shfl_xor_sync(0xffffffffu, acc[j][tt], off);
    if (lane < nt) {
      float v = acc[j][0];
#pragma unroll
      for (int tt = 1; tt < DG; ++tt)
        if (lane == tt) v = acc[j][tt];
      part[((int64_t)z * T + t0 + lane) * E + e] = v;
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    if (*s_abort)  // copies may still be in flight: give them the wait limit
      for (int c = 0; c < nch; ++c) {
        const uint64_t tw = ptx::global_timer_ns();
        while (!ptx::mbar_try_wait(ptx::smem_addr(&bars[c]), 0))
          if (ptx::global_timer_ns() - tw > kSmallWaitNs) break;
      }
    *s_last = atomicAdd(&counter[g], 1) == (int)(gridDim.y * gridDim.z) - 1;
  }
  __syncthreads();
  if (!*s_last) return;
  __threadfence();
  // split sums of the group's tokens into shared memory (the chunks are
  // done): (token, expert) elements spread over the threads, each added in
  // ascending split order; a thread has the loads of 8 elements x 4 splits in
  // flight at once, so a group of up to 2048 elements takes one round trip
  // per 4 splits
  float* lgs = reinterpret_cast<float*>(chunks);  // [DG][E]
  const int nz = (int)gridDim.z;
  const int nel = nt * E;
  const int64_t zstride = (int64_t)T * E;
  const float* pbase = part + (int64_t)t0 * E;  // rows t0.. are contiguous
  for (int el0 = threadIdx.x; el0 < nel; el0 += 8 * blockDim.x) {
    float sum[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) sum[r] = 0.f;
    for (int z0 = 0; z0 < nz; z0 += 4) {
      float v[8][4];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int el = el0 + r * (int)blockDim.x;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          v[r][q] = (el < nel && z0 + q < nz) ? __ldcg(pbase + (z0 + q) * zstride + el) : 0.f;
      }
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (z0 + q < nz) sum[r] += v[r][q];
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int el = el0 + r * (int)blockDim.x;
      if (el < nel) lgs[el] = sum[r];
    }
  }
  __syncthreads();
  if (warp < nt) {
    float lg[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) lg[i] = (lane + 32 * i < E) ? lgs[warp * E + lane + 32 * i] : 0.f;
    warp_select_token<PL>(lg, bv, logits_out, idx_out, gate_out, flags, t0 + warp, E, k, lane);
  }
  if (threadIdx.x == 0) counter[g] = 0;
}

// Row of plane p (0 hi, 1 mid, 2 lo) of expert e in the tensor-core router's
// A operand: each 32-row quarter of a 128-row tile holds the three planes of
// 10 experts side by side (rows 3j, 3j + 1, 3j + 2; rows 30 and 31 are
// zeros), so the GEMM's epilogue adds an expert's planes inside one warp.
__host__ __device__ __forceinline__ int64_t plane_row(int64_t e, int p) {
  return (e / 40) * 128 + ((e % 40) / 10) * 32 + 3 * (e % 10) + p;
}

// Exact three-way split of the fp32 router weights into bf16 planes for the
// tensor-core router: hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid)
// (each difference is exact in fp32), so hi + mid + lo carries the 24 bits of
// w and x . w = x . hi + x . mid + x . lo with x in bf16 and every product
// exact in fp32. Plane p of expert e goes to row plane_row(e, p); every other
// row up to Ep is zeros. Also writes the one-expert plan of the GEMM.
__global__ void __launch_bounds__(256)
    router_split_kernel(const float4* __restrict__ w_r, int64_t E, int64_t d, int64_t Ep,
                        uint2* __restrict__ planes, int32_t* __restrict__ plan,
                        int64_t T, int tile) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t q = d / 4;  // float4 per row
  // one row of A per block at a time: expert rows are split, padding rows
  // (rows 30 and 31 of a quarter, and the unused experts of the last tile)
  // zeroed
  for (int64_t r = blockIdx.x; r < Ep; r += gridDim.x) {
    const int64_t l = r % 32;  // row inside its quarter
    const int64_t e = (r / 128) * 40 + ((r % 128) / 32) * 10 + l / 3;
    if (l >= 30 || e >= E)
      for (int64_t c4 = threadIdx.x; c4 < q; c4 += blockDim.x)
        planes[r * q + c4] = make_uint2(0u, 0u);
  }
  for (int64_t e = blockIdx.x; e < E; e += gridDim.x) {
    const int64_t hi_row = plane_row(e, 0) * q, mid_row = plane_row(e, 1) * q,
                  lo_row = plane_row(e, 2) * q;
    for (int64_t c4 = threadIdx.x; c4 < q; c4 += blockDim.x) {
      const float4 w = w_r[e * q + c4];
      const float v[4] = {w.x, w.y, w.z, w.w};
      uint16_t hb[4], mb[4], lb[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat16 h = __float2bfloat16_rn(v[j]);
        const float r1 = v[j] - __bfloat162float(h);
        const __nv_bfloat16 m = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(m);
        const __nv_bfloat16 l = __float2bfloat16_rn(r2);
        hb[j] = __bfloat16_as_ushort(h);
        mb[j] = __bfloat16_as_ushort(m);
        lb[j] = __bfloat16_as_ushort(l);
      }
      auto pack = [](const uint16_t* b) {
        return make_uint2((uint32_t)b[0] | ((uint32_t)b[1] << 16),
                          (uint32_t)b[2] | ((uint32_t)b[3] << 16));
      };
      planes[hi_row + c4] = pack(hb);
      planes[mid_row + c4] = pack(mb);
      planes[lo_row + c4] = pack(lb);
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    plan[0] = 0;
    plan[1] = (int32_t)T;
    plan[2] = 0;
    plan[3] = (int32_t)((T + tile - 1) / tile);
  }
}

}  // namespace

// The router runs on the tensor cores (three bf16 planes, fp32 accumulation)
// for bf16 batches large enough to fill the GPU; small batches and fp32
// activations use the CUDA-core split-K kernel.
constexpr int64_t kTcRouterMinTokens = 512;

int64_t router_planes_rows(const Shape& sh) { return (sh.E + 39) / 40 * 128; }

// The tensor-core router restarts its fp32 accumulation every 1024 contraction
// elements (16 blocks of 64), a chain of 64 MMA steps per partial.
static int router_kb_chunk(const Shape& sh) {
  const int kb = (int)(sh.d / 64);
  if (kb < 1) return 1;  // d < 64: the tensor-core router is not used, but sizes stay defined
  int c = kb < 16 ? kb : 16;
  while (kb % c != 0) --c;
  return c;
}

int router_tc_chunks(const Shape& sh) { return (int)(sh.d / 64) / router_kb_chunk(sh); }

bool router_uses_tensor_cores(const Shape& sh) {
  return sh.bf16 && sh.d % 128 == 0 && sh.T >= kTcRouterMinTokens &&
         router_planes_rows(sh) <= 4096;
}

constexpr int64_t kSmallRouterMaxTokens = 256;

bool router_uses_small_kernel(const Shape& sh) { return sh.T <= kSmallRouterMaxTokens; }

// Contraction split of the small-batch router: as many splits as fill the
// SMs once with the (token group, expert tile) pairs, at least enough that a
// CTA's rows fit its shared-memory budget, and at most one per 256 elements.
// Returns the number of splits; *ksplit (if given) gets their length.
int small_chunk_bytes(const Shape& sh) {
  return DE * kSmallChunk * 4 + DG * kSmallChunk * (sh.bf16 ? 2 : 4);
}

int router_small_plan(const Shape& sh, int* ksplit_out) {
  int64_t base = ((sh.T + DG - 1) / DG) * ((sh.E + DE - 1) / DE);
  if (base < 1) base = 1;  // an empty batch still gets a valid plan
  int64_t chunks = (kSmallMaxBytes - kSmallHeader) / small_chunk_bytes(sh);
  if (chunks > kSmallMaxChunks) chunks = kSmallMaxChunks;
  const int64_t kmax = chunks * kSmallChunk;
  int64_t n = num_sms() / base;
  const int64_t n_min = (sh.d + kmax - 1) / kmax;
  const int64_t n_max = (sh.d + kSmallChunk - 1) / kSmallChunk;
  if (n > n_max) n = n_max;
  if (n < n_min) n = n_min;
  if (n < 1) n = 1;
  int64_t ks = (sh.d + n - 1) / n;
  ks = (ks + 31) / 32 * 32;
  if (ksplit_out) *ksplit_out = (int)ks;
  return (int)((sh.d + ks - 1) / ks);
}

int router_small_splits(const Shape& sh) { return router_small_plan(sh, nullptr); }

// The CUDA-core logits GEMM puts token tiles of RT on grid.y (at most 65535).
bool router_simt_grid_fits(const Shape& sh) { return (sh.T + RT - 1) / RT <= 65535; }

bool router_grid_fits(const Shape& sh) {
  if (router_uses_tensor_cores(sh) || router_uses_small_kernel(sh)) return true;
  return router_simt_grid_fits(sh);
}

int router_launch_count(const Shape& sh) {
  return router_uses_tensor_cores(sh) ? 3 : (router_uses_small_kernel(sh) ? 1 : 2);
}

// Number of contraction splits so that the logits GEMM has >= ~2 CTAs per SM.
int router_splits(const Shape& sh) {
  int64_t tiles = ((sh.E + RE - 1) / RE) * ((sh.T + RT - 1) / RT);
  if (tiles < 1) tiles = 1;  // an empty batch still gets a valid plan
  int64_t want = (2 * num_sms() + tiles - 1) / tiles;
  int64_t max_split = (sh.d + 255) / 256;  // >= 256 k per split
  if (max_split > 16) max_split = 16;
  if (want > max_split) want = max_split;
  if (want < 1) want = 1;
  return (int)want;
}

PFN_cuTensorMapEncodeTiled_v12000 router_map_encoder() {
  static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
  if (!fn.load()) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn.store(reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p));
  }
  return fn.load();
}

// Tensor maps of the small-batch router: router rows [E, d] fp32 in boxes of
// 32 rows x 256 columns, x [T, d] in boxes of 8 rows x 256 columns; no
// swizzle, out-of-range elements read as zero.
bool make_router_maps(const Shape& sh, const void* x, const float* w_r, CUtensorMap* tm_w,
                      CUtensorMap* tm_x) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = router_map_encoder();
  if (!enc) return false;
  const cuuint32_t estr[2] = {1, 1};
  const cuuint64_t wdims[2] = {(cuuint64_t)sh.d, (cuuint64_t)sh.E};
  const cuuint64_t wstr[1] = {(cuuint64_t)sh.d * 4};
  const cuuint32_t wbox[2] = {(cuuint32_t)kSmallChunk, (cuuint32_t)DE};
  if (enc(tm_w, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(w_r), wdims, wstr, wbox,
          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  const int es = sh.bf16 ? 2 : 4;
  const cuuint64_t xdims[2] = {(cuuint64_t)sh.d, (cuuint64_t)sh.T};
  const cuuint64_t xstr[1] = {(cuuint64_t)sh.d * es};
  const cuuint32_t xbox[2] = {(cuuint32_t)kSmallChunk, (cuuint32_t)DG};
  return enc(tm_x, sh.bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
             2, const_cast<void*>(x), xdims, xstr, xbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename XT, int PL>
cudaError_t launch_small(dim3 grid, size_t smem, cudaStream_t st, const CUtensorMap& tm_w,
                         const CUtensorMap& tm_x, const float* bias, float* part, int32_t* counter, int32_t* err,
                         float* logits_out, int32_t* idx, float* gate, uint8_t* flags, int T,
                         int d, int E, int k, int ksplit) {
  static std::atomic<uint64_t> attr_set{0};
  const cudaError_t a = raise_smem_once(attr_set, router_small_kernel<XT, PL>, kSmallMaxBytes);
  if (a != cudaSuccess) return a;
  return launch_pdl(router_small_kernel<XT, PL>, grid, dim3(256), smem, st, tm_w, tm_x, bias,
                    part, counter, err, logits_out, idx, gate, flags, T, d, E, k, ksplit);
}

cudaError_t launch_router(const Shape& sh, const void* x, const float* w_r,
                          const float* bias, float* part, int32_t* idx,
                          float* gate, uint8_t* flags, float* logits_out,
                          void* planes, int32_t* plan, int32_t* err,
                          cudaStream_t st) {
  int n_outer, n_inner;
  int64_t outer_stride, inner_stride, row_stride;
  cudaError_t e;
  if (router_uses_small_kernel(sh)) {
    // one launch: logits, split sums and top-k; the group counters live in
    // the workspace header after the error word (zero between calls)
    int ksplit = 0;
    const int nsplit = router_small_plan(sh, &ksplit);
    const dim3 grid((unsigned)((sh.T + DG - 1) / DG), (unsigned)((sh.E + DE - 1) / DE),
                    (unsigned)nsplit);
    const size_t smem = (size_t)kSmallHeader +
                        (size_t)((ksplit + kSmallChunk - 1) / kSmallChunk) * small_chunk_bytes(sh);
    CUtensorMap tm_w, tm_x;
    if (!make_router_maps(sh, x, w_r, &tm_w, &tm_x)) return cudaErrorInvalidValue;
    int32_t* counter = err + 2;
    const int pl = (int)((sh.E + 31) / 32);
    const int E = (int)sh.E, k = (int)sh.k;
#define MOE_SMALL(XT, P)                                                                \
  launch_small<XT, P>(grid, smem, st, tm_w, tm_x, bias, part, counter, err, logits_out, idx, \
                      gate, flags, (int)sh.T, (int)sh.d, E, k, ksplit)
#define MOE_SMALL_PL(XT)                    \
  (pl <= 1    ? MOE_SMALL(XT, 1)            \
   : pl <= 2  ? MOE_SMALL(XT, 2)            \
   : pl <= 4  ? MOE_SMALL(XT, 4)            \
   : pl <= 8  ? MOE_SMALL(XT, 8)            \
   : pl <= 16 ? MOE_SMALL(XT, 16)           \
              : MOE_SMALL(XT, 32))
    e = sh.bf16 ? MOE_SMALL_PL(__nv_bfloat16) : MOE_SMALL_PL(float);
#undef MOE_SMALL_PL
#undef MOE_SMALL
    return e;
  }
  if (router_uses_tensor_cores(sh)) {
    const int64_t Ep = router_planes_rows(sh);
    int64_t blocks = Ep;  // rows of the planes, one block per row at a time
    if (blocks > 4 * num_sms()) blocks = 4 * num_sms();
    e = launch_pdl(router_split_kernel, dim3((unsigned)blocks), dim3(256), 0, st,
                   reinterpret_cast<const float4*>(w_r), sh.E, sh.d, Ep,
                   static_cast<uint2*>(planes), plan, sh.T, kRouterGemmTile);
    if (e != cudaSuccess) return e;
    e = launch_dense_gemm_tc(planes, Ep, x, sh.T, sh.d, router_kb_chunk(sh), sh.E, part,
                             plan, err, st);
    if (e != cudaSuccess) return e;
    // part[t, c * E + e]: chunk c, the three planes already added
    n_outer = router_tc_chunks(sh);
    outer_stride = sh.E;
    n_inner = 1;
    inner_stride = 0;
    row_stride = (int64_t)n_outer * sh.E;
  } else {
    const int nsplit = router_splits(sh);
    int64_t kps = (sh.d + nsplit - 1) / nsplit;
    kps = (kps + RK - 1) / RK * RK;
    dim3 grid((unsigned)((sh.E + RE - 1) / RE), (unsigned)((sh.T + RT - 1) / RT),
              (unsigned)nsplit);
    if (sh.bf16)
      e = launch_pdl(router_logits_kernel<__nv_bfloat16>, grid, dim3(kRouterThreads), 0, st,
                     static_cast<const __nv_bfloat16*>(x), w_r, part, sh.T, sh.d, sh.E,
                     kps);
    else
      e = launch_pdl(router_logits_kernel<float>, grid, dim3(kRouterThreads), 0, st,
                     static_cast<const float*>(x), w_r, part, sh.T, sh.d, sh.E, kps);
    if (e != cudaSuccess) return e;
    n_outer = nsplit;
    outer_stride = sh.T * sh.E;
    n_inner = 1;
    inner_stride = 0;
    row_stride = sh.E;
  }
  const int pl = (int)((sh.E + 31) / 32);
  const int E = (int)sh.E, k = (int)sh.k;
#define MOE_TOPK(P)                                                                 \
  launch_topk<P>(part, n_outer, outer_stride, n_inner, inner_stride, row_stride, bias, \
                 logits_out, idx, gate, flags, sh.T, E, k, st)
  if (pl <= 1)
    MOE_TOPK(1);
  else if (pl <= 2)
    MOE_TOPK(2);
  else if (pl <= 4)
    MOE_TOPK(4);
  else if (pl <= 8)
    MOE_TOPK(8);
  else if (pl <= 16)
    MOE_TOPK(16);
  else
    MOE_TOPK(32);
#undef MOE_TOPK
  return cudaGetLastError();
}

// The CUDA-core router with a caller-chosen number of contraction splits and
// caller-provided scratch `part` of nsplit * T * E floats (used by the
// entry point that allocates nothing).
cudaError_t launch_router_simt(const Shape& sh, const void* x, const float* w_r,
                               const float* bias, float* part, int nsplit,
                               int32_t* idx, float* gate, uint8_t* flags,
                               float* logits_out, cudaStream_t st) {
  int64_t kps = (sh.d + nsplit - 1) / nsplit;
  kps = (kps + RK - 1) / RK * RK;
  dim3 grid((unsigned)((sh.E + RE - 1) / RE), (unsigned)((sh.T + RT - 1) / RT),
            (unsigned)nsplit);
  cudaError_t e;
  if (sh.bf16)
    e = launch_pdl(router_logits_kernel<__nv_bfloat16>, grid, dim3(kRouterThreads), 0, st,
                   static_cast<const __nv_bfloat16*>(x), w_r, part, sh.T, sh.d, sh.E, kps);
  else
    e = launch_pdl(router_logits_kernel<float>, grid, dim3(kRouterThreads), 0, st,
                   static_cast<const float*>(x), w_r, part, sh.T, sh.d, sh.E, kps);
  if (e != cudaSuccess) return e;
  const int64_t split_stride = sh.T * sh.E;
  const int pl = (int)((sh.E + 31) / 32);
  const int E = (int)sh.E, k = (int)sh.k;
#define MOE_TOPK_S(P)                                                                 \
  launch_topk<P>(part, nsplit, split_stride, 1, 0, sh.E, bias, logits_out, idx, gate, \
                 flags, sh.T, E, k, st)
  if (pl <= 1)
    MOE_TOPK_S(1);
  else if (pl <= 2)
    MOE_TOPK_S(2);
  else if (pl <= 4)
    MOE_TOPK_S(4);
  else if (pl <= 8)
    MOE_TOPK_S(8);
  else if (pl <= 16)
    MOE_TOPK_S(16);
  else
    MOE_TOPK_S(32);
#undef MOE_TOPK_S
  return cudaGetLastError();
}

}  // namespace moe
