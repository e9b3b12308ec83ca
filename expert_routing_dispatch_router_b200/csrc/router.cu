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
// Kernel 1 (router_logits_kernel): CUDA-core GEMM in fp32. The contraction is
// split over blockIdx.z so that a decode batch (T ~ 64) still spreads the
// router weights over many SMs; each split writes its partial sums to the
// workspace and kernel 2 adds them in a fixed order, so results are
// bit-reproducible run to run.
//
// Kernel 2 (topk_kernel): one warp per token. The E keys sit in registers,
// ceil(E/32) per lane. k+1 rounds of a warp arg-max (ties to the lower id)
// give the selection in descending key order and the margin between the k-th
// and (k+1)-th key.
#include <float.h>
#include <math.h>

#include "moe_internal.cuh"

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

// Top-k of one token by one warp, from its logits lg[i] of experts
// lane + 32 i: keys = logits + bias, k+1 rounds of a warp arg-max (ties to the
// lower id), gates = softmax of the selected raw logits, and the near-tie flag.
// Writes logits_out (if given), idx_out, gate_out and flags (if given) of t.
template <int PL>
__device__ __forceinline__ void warp_select_token(const float (&lg)[PL],
                                                  const float* __restrict__ bias,
                                                  float* __restrict__ logits_out,
                                                  int32_t* __restrict__ idx_out,
                                                  float* __restrict__ gate_out,
                                                  uint8_t* __restrict__ flags, int64_t t,
                                                  int E, int k, int lane) {
  float key[PL];
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const int e = lane + 32 * i;
    key[i] = -INFINITY;
    if (e < E) {
      const float kv = lg[i] + bias[e];
      key[i] = (kv != kv) ? -INFINITY : kv;  // a NaN key never wins
      if (logits_out) logits_out[t * E + e] = lg[i];
    }
  }

  // Each round: every lane takes its best remaining key (ascending ids, so the
  // lower id wins ties), then two warp reductions pick the largest key and,
  // among lanes holding it, the lowest id.
  uint32_t taken = 0;  // bit i: expert lane + 32 i already selected
  float kth_key = 0.f, next_key = -INFINITY;
  float my_logit = 0.f;
  int my_e = 0;
  const int rounds = (k < E) ? k + 1 : k;
  for (int j = 0; j < rounds; ++j) {
    uint32_t bo = 0u;
    int be = 0x7fffffff;
    float bk = -INFINITY, bl = 0.f;
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      const int e = lane + 32 * i;
      const uint32_t o = ord_key(key[i]);
      if (e < E && !((taken >> i) & 1u) && (be == 0x7fffffff || o > bo)) {
        bo = o;
        be = e;
        bk = key[i];
        bl = lg[i];
      }
    }
    const uint32_t mo = __reduce_max_sync(0xffffffffu, bo);
    const int we = (int)__reduce_min_sync(0xffffffffu,
                                          (be != 0x7fffffff && bo == mo) ? (uint32_t)be
                                                                        : 0x7fffffffu);
    const float wk = __shfl_sync(0xffffffffu, bk, we & 31);
    const float wl = __shfl_sync(0xffffffffu, bl, we & 31);
    if (j < k) {
      if (lane == (we & 31)) taken |= 1u << (we >> 5);
      if (lane == j) {
        my_logit = wl;
        my_e = we;
      }
      kth_key = wk;
    } else {
      next_key = wk;
    }
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
    const float margin = (k < E) ? kth_key - next_key : INFINITY;
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
  warp_select_token<PL>(lg, bias, logits_out, idx_out, gate_out, flags, t, E, k, lane);
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
// group g, the 32 experts of tile et and contraction split z (<= 1024
// elements). Its x rows sit in shared memory as fp32; each warp streams 4
// router rows from global memory, lanes along the contraction (coalesced).
// A lane sums its 32-element share, a warp tree adds the lanes, and the
// partial sums of the splits go to the workspace. The last CTA to finish a
// token group (a counter per group, incremented after a fence) adds the
// partials of its 8 tokens in split order and runs their top-k, then resets
// the counter to zero for the next call. No CTA waits for another.
//
// Weight prefetch (the fused layer call at T <= 64): while the router and
// dispatch run, HBM would sit idle, so the router's CTAs first ask L2 to fetch
// the weight tiles the gate/up GEMM reads first. At T <= 64 every touched
// expert is one token tile, and the GEMM's units run expert by expert, so
// unit u is (expert u / m_tiles, rows (u % m_tiles) * 128) when every expert is
// touched; the first pf_units such tiles of W_gate and W_up are requested.
// This only moves bytes earlier; a wrong guess costs idle bandwidth.
struct WeightPrefetch {
  const uint8_t* w_gate = nullptr;  // [N, F, d] bf16, or null for none
  const uint8_t* w_up = nullptr;
  int64_t expert_bytes = 0;  // F * d * 2
  int64_t tile_bytes = 0;    // 128 rows * d * 2 (contiguous)
  int m_tiles = 0;           // F / 128
  int units = 0;             // tiles of each matrix to request
};
// Bring `bytes` (16-byte aligned, a multiple of 16) of global memory into L2,
// asynchronously; nothing waits for it.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                   reinterpret_cast<uint64_t>(p)),
               "r"(bytes)
               : "memory");
}

constexpr int DG = 8;    // tokens per group
constexpr int DE = 32;   // experts per CTA (8 warps x 4)

template <typename XT>
__device__ __forceinline__ void load_x8(const XT* x, int64_t off, float* dst);
template <>
__device__ __forceinline__ void load_x8<__nv_bfloat16>(const __nv_bfloat16* x, int64_t off,
                                                       float* dst) {
  const uint4 v = *reinterpret_cast<const uint4*>(x + off);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    dst[2 * i] = __uint_as_float(w[i] << 16);
    dst[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
template <>
__device__ __forceinline__ void load_x8<float>(const float* x, int64_t off, float* dst) {
  const float4 a = *reinterpret_cast<const float4*>(x + off);
  const float4 b = *reinterpret_cast<const float4*>(x + off + 4);
  dst[0] = a.x; dst[1] = a.y; dst[2] = a.z; dst[3] = a.w;
  dst[4] = b.x; dst[5] = b.y; dst[6] = b.z; dst[7] = b.w;
}

// ITER: 128-element steps per lane in one split (ksplit = 128 * ITER), a
// compile-time count so that all of a warp's router-row loads are in flight
// together instead of one round trip per step.
template <typename XT, int PL, int ITER>
__global__ void __launch_bounds__(256)
    router_small_kernel(const XT* __restrict__ x, const float* __restrict__ w_r,
                        const float* __restrict__ bias, float* __restrict__ part,
                        int32_t* __restrict__ counter, float* __restrict__ logits_out,
                        int32_t* __restrict__ idx_out, float* __restrict__ gate_out,
                        uint8_t* __restrict__ flags, int64_t T, int64_t d, int E, int k,
                        int64_t ksplit, const WeightPrefetch pf) {
  extern __shared__ float xs[];  // [DG][ksplit]
  __shared__ int s_last;
  griddep_wait();
  griddep_launch_dependents();
  if (pf.units > 0 && threadIdx.x == 0) {
    const int nctas = gridDim.x * gridDim.y * gridDim.z;
    const int c = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    for (int u = c; u < pf.units; u += nctas) {
      const int64_t off = (int64_t)(u / pf.m_tiles) * pf.expert_bytes +
                          (int64_t)(u % pf.m_tiles) * pf.tile_bytes;
      prefetch_l2_bulk(pf.w_gate + off, (uint32_t)pf.tile_bytes);
      prefetch_l2_bulk(pf.w_up + off, (uint32_t)pf.tile_bytes);
    }
  }
  const int g = blockIdx.x, et = blockIdx.y, z = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t0 = (int64_t)g * DG;
  const int64_t kbeg = (int64_t)z * ksplit;
  const int64_t klen = min(d, kbeg + ksplit) - kbeg;
  const int64_t v8 = klen / 8;
  for (int64_t i = threadIdx.x; i < DG * v8; i += blockDim.x) {
    const int tt = (int)(i / v8);
    const int64_t kk = (i - tt * v8) * 8;
    float* dst = xs + tt * ksplit + kk;
    if (t0 + tt < T) {
      load_x8<XT>(x, (t0 + tt) * d + kbeg + kk, dst);
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) dst[q] = 0.f;
    }
  }
  __syncthreads();
  // the 4 experts of this warp: all their router-row loads first
  float4 wv[4][ITER];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = et * DE + warp * 4 + j;
    const float* wr = w_r + (int64_t)e * d + kbeg;
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
      const int64_t kk = 4 * lane + 128 * it;
      wv[j][it] = (e < E && kk < klen) ? *reinterpret_cast<const float4*>(wr + kk)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = et * DE + warp * 4 + j;
    if (e >= E) break;
    float acc[DG];
#pragma unroll
    for (int tt = 0; tt < DG; ++tt) acc[tt] = 0.f;
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
      const int64_t kk = 4 * lane + 128 * it;
      if (kk >= klen) break;
      const float4 w4 = wv[j][it];
#pragma unroll
      for (int tt = 0; tt < DG; ++tt) {
        const float4 xv = *reinterpret_cast<const float4*>(xs + tt * ksplit + kk);
        acc[tt] = fmaf(w4.x, xv.x, acc[tt]);
        acc[tt] = fmaf(w4.y, xv.y, acc[tt]);
        acc[tt] = fmaf(w4.z, xv.z, acc[tt]);
        acc[tt] = fmaf(w4.w, xv.w, acc[tt]);
      }
    }
#pragma unroll
    for (int tt = 0; tt < DG; ++tt)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        acc[tt] += __shfl_xor_sync(0xffffffffu, acc[tt], off);
    if (lane < DG && t0 + lane < T) {
      float v = acc[0];
#pragma unroll
      for (int tt = 1; tt < DG; ++tt)
        if (lane == tt) v = acc[tt];
      part[((int64_t)z * T + t0 + lane) * E + e] = v;
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0)
    s_last = atomicAdd(&counter[g], 1) == (int)(gridDim.y * gridDim.z) - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int64_t t = t0 + warp;
  if (t < T) {
    float lg[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) lg[i] = 0.f;
    for (int zz = 0; zz < (int)gridDim.z; ++zz) {
      const float* pz = part + ((int64_t)zz * T + t) * E + lane;
#pragma unroll
      for (int i = 0; i < PL; ++i)
        if (lane + 32 * i < E) lg[i] += __ldcg(pz + 32 * i);
    }
    warp_select_token<PL>(lg, bias, logits_out, idx_out, gate_out, flags, t, E, k, lane);
  }
  if (threadIdx.x == 0) counter[g] = 0;
}

// Exact three-way split of the fp32 router weights into bf16 planes for the
// tensor-core router: hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid)
// (each difference is exact in fp32), so hi + mid + lo carries the 24 bits of
// w and x . w = x . hi + x . mid + x . lo with x in bf16 and every product
// exact in fp32. Rows [0,E) of `planes` get hi, [E,2E) mid, [2E,3E) lo, the
// padding rows up to Ep zeros. Also writes the one-expert plan of the GEMM.
__global__ void __launch_bounds__(256)
    router_split_kernel(const float4* __restrict__ w_r, int64_t E, int64_t d, int64_t Ep,
                        uint2* __restrict__ planes, int32_t* __restrict__ plan,
                        int64_t T, int tile) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t q = d / 4;  // float4 per row
  const int64_t n = E * q;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const float4 w = w_r[i];
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
    planes[i] = pack(hb);
    planes[n + i] = pack(mb);
    planes[2 * n + i] = pack(lb);
  }
  for (int64_t i = 3 * n + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < Ep * q;
       i += stride)
    planes[i] = make_uint2(0u, 0u);
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

int64_t router_planes_rows(const Shape& sh) { return (3 * sh.E + 127) / 128 * 128; }

// The tensor-core router restarts its fp32 accumulation every 1024 contraction
// elements (16 blocks of 64), a chain of 64 MMA steps per partial.
static int router_kb_chunk(const Shape& sh) {
  const int kb = (int)(sh.d / 64);
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
constexpr int64_t kPrefetchBytes = 96ll << 20;  // L2 prefetch budget of a decode call

bool router_uses_small_kernel(const Shape& sh) { return sh.T <= kSmallRouterMaxTokens; }

// Contraction splits of the small-batch router (<= 1024 elements each).
int router_small_splits(const Shape& sh) { return (int)((sh.d + 1023) / 1024); }

int router_launch_count(const Shape& sh) {
  return router_uses_tensor_cores(sh) ? 3 : (router_uses_small_kernel(sh) ? 1 : 2);
}

// Number of contraction splits so that the logits GEMM has >= ~2 CTAs per SM.
int router_splits(const Shape& sh) {
  const int64_t tiles = ((sh.E + RE - 1) / RE) * ((sh.T + RT - 1) / RT);
  int64_t want = (2 * num_sms() + tiles - 1) / tiles;
  int64_t max_split = (sh.d + 255) / 256;  // >= 256 k per split
  if (max_split > 16) max_split = 16;
  if (want > max_split) want = max_split;
  if (want < 1) want = 1;
  return (int)want;
}

cudaError_t launch_router(const Shape& sh, const void* x, const float* w_r,
                          const float* bias, float* part, int32_t* idx,
                          float* gate, uint8_t* flags, float* logits_out,
                          void* planes, int32_t* plan, int32_t* err,
                          const void* prefetch_gate, const void* prefetch_up,
                          cudaStream_t st) {
  int n_outer, n_inner;
  int64_t outer_stride, inner_stride, row_stride;
  cudaError_t e;
  if (router_uses_small_kernel(sh)) {
    // one launch: logits, split sums and top-k; the group counters live in
    // the workspace header after the error word (zero between calls)
    const int nsplit = router_small_splits(sh);
    const int64_t steps = ((sh.d + nsplit - 1) / nsplit + 127) / 128;  // <= 8
    const int iter = steps <= 1 ? 1 : steps <= 2 ? 2 : steps <= 4 ? 4 : 8;
    const int64_t ksplit = 128 * (int64_t)iter;
    const dim3 grid((unsigned)((sh.T + DG - 1) / DG), (unsigned)((sh.E + DE - 1) / DE),
                    (unsigned)nsplit);
    const size_t smem = (size_t)DG * ksplit * sizeof(float);
    int32_t* counter = err + 2;
    WeightPrefetch pf;
    const bool aligned = ((reinterpret_cast<uintptr_t>(prefetch_gate) |
                           reinterpret_cast<uintptr_t>(prefetch_up)) & 15) == 0;
    if (prefetch_gate && prefetch_up && aligned && sh.T <= 64 && sh.N > 0 &&
        expert_ffn_uses_tensor_cores(sh)) {
      pf.w_gate = static_cast<const uint8_t*>(prefetch_gate);
      pf.w_up = static_cast<const uint8_t*>(prefetch_up);
      pf.expert_bytes = sh.F * sh.d * 2;
      pf.tile_bytes = 128 * sh.d * 2;
      pf.m_tiles = (int)(sh.F / 128);
      const int64_t budget = kPrefetchBytes / (2 * pf.tile_bytes);  // tiles per matrix
      const int64_t all = sh.N * pf.m_tiles;
      pf.units = (int)(budget < all ? budget : all);
    }
    const int pl = (int)((sh.E + 31) / 32);
    const int E = (int)sh.E, k = (int)sh.k;
#define MOE_SMALL_IT(XT, P, I)                                                        \
  launch_pdl(router_small_kernel<XT, P, I>, grid, dim3(256), smem, st,                \
             static_cast<const XT*>(x), w_r, bias, part, counter, logits_out, idx, gate, \
             flags, sh.T, sh.d, E, k, ksplit, pf)
#define MOE_SMALL(XT, P)                                          \
  (iter == 1 ? MOE_SMALL_IT(XT, P, 1)                             \
   : iter == 2 ? MOE_SMALL_IT(XT, P, 2)                           \
   : iter == 4 ? MOE_SMALL_IT(XT, P, 4) : MOE_SMALL_IT(XT, P, 8))
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
#undef MOE_SMALL_IT
    return e;
  }
  if (router_uses_tensor_cores(sh)) {
    const int64_t Ep = router_planes_rows(sh);
    const int64_t n4 = sh.E * sh.d / 4;
    int64_t blocks = (n4 + 255) / 256;
    if (blocks > 4 * num_sms()) blocks = 4 * num_sms();
    e = launch_pdl(router_split_kernel, dim3((unsigned)blocks), dim3(256), 0, st,
                   reinterpret_cast<const float4*>(w_r), sh.E, sh.d, Ep,
                   static_cast<uint2*>(planes), plan, sh.T, kTileDown);
    if (e != cudaSuccess) return e;
    e = launch_dense_gemm_tc(planes, Ep, x, sh.T, sh.d, router_kb_chunk(sh), part, plan,
                             err, st);
    if (e != cudaSuccess) return e;
    // part[t, c * Ep + p * E + e]: chunk c, plane p (hi, mid, lo)
    n_outer = router_tc_chunks(sh);
    outer_stride = Ep;
    n_inner = 3;
    inner_stride = sh.E;
    row_stride = (int64_t)n_outer * Ep;
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
