// Combine: gate-weighted sum of each token's expert outputs, with the identity
// contribution of zero experts.
//
// Ascend LongCat-2.0 deployment article (10100.com), "底层定制算子深度优化":
// a Combine operator that supports zero-computation experts. LongCat-2.0 model
// card (archdb), "Routed scaling factor": a multiplier on the combined
// routed-expert output; the library applies it to the routed part only and
// leaves the identity part of zero experts unscaled.
//
//   out[t] = s * sum_{j: idx<N} gate[t,j] * y_perm[slot_row[t,j]]
//              + sum_{j: idx>=N} gate[t,j] * x[t]
//
// y_perm is in the activation type, like x and out. Both sums run in fp32 in
// slot order j = 0..k-1 and the result is rounded once, so the output does not
// depend on thread timing. When the fused layer split the down GEMM's
// contraction (tiny batches), y holds ysplit fp32 partial rows per slot row:
// they are added in split order and rounded to the activation type, the same
// arithmetic as reducing them into y_perm and combining that.
// Grid: one block row per token, 16-byte vectors along d; the y loads of up to
// eight slots are in flight together (each kept as loaded until it is added).
#include "moe_internal.cuh"

namespace moe {
namespace {

template <typename AT>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ static void load(const __nv_bfloat16* p, float* v) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ static void store(__nv_bfloat16* p, const float* v) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};
template <>
struct Vec<float> {
  static constexpr int n = 4;
  __device__ static void load(const float* p, float* v) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    v[0] = u.x;
    v[1] = u.y;
    v[2] = u.z;
    v[3] = u.w;
  }
  __device__ static void store(float* p, const float* v) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

// the value a stored activation would have: v rounded to AT
template <typename AT>
__device__ __forceinline__ float round_to(float v);
template <>
__device__ __forceinline__ float round_to<float>(float v) { return v; }
template <>
__device__ __forceinline__ float round_to<__nv_bfloat16>(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

// One 16-byte vector of y or x as loaded (8 bf16 or 4 fp32 values), kept in
// that form until it is used: fewer registers per load in flight.
template <typename AT>
struct Raw;
template <>
struct Raw<__nv_bfloat16> {
  uint4 u;
  __device__ void load(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ void zero() { u = make_uint4(0, 0, 0, 0); }
  __device__ float get(int i) const {  // element i < 8, widened exactly
    const uint32_t w = i < 2 ? u.x : (i < 4 ? u.y : (i < 6 ? u.z : u.w));
    return (i & 1) ? __uint_as_float(w & 0xffff0000u) : __uint_as_float(w << 16);
  }
};
template <>
struct Raw<float> {
  float4 f;
  __device__ void load(const float* p) { f = __ldg(reinterpret_cast<const float4*>(p)); }
  __device__ void zero() { f = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ float get(int i) const { return i == 0 ? f.x : (i == 1 ? f.y : (i == 2 ? f.z : f.w)); }
};

// Slots per group of y loads issued together before any of them is added.
constexpr int kCombineGroup = 8;

// Slot metadata of token t in shared memory: y row, gate, zero-expert flag.
__device__ __forceinline__ void load_slots(const int32_t* __restrict__ idx,
                                           const float* __restrict__ gate,
                                           const int32_t* __restrict__ slot_row, int64_t t,
                                           int N, int k, int32_t* s_row, float* s_gate,
                                           int32_t* s_zero) {
  if ((int)threadIdx.x < k) {
    const int e = idx[t * k + threadIdx.x];
    s_row[threadIdx.x] = slot_row[t * k + threadIdx.x];
    s_gate[threadIdx.x] = gate[t * k + threadIdx.x];
    s_zero[threadIdx.x] = (e >= N) ? 1 : 0;
  }
}

template <typename AT>
__global__ void __launch_bounds__(128)
    combine_kernel(const AT* __restrict__ x, const AT* __restrict__ y,
                   const int32_t* __restrict__ idx, const float* __restrict__ gate,
                   const int32_t* __restrict__ slot_row, AT* __restrict__ out, int64_t d,
                   int N, int k, float s) {
  constexpr int V = Vec<AT>::n;
  __shared__ int32_t s_row[kMaxTopK];
  __shared__ float s_gate[kMaxTopK];
  __shared__ int32_t s_zero[kMaxTopK];
  griddep_wait();
  griddep_launch_dependents();
  const int64_t t = blockIdx.x;
  const int64_t col = ((int64_t)blockIdx.y * blockDim.x + threadIdx.x) * V;
  load_slots(idx, gate, slot_row, t, N, k, s_row, s_gate, s_zero);
  // the token's own row, for the identity term, is fetched while the slot
  // table arrives (most tokens send a slot to a zero expert)
  Raw<AT> xr;
  if (col < d)
    xr.load(x + t * d + col);
  else
    xr.zero();
  __syncthreads();
  if (col >= d) return;
  float racc[V], zacc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) racc[i] = zacc[i] = 0.f;
  // y rows of kCombineGroup slots in flight at once, then added in slot order
  for (int j0 = 0; j0 < k; j0 += kCombineGroup) {
    Raw<AT> yr[kCombineGroup];
#pragma unroll
    for (int q = 0; q < kCombineGroup; ++q) {
      const int j = j0 + q;
      if (j < k && !s_zero[j])
        yr[q].load(y + (int64_t)s_row[j] * d + col);
      else
        yr[q].zero();
    }
#pragma unroll
    for (int q = 0; q < kCombineGroup; ++q) {
      const int j = j0 + q;
      if (j >= k) continue;
      const float g = s_gate[j];
      if (s_zero[j]) {
#pragma unroll
        for (int i = 0; i < V; ++i) zacc[i] = fmaf(g, xr.get(i), zacc[i]);
      } else {
#pragma unroll
        for (int i = 0; i < V; ++i) racc[i] = fmaf(g, yr[q].get(i), racc[i]);
      }
    }
  }
  float v[V];
#pragma unroll
  for (int i = 0; i < V; ++i) v[i] = fmaf(s, racc[i], zacc[i]);
  Vec<AT>::store(out + t * d + col, v);
}

// The same when the fused layer split the down GEMM's contraction (tiny
// batches): y holds ysplit fp32 partial rows per slot row, added in split
// order and rounded as a stored y_perm row would be, four slots at a time.
template <typename AT>
__global__ void __launch_bounds__(128)
    combine_split_kernel(const AT* __restrict__ x, const float* __restrict__ y,
                         const int32_t* __restrict__ idx, const float* __restrict__ gate,
                         const int32_t* __restrict__ slot_row, AT* __restrict__ out,
                         int64_t d, int N, int k, float s, int ysplit) {
  constexpr int V = Vec<AT>::n;
  __shared__ int32_t s_row[kMaxTopK];
  __shared__ float s_gate[kMaxTopK];
  __shared__ int32_t s_zero[kMaxTopK];
  griddep_wait();
  griddep_launch_dependents();
  const int64_t t = blockIdx.x;
  const int64_t col = ((int64_t)blockIdx.y * blockDim.x + threadIdx.x) * V;
  load_slots(idx, gate, slot_row, t, N, k, s_row, s_gate, s_zero);
  Raw<AT> xr;
  if (col < d)
    xr.load(x + t * d + col);
  else
    xr.zero();
  __syncthreads();
  if (col >= d) return;
  float racc[V], zacc[V], v[V];
#pragma unroll
  for (int i = 0; i < V; ++i) racc[i] = zacc[i] = 0.f;
  for (int j0 = 0; j0 < k; j0 += 4) {
    float yv[4][V];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = j0 + q;
      if (j < k && !s_zero[j]) {
        const float* yr = y + (int64_t)s_row[j] * ysplit * d + col;
#pragma unroll
        for (int i = 0; i < V; i += 4) Vec<float>::load(yr + i, yv[q] + i);
        for (int c = 1; c < ysplit; ++c) {
#pragma unroll
          for (int i = 0; i < V; i += 4) Vec<float>::load(yr + (int64_t)c * d + i, v + i);
#pragma unroll
          for (int i = 0; i < V; ++i) yv[q][i] += v[i];
        }
#pragma unroll
        for (int i = 0; i < V; ++i) yv[q][i] = round_to<AT>(yv[q][i]);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = j0 + q;
      if (j >= k) continue;
      const float g = s_gate[j];
      if (s_zero[j]) {
#pragma unroll
        for (int i = 0; i < V; ++i) zacc[i] = fmaf(g, xr.get(i), zacc[i]);
      } else {
#pragma unroll
        for (int i = 0; i < V; ++i) racc[i] = fmaf(g, yv[q][i], racc[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < V; ++i) v[i] = fmaf(s, racc[i], zacc[i]);
  Vec<AT>::store(out + t * d + col, v);
}

}  // namespace

cudaError_t launch_combine(const Shape& sh, const void* x, const void* y_perm,
                           const int32_t* idx, const float* gate,
                           const int32_t* slot_row, void* out, cudaStream_t st,
                           int ysplit) {
  const int V = sh.bf16 ? 8 : 4;
  const int64_t vecs = sh.d / V;
  const int threads = 128;
  dim3 grid((unsigned)sh.T, (unsigned)((vecs + threads - 1) / threads));
  const int N = (int)sh.N, k = (int)sh.k;
  if (ysplit > 1) {
    if (sh.bf16)
      launch_pdl(combine_split_kernel<__nv_bfloat16>, grid, dim3(threads), 0, st,
                 static_cast<const __nv_bfloat16*>(x), static_cast<const float*>(y_perm), idx,
                 gate, slot_row, static_cast<__nv_bfloat16*>(out), sh.d, N, k, sh.s, ysplit);
    else
      launch_pdl(combine_split_kernel<float>, grid, dim3(threads), 0, st,
                 static_cast<const float*>(x), static_cast<const float*>(y_perm), idx, gate,
                 slot_row, static_cast<float*>(out), sh.d, N, k, sh.s, ysplit);
  } else if (sh.bf16) {
    launch_pdl(combine_kernel<__nv_bfloat16>, grid, dim3(threads), 0, st,
               static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(y_perm),
               idx, gate, slot_row, static_cast<__nv_bfloat16*>(out), sh.d, N, k, sh.s);
  } else {
    launch_pdl(combine_kernel<float>, grid, dim3(threads), 0, st, static_cast<const float*>(x),
               static_cast<const float*>(y_perm), idx, gate, slot_row,
               static_cast<float*>(out), sh.d, N, k, sh.s);
  }
  return cudaGetLastError();
}

}  // namespace moe
