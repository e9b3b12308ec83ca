// Internal declarations shared by the CUDA sources of the MoE library:
// workspace layout, launcher prototypes and small device helpers.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "../../include/moe_api.h"

namespace moe {

constexpr int kMaxExperts = 1024;  // top-k keeps E/32 keys per lane
constexpr int kMaxTopK = 32;       // one gate per lane
constexpr int kChunkTokens = 256;  // tokens per dispatch block
constexpr int kRouterGemmTile = 256;  // token tile of the tensor-core router GEMM
constexpr int kWsAlign = 1024;

// Device error codes written into the workspace header.
constexpr int kErrWaitTimeout = 1;
constexpr int kErrBadExpertId = 2;

// Layout of the workspace (byte offsets from its base). Built on the host
// from the config alone; every region is kWsAlign-aligned.
struct WsLayout {
  size_t header;       // int32[64]: [0] error code, [1] detail, [2..33] router
                       // group counters (zero between calls)
  size_t logits;       // float router partials: [splits, T, E] or [T, 3E pad]
  size_t planes;       // bf16 [3E pad, d] router weights split in 3 planes
  size_t router_plan;  // int32 [4] plan of the tensor-core router GEMM
  size_t topk_idx;     // int32 [T, k]
  size_t topk_gate;    // float [T, k]
  size_t chunk_base;   // int32 [nchunks, E]
  size_t counts;       // int32 [E]
  size_t offsets;      // int32 [N + 1]
  size_t row_token;    // int32 [T*k]
  size_t slot_row;     // int32 [T*k]
  size_t tile_start;   // int32 [2 (N + 1) + 2]: the expert GEMMs' plans, then
                       // the CTA-pair GEMMs' unit counters
  size_t x_perm;       // act   [T*k, d]
  size_t h;            // act   [T*k, F]
  size_t y_perm;       // act [T*k, d]
  size_t ffn_part;     // float split-contraction partials of the expert GEMMs
                       // (tiny batches only; else empty)
  size_t x_stage;      // act   [T, d]   (host-buffer entry point)
  size_t out_stage;    // act   [T, d]
  size_t total;
};

struct Shape {
  int64_t T, d, N, Z, E, k, F;
  int es;  // bytes per activation element
  float s;
  bool bf16;
  int64_t nchunks;
};

WsLayout ws_layout(const Shape& sh);

// ---- launchers (each returns cudaGetLastError() after its launches) ----
int router_splits(const Shape& sh);
cudaError_t launch_router(const Shape& sh, const void* x, const float* w_r,
                          const float* bias, float* part, int32_t* idx,
                          float* gate, uint8_t* flags, float* logits_out,
                          void* planes, int32_t* plan, int32_t* err,
                          cudaStream_t st);
// x_perm null: the rows are not gathered (the gate/up GEMM gathers them).
// tile_start given and dispatch_plans_tiles(sh): the one-block dispatch also
// writes the expert GEMMs' token-tile prefixes for tiles tile_gu and tile_dn.
cudaError_t launch_dispatch(const Shape& sh, const void* x, const int32_t* idx,
                            int32_t* chunk_base, int32_t* counts,
                            int32_t* offsets, int32_t* row_token,
                            int32_t* slot_row, void* x_perm, int32_t* err,
                            cudaStream_t st, int32_t* tile_start = nullptr,
                            int tile_gu = 0, int tile_dn = 0);
bool dispatch_plans_tiles(const Shape& sh);
// The one-block dispatch also gathers x_perm, in the same launch.
bool dispatch_gathers_in_sort(const Shape& sh);
// With x_src and row_token given (the fused layer, where expert_ffn_gathers
// holds), the gate/up GEMM reads token rows from x by row_token and x_perm is
// not used.
cudaError_t launch_expert_ffn(const Shape& sh, const void* x_perm,
                              const int32_t* offsets, const void* w_gate,
                              const void* w_up, const void* w_down, void* h,
                              void* y_perm, int32_t* tile_start, int32_t* err,
                              cudaStream_t st, const void* x_src = nullptr,
                              const int32_t* row_token = nullptr, bool plan_ready = false,
                              float* part = nullptr, bool leave_y_split = false);
// Contraction splits of the expert GEMMs (1 unless the batch is tiny) and the
// fp32 scratch they need (floats; 0 without splits). With leave_y_split the
// down GEMM's split partials stay in `part` ([row][split][d]) for the combine
// to add; otherwise they are added into y_perm.
int expert_ffn_split(const Shape& sh, bool gateup);
int64_t expert_ffn_part_floats(const Shape& sh);
bool expert_ffn_gathers(const Shape& sh);
// Token tiles of the gate/up and down GEMMs on the tensor-core path.
void expert_ffn_tiles(const Shape& sh, int* tile_gu, int* tile_dn);
// y_perm rows hold ysplit partial rows of d floats each ([row][split][d]),
// added in split order before the gate weighting (1 for a plain y_perm).
cudaError_t launch_combine(const Shape& sh, const void* x, const void* y_perm,
                           const int32_t* idx, const float* gate,
                           const int32_t* slot_row, void* out, cudaStream_t st,
                           int ysplit = 1);
// plane_experts > 0: A holds the router's three bf16 planes of that many
// experts (router_planes_rows layout) and out gets their per-chunk sums,
// [T][chunks][plane_experts]; otherwise out is [T][chunks][M].
cudaError_t launch_dense_gemm_tc(const void* a, int64_t M, const void* b, int64_t T,
                                 int64_t K, int kb_chunk, int64_t plane_experts, float* out,
                                 const int32_t* plan, int32_t* err, cudaStream_t st);
bool router_uses_tensor_cores(const Shape& sh);
int64_t router_planes_rows(const Shape& sh);   // 128 per 40 experts
int router_tc_chunks(const Shape& sh);         // contraction chunks of that router
int router_launch_count(const Shape& sh);
// False when the batch is too large for the router path it would take (the
// CUDA-core router tiles tokens along gridDim.y, at most 65535 tiles).
bool router_grid_fits(const Shape& sh);
int router_small_splits(const Shape& sh);
int expert_ffn_launch_count(const Shape& sh);
// Expert parallelism over G ranks (csrc/expert_parallel.cu).
int ep_local_experts(int rank, int N, int G);
int ep_first_expert(int rank, int N, int G);
cudaError_t launch_ep_plan(const Shape& sh, int rank, int G, const int32_t* counts_all,
                           int32_t* dest_row, int32_t* recv_offsets, cudaStream_t st);
cudaError_t launch_ep_dispatch(const Shape& sh, int G, const void* x, const int32_t* offsets,
                               const int32_t* row_token, const int32_t* dest_row,
                               void* const* recv, cudaStream_t st);
cudaError_t launch_ep_return(const Shape& sh, int rank, int G, const void* y_recv,
                             const int32_t* recv_offsets, const int32_t* counts_all,
                             const int32_t* offsets_all, void* const* home, cudaStream_t st);
cudaError_t launch_bias_pid(const Shape& sh, const int32_t* counts, float* bias,
                            double* state, double target, double kp, double ki,
                            double kd, double max_step, cudaStream_t st);
int dispatch_launch_count(const Shape& sh);
cudaError_t launch_wait_limit_selftest(int32_t* err, cudaStream_t st);
bool expert_ffn_uses_tensor_cores(const Shape& sh);
int num_sms();

// Raises a kernel's dynamic shared-memory limit once per device (the
// attribute is per device; one process may drive several GPUs). `done` is the
// calling launcher's set of devices already done; racing threads only repeat
// the idempotent call.
template <typename Kernel>
cudaError_t raise_smem_once(std::atomic<uint64_t>& done, Kernel kernel, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load() & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit);
  return e;
}

// Launch with programmatic dependent launch allowed: the kernel may start
// while its predecessor on the stream drains, and must call griddep_wait()
// before it reads or writes anything the predecessor touches.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---- device helpers ----
// Wait until the previous kernel on the stream has completed and its memory
// is visible (no-op when launched without programmatic dependencies).
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Allow the next kernel on the stream to be scheduled.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

}  // namespace moe
