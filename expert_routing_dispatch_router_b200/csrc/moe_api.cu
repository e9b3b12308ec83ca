// C ABI of the MoE library: argument checks, workspace layout and the launch
// sequence of each call. Every check runs on the host before the first launch;
// nothing here allocates, frees or synchronises (moe_read_device_error waits on
// the stream it is given, by design).
#include <math.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

#include "moe_internal.cuh"

namespace moe {

// NVTX range over a host-side scope: each call and each stage of the fused
// layer shows up by name in a profiler's timeline (header-only NVTX; without
// a profiler attached a push or pop is one check of a null hook).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

static size_t align_up(size_t v) {
  return (v + kWsAlign - 1) / kWsAlign * kWsAlign;
}

WsLayout ws_layout(const Shape& sh) {
  WsLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  const size_t Tk = (size_t)(sh.T * sh.k);
  L.header = take(256);
  const int splits = router_splits(sh) > router_small_splits(sh) ? router_splits(sh)
                                                                 : router_small_splits(sh);
  size_t part = (size_t)splits * sh.T * sh.E;
  const size_t tc_part = (size_t)sh.T * router_tc_chunks(sh) * sh.E;
  if (router_uses_tensor_cores(sh) && tc_part > part) part = tc_part;
  L.logits = take(part * sizeof(float));
  L.planes = take(router_uses_tensor_cores(sh)
                      ? (size_t)router_planes_rows(sh) * sh.d * sizeof(uint16_t)
                      : 0);
  L.router_plan = take(4 * sizeof(int32_t));
  L.topk_idx = take(Tk * sizeof(int32_t));
  L.topk_gate = take(Tk * sizeof(float));
  L.chunk_base = take((size_t)sh.nchunks * sh.E * sizeof(int32_t));
  L.counts = take((size_t)sh.E * sizeof(int32_t));
  L.offsets = take((size_t)(sh.N + 1) * sizeof(int32_t));
  L.row_token = take(Tk * sizeof(int32_t));
  L.slot_row = take(Tk * sizeof(int32_t));
  L.tile_start = take((2 * (size_t)(sh.N + 1) + 2) * sizeof(int32_t));
  L.x_perm = take(Tk * sh.d * sh.es);
  L.h = take(Tk * sh.F * sh.es);
  L.y_perm = take(Tk * sh.d * sh.es);
  L.ffn_part = take(sh.N > 0 ? (size_t)expert_ffn_part_floats(sh) * sizeof(float) : 0);
  L.x_stage = take((size_t)sh.T * sh.d * sh.es);
  L.out_stage = take((size_t)sh.T * sh.d * sh.es);
  L.total = off;
  return L;
}

}  // namespace moe

using namespace moe;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Required device pointer: non-null and 16-byte aligned.
bool dev_ok(const void* p) { return p != nullptr && aligned16(p); }
// Optional device pointer: null, or 16-byte aligned.
bool opt_ok(const void* p) { return p == nullptr || aligned16(p); }

moe_status_t make_shape(const moe_config_t* c, Shape* sh) {
  if (c == nullptr) return MOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->d <= 0 || c->n_routed < 0 || c->n_zero < 0 || c->top_k <= 0 ||
      c->ffn <= 0)
    return MOE_ERR_INVALID_ARG;
  if (c->act_dtype != MOE_F32 && c->act_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  const int64_t E = (int64_t)c->n_routed + c->n_zero;
  if (E <= 0 || c->top_k > E) return MOE_ERR_INVALID_ARG;
  if (!isfinite(c->routed_scale)) return MOE_ERR_INVALID_ARG;
  if (c->top_k > kMaxTopK || E > kMaxExperts) return MOE_ERR_UNSUPPORTED;
  if (c->d % 8 != 0 || c->ffn % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if ((int64_t)c->T * c->top_k >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
  sh->T = c->T;
  sh->d = c->d;
  sh->N = c->n_routed;
  sh->Z = c->n_zero;
  sh->E = E;
  sh->k = c->top_k;
  sh->F = c->ffn;
  sh->bf16 = c->act_dtype == MOE_BF16;
  sh->es = sh->bf16 ? 2 : 4;
  sh->s = c->routed_scale;
  sh->nchunks = (sh->T + kChunkTokens - 1) / kChunkTokens;
  if (!router_grid_fits(*sh)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status_t check_ws(const Shape& sh, const void* ws, size_t ws_bytes) {
  if (ws == nullptr || ws_bytes < ws_layout(sh).total) return MOE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// The fused sequence with every intermediate in ws (arguments already checked).
moe_status_t run_layer(const Shape& sh, const void* x, const float* w_router,
                       const float* bias, const void* w_gate, const void* w_up,
                       const void* w_down, void* out, int32_t* counts, void* ws,
                       cudaStream_t st) {
  const WsLayout L = ws_layout(sh);
  int32_t* err = at<int32_t>(ws, L.header);
  int32_t* idx = at<int32_t>(ws, L.topk_idx);
  float* gate = at<float>(ws, L.topk_gate);
  int32_t* slot_row = at<int32_t>(ws, L.slot_row);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  void* x_perm = at<void>(ws, L.x_perm);
  void* y_perm = at<void>(ws, L.y_perm);
  cudaError_t e;
  {
    NvtxRange r("moe.route");
    e = launch_router(sh, x, w_router, bias, at<float>(ws, L.logits), idx, gate, nullptr,
                      nullptr, at<void>(ws, L.planes), at<int32_t>(ws, L.router_plan), err, st);
  }
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  // where the gate/up GEMM gathers token rows itself, x_perm is never written
  const bool gather = expert_ffn_gathers(sh);
  // the one-block dispatch also writes the expert GEMMs' plans
  const bool plan = sh.N > 0 && expert_ffn_uses_tensor_cores(sh) && dispatch_plans_tiles(sh);
  int tgu = 0, tdn = 0;
  expert_ffn_tiles(sh, &tgu, &tdn);
  int32_t* row_token = at<int32_t>(ws, L.row_token);
  int32_t* tile_start = at<int32_t>(ws, L.tile_start);
  {
    NvtxRange r("moe.dispatch");
    e = launch_dispatch(sh, x, idx, at<int32_t>(ws, L.chunk_base),
                        counts ? counts : at<int32_t>(ws, L.counts), offsets, row_token,
                        slot_row, gather ? nullptr : x_perm, err, st,
                        plan ? tile_start : nullptr, tgu, tdn);
  }
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  // with a split down GEMM, the combine adds its partials itself
  const int ysplit = sh.N > 0 ? expert_ffn_split(sh, false) : 1;
  float* part = at<float>(ws, L.ffn_part);
  {
    NvtxRange r("moe.expert_ffn");
    e = launch_expert_ffn(sh, x_perm, offsets, w_gate, w_up, w_down, at<void>(ws, L.h),
                          y_perm, tile_start, err, st, gather ? x : nullptr,
                          gather ? row_token : nullptr, plan, part, true);
  }
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  NvtxRange r("moe.combine");
  e = launch_combine(sh, x, ysplit > 1 ? static_cast<void*>(part) : y_perm, idx, gate,
                     slot_row, out, st, ysplit);
  return cuda_status(e);
}

}  // namespace

namespace moe {
// Configuration checks shared with the entry points defined in other files.
moe_status_t shape_from_config(const moe_config_t* c, Shape* sh) { return make_shape(c, sh); }
}  // namespace moe

extern "C" {

size_t moe_workspace_size(const moe_config_t* cfg) {
  Shape sh;
  if (make_shape(cfg, &sh) != MOE_OK) return 0;
  return ws_layout(sh).total;
}

moe_status_t moe_route(const moe_config_t* cfg, const void* x, const float* w_router,
                       const float* bias, float* logits, int32_t* topk_idx,
                       float* topk_gate, uint8_t* flags, void* ws, size_t ws_bytes,
                       moe_stream_t stream) {
  NvtxRange range("moe_route");
  Shape sh;
  moe_status_t s = make_shape(cfg, &sh);
  if (s != MOE_OK) return s;
  if (sh.T == 0) return MOE_OK;  // empty batch: nothing is read or written
  if (!dev_ok(x) || !dev_ok(w_router) || !dev_ok(bias) || !dev_ok(topk_idx) ||
      !dev_ok(topk_gate) || !opt_ok(logits) || !opt_ok(flags))
    return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(sh, ws, ws_bytes)) != MOE_OK) return s;
  const WsLayout L = ws_layout(sh);
  return cuda_status(launch_router(sh, x, w_router, bias, at<float>(ws, L.logits),
                                   topk_idx, topk_gate, flags, logits,
                                   at<void>(ws, L.planes), at<int32_t>(ws, L.router_plan),
                                   at<int32_t>(ws, L.header),
                                   reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                          int32_t* counts, int32_t* offsets, int32_t* row_token,
                          int32_t* slot_row, void* x_perm, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
  NvtxRange range("moe_dispatch");
  Shape sh;
  moe_status_t s = make_shape(cfg, &sh);
  if (s != MOE_OK) return s;
  if (sh.T == 0) return MOE_OK;  // empty batch: nothing is read or written
  if (!dev_ok(x) || !dev_ok(topk_idx) || !dev_ok(counts) || !dev_ok(offsets) ||
      !dev_ok(row_token) || !dev_ok(slot_row) || !dev_ok(x_perm))
    return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(sh, ws, ws_bytes)) != MOE_OK) return s;
  const WsLayout L = ws_layout(sh);
  return cuda_status(launch_dispatch(sh, x, topk_idx, at<int32_t>(ws, L.chunk_base),
                                     counts, offsets, row_token, slot_row, x_perm,
                                     at<int32_t>(ws, L.header),
                                     reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_expert_ffn(const moe_config_t* cfg, const void* x_perm,
                            const int32_t* offsets, const void* w_gate, const void* w_up,
                            const void* w_down, void* y_perm, void* ws, size_t ws_bytes,
                            moe_stream_t stream) {
  NvtxRange range("moe_expert_ffn");
  Shape sh;
  moe_status_t s = make_shape(cfg, &sh);
  if (s != MOE_OK) return s;
  if (sh.T == 0) return MOE_OK;  // empty batch: nothing is read or written
  if (!dev_ok(x_perm) || !dev_ok(offsets) || !dev_ok(y_perm)) return MOE_ERR_INVALID_ARG;
  if (sh.N > 0 && (!dev_ok(w_gate) || !dev_ok(w_up) || !dev_ok(w_down)))
    return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(sh, ws, ws_bytes)) != MOE_OK) return s;
  const WsLayout L = ws_layout(sh);
  return cuda_status(launch_expert_ffn(sh, x_perm, offsets, w_gate, w_up, w_down,
                                       at<void>(ws, L.h), y_perm,
                                       at<int32_t>(ws, L.tile_start),
                                       at<int32_t>(ws, L.header),
                                       reinterpret_cast<cudaStream_t>(stream), nullptr,
                                       nullptr, false, at<float>(ws, L.ffn_part), false));
}

moe_status_t moe_combine(const moe_config_t* cfg, const void* x, const void* y_perm,
                         const int32_t* topk_idx, const float* topk_gate,
                         const int32_t* slot_row, void* out, moe_stream_t stream) {
  NvtxRange range("moe_combine");
  Shape sh;
  moe_status_t s = make_shape(cfg, &sh);
  if (s != MOE_OK) return s;
  if (sh.T == 0) return MOE_OK;  // empty batch: nothing is read or written
  if (!dev_ok(x) || !dev_ok(y_perm) || !dev_ok(topk_idx) || !dev_ok(topk_gate) ||
      !dev_ok(slot_row) || !dev_ok(out))
    return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_combine(sh, x, y_perm, topk_idx, topk_gate, slot_row, out,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_layer_forward(const moe_config_t* cfg, const void* x,
                               const float* w_router, const float* bias,
                               const void* w_gate, const void* w_up, const void* w_down,
                               void* out, int32_t* counts, void* ws, size_t ws_bytes,
                               moe_stream_t stream) {
  NvtxRange range("moe_layer_forward");
  Shape sh;
  moe_status_t s = make_shape(cfg, &sh);
  if (s != MOE_OK) return s;
  if (sh.T == 0) return MOE_OK;  // empty batch: nothing is read or written
  if (!dev_ok(x) || !dev_ok(w_router) || !dev_ok(bias) || !dev_ok(out) ||
      !opt_ok(counts))
    return MOE_ERR_INVALID_ARG;
  if (sh.N > 0 && (!dev_ok(w_gate) || !dev_ok(w_up) || !dev_ok(w_down)))
    return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(sh, ws, ws_bytes)) != MOE_OK) return s;
  return run_layer(sh, x, w_router, bias, w_gate, w_up, w_down, out, counts, ws,
                   reinterpret_cast<cudaStream_t>(stream));
}

moe_status_t moe_layer_forward_host(const moe_config_t* cfg, const void* x_host,
                                    const float* w_router, const float* bias,
                                    const void* w_gate, const void* w_up,
                                    const void* w_down, void* out_host,
                                    int32_t* counts_host, void* ws, size_t ws_bytes,
                                    moe_stream_t stream) {
  NvtxRange range("moe_layer_forward_host");
  Shape sh;
  moe_status_t s = make_shape(cfg, &sh);
  if (s != MOE_OK) return s;
  if (sh.T == 0) return MOE_OK;  // empty batch: nothing is read or written
  if (x_host == nullptr || out_host == nullptr || !dev_ok(w_router) || !dev_ok(bias))
    return MOE_ERR_INVALID_ARG;
  if (sh.N > 0 && (!dev_ok(w_gate) || !dev_ok(w_up) || !dev_ok(w_down)))
    return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(sh, ws, ws_bytes)) != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(sh);
  const size_t act_bytes = (size_t)sh.T * sh.d * sh.es;
  void* xd = at<void>(ws, L.x_stage);
  void* od = at<void>(ws, L.out_stage);
  int32_t* cd = at<int32_t>(ws, L.counts);
  if (cudaMemcpyAsync(xd, x_host, act_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  s = run_layer(sh, xd, w_router, bias, w_gate, w_up, w_down, od, cd, ws, st);
  if (s != MOE_OK) return s;
  if (cudaMemcpyAsync(out_host, od, act_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (counts_host &&
      cudaMemcpyAsync(counts_host, cd, (size_t)sh.E * sizeof(int32_t),
                      cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status_t moe_bias_pid_update(const moe_config_t* cfg, const int32_t* counts,
                                 float* bias, double* state,
                                 const moe_pid_params_t* params, moe_stream_t stream) {
  NvtxRange range("moe_bias_pid_update");
  Shape sh;
  moe_status_t s = make_shape(cfg, &sh);
  if (s != MOE_OK) return s;
  if (!dev_ok(counts) || !dev_ok(bias) || !dev_ok(state) || params == nullptr)
    return MOE_ERR_INVALID_ARG;
  const moe_pid_params_t& p = *params;
  if (!(p.target_routed_share >= 0.f && p.target_routed_share <= 1.f)) return MOE_ERR_INVALID_ARG;
  const float g[4] = {p.kp, p.ki, p.kd, p.max_step};
  for (float v : g)
    if (!isfinite(v) || v < 0.f) return MOE_ERR_INVALID_ARG;
  if (sh.T == 0) return MOE_OK;
  return cuda_status(launch_bias_pid(sh, counts, bias, state, p.target_routed_share, p.kp,
                                     p.ki, p.kd, p.max_step,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

int32_t moe_ep_local_experts(const moe_config_t* cfg, int32_t rank, int32_t world) {
  Shape sh;
  if (make_shape(cfg, &sh) != MOE_OK || world < 1 || rank < 0 || rank >= world) return -1;
  return ep_local_experts(rank, (int)sh.N, world);
}

moe_status_t moe_ep_plan(const moe_config_t* cfg, int32_t rank, int32_t world,
                         const int32_t* counts_all, int32_t* dest_row, int32_t* recv_offsets,
                         moe_stream_t stream) {
  NvtxRange range("moe_ep_plan");
  Shape sh;
  moe_status_t s = make_shape(cfg, &sh);
  if (s != MOE_OK) return s;
  if (world < 1 || rank < 0 || rank >= world || sh.N < 1) return MOE_ERR_INVALID_ARG;
  if (!dev_ok(counts_all) || !dev_ok(dest_row) || !dev_ok(recv_offsets))
    return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_ep_plan(sh, rank, world, counts_all, dest_row, recv_offsets,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_dispatch(const moe_config_t* cfg, int32_t world, const void* x,
                             const int32_t* offsets, const int32_t* row_token,
                             const int32_t* dest_row, void* const* recv_x,
                             moe_stream_t stream) {
  NvtxRange range("moe_ep_dispatch");
  Shape sh;
  moe_status_t s = make_shape(cfg, &sh);
  if (s != MOE_OK) return s;
  if (world < 1 || sh.N < 1) return MOE_ERR_INVALID_ARG;
  if (sh.T == 0) return MOE_OK;  // empty batch: nothing is read or written
  if (!dev_ok(x) || !dev_ok(offsets) || !dev_ok(row_token) || !dev_ok(dest_row) ||
      !dev_ok(recv_x))
    return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_ep_dispatch(sh, world, x, offsets, row_token, dest_row, recv_x,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_return(const moe_config_t* cfg, int32_t rank, int32_t world,
                           const void* y_recv, const int32_t* recv_offsets,
                           const int32_t* counts_all, const int32_t* offsets_all,
                           void* const* y_home, moe_stream_t stream) {
  NvtxRange range("moe_ep_return");
  Shape sh;
  moe_status_t s = make_shape(cfg, &sh);
  if (s != MOE_OK) return s;
  if (world < 1 || rank < 0 || rank >= world || sh.N < 1) return MOE_ERR_INVALID_ARG;
  if (!dev_ok(y_recv) || !dev_ok(recv_offsets) || !dev_ok(counts_all) ||
      !dev_ok(offsets_all) || !dev_ok(y_home))
    return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_ep_return(sh, rank, world, y_recv, recv_offsets, counts_all,
                                      offsets_all, y_home,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_selftest_wait_limit(void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (ws == nullptr || ws_bytes < 256 || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return MOE_ERR_WORKSPACE;
  return cuda_status(launch_wait_limit_selftest(static_cast<int32_t*>(ws),
                                                reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_read_device_error(void* ws, int32_t* code_out, moe_stream_t stream) {
  if (ws == nullptr) return MOE_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t code = 0;
  if (cudaMemcpyAsync(&code, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (code != 0) {
    if (cudaMemsetAsync(ws, 0, sizeof(int32_t), st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (code_out) *code_out = code;
  return code == 0 ? MOE_OK : MOE_ERR_DEVICE_CHECK;
}

int32_t moe_layer_launch_count(const moe_config_t* cfg) {
  Shape sh;
  if (make_shape(cfg, &sh) != MOE_OK || sh.T == 0) return 0;
  int32_t n = router_launch_count(sh);  // (split + GEMM | logits) + top-k
  n += dispatch_launch_count(sh);  // (count, scan, scatter | small) + gather
  if (sh.N > 0 && expert_ffn_gathers(sh) && !dispatch_gathers_in_sort(sh))
    n -= 1;  // the gate/up GEMM gathers
  n += expert_ffn_launch_count(sh);
  if (sh.N > 0 && expert_ffn_uses_tensor_cores(sh) && dispatch_plans_tiles(sh))
    n -= 1;  // the one-block dispatch writes the GEMM plans
  n += 1;                         // combine
  return n;
}

const char* moe_status_string(moe_status_t status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_CUDA: return "CUDA launch or copy failed";
    case MOE_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

}  // extern "C"
