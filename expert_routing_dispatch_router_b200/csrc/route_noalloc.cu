// moe_route_noalloc: the router + top-k call for callers that cannot allocate
// device memory.
//
// Who needs it: code that runs where cudaMalloc is not allowed or not safe,
// for example inside a memory pool that owns every byte of the device, in a
// plugin whose host framework forbids allocations after start-up, or in a
// latency-critical path that must never hit the allocator. Such callers can
// pass inputs and outputs but no workspace.
//
// How: the split-K partial sums that moe_route keeps in its workspace live
// here in one file-scope device array, kNoAllocScratchFloats floats (16 MiB),
// which every GPU that loads this library holds until the process exits. The
// first call on a device, with that device current, looks up the array's
// device address once (cudaGetSymbolAddress) and remembers it. The remembered
// address belongs
// to the device's primary context: after cudaDeviceReset on that device the
// process must not call this entry point again. Every call on a device shares
// the one array and leaves the last call's partial sums in it. Nothing has to
// start at zero: each call writes every partial sum it later reads. Calls
// whose work overlaps on the GPU (other streams, other host threads) race on
// the array, so the caller orders them.
#include <mutex>

#include "moe_internal.cuh"

namespace moe {
cudaError_t launch_router_simt(const Shape& sh, const void* x, const float* w_r,
                               const float* bias, float* part, int nsplit,
                               int32_t* idx, float* gate, uint8_t* flags,
                               float* logits_out, cudaStream_t st);
int router_splits(const Shape& sh);
bool router_simt_grid_fits(const Shape& sh);
moe_status_t shape_from_config(const moe_config_t* c, Shape* sh);
}  // namespace moe

namespace {

constexpr int64_t kNoAllocScratchFloats = 4 * 1024 * 1024;  // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_route_scratch[kNoAllocScratchFloats];

std::mutex g_setup_mutex;
float* g_scratch_ptr[kMaxDevices] = {};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of the scratch array on the current device (looked up once).
cudaError_t scratch_for_current_device(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" moe_status_t moe_route_noalloc(const moe_config_t* cfg, const void* x,
                                          const float* w_router, const float* bias,
                                          float* logits, int32_t* topk_idx,
                                          float* topk_gate, uint8_t* flags,
                                          moe_stream_t stream) {
  using namespace moe;
  Shape sh;
  const moe_status_t s = shape_from_config(cfg, &sh);  // the checks of every call
  if (s != MOE_OK) return s;
  if (sh.T == 0) return MOE_OK;  // empty batch: nothing is read or written
  if (x == nullptr || w_router == nullptr || bias == nullptr || topk_idx == nullptr ||
      topk_gate == nullptr || !aligned16(x) || !aligned16(w_router) || !aligned16(bias) ||
      !aligned16(topk_idx) || !aligned16(topk_gate) || !aligned16(logits) ||
      !aligned16(flags))
    return MOE_ERR_INVALID_ARG;
  // this call always runs the CUDA-core router, whatever path moe_route would
  // take for the shape, so its grid limit is checked here too; the partial
  // sums of one split need T * E floats
  const int64_t per_split = sh.T * sh.E;
  if (per_split > kNoAllocScratchFloats || !router_simt_grid_fits(sh))
    return MOE_ERR_UNSUPPORTED;
  // router_splits keeps nsplit * T * E near 2 * SMs * RT * RE (~0.6 M floats),
  // so this clamp only guards the array against a future split rule
  int nsplit = router_splits(sh);
  if ((int64_t)nsplit * per_split > kNoAllocScratchFloats)
    nsplit = (int)(kNoAllocScratchFloats / per_split);
  float* part = nullptr;
  if (scratch_for_current_device(&part) != cudaSuccess) return MOE_ERR_CUDA;
  const cudaError_t e =
      launch_router_simt(sh, x, w_router, bias, part, nsplit, topk_idx, topk_gate, flags,
                         logits, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
