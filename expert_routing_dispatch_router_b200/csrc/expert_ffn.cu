// Routed experts over the dispatched rows: a grouped SwiGLU FFN,
//   h = silu(x W_gate[e]^T) * (x W_up[e]^T),   y = h W_down[e]^T,
// for every expert e over its contiguous segment of rows [offsets[e],
// offsets[e+1]). LongCat-2.0 model card (archdb), "Mixture of experts" (expert
// dim) and "Feed-forward" (activation not disclosed; SwiGLU is the reading).
//
// Tensor-core path (bf16, d and F multiples of 128): one persistent kernel per
// GEMM (gate/up, then down), warp-specialised for sm_100a:
//   warp 0      TMA producer: weight tiles and token tiles -> smem ring
//   warp 1      MMA issuer: tcgen05.mma into TMEM (fp32), tcgen05.commit
//   warps 2..9  epilogue: tcgen05.ld from TMEM, SwiGLU, bf16 stores (two
//               warps per TMEM lane quarter, each taking every other
//               32-column chunk)
// The operands are swapped relative to the usual token-major GEMM: 128 rows
// of an expert's weight matrix fill the MMA's M = 128 and the expert's tokens
// (up to 128 per tile, rounded up to a multiple of 16) are its N. A decode
// batch gives an expert ~3 tokens, so this keeps the tensor work at N = 16
// instead of padding tokens to M = 128, and the kernel streams weights at
// HBM speed. The gate/up kernel loads the W_gate and W_up tiles of the same
// 128 rows and issues two MMAs against one token tile, so the epilogue has
// both accumulators of a row at hand. TMEM holds two accumulator buffers so
// the epilogue of one tile overlaps the MMAs of the next.
//
// Work unit = (expert, 128-row weight tile m, token tile). Units are numbered
// expert-major, then m, then token tile, so CTAs that run at the same time
// share weight tiles through L2. A tiny plan kernel turns offsets[] into
// per-expert token-tile prefix sums on the device; no host sync is needed.
//
// Every mbarrier wait is bounded (about 2 s); on expiry the kernel records an
// error code in the workspace, the other roles stop, outstanding TMA loads and
// MMAs are waited for (again bounded), TMEM is freed and the kernel returns.
//
// Rounding points: h is stored in the activation type (bf16 feeds the tensor
// cores); y is written in fp32 so that the combine rounds the output only once.
//
// CUDA-core path (f32, or shapes the tensor-core path does not take): one warp
// per output element, fp32 accumulation, same rounding points.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

// ------------------------------------------------------------------ plan --
// For token tiles of `tile` rows: tile_start[e] = sum over routed e' < e of
// ceil(count[e'] / tile); tile_start[N] = total token tiles. One block; N <= 1024.
__device__ __forceinline__ void tile_prefix(const int32_t* __restrict__ offsets, int N,
                                            int tile, int32_t* __restrict__ tile_start,
                                            int32_t* warp_sums) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int32_t v = 0;
  if ((int)threadIdx.x < N) {
    const int32_t n = offsets[threadIdx.x + 1] - offsets[threadIdx.x];
    v = (n + tile - 1) / tile;
  }
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
  const int32_t before = (wid > 0 ? warp_sums[wid - 1] : 0) + incl - v;
  if ((int)threadIdx.x < N) tile_start[threadIdx.x] = before;
  if (threadIdx.x == 0) tile_start[N] = warp_sums[31];
  __syncthreads();
}

// Plans of both expert GEMMs: gate/up tiles of tile_gu tokens into
// tile_start[0..N], down tiles of tile_dn tokens into tile_start[N+1..2N+1].
__global__ void __launch_bounds__(1024)
    gemm_plan_kernel(const int32_t* __restrict__ offsets, int N, int tile_gu, int tile_dn,
                     int32_t* __restrict__ tile_start) {
  __shared__ int32_t warp_sums[32];
  griddep_wait();
  griddep_launch_dependents();
  tile_prefix(offsets, N, tile_gu, tile_start, warp_sums);
  tile_prefix(offsets, N, tile_dn, tile_start + N + 1, warp_sums);
  if (threadIdx.x == 0) {  // the CTA-pair GEMMs' unit counters
    tile_start[2 * N + 2] = 0;
    tile_start[2 * N + 3] = 0;
  }
}

// ------------------------------------------------------- tensor-core path --
constexpr int BM = 128;  // weight rows per tile (MMA M)
constexpr int BK = 64;   // contraction elements per stage: 128-byte rows
// warp 0: TMA producer, warp 1: MMA issuer, warps 2..9: epilogue (two warps
// per TMEM lane quarter, splitting the accumulator columns)
constexpr int kThreads = 320;
constexpr int kEpiWarps = 8;
// CTA pairs: unit ring depth and readers of each slot (leader MMA thread,
// leader epilogue warps, peer producer, peer epilogue warps)
constexpr int kRing = 4;
constexpr int kRingReaders = 1 + kEpiWarps + 1 + kEpiWarps;
constexpr uint32_t kTileBytes = BM * BK * 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccStride = 256;  // TMEM columns per accumulator buffer (2 buffers)
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Gate/up: two weight tiles (W_gate, W_up rows) x up to BN tokens, two fp32
// accumulators of BN columns. Down: one weight tile x up to BN tokens, one
// accumulator of BN columns. When one accumulator set fits in 256 TMEM
// columns there are two sets, so the epilogue of a tile overlaps the MMAs of
// the next; the 256-token gate/up tile fills all 512 columns with one set and
// the MMAs wait for its epilogue (short against its 64-block main loop).
// Token tiles are sized to the batch on the host (an expert sees at most T
// rows): small tiles leave room for more stages, so a decode step keeps more
// weight bytes in flight, and large tiles halve the bytes each FLOP needs.
template <bool GATEUP, int BN_>
struct Cfg {
  static constexpr int kNumA = GATEUP ? 2 : 1;
  static constexpr int BN = BN_;  // max MMA N
  static_assert(BN % 16 == 0 && BN <= 256, "token tile");
  static constexpr uint32_t kAccCols = kNumA * BN;  // columns of one accumulator set
  static constexpr int kAccBufs = kAccCols <= kAccStride ? 2 : 1;
  static constexpr uint32_t kBBytes = BN * BK * 2;
  static constexpr uint32_t kStageBytes = kNumA * kTileBytes + kBBytes;
  static constexpr int kStages =
      (204800 / kStageBytes) > 8 ? 8 : (int)(204800 / kStageBytes);
  static constexpr uint32_t kBarOff = kStages * kStageBytes;
  static constexpr uint32_t kTabOff = kBarOff + 256;
  static constexpr uint32_t kSmemBytes =
      1024 + kTabOff + 2 * 4 * (kMaxExperts + 1);
};

struct GemmArgs {
  const int32_t* offsets;     // [N+1] row offsets per expert
  const int32_t* tile_start;  // [N+1] token-tile prefix per expert
  void* out;                  // [rows_cap, out_cols]: bf16 h, bf16 y or fp32 rows
  int32_t* err;               // workspace error word
  int N;
  int num_kb;    // contraction length / BK
  int out_cols;  // output row stride: F for gate/up, d for down
  int m_tiles;   // out_cols / BM
  int a_rows;    // rows of A per expert (A row = e * a_rows + (m % mt_chunk) * BM)
  int mt_chunk;  // m-tiles per contraction chunk: m-tile m covers k-blocks
  int kb_chunk;  // [(m / mt_chunk) * kb_chunk, +kb_chunk) with a fresh accumulator
  // Gate/up of the fused layer (single-CTA path): when set, token rows are
  // gathered from x by row_token with TMA gather4 (tmB16 is then x's map with
  // a one-row box) instead of being read from x_perm; oob_row is a row outside
  // x, which reads as zeros, for the padding rows of a tile.
  const int32_t* row_token = nullptr;
  int oob_row = 0;
  // Gate/up with a split contraction (tiny batches): when set, the epilogue
  // writes the raw fp32 gate and up sums of split m / mt_chunk to
  // part[row][split][0 or 1][F] (part_stride floats per row) instead of h; a
  // fixup kernel adds the splits and applies SwiGLU.
  float* part = nullptr;
  int64_t part_stride = 0;
  // CTA pairs: units are handed out in order from this counter (zeroed with
  // the tile plan before the launch)
  int* unit_counter = nullptr;
  // Down GEMM: output rows in bf16 (the expert outputs y_perm) instead of
  // fp32 (the router's logits and split-contraction partials)
  bool out_bf16 = false;
  // Tensor-core router: when > 0, the A rows are the three bf16 planes of
  // this many experts, each 32-row quarter of an m-tile holding hi, mid and
  // lo of 10 experts in rows 3j, 3j + 1, 3j + 2; the epilogue adds the three
  // planes of an expert (hi + mid, then + lo, in fp32) and writes
  // out[token][chunk * plane_experts + e]
  int plane_experts = 0;
};

struct Unit {
  int e, m, row0, n_valid, n_mma, ntiles;
};

template <int BN>
__device__ __forceinline__ Unit decode_unit(int u, const int* s_tiles,
                                            const int* s_offs, int N,
                                            int m_tiles) {
  int lo = 0, hi = N - 1;  // largest e with m_tiles * tile_start[e] <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (m_tiles * s_tiles[mid] <= u)
      lo = mid;
    else
      hi = mid - 1;
  }
  Unit un;
  un.e = lo;
  const int ntiles = s_tiles[lo + 1] - s_tiles[lo];
  un.ntiles = ntiles;
  const int local = u - m_tiles * s_tiles[lo];
  un.m = local / ntiles;
  const int tt = local - un.m * ntiles;
  un.row0 = s_offs[lo] + tt * BN;
  const int rem = s_offs[lo + 1] - un.row0;
  un.n_valid = rem < BN ? rem : BN;
  un.n_mma = (un.n_valid + 15) & ~15;
  return un;
}

// Bounded wait on an mbarrier phase. Returns false when the CTA was told to
// stop or when the limit ran out (then it tells the CTA to stop and records
// the error).
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity,
                                             volatile int* abort_flag,
                                             int32_t* err) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::global_timer_ns();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (ptx::global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicCAS(err, 0, kErrWaitTimeout);
      return false;
    }
  }
}

// wait_bounded with cluster-scope acquire (phases completed by the other CTA).
__device__ __forceinline__ bool wait_bounded_cluster(uint32_t bar, uint32_t parity,
                                                     volatile int* abort_flag,
                                                     int32_t* err) {
  if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = ptx::global_timer_ns();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
    if (*abort_flag) return false;
    if (ptx::global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicCAS(err, 0, kErrWaitTimeout);
      return false;
    }
  }
}

// Bounded wait that ignores the stop flag (used while cleaning up).
__device__ __forceinline__ void wait_cleanup(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = ptx::global_timer_ns();
  while (!ptx::mbar_try_wait(bar, parity))
    if (ptx::global_timer_ns() - t0 > kWaitLimitNs) return;
}

// silu(z) = z / (1 + e^-z); the fast divide's 2-ulp error is far below the
// bf16 rounding of h that follows (and it returns 0 once 1 + e^-z overflows,
// where silu is 0 to fp32 precision anyway)
__device__ __forceinline__ float silu_f(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// SwiGLU epilogue of one epilogue warp's share of a gate/up accumulator: its
// 32-column chunks c0 = 32 eh + 64 q (q < NQ, c0 < n_cols) are read from TMEM
// (gate at column c0, up at bn_off + c0) and become bf16 h in registers. Then
// release() hands the accumulator back to the MMA warp, and only after that
// are the rows stored: the next unit's MMAs do not wait for the stores.
template <int NQ, typename Release>
__device__ __forceinline__ void swiglu_epilogue(uint32_t tb, uint32_t bn_off, int eh,
                                                int n_cols, int n_valid, __nv_bfloat16* outp,
                                                int64_t out_cols, Release release) {
  uint32_t hb[NQ][16];
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int c0 = 32 * eh + 64 * q;
    if (c0 < n_cols) {  // warp-uniform
      float g[32], v[32];
      ptx::tmem_ld32x2(tb + c0, tb + bn_off + c0, g, v);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const __nv_bfloat162 p = __floats2bfloat162_rn(silu_f(g[2 * c]) * v[2 * c],
                                                       silu_f(g[2 * c + 1]) * v[2 * c + 1]);
        hb[q][c] = *reinterpret_cast<const uint32_t*>(&p);
      }
    }
  }
  release();
  uint16_t* o16 = reinterpret_cast<uint16_t*>(outp);
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int c0 = 32 * eh + 64 * q;
    if (c0 < n_cols) {
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (c0 + c < n_valid)
          o16[(int64_t)(c0 + c) * out_cols] =
              (c & 1) ? (uint16_t)(hb[q][c >> 1] >> 16) : (uint16_t)(hb[q][c >> 1] & 0xffffu);
    }
  }
}

template <bool GATEUP, int BN_>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA0,
                           const __grid_constant__ CUtensorMap tmA1,
                           const __grid_constant__ CUtensorMap tmB16,
                           const __grid_constant__ CUtensorMap tmB128,
                           const GemmArgs args) {
  using C = Cfg<GATEUP, BN_>;
  constexpr int S = C::kStages;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = ptx::smem_addr(smem);
  const uint32_t bars = sbase + C::kBarOff;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (S + s); };
  auto tfull_bar = [&](int b) { return bars + 8u * (2 * S + b); };
  auto tempty_bar = [&](int b) { return bars + 8u * (2 * S + 2 + b); };
  const uint32_t mma_done_bar = bars + 8u * (2 * S + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + 8 * (2 * S + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_tiles = reinterpret_cast<int*>(smem + C::kTabOff);
  int* s_offs = s_tiles + (kMaxExperts + 1);
  __shared__ int s_ids[BN_];  // token ids of the current unit's rows (gather)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = args.N;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(tfull_bar(b), 1);
      ptx::mbar_init(tempty_bar(b), kEpiWarps);
    }
    ptx::mbar_init(mma_done_bar, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tensormap(&tmA0);
    if (GATEUP) ptx::prefetch_tensormap(&tmA1);
    ptx::prefetch_tensormap(&tmB16);
    ptx::prefetch_tensormap(&tmB128);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_addr(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  // everything above overlaps the previous kernel's tail; the plan and the
  // operands are read only after it has completed
  griddep_wait();
  griddep_launch_dependents();
  for (int i = threadIdx.x; i <= N; i += blockDim.x) {
    s_tiles[i] = args.tile_start[i];
    s_offs[i] = args.offsets[i];
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  const int total_units = s_tiles[N] * args.m_tiles;

  if (warp == 0) {
    // ---------------------------------------------------- TMA producer --
    // Lane 0 issues the copies. When the token rows are gathered from x, the
    // whole warp fetches the token ids one unit ahead (lane + 32 i of the next
    // unit's rows), so the copies never wait for them.
    const bool gather = GATEUP && args.row_token != nullptr;
    constexpr int kIds = BN / 32;
    int nxt[kIds];
    auto fetch_ids = [&](int u) {
      if (u < total_units) {
        const Unit nu = decode_unit<BN>(u, s_tiles, s_offs, N, args.m_tiles);
#pragma unroll
        for (int i = 0; i < kIds; ++i) {
          const int j = lane + 32 * i;  // padding rows read a row outside x: zeros
          nxt[i] = j < nu.n_valid ? __ldg(args.row_token + nu.row0 + j) : args.oob_row;
        }
      }
    };
    if (gather) fetch_ids(blockIdx.x);
    // L2 policy per unit: an expert with a single token tile reads each
    // weight tile once (a decode step), so its weights are streamed
    // evict-first and its few token rows kept evict-last. An expert with
    // several token tiles reuses every weight tile once per token tile, so
    // both operands use the normal policy.
    const uint64_t pol_first = ptx::policy_evict_first();
    const uint64_t pol_last = ptx::policy_evict_last();
    const uint64_t pol_normal = ptx::policy_evict_normal();
    int stage = 0;
    uint32_t phase = 0, armed = 0, armed_par = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
      const Unit un = decode_unit<BN>(u, s_tiles, s_offs, N, args.m_tiles);
      if (gather) {
#pragma unroll
        for (int i = 0; i < kIds; ++i) s_ids[lane + 32 * i] = nxt[i];
        __syncwarp();
        fetch_ids(u + (int)gridDim.x);
      }
      if (lane == 0) {
        const int arow = un.e * args.a_rows + (un.m % args.mt_chunk) * BM;
        const int kb0 = (un.m / args.mt_chunk) * args.kb_chunk;
        const uint32_t bytes = C::kNumA * kTileBytes + (uint32_t)un.n_mma * 128u;
        const uint64_t pol_w = un.ntiles == 1 ? pol_first : pol_normal;
        const uint64_t pol_x = un.ntiles == 1 ? pol_last : pol_normal;
        for (int kb = kb0; kb < kb0 + args.kb_chunk; ++kb) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, args.err)) {
            ok = false;
            break;
          }
          const uint32_t fb = full_bar(stage);
          ptx::mbar_arrive_expect_tx(fb, bytes);
          const uint32_t a0 = sbase + stage * C::kStageBytes;
          ptx::tma_load_2d(&tmA0, a0, fb, kb * BK, arow, pol_w);
          if (GATEUP) ptx::tma_load_2d(&tmA1, a0 + kTileBytes, fb, kb * BK, arow, pol_w);
          // token rows: 128-row boxes while 128 or more remain, then 16-row
          // boxes; or, gathering from x, four rows per request
          const uint32_t b0 = a0 + C::kNumA * kTileBytes;
          if (gather) {
            for (int j = 0; j < un.n_mma; j += 4)
              ptx::tma_gather4_2d(&tmB16, b0 + j * 128u, fb, kb * BK, s_ids[j], s_ids[j + 1],
                                  s_ids[j + 2], s_ids[j + 3], pol_x);
          } else {
            int j = 0;
            for (; j + 128 <= un.n_mma; j += 128)
              ptx::tma_load_2d(&tmB128, b0 + j * 128u, fb, kb * BK, un.row0 + j, pol_x);
            for (; j < un.n_mma; j += 16)
              ptx::tma_load_2d(&tmB16, b0 + j * 128u, fb, kb * BK, un.row0 + j, pol_x);
          }
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every lane follows lane 0 (and keeps s_ids until its copies are issued)
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (lane == 0 && !ok) {  // let our own loads land before the CTA goes away
      for (int s = 0; s < S; ++s)
        if ((armed >> s) & 1u) wait_cleanup(full_bar(s), (armed_par >> s) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer --
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true, issued = false;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        const Unit un = decode_unit<BN>(u, s_tiles, s_offs, N, args.m_tiles);
        if (!wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag, args.err)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t idesc = ptx::idesc_bf16_f32(BM, un.n_mma);
        const uint32_t d0 = tmem_base + (uint32_t)acc * kAccStride;  // acc = 0 if one set
        for (int kb = 0; kb < args.kb_chunk; ++kb) {
          if (!wait_bounded(full_bar(stage), phase, abort_flag, args.err)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a0 = sbase + stage * C::kStageBytes;
          const uint32_t b0 = a0 + C::kNumA * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bdesc = ptx::desc_k_sw128(b0 + kk * 32);
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            ptx::mma_bf16(d0, ptx::desc_k_sw128(a0 + kk * 32), bdesc, idesc, accum);
            if (GATEUP)
              ptx::mma_bf16(d0 + BN, ptx::desc_k_sw128(a0 + kTileBytes + kk * 32),
                            bdesc, idesc, accum);
          }
          issued = true;
          ptx::mma_commit(empty_bar(stage));
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        ptx::mma_commit(tfull_bar(acc));
        if (++acc == C::kAccBufs) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok && issued) {  // the MMAs already issued must finish before TMEM is freed
        ptx::mma_commit(mma_done_bar);
        wait_cleanup(mma_done_bar, 0);
      }
    }
  } else {
    // -------------------------------------------------------- epilogue --
    const int ew = warp & 3;          // TMEM lane quarter this warp may access
    const int eh = (warp - 2) >> 2;   // which half of the column chunks
    const int lrow = ew * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
      const Unit un = decode_unit<BN>(u, s_tiles, s_offs, N, args.m_tiles);
      const bool ok = wait_bounded(tfull_bar(acc), acc_phase, abort_flag, args.err);
      if (!__all_sync(0xffffffffu, ok)) break;
      ptx::tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) +
                          (uint32_t)acc * kAccStride;
      const int64_t col = (int64_t)un.m * BM + lrow;
      const int64_t obase = (int64_t)un.row0 * args.out_cols + col;
      // 32-column chunks, alternating between the two warps of this quarter
      auto release = [&]() {
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(tempty_bar(acc));
      };
      if (GATEUP && BN == 64 && args.part != nullptr) {  // splits only at T <= 64
        const int split = un.m / args.mt_chunk;
        float* pp = args.part + (int64_t)un.row0 * args.part_stride +
                    (int64_t)split * 2 * args.out_cols +
                    (int64_t)(un.m % args.mt_chunk) * BM + lrow;
        for (int c0 = 32 * eh; c0 < un.n_mma; c0 += 64) {
          float g[32], v[32];
          ptx::tmem_ld32x2(tb + c0, tb + BN + c0, g, v);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c0 + c < un.n_valid) {
              pp[(int64_t)(c0 + c) * args.part_stride] = g[c];
              pp[(int64_t)(c0 + c) * args.part_stride + args.out_cols] = v[c];
            }
        }
        release();
      } else if (GATEUP) {
        swiglu_epilogue<BN / 64>(tb, BN, eh, un.n_mma, un.n_valid,
                                 static_cast<__nv_bfloat16*>(args.out) + obase, args.out_cols,
                                 release);
      } else {
        for (int c0 = 32 * eh; c0 < un.n_mma; c0 += 64) {
          float g[32];
          ptx::tmem_ld32(tb + c0, g);
          if (args.out_bf16) {
            __nv_bfloat16* outp = static_cast<__nv_bfloat16*>(args.out) + obase;
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c0 + c < un.n_valid)
                outp[(int64_t)(c0 + c) * args.out_cols] = __float2bfloat16_rn(g[c]);
          } else if (args.plane_experts > 0) {
            const int64_t e =
                (int64_t)(un.m % args.mt_chunk) * 40 + (int64_t)ew * 10 + lane / 3;
            const bool writer = lane < 30 && lane % 3 == 0 && e < args.plane_experts;
            float* outp = static_cast<float*>(args.out) + (int64_t)un.row0 * args.out_cols +
                          (int64_t)(un.m / args.mt_chunk) * args.plane_experts + e;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float mid = __shfl_down_sync(0xffffffffu, g[c], 1);
              const float lo = __shfl_down_sync(0xffffffffu, g[c], 2);
              if (writer && c0 + c < un.n_valid)
                outp[(int64_t)(c0 + c) * args.out_cols] = (g[c] + mid) + lo;
            }
          } else {
            float* outp = static_cast<float*>(args.out) + obase;
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c0 + c < un.n_valid) outp[(int64_t)(c0 + c) * args.out_cols] = g[c];
          }
        }
        release();
      }
      if (++acc == C::kAccBufs) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------- split contraction (tiny batches) --
// h[r, f] = silu(sum_c gate_c[r, f]) * sum_c up_c[r, f] for the routed rows
// r < R, the split partials added in order c = 0..s-1 (part as written by the
// split gate/up epilogue: [row][c][gate | up][F] fp32).
__global__ void __launch_bounds__(256)
    swiglu_split_fixup_kernel(const float* __restrict__ part, int s, int64_t F,
                              const int32_t* __restrict__ offsets, int N,
                              __nv_bfloat16* __restrict__ h) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t R = offsets[N];
  const int64_t fv = F / 4;
  const int64_t stride = (int64_t)s * 2 * F;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < R * fv;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / fv, f = (i - r * fv) * 4;
    const float* p = part + r * stride + f;
    float4 g = *reinterpret_cast<const float4*>(p);
    float4 u = *reinterpret_cast<const float4*>(p + F);
    for (int c = 1; c < s; ++c) {
      const float4 gc = *reinterpret_cast<const float4*>(p + (int64_t)c * 2 * F);
      const float4 uc = *reinterpret_cast<const float4*>(p + (int64_t)c * 2 * F + F);
      g.x += gc.x; g.y += gc.y; g.z += gc.z; g.w += gc.w;
      u.x += uc.x; u.y += uc.y; u.z += uc.z; u.w += uc.w;
    }
    const __nv_bfloat162 a = __floats2bfloat162_rn(silu_f(g.x) * u.x, silu_f(g.y) * u.y);
    const __nv_bfloat162 b = __floats2bfloat162_rn(silu_f(g.z) * u.z, silu_f(g.w) * u.w);
    uint2 o;
    o.x = *reinterpret_cast<const uint32_t*>(&a);
    o.y = *reinterpret_cast<const uint32_t*>(&b);
    *reinterpret_cast<uint2*>(h + r * F + f) = o;
  }
}

// y[r, :] = bf16(sum_c part[r][c][:]), the sum in fp32 in order c = 0..s-1,
// for the routed rows r < R (the down GEMM's split partials, [row][c][d]).
__global__ void __launch_bounds__(256)
    split_reduce_kernel(const float* __restrict__ part, int s, int64_t d,
                        const int32_t* __restrict__ offsets, int N,
                        __nv_bfloat16* __restrict__ y) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t R = offsets[N];
  const int64_t dv = d / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < R * dv;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / dv, col = (i - r * dv) * 4;
    const float* p = part + r * s * d + col;
    float4 v = *reinterpret_cast<const float4*>(p);
    for (int c = 1; c < s; ++c) {
      const float4 w = *reinterpret_cast<const float4*>(p + (int64_t)c * d);
      v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
    }
    const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    const __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 o;
    o.x = *reinterpret_cast<const uint32_t*>(&a);
    o.y = *reinterpret_cast<const uint32_t*>(&b);
    *reinterpret_cast<uint2*>(y + r * d + col) = o;
  }
}

// -------------------------------------------- CTA-pair path (cta_group::2) --
// For batches with many rows per expert the same GEMMs run on pairs of CTAs
// (a 2-CTA cluster on one GPC). A unit is (expert, 256 weight rows, up to 256
// tokens): each CTA loads 128 of the weight rows and half of the token rows,
// the leader issues M = 256 MMAs that read both CTAs' shared memory, and each
// CTA's TMEM receives the accumulators of its own 128 weight rows for all the
// unit's tokens. Per FLOP this loads half the shared-memory bytes of the
// single-CTA kernel, and the two CTAs that share every tile sit on one die.
//
// Protocol (barriers at the same offsets in both CTAs):
//   full[s]   leader's: armed by the leader's producer with both CTAs' bytes;
//             both CTAs' TMA loads complete on it (cta_group::2 loads)
//   empty[s]  both: the leader's MMA commit arrives on both (multicast commit)
//   tfull[b]  both: the leader's commit after a unit's last MMA
//   tempty[b] leader's, 16 arrivals: 8 epilogue warps here + 8 in the peer
template <bool GATEUP>
struct PairCfg {
  static constexpr int kNumA = GATEUP ? 2 : 1;
  static constexpr int BN = 256;   // token columns of a unit (both CTAs)
  static constexpr int BNH = 128;  // token rows one CTA loads, at most
  static constexpr uint32_t kStageBytes = kNumA * kTileBytes + BNH * BK * 2;
  static constexpr int kStages = (int)(204800 / kStageBytes);  // 4 or 6
  static constexpr uint32_t kAccCols = kNumA * BN;             // 512 or 256
  static constexpr int kAccBufs = kAccCols <= kAccStride ? 2 : 1;
  static constexpr uint32_t kBarOff = kStages * kStageBytes;
  static constexpr uint32_t kTabOff = kBarOff + 256;
  static constexpr uint32_t kSmemBytes = 1024 + kTabOff + 2 * 4 * (kMaxExperts + 1);
};

// Busy wait of about `ns` nanoseconds (lets in-flight copies land on abort).
__device__ __forceinline__ void settle_ns(uint64_t ns) {
  const uint64_t t0 = ptx::global_timer_ns();
  while (ptx::global_timer_ns() - t0 < ns) {
  }
}

template <bool GATEUP>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0,
                             const __grid_constant__ CUtensorMap tmA1,
                             const __grid_constant__ CUtensorMap tmB16,
                             const __grid_constant__ CUtensorMap tmB128,
                             const GemmArgs args) {
  using C = PairCfg<GATEUP>;
  constexpr int S = C::kStages;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = ptx::smem_addr(smem);
  const uint32_t bars = sbase + C::kBarOff;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (S + s); };
  auto tfull_bar = [&](int b) { return bars + 8u * (2 * S + b); };
  auto tempty_bar = [&](int b) { return bars + 8u * (2 * S + 2 + b); };
  const uint32_t mma_done_bar = bars + 8u * (2 * S + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + 8 * (2 * S + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // unit ring: the leader's producer hands each unit id to both CTAs
  auto ring_full = [&](int r) { return bars + 160u + 8u * r; };
  auto ring_empty = [&](int r) { return bars + 192u + 8u * r; };
  volatile int* s_ring = reinterpret_cast<volatile int*>(smem + C::kBarOff + 224);
  int* s_tiles = reinterpret_cast<int*>(smem + C::kTabOff);
  int* s_offs = s_tiles + (kMaxExperts + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = args.N;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(tfull_bar(b), 1);
      ptx::mbar_init(tempty_bar(b), 2 * kEpiWarps);
    }
    ptx::mbar_init(mma_done_bar, 1);
    for (int r = 0; r < kRing; ++r) {
      ptx::mbar_init(ring_full(r), 1);
      ptx::mbar_init(ring_empty(r), kRingReaders);
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tensormap(&tmA0);
    if (GATEUP) ptx::prefetch_tensormap(&tmA1);
    ptx::prefetch_tensormap(&tmB16);
    ptx::prefetch_tensormap(&tmB128);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(ptx::smem_addr(tmem_slot), kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  griddep_wait();
  griddep_launch_dependents();
  for (int i = threadIdx.x; i <= N; i += blockDim.x) {
    s_tiles[i] = args.tile_start[i];
    s_offs[i] = args.offsets[i];
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // both CTAs' barriers exist before any remote arrive
  ptx::tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  const int total_units = s_tiles[N] * args.m_tiles;
  // Dynamic schedule: the leader's producer takes the next unit from the
  // global counter (-1 once none are left) and publishes it in ring slot
  // seq % kRing of both CTAs; every other role reads its units from there, in
  // the same order. A slot is reused once its kRingReaders readers (the
  // leader's MMA thread and epilogue warps, the peer's producer and epilogue
  // warps) have arrived on the leader's ring_empty.
  auto publish = [&](int seq, int u) -> bool {
    const int r = seq % kRing;
    const uint32_t par = (uint32_t)(seq / kRing) & 1u;
    if (!wait_bounded(ring_empty(r), par ^ 1u, abort_flag, args.err)) return false;
    s_ring[r] = u;
    ptx::st_shared_cluster_u32(ptx::map_to_rank(ptx::smem_addr((const void*)(s_ring + r)), 1),
                               (uint32_t)u);
    ptx::mbar_arrive(ring_full(r));
    ptx::mbar_arrive_remote(ptx::map_to_rank(ring_full(r), 1));
    return true;
  };
  auto take = [&](int seq, int* u) -> bool {
    const int r = seq % kRing;
    const uint32_t par = (uint32_t)(seq / kRing) & 1u;
    if (!wait_bounded_cluster(ring_full(r), par, abort_flag, args.err)) return false;
    *u = s_ring[r];
    if (leader)
      ptx::mbar_arrive(ring_empty(r));
    else
      ptx::mbar_arrive_remote(ptx::map_to_rank(ring_empty(r), 0));
    return true;
  };

  if (warp == 0) {
    // ---------------------------------------------------- TMA producer --
    if (lane == 0) {
      const uint64_t pol_first = ptx::policy_evict_first();
      const uint64_t pol_last = ptx::policy_evict_last();
      const uint64_t pol_normal = ptx::policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_par = 0;
      bool ok = true, issued = false;
      for (int seq = 0; ok; ++seq) {
        int u = -1;
        if (leader) {
          u = atomicAdd(args.unit_counter, 1);
          if (u >= total_units) u = -1;
          ok = publish(seq, u);
        } else {
          ok = take(seq, &u);
        }
        if (!ok || u < 0) break;
        const Unit un = decode_unit<BN>(u, s_tiles, s_offs, N, args.m_tiles);
        const int n_pair = (un.n_valid + 31) & ~31;  // MMA N; each CTA holds half
        const int half = n_pair >> 1;
        const int arow = un.e * args.a_rows + un.m * 2 * BM + (int)rank * BM;
        const int brow = un.row0 + (int)rank * half;
        const uint32_t bytes = 2u * (C::kNumA * kTileBytes + (uint32_t)half * 128u);
        const uint64_t pol_w = un.ntiles == 1 ? pol_first : pol_normal;
        const uint64_t pol_x = un.ntiles == 1 ? pol_last : pol_normal;
        for (int kb = 0; kb < args.num_kb; ++kb) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, args.err)) {
            ok = false;
            break;
          }
          if (leader) ptx::mbar_arrive_expect_tx(full_bar(stage), bytes);
          const uint32_t lbar = ptx::map_to_rank(full_bar(stage), 0);
          const uint32_t a0 = sbase + stage * C::kStageBytes;
          ptx::tma_load_2d_pair(&tmA0, a0, lbar, kb * BK, arow, pol_w);
          if (GATEUP) ptx::tma_load_2d_pair(&tmA1, a0 + kTileBytes, lbar, kb * BK, arow, pol_w);
          const uint32_t b0 = a0 + C::kNumA * kTileBytes;
          int j = 0;
          for (; j + 128 <= half; j += 128)
            ptx::tma_load_2d_pair(&tmB128, b0 + j * 128u, lbar, kb * BK, brow + j, pol_x);
          for (; j < half; j += 16)
            ptx::tma_load_2d_pair(&tmB16, b0 + j * 128u, lbar, kb * BK, brow + j, pol_x);
          issued = true;
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // let our own loads land before the CTA goes away: the leader can see
        // them on its full barriers, the peer's complete on the leader's
        if (leader) {
          for (int s = 0; s < S; ++s)
            if ((armed >> s) & 1u) wait_cleanup(full_bar(s), (armed_par >> s) & 1u);
        } else if (issued) {
          settle_ns(2000000);
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------- MMA issuer (leader) --
    if (lane == 0 && leader) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true, issued = false;
      for (int seq = 0; ok; ++seq) {
        int u = -1;
        ok = take(seq, &u);
        if (!ok || u < 0) break;
        const Unit un = decode_unit<BN>(u, s_tiles, s_offs, N, args.m_tiles);
        const int n_pair = (un.n_valid + 31) & ~31;
        if (!wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag, args.err)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t idesc = ptx::idesc_bf16_f32(2 * BM, n_pair);
        const uint32_t d0 = tmem_base + (uint32_t)acc * kAccStride;
        for (int kb = 0; kb < args.num_kb; ++kb) {
          if (!wait_bounded(full_bar(stage), phase, abort_flag, args.err)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a0 = sbase + stage * C::kStageBytes;
          const uint32_t b0 = a0 + C::kNumA * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bdesc = ptx::desc_k_sw128(b0 + kk * 32);
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            ptx::mma_bf16_pair(d0, ptx::desc_k_sw128(a0 + kk * 32), bdesc, idesc, accum);
            if (GATEUP)
              ptx::mma_bf16_pair(d0 + BN, ptx::desc_k_sw128(a0 + kTileBytes + kk * 32),
                                 bdesc, idesc, accum);
          }
          issued = true;
          ptx::mma_commit_pair(empty_bar(stage));
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        ptx::mma_commit_pair(tfull_bar(acc));
        if (++acc == C::kAccBufs) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok && issued) {  // MMAs already issued must finish before TMEM is freed
        ptx::mma_commit_pair(mma_done_bar);
        wait_cleanup(mma_done_bar, 0);
      }
    }
  } else {
    // -------------------------------------------------------- epilogue --
    const int ew = warp & 3;          // TMEM lane quarter
    const int eh = (warp - 2) >> 2;   // which half of the column chunks
    const int lrow = ew * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int seq = 0;; ++seq) {
      int u = -1;
      bool got = true;
      if (lane == 0) got = take(seq, &u);
      got = __shfl_sync(0xffffffffu, got, 0);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (!got || u < 0) break;
      const Unit un = decode_unit<BN>(u, s_tiles, s_offs, N, args.m_tiles);
      const int n_pair = (un.n_valid + 31) & ~31;
      const bool ok = wait_bounded(tfull_bar(acc), acc_phase, abort_flag, args.err);
      if (!__all_sync(0xffffffffu, ok)) break;
      ptx::tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) +
                          (uint32_t)acc * kAccStride;
      const int64_t col = (int64_t)un.m * 2 * BM + (int64_t)rank * BM + lrow;
      const int64_t obase = (int64_t)un.row0 * args.out_cols + col;
      auto release = [&]() {
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (leader)
            ptx::mbar_arrive(tempty_bar(acc));
          else
            ptx::mbar_arrive_remote(ptx::map_to_rank(tempty_bar(acc), 0));
        }
      };
      if (GATEUP) {
        swiglu_epilogue<BN / 64>(tb, BN, eh, n_pair, un.n_valid,
                                 static_cast<__nv_bfloat16*>(args.out) + obase, args.out_cols,
                                 release);
      } else {  // pairs run only the expert GEMMs: y in bf16
        __nv_bfloat16* outp = static_cast<__nv_bfloat16*>(args.out) + obase;
        for (int c0 = 32 * eh; c0 < n_pair; c0 += 64) {
          float g[32];
          ptx::tmem_ld32(tb + c0, g);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c0 + c < un.n_valid)
              outp[(int64_t)(c0 + c) * args.out_cols] = __float2bfloat16_rn(g[c]);
        }
        release();
      }
      if (++acc == C::kAccBufs) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // neither CTA frees TMEM or exits while the pair works
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  // looked up once; callers on several host threads may race to store the
  // same pointer, hence the atomic
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

// Row-major bf16 matrix [rows, cols] seen as a 2-D tensor, box = 64 columns
// (128 bytes, 128-byte swizzle) x box_rows rows. Rows past `rows` read as 0.
bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
              uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool GATEUP, int BN>
cudaError_t launch_tc(const CUtensorMap& a0, const CUtensorMap& a1,
                      const CUtensorMap& b16, const CUtensorMap& b128,
                      const GemmArgs& args, cudaStream_t st) {
  using C = Cfg<GATEUP, BN>;
  static std::atomic<uint64_t> attr_set{0};
  const cudaError_t e =
      raise_smem_once(attr_set, grouped_gemm_tc_kernel<GATEUP, BN>, (int)C::kSmemBytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(grouped_gemm_tc_kernel<GATEUP, BN>, dim3(num_sms()), dim3(kThreads),
                    C::kSmemBytes, st, a0, a1, b16, b128, args);
}

// CTA-pair launch: clusters of 2 with programmatic dependent launch, as many
// pairs as can be resident at once (so the persistent schedule has no tail).
template <bool GATEUP>
cudaError_t launch_pair(const CUtensorMap& a0, const CUtensorMap& a1,
                        const CUtensorMap& b16, const CUtensorMap& b128,
                        const GemmArgs& args, cudaStream_t st) {
  using C = PairCfg<GATEUP>;
  static std::atomic<uint64_t> attr_set{0};
  static std::atomic<int> grids[64];  // resident pairs x 2, per device
  int dev = 0;
  cudaError_t e0 = cudaGetDevice(&dev);
  if (e0 != cudaSuccess) return e0;
  e0 = raise_smem_once(attr_set, grouped_gemm_pair_kernel<GATEUP>, (int)C::kSmemBytes);
  if (e0 != cudaSuccess) return e0;
  int grid = grids[dev & 63].load();
  if (grid == 0) {
    cudaError_t e = cudaSuccess;
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(num_sms());
    q.blockDim = dim3(kThreads);
    q.dynamicSmemBytes = C::kSmemBytes;
    cudaLaunchAttribute ca[1];
    ca[0].id = cudaLaunchAttributeClusterDimension;
    ca[0].val.clusterDim.x = 2;
    ca[0].val.clusterDim.y = 1;
    ca[0].val.clusterDim.z = 1;
    q.attrs = ca;
    q.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, grouped_gemm_pair_kernel<GATEUP>, &q);
    if (e != cudaSuccess) return e;
    if (clusters < 1) return cudaErrorInvalidConfiguration;
    const int most = num_sms() / 2;
    grid = 2 * (clusters < most ? clusters : most);
    grids[dev & 63].store(grid);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, grouped_gemm_pair_kernel<GATEUP>, a0, a1, b16, b128,
                            args);
}

// Token tiles of the two expert GEMMs for a batch of T tokens (an expert sees
// at most T rows, so a small batch gets small tiles and a deeper ring).
int tile_gateup_for(int64_t T) { return T <= 64 ? 64 : (T <= 1024 ? 128 : 256); }

// Batches with many rows per expert run both expert GEMMs on CTA pairs
// (256 weight rows per unit, so F and d must be multiples of 256).
bool use_pairs(const Shape& sh) {
  return sh.T > 1024 && sh.F % 256 == 0 && sh.d % 256 == 0;
}
int tile_down_for(int64_t T) { return T <= 64 ? 64 : (T <= 128 ? 128 : 256); }

// --------------------------------------------------------- CUDA-core path --
__device__ __forceinline__ int expert_of_row(const int32_t* offsets, int N, int64_t r) {
  int lo = 0, hi = N - 1;  // largest e with offsets[e] <= r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offsets[mid] <= r)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

template <typename AT>
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// h[r, f] = silu(x_perm[r] . w_gate[e, f]) * (x_perm[r] . w_up[e, f])
template <typename AT>
__global__ void __launch_bounds__(256)
    ffn_gateup_simt_kernel(const AT* __restrict__ x, const int32_t* __restrict__ offsets,
                           int N, const AT* __restrict__ wg, const AT* __restrict__ wu,
                           AT* __restrict__ h, int64_t d, int64_t F) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t R = offsets[N];
  const int lane = threadIdx.x & 31;
  const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       w < R * F; w += nw) {
    const int64_t r = w / F, f = w - (w / F) * F;
    const int e = expert_of_row(offsets, N, r);
    const AT* xr = x + r * d;
    const AT* gr = wg + ((int64_t)e * F + f) * d;
    const AT* ur = wu + ((int64_t)e * F + f) * d;
    float a = 0.f, u = 0.f;
    for (int64_t i = lane; i < d; i += 32) {
      const float xv = to_f32(xr[i]);
      a = fmaf(to_f32(gr[i]), xv, a);
      u = fmaf(to_f32(ur[i]), xv, u);
    }
    a = warp_sum<AT>(a);
    u = warp_sum<AT>(u);
    if (lane == 0) h[r * F + f] = from_f32<AT>(a / (1.0f + expf(-a)) * u);
  }
}

// y[r, n] = h[r] . w_down[e, n]   (fp32 sum, stored in the activation type)
template <typename AT>
__global__ void __launch_bounds__(256)
    ffn_down_simt_kernel(const AT* __restrict__ h, const int32_t* __restrict__ offsets,
                         int N, const AT* __restrict__ wd, AT* __restrict__ y,
                         int64_t d, int64_t F) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t R = offsets[N];
  const int lane = threadIdx.x & 31;
  const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       w < R * d; w += nw) {
    const int64_t r = w / d, n = w - (w / d) * d;
    const int e = expert_of_row(offsets, N, r);
    const AT* hr = h + r * F;
    const AT* dr = wd + ((int64_t)e * d + n) * F;
    float acc = 0.f;
    for (int64_t f = lane; f < F; f += 32) acc = fmaf(to_f32(dr[f]), to_f32(hr[f]), acc);
    acc = warp_sum<AT>(acc);
    if (lane == 0) y[r * d + n] = from_f32<AT>(acc);
  }
}

template <typename AT>
cudaError_t launch_simt(const Shape& sh, const void* x_perm, const int32_t* offsets,
                        const void* wg, const void* wu, const void* wd, void* h,
                        void* y, cudaStream_t st) {
  const unsigned blocks = (unsigned)num_sms() * 16;
  cudaError_t e = launch_pdl(ffn_gateup_simt_kernel<AT>, dim3(blocks), dim3(256), 0, st,
                             static_cast<const AT*>(x_perm), offsets, (int)sh.N,
                             static_cast<const AT*>(wg), static_cast<const AT*>(wu),
                             static_cast<AT*>(h), sh.d, sh.F);
  if (e != cudaSuccess) return e;
  return launch_pdl(ffn_down_simt_kernel<AT>, dim3(blocks), dim3(256), 0, st,
                    static_cast<const AT*>(h), offsets, (int)sh.N,
                    static_cast<const AT*>(wd), static_cast<AT*>(y), sh.d, sh.F);
}

}  // namespace

// Chunked dense GEMM on the tensor cores, run as one "expert" of the grouped
// kernel's down variant: for each contraction chunk c of kb_chunk * 64
// elements, out[t, c * M + i] = sum over k in chunk c of b[t, k] * a[i, k]
// (fp32, bf16 inputs). M is a multiple of 128 and K of kb_chunk * 64. Every
// chunk starts a fresh accumulator, which bounds the accumulation chain the
// tensor cores' fp32 adder runs through. plan is a device int32[4] holding
// {0, T, 0, ceil(T / kRouterGemmTile)} (the expert's rows, then its token tiles).
cudaError_t launch_dense_gemm_tc(const void* a, int64_t M, const void* b, int64_t T,
                                 int64_t K, int kb_chunk, int64_t plane_experts, float* out,
                                 const int32_t* plan, int32_t* err, cudaStream_t st) {
  CUtensorMap am, b16, b128;
  if (!make_map(&am, a, (uint64_t)M, (uint64_t)K, BM) ||
      !make_map(&b16, b, (uint64_t)T, (uint64_t)K, 16) ||
      !make_map(&b128, b, (uint64_t)T, (uint64_t)K, 128))
    return cudaErrorInvalidValue;
  const int chunks = (int)(K / BK) / kb_chunk;
  GemmArgs g;
  g.offsets = plan;
  g.tile_start = plan + 2;
  g.out = out;
  g.err = err;
  g.N = 1;
  g.num_kb = (int)(K / BK);
  g.out_cols = (int)(plane_experts > 0 ? plane_experts : M) * chunks;
  g.plane_experts = (int)plane_experts;
  g.m_tiles = (int)(M / BM) * chunks;
  g.a_rows = (int)M;
  g.mt_chunk = (int)(M / BM);
  g.kb_chunk = kb_chunk;
  return launch_tc<false, kRouterGemmTile>(am, am, b16, b128, g, st);
}

bool expert_ffn_uses_tensor_cores(const Shape& sh) {
  return sh.bf16 && sh.d % 128 == 0 && sh.F % 128 == 0 && sh.N <= kMaxExperts;
}

int expert_ffn_launch_count(const Shape& sh) {
  if (sh.N == 0) return 0;
  if (!expert_ffn_uses_tensor_cores(sh)) return 2;
  return 3 + (expert_ffn_split(sh, true) > 1 ? 1 : 0);  // plan, GEMMs, fixup
}

void expert_ffn_tiles(const Shape& sh, int* tile_gu, int* tile_dn) {
  const bool pairs = use_pairs(sh);
  *tile_gu = pairs ? 256 : tile_gateup_for(sh.T);
  *tile_dn = pairs ? 256 : tile_down_for(sh.T);
}

bool expert_ffn_gathers(const Shape& sh) {
  return expert_ffn_uses_tensor_cores(sh) && !use_pairs(sh) && tile_gateup_for(sh.T) <= 128;
}

// Contraction splits of the single-CTA expert GEMMs for tiny batches. With
// one or a few tokens, a handful of experts gives about one 128-row unit per
// SM, so the last units run on few SMs. Each GEMM is split so that the most
// units the batch can have fill the SMs about four times. At most 4 splits,
// and a divisor of the k-blocks. It stays 1 for the CTA-pair path and for
// batches whose units already fill the SMs (decode at T = 64 among them).
int expert_ffn_split(const Shape& sh, bool gateup) {
  if (!expert_ffn_uses_tensor_cores(sh) || use_pairs(sh) || tile_gateup_for(sh.T) > 64)
    return 1;
  const int64_t experts = sh.N < sh.T * sh.k ? sh.N : sh.T * sh.k;
  const int64_t units = experts * ((gateup ? sh.F : sh.d) / BM);
  const int nkb = (int)((gateup ? sh.d : sh.F) / BK);
  const int64_t want = 4ll * num_sms();
  for (int s = 1; s <= 4; ++s)
    if (nkb % s == 0 && units * s >= want) return s;
  for (int s = 4; s > 1; --s)
    if (nkb % s == 0) return s;
  return 1;
}

int64_t expert_ffn_part_floats(const Shape& sh) {
  const int sg = expert_ffn_split(sh, true), sd = expert_ffn_split(sh, false);
  if (sg == 1 && sd == 1) return 0;
  const int64_t a = sg > 1 ? (int64_t)sg * 2 * sh.F : 0;
  const int64_t b = sd > 1 ? (int64_t)sd * sh.d : 0;
  return sh.T * sh.k * (a > b ? a : b);
}

cudaError_t launch_expert_ffn(const Shape& sh, const void* x_perm,
                              const int32_t* offsets, const void* w_gate,
                              const void* w_up, const void* w_down, void* h,
                              void* y_perm, int32_t* tile_start, int32_t* err,
                              cudaStream_t st, const void* x_src,
                              const int32_t* row_token, bool plan_ready, float* part,
                              bool leave_y_split) {
  if (sh.N == 0 || sh.T == 0) return cudaSuccess;
  if (!expert_ffn_uses_tensor_cores(sh)) {
    if (sh.bf16)
      return launch_simt<__nv_bfloat16>(sh, x_perm, offsets, w_gate, w_up, w_down, h,
                                        y_perm, st);
    return launch_simt<float>(sh, x_perm, offsets, w_gate, w_up, w_down, h, y_perm, st);
  }
  const uint64_t rows_cap = (uint64_t)(sh.T * sh.k);
  CUtensorMap wg_map, wu_map, wd_map, x16, x128, h16, h128;
  const bool ok =
      make_map(&wg_map, w_gate, (uint64_t)(sh.N * sh.F), (uint64_t)sh.d, BM) &&
      make_map(&wu_map, w_up, (uint64_t)(sh.N * sh.F), (uint64_t)sh.d, BM) &&
      make_map(&wd_map, w_down, (uint64_t)(sh.N * sh.d), (uint64_t)sh.F, BM) &&
      make_map(&x16, x_perm, rows_cap, (uint64_t)sh.d, 16) &&
      make_map(&x128, x_perm, rows_cap, (uint64_t)sh.d, 128) &&
      make_map(&h16, h, rows_cap, (uint64_t)sh.F, 16) &&
      make_map(&h128, h, rows_cap, (uint64_t)sh.F, 128);
  if (!ok) return cudaErrorInvalidValue;

  const bool pairs = use_pairs(sh);
  int tgu = 0, tdn = 0;
  expert_ffn_tiles(sh, &tgu, &tdn);
  cudaError_t e = cudaSuccess;
  if (!plan_ready) {
    e = launch_pdl(gemm_plan_kernel, dim3(1), dim3(1024), 0, st, offsets, (int)sh.N, tgu, tdn,
                   tile_start);
    if (e != cudaSuccess) return e;
  }

  GemmArgs gu;
  gu.offsets = offsets;
  gu.tile_start = tile_start;
  gu.out = h;
  gu.err = err;
  gu.N = (int)sh.N;
  gu.num_kb = (int)(sh.d / BK);
  gu.out_cols = (int)sh.F;
  gu.m_tiles = (int)(sh.F / BM);
  gu.a_rows = gu.out_cols;
  gu.mt_chunk = gu.m_tiles;
  gu.kb_chunk = gu.num_kb;
  if (x_src && row_token) {
    // token rows straight from x: x16 becomes x's one-row-box map
    if (!expert_ffn_gathers(sh) || !make_map(&x16, x_src, (uint64_t)sh.T, (uint64_t)sh.d, 1))
      return cudaErrorInvalidValue;
    gu.row_token = row_token;
    gu.oob_row = (int)sh.T;
  }
  if (pairs) {
    GemmArgs gp = gu;
    gp.m_tiles = (int)(sh.F / 256);  // pairs of 128-row tiles
    gp.unit_counter = tile_start + 2 * sh.N + 2;
    e = launch_pair<true>(wg_map, wu_map, x16, x128, gp, st);
    if (e != cudaSuccess) return e;
    GemmArgs dp = gu;
    dp.row_token = nullptr;  // the down GEMM reads h, already in row order
    dp.unit_counter = tile_start + 2 * sh.N + 3;
    dp.tile_start = tile_start + sh.N + 1;
    dp.out = y_perm;
    dp.out_bf16 = true;
    dp.num_kb = (int)(sh.F / BK);
    dp.out_cols = (int)sh.d;
    dp.a_rows = (int)sh.d;
    dp.m_tiles = (int)(sh.d / 256);
    dp.mt_chunk = dp.m_tiles;
    dp.kb_chunk = dp.num_kb;
    return launch_pair<false>(wd_map, wd_map, h16, h128, dp, st);
  }
  // tiny batches: split contractions, fp32 partials in `part`
  const int sg = expert_ffn_split(sh, true), sd = expert_ffn_split(sh, false);
  if ((sg > 1 || sd > 1) && part == nullptr) return cudaErrorInvalidValue;
  if (sg > 1) {
    gu.m_tiles = (int)(sh.F / BM) * sg;
    gu.kb_chunk = gu.num_kb / sg;
    gu.part = part;
    gu.part_stride = (int64_t)sg * 2 * sh.F;
  }
  e = tgu == 64    ? launch_tc<true, 64>(wg_map, wu_map, x16, x128, gu, st)
      : tgu == 128 ? launch_tc<true, 128>(wg_map, wu_map, x16, x128, gu, st)
                   : launch_tc<true, 256>(wg_map, wu_map, x16, x128, gu, st);
  if (e != cudaSuccess) return e;
  const unsigned fix_blocks = (unsigned)(2 * num_sms());
  if (sg > 1) {
    e = launch_pdl(swiglu_split_fixup_kernel, dim3(fix_blocks), dim3(256), 0, st,
                   static_cast<const float*>(part), sg, sh.F, offsets, (int)sh.N,
                   static_cast<__nv_bfloat16*>(h));
    if (e != cudaSuccess) return e;
  }

  GemmArgs dn = gu;
  dn.row_token = nullptr;  // the down GEMM reads h, already in row order
  dn.part = nullptr;
  dn.tile_start = tile_start + sh.N + 1;
  dn.out = sd > 1 ? static_cast<void*>(part) : y_perm;
  dn.out_bf16 = sd == 1;  // split partials stay fp32 until they are added
  dn.num_kb = (int)(sh.F / BK);
  dn.out_cols = (int)sh.d * sd;  // split c writes columns [c d, (c + 1) d)
  dn.m_tiles = (int)(sh.d / BM) * sd;
  dn.a_rows = (int)sh.d;
  dn.mt_chunk = (int)(sh.d / BM);
  dn.kb_chunk = dn.num_kb / sd;
  e = tdn == 64    ? launch_tc<false, 64>(wd_map, wd_map, h16, h128, dn, st)
      : tdn == 128 ? launch_tc<false, 128>(wd_map, wd_map, h16, h128, dn, st)
                   : launch_tc<false, 256>(wd_map, wd_map, h16, h128, dn, st);
  if (e != cudaSuccess || sd == 1 || leave_y_split) return e;
  return launch_pdl(split_reduce_kernel, dim3(fix_blocks), dim3(256), 0, st,
                    static_cast<const float*>(part), sd, sh.d, offsets, (int)sh.N,
                    static_cast<__nv_bfloat16*>(y_perm));
}

}  // namespace moe
