/*
 * moe_api.h - C ABI of the B200 (sm_100a) library for the forward pass of a
 * mixture-of-experts FFN layer with zero-computation (identity) experts.
 *
 * The layer (LongCat-2.0 model card (archdb), section "Mixture of experts";
 * "Meituan lancerer LongCat-2.0" (snilld.dk), section "MoE i praksis og
 * prisen for fleksibilitet"; Ascend LongCat-2.0 deployment article
 * (10100.com), section "底层定制算子深度优化"):
 *
 *   logits[t,e] = x[t,:] . w_router[e,:]              e < E = N + Z
 *   S_t         = the top_k experts by key logits[t,e] + bias[e]
 *                 (ties to the lower id; emitted in descending key order)
 *   gate[t,j]   = softmax over j of logits[t, S_t[j]]  (bias not included)
 *   y_e(x)      = W_down[e] (silu(W_gate[e] x) * (W_up[e] x))     e < N
 *   out[t,:]    = s * sum_{j: S_t[j] <  N} gate[t,j] * y_{S_t[j]}(x[t,:])
 *                   + sum_{j: S_t[j] >= N} gate[t,j] * x[t,:]
 *
 * Expert ids 0..N-1 are routed experts, N..E-1 are zero experts. The bias is
 * the per-expert correction bias that the pages' PID controller adjusts; here
 * it is an input.
 *
 * Conventions shared by every call
 *  - Ownership: the caller owns every buffer. The library allocates, frees and
 *    synchronises nothing (moe_read_device_error is the one call that waits,
 *    and only on the stream it is given).
 *  - Pointers are device pointers unless the name ends in _host. All tensors
 *    are dense row-major. Every pointer must be 16-byte aligned. The device
 *    pointers of a call must all be memory of the current CUDA device, the
 *    one `stream` belongs to: kernels run there and read them directly.
 *  - act_dtype is the type of x, out, the expert weights, x_perm, h and the
 *    expert outputs y_perm: MOE_F32 (float) or MOE_BF16 (bfloat16).
 *    w_router, bias and topk_gate are always float; indices are int32.
 *  - Every call is asynchronous on `stream` (0 = legacy default stream) and
 *    issues no host synchronisation.
 *  - Buffers that depend on the routing are sized for the worst case T*top_k
 *    rows, because the number R of routed rows is only known on the device.
 *  - Errors: argument errors are found on the host before anything is
 *    launched and leave every buffer untouched. A launch failure returns
 *    MOE_ERR_CUDA. Device-side checks (a bounded wait in the router or an
 *    expert GEMM that ran out; an invalid expert id given to the dispatch)
 *    are recorded in the workspace and reported by moe_read_device_error.
 *  - Limits: 1 <= top_k <= min(E, 32), E <= 1024, d and ffn multiples of 8,
 *    T*top_k < 2^31, and T <= 4194240 where the router runs on CUDA cores
 *    (f32 activations above 256 tokens, or d not a multiple of 128). Outside them a call returns MOE_ERR_UNSUPPORTED (or
 *    MOE_ERR_INVALID_ARG for nonsensical values). T == 0 is a no-op: once
 *    the config passes its checks the call returns MOE_OK without looking
 *    at any pointer (empty buffers may be null) and launches nothing.
 *  - Workspace: every call that takes `ws` needs ws_bytes >=
 *    moe_workspace_size(cfg) and a 256-byte aligned `ws`; the same workspace
 *    serves all calls of one config. Its first 256 bytes hold the device
 *    error word and small counters that the kernels return to zero; they
 *    must be zero before first use (cudaMemset once). moe_read_device_error
 *    clears the error word again. Calls that share a workspace must
 *    be ordered on one stream.
 */
#ifndef MOE_API_H
#define MOE_API_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* same handle as cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or config */
  MOE_ERR_UNSUPPORTED = 2,  /* valid but outside the limits listed above */
  MOE_ERR_WORKSPACE = 3,    /* ws is NULL or ws_bytes too small */
  MOE_ERR_CUDA = 4,         /* a CUDA launch or copy failed */
  MOE_ERR_DEVICE_CHECK = 5  /* a device-side check failed (see below) */
} moe_status_t;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype_t;

typedef struct {
  int32_t T;            /* tokens */
  int32_t d;            /* hidden size */
  int32_t n_routed;     /* N: routed (SwiGLU) experts, ids 0..N-1 */
  int32_t n_zero;       /* Z: zero-computation (identity) experts, ids N..E-1 */
  int32_t top_k;        /* k: experts per token */
  int32_t ffn;          /* F: routed expert FFN width */
  moe_dtype_t act_dtype;
  float routed_scale;   /* s: multiplies the routed part only (card: 9) */
} moe_config_t;

/* Bytes of workspace every call of this config needs (0 if cfg is invalid). */
size_t moe_workspace_size(const moe_config_t* cfg);

/* Router + top-k selection + gates.
 * Model card (archdb), "Mixture of experts": router classifier [E, d] with
 * e_score_correction_bias; "Experts per token".
 *  x         [T, d] act_dtype
 *  w_router  [E, d] float;  bias [E] float
 *  logits    [T, E] float, or NULL (then kept in ws). fp32 accumulation.
 *  topk_idx  [T, k] int32  expert ids in descending key order
 *  topk_gate [T, k] float  softmax of the selected raw logits (sums to 1)
 *  flags     [T] uint8 or NULL: 1 when key_(k) - key_(k+1) < 1e-4 (a near
 *            tie whose selection depends on rounding), else 0. */
moe_status_t moe_route(const moe_config_t* cfg, const void* x,
                       const float* w_router, const float* bias, float* logits,
                       int32_t* topk_idx, float* topk_gate, uint8_t* flags,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

/* Dispatch: group routed slots by expert; zero-expert slots are counted but
 * not copied. Ascend deployment article, "底层定制算子深度优化" (Dispatch
 * operator supporting zero-computation experts); deterministic order as the
 * Portuguese op-ed ("A Primeira Parede") describes.
 *  topk_idx  [T, k] int32 (a slot id outside [0, E), or an id repeated
 *            inside one token, is skipped and recorded as device error 2)
 *  counts    [E] int32    slots per expert, zero experts included
 *  offsets   [N+1] int32  start row of each routed expert; offsets[N] = R
 *  row_token [T*k] int32  token of row r (rows ordered by expert, then
 *                         token); -1 for r >= R
 *  slot_row  [T*k] int32  row of slot (t, j), -1 for a zero-expert slot
 *  x_perm    [T*k, d] act_dtype: x_perm[r] = x[row_token[r]] for r < R;
 *            rows >= R are left as they were. */
moe_status_t moe_dispatch(const moe_config_t* cfg, const void* x,
                          const int32_t* topk_idx, int32_t* counts,
                          int32_t* offsets, int32_t* row_token,
                          int32_t* slot_row, void* x_perm, void* ws,
                          size_t ws_bytes, moe_stream_t stream);

/* Routed experts over the dispatched rows (grouped SwiGLU GEMM).
 * Model card, "Mixture of experts": expert dim; activation taken as SwiGLU.
 *  x_perm  [T*k, d] act_dtype;  offsets [N+1] int32 (as from moe_dispatch)
 *  w_gate, w_up [N, F, d] act_dtype;  w_down [N, d, F] act_dtype
 *  y_perm  [T*k, d] act_dtype: y_perm[r] = y_e(x_perm[r]) for r < R, e the
 *          expert owning row r; rows >= R are left as they were.
 *  bf16 with d and F multiples of 128 runs on tcgen05 tensor cores (fp32
 *  accumulation in TMEM, h and y rounded to bf16); other shapes and f32 run on a
 *  CUDA-core path with fp32 accumulation. */
moe_status_t moe_expert_ffn(const moe_config_t* cfg, const void* x_perm,
                            const int32_t* offsets, const void* w_gate,
                            const void* w_up, const void* w_down, void* y_perm,
                            void* ws, size_t ws_bytes, moe_stream_t stream);

/* Combine: out[t] = s * sum_routed gate * y_perm[slot_row] + sum_zero gate * x[t],
 * summed in fp32 in slot order j = 0..k-1 and rounded once (deterministic).
 * Ascend deployment article, "底层定制算子深度优化" (Combine operator);
 * model card, "Routed scaling factor".
 *  x [T, d], out [T, d], y_perm [T*k, d] act_dtype; topk_idx,
 *  topk_gate, slot_row as above. */
moe_status_t moe_combine(const moe_config_t* cfg, const void* x,
                         const void* y_perm, const int32_t* topk_idx,
                         const float* topk_gate, const int32_t* slot_row,
                         void* out, moe_stream_t stream);

/* The whole layer: route -> dispatch -> expert FFN -> combine, with every
 * intermediate kept in ws. counts [E] int32 may be NULL (per-expert slot
 * counts, the per-expert observability the snilld.dk piece asks for in
 * "Hvad det betyder i drift"). Results equal the four separate calls bit for
 * bit. Where the gate/up GEMM runs on single CTAs (bf16, d and F multiples of
 * 128, T <= 1024) it reads the token rows from x by row_token itself, so
 * x_perm is not written; where the dispatch fits one block (T <= 4096) it also
 * writes the expert GEMMs' tile plans. */
moe_status_t moe_layer_forward(const moe_config_t* cfg, const void* x,
                               const float* w_router, const float* bias,
                               const void* w_gate, const void* w_up,
                               const void* w_down, void* out, int32_t* counts,
                               void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_layer_forward with x and out in HOST memory (pinned memory lets the
 * copies run asynchronously): copies x_host to the device, runs the layer and
 * copies the result to out_host, all on `stream`. counts_host [E] may be
 * NULL. The caller synchronises the stream before reading out_host. */
moe_status_t moe_layer_forward_host(const moe_config_t* cfg, const void* x_host,
                                    const float* w_router, const float* bias,
                                    const void* w_gate, const void* w_up,
                                    const void* w_down, void* out_host,
                                    int32_t* counts_host, void* ws,
                                    size_t ws_bytes, moe_stream_t stream);

/* moe_route without a workspace, for callers that cannot allocate device
 * memory: code running inside an allocator or memory pool that owns the whole
 * device, plugins whose host forbids allocation after start-up, and paths
 * that must never wait on an allocator. The pages have no counterpart of this
 * call; it exists for those callers only.
 *  Same arguments, layouts and results as moe_route, minus ws/ws_bytes (it
 *  always runs the CUDA-core router). It allocates nothing: its scratch is
 *  one 16 MiB array inside the library, held by every GPU that loads the
 *  library until the process exits.
 *  Limits: T * (n_routed + n_zero) <= 4194304, and T <= 65535 * 64 (the
 *  CUDA-core router's grid); larger problems return MOE_ERR_UNSUPPORTED
 *  before anything is launched.
 *  The first call on a device (with that device current) looks up the
 *  array's address once. The address is kept for the life of the process: after cudaDeviceReset
 *  on a device, do not call this entry point on it again.
 *  All calls on a device share the array: calls that overlap on the GPU
 *  (other streams or host threads) race and must be ordered by the caller. */
moe_status_t moe_route_noalloc(const moe_config_t* cfg, const void* x,
                               const float* w_router, const float* bias,
                               float* logits, int32_t* topk_idx,
                               float* topk_gate, uint8_t* flags,
                               moe_stream_t stream);

/* Expert parallelism across `world` ranks, one GPU each. Ascend deployment
 * article (10100.com), "Decode节点：EP128超大专家并行" and "多场景模型分层切分优化"
 * (experts sharded over the cards of a decode instance, DP + EP) and
 * "底层定制算子深度优化" (Dispatch/Combine operators that support zero experts).
 * Rank r owns the routed experts [lo_r, lo_r + n_r): an even split of the N
 * routed ids, the first N % world ranks taking one more (moe_ep_local_experts
 * gives n_r; lo_r = sum of n_r' over r' < r). Zero experts belong to no rank:
 * their slots never leave the token's rank. One step on rank s:
 *  1. moe_route and moe_dispatch on s's own T tokens (counts [E], offsets
 *     [N+1], row_token; x_perm is not needed);
 *  2. gather every rank's counts and offsets on every rank (the caller's
 *     collective): counts_all [world, E] and offsets_all [world, N+1] int32;
 *  3. moe_ep_plan, then moe_ep_dispatch: s's routed rows go straight into
 *     their owners' receive buffers, expert-major (expert, source rank,
 *     source order);
 *  4. after a barrier, each owner runs moe_expert_ffn on its buffer with the
 *     recv_offsets of step 3 and its slice of the expert weights (a config
 *     with n_routed = n_r and T * top_k >= the buffer's rows);
 *  5. moe_ep_return: each owner sends its output rows back into the sources'
 *     y_perm, at the rows their dispatches gave them;
 *  6. after a barrier, moe_combine on each source, as on one GPU.
 * recv_x and y_home are device arrays of `world` device pointers (the ranks'
 * receive buffers [rows, d] and y_perm [T*k, d], act_dtype); on one node
 * these are peer addresses, written with plain stores. A receive buffer
 * needs room for every row its experts get, at most world * T * top_k.
 * The calls only order their own work on `stream`: the barriers between the
 * steps are the caller's. They return MOE_ERR_INVALID_ARG for a bad rank,
 * world or pointer, and need N >= 1. */
int32_t moe_ep_local_experts(const moe_config_t* cfg, int32_t rank, int32_t world);

/*  dest_row [N] int32: the first row of rank `rank`'s block of expert e in
 *  e's owner's receive buffer; recv_offsets [n_rank + 1] int32: rank's own
 *  receive layout over its experts (the offsets its expert FFN takes). */
moe_status_t moe_ep_plan(const moe_config_t* cfg, int32_t rank, int32_t world,
                         const int32_t* counts_all, int32_t* dest_row,
                         int32_t* recv_offsets, moe_stream_t stream);

/*  Copies x[row_token[j]] for every routed row j < offsets[N] of this rank
 *  to recv_x[owner(e)] row dest_row[e] + (j - offsets[e]), e the expert of
 *  row j. */
moe_status_t moe_ep_dispatch(const moe_config_t* cfg, int32_t world,
                             const void* x, const int32_t* offsets,
                             const int32_t* row_token, const int32_t* dest_row,
                             void* const* recv_x, moe_stream_t stream);

/*  Copies each row i < recv_offsets[n_rank] of y_recv (this rank's expert
 *  outputs, in its receive order) to y_home[s] row offsets_all[s][e] + its
 *  order among source s's rows of expert e. */
moe_status_t moe_ep_return(const moe_config_t* cfg, int32_t rank, int32_t world,
                           const void* y_recv, const int32_t* recv_offsets,
                           const int32_t* counts_all, const int32_t* offsets_all,
                           void* const* y_home, moe_stream_t stream);

/* PID controller on the zero experts' router bias, run between layer calls.
 * "Meituan lancerer LongCat-2.0" (snilld.dk), "MoE i praksis og prisen for
 * fleksibilitet": a PID controller adjusts the router bias so that the
 * activated parameters stay in the wanted range. From the per-expert counts of
 * the last call (moe_layer_forward or moe_dispatch):
 *   share = sum_{e<N} counts[e] / (T*k)   (slots that ran a routed expert)
 *   err   = share - target_routed_share
 *   u     = kp*err + ki*(I + err) + kd*(err - prev), clamped to +-max_step
 *   bias[e] += u for every zero expert e >= N (routed experts untouched)
 *   state = {I + err, err}
 * A share above the target raises the zero experts' keys, so the next call
 * sends more slots to them. The pages give no gains or set-point.
 *  counts [E] int32 (device), bias [E] float (device, updated in place),
 *  state [2] double (device; start from zeros), params on the host.
 *  cfg->T and top_k must be those of the call that produced counts.
 *  Returns MOE_ERR_INVALID_ARG for a NULL pointer, a misaligned pointer, a
 *  target outside [0, 1], or a negative or non-finite gain or max_step. */
typedef struct {
  float target_routed_share;
  float kp, ki, kd;
  float max_step;
} moe_pid_params_t;

moe_status_t moe_bias_pid_update(const moe_config_t* cfg, const int32_t* counts,
                                 float* bias, double* state,
                                 const moe_pid_params_t* params, moe_stream_t stream);

/* Waits for `stream`, then reads and clears the device-side error word in ws.
 * *code_out (may be NULL) gets 0 when no check failed, else a nonzero code:
 *   1 = a bounded wait in the router or an expert GEMM ran out (2 s);
 *   2 = a routing slot held an expert id outside [0, E), or one token listed
 *       an expert twice; such slots are skipped.
 * Returns MOE_ERR_DEVICE_CHECK when the code is nonzero, MOE_ERR_WORKSPACE
 * for a NULL ws. */
moe_status_t moe_read_device_error(void* ws, int32_t* code_out,
                                   moe_stream_t stream);

/* Self-test of the device-side failure detection, for tests and health
 * checks; it has no counterpart in the method. Launches one small kernel whose
 * mbarrier wait can never complete. After the 2 s limit that every wait in
 * the library has, the kernel records code 1 in the workspace error word and
 * returns, so the context stays usable; moe_read_device_error then reports
 * (and clears) it. Only the first 256 bytes of `ws` are used, and ws must be
 * 256-byte aligned (else MOE_ERR_WORKSPACE). */
moe_status_t moe_selftest_wait_limit(void* ws, size_t ws_bytes, moe_stream_t stream);

/* Number of kernel launches one moe_layer_forward call makes for cfg. */
int32_t moe_layer_launch_count(const moe_config_t* cfg);

const char* moe_status_string(moe_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_API_H */
