/*
 * CPU oracle: forward pass of a mixture-of-experts FFN layer with
 * zero-computation (identity) experts.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the plain, slow, obviously correct
 * definition that the CUDA library is checked against. Only the tests, the
 * smoke check and the bench's CPU-baseline leg may load it. It shares no code,
 * header, table or helper with the CUDA library, and it never reads anything
 * the CUDA library produced.
 *
 * Arithmetic: every floating-point step runs in fp64 (double). Inputs arrive
 * in their stored types (fp32, or bf16 as raw 16-bit patterns) and are widened
 * exactly. Loops are written in the order of the definition, one token at a
 * time; OpenMP only spreads independent tokens (or experts) over threads.
 *
 * Sources (page title, section):
 *  - LongCat-2.0 model card (archdb), "Mixture of experts": 768 routed experts
 *    plus 128 identity zero-experts, scored together by one router classifier
 *    [896, 8192] with an e_score_correction_bias; 12 experts per token; expert
 *    width 2048; a routed scaling factor applied to the combined routed-expert
 *    output. Router score and top-k renormalisation are "Not disclosed".
 *  - same card, "Feed-forward": activation "Not disclosed".
 *  - "Meituan lancerer LongCat-2.0" (snilld.dk), "MoE i praksis og prisen for
 *    fleksibilitet": zero-computation experts; a PID controller adjusts the
 *    router bias (taken here as an input).
 *  - Ascend LongCat-2.0 deployment article (10100.com), section
 *    "底层定制算子深度优化": Dispatch/Combine operators that support
 *    zero-computation experts.
 *
 * Readings taken where the pages are silent or ambiguous:
 *  R1 expert ids 0..N-1 are routed, N..E-1 are zero experts;
 *  R2 the correction bias is added to the logits for selection only;
 *  R3 the selected set is the k largest keys, ties to the lower id, emitted in
 *     descending key order;
 *  R4 gates are the softmax of the raw logits over the selected set (they sum
 *     to 1);
 *  R5 a routed expert is a SwiGLU FFN without biases:
 *     y = W_d (silu(W_g x) * (W_u x)), silu(z) = z / (1 + exp(-z));
 *  R6 a zero expert returns the token's input x;
 *  R7 the routed scaling factor s multiplies the routed part only:
 *     out = s * sum_{routed j} g_j y_j + sum_{zero j} g_j x;
 *  R8 dispatch orders routed slots by (expert ascending, token ascending).
 *
 * Parity pins: every function here is checked by the CPU tests against
 * library routines, closed forms, invariants and a brute force; none is
 * "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_F32 0
#define ORACLE_BF16 1

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Exact widening of one stored element to double. A bf16 value is the upper
 * half of an IEEE binary32 pattern. */
static double elem(const void* base, int dtype, int64_t i) {
  if (dtype == ORACLE_F32) return (double)((const float*)base)[i];
  uint32_t bits = ((uint32_t)((const uint16_t*)base)[i]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* ---------------------------------------------------------------- router -- */

/* logits[t,e] = sum_i x[t,i] * w_r[e,i]   (router classifier [E, d]) */
void oracle_router_logits(int64_t T, int64_t d, int64_t E, int x_dtype,
                          const void* x, const float* w_r, double* logits) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int64_t i = 0; i < d; ++i)
        acc += elem(x, x_dtype, t * d + i) * (double)w_r[e * d + i];
      logits[t * E + e] = acc;
    }
  }
}

/* Selection and gates for one token, readings R2-R4.
 * key_e = logit_e + bias_e; pick the k largest keys one after another (ties go
 * to the lower id); margin = (k-th key) - ((k+1)-th key), +inf when k == E;
 * gate_j = exp(l_j - m) / sum_j' exp(l_j' - m) over the selected raw logits,
 * m = the largest selected raw logit. */
static void select_token(int64_t E, int64_t k, const double* logit,
                         const float* bias, int32_t* idx, double* gate,
                         double* margin, unsigned char* taken) {
  memset(taken, 0, (size_t)E);
  double kth_key = 0.0;
  for (int64_t j = 0; j < k; ++j) {
    int64_t best = -1;
    double best_key = 0.0;
    for (int64_t e = 0; e < E; ++e) {
      if (taken[e]) continue;
      double key = logit[e] + (double)bias[e];
      if (best < 0 || key > best_key) {
        best = e;
        best_key = key;
      }
    }
    taken[best] = 1;
    idx[j] = (int32_t)best;
    kth_key = best_key;
  }
  if (margin) {
    if (k == E) {
      *margin = INFINITY;
    } else {
      double next = -INFINITY;
      for (int64_t e = 0; e < E; ++e) {
        if (taken[e]) continue;
        double key = logit[e] + (double)bias[e];
        if (key > next) next = key;
      }
      *margin = kth_key - next;
    }
  }
  double m = -INFINITY;
  for (int64_t j = 0; j < k; ++j)
    if (logit[idx[j]] > m) m = logit[idx[j]];
  double z = 0.0;
  for (int64_t j = 0; j < k; ++j) z += exp(logit[idx[j]] - m);
  for (int64_t j = 0; j < k; ++j) gate[j] = exp(logit[idx[j]] - m) / z;
}

/* Top-k selection from given logits (fp64). idx [T,k], gate [T,k],
 * margin [T] (may be NULL). */
void oracle_select(int64_t T, int64_t E, int64_t k, const double* logits,
                   const float* bias, int32_t* idx, double* gate,
                   double* margin) {
#pragma omp parallel
  {
    unsigned char* taken = (unsigned char*)malloc((size_t)E);
#pragma omp for schedule(static)
    for (int64_t t = 0; t < T; ++t)
      select_token(E, k, logits + t * E, bias, idx + t * k, gate + t * k,
                   margin ? margin + t : NULL, taken);
    free(taken);
  }
}

/* Gates of a GIVEN selection (used to build the valid alternative answers for
 * near-tied tokens): softmax of the raw logits over idx[t, :]. */
void oracle_gates_of(int64_t T, int64_t E, int64_t k, const double* logits,
                     const int32_t* idx, double* gate) {
  for (int64_t t = 0; t < T; ++t) {
    const double* l = logits + t * E;
    const int32_t* s = idx + t * k;
    double m = -INFINITY;
    for (int64_t j = 0; j < k; ++j)
      if (l[s[j]] > m) m = l[s[j]];
    double z = 0.0;
    for (int64_t j = 0; j < k; ++j) z += exp(l[s[j]] - m);
    for (int64_t j = 0; j < k; ++j) gate[t * k + j] = exp(l[s[j]] - m) / z;
  }
}

/* Whole router: logits, selection, gates, margin. */
void oracle_route(int64_t T, int64_t d, int64_t E, int64_t k, int x_dtype,
                  const void* x, const float* w_r, const float* bias,
                  double* logits, int32_t* idx, double* gate, double* margin) {
  oracle_router_logits(T, d, E, x_dtype, x, w_r, logits);
  oracle_select(T, E, k, logits, bias, idx, gate, margin);
}

/* -------------------------------------------------------------- dispatch -- */

/* Counting sort of the routing slots, reading R8.
 * counts[e]    = number of slots (t, j) with idx[t,j] == e, for all E experts;
 * offsets[e]   = sum of counts over routed experts e' < e, e = 0..N
 *                (offsets[N] = R, the number of routed slots);
 * row_token[r] = token of the r-th routed row, rows ordered by (expert, token);
 * slot_row[t*k+j] = row of slot (t, j), or -1 when it goes to a zero expert.
 * row_token must hold T*k entries; entries r >= R are set to -1. */
void oracle_dispatch(int64_t T, int64_t k, int64_t N, int64_t E,
                     const int32_t* idx, int32_t* counts, int32_t* offsets,
                     int32_t* row_token, int32_t* slot_row) {
  for (int64_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t s = 0; s < T * k; ++s) counts[idx[s]] += 1;
  offsets[0] = 0;
  for (int64_t e = 0; e < N; ++e) offsets[e + 1] = offsets[e] + counts[e];
  for (int64_t s = 0; s < T * k; ++s) {
    slot_row[s] = -1;
    row_token[s] = -1;
  }
  int64_t r = 0;
  for (int64_t e = 0; e < N; ++e)
    for (int64_t t = 0; t < T; ++t)
      for (int64_t j = 0; j < k; ++j)
        if (idx[t * k + j] == e) {
          row_token[r] = (int32_t)t;
          slot_row[t * k + j] = (int32_t)r;
          ++r;
        }
}

/* ------------------------------------------------------------ expert FFN -- */

/* One routed expert on one input row, reading R5.
 * a = W_g[e] x, u = W_u[e] x (W_g, W_u are [N, F, d]); h = silu(a) * u;
 * y = W_d[e] h (W_d is [N, d, F]). h_out may be NULL. */
static void expert_row(int64_t d, int64_t F, int w_dtype, const void* w_gate,
                       const void* w_up, const void* w_down, int64_t e,
                       const double* x, double* y, double* h) {
  for (int64_t f = 0; f < F; ++f) {
    double a = 0.0, u = 0.0;
    int64_t base = (e * F + f) * d;
    for (int64_t i = 0; i < d; ++i) {
      a += elem(w_gate, w_dtype, base + i) * x[i];
      u += elem(w_up, w_dtype, base + i) * x[i];
    }
    h[f] = a / (1.0 + exp(-a)) * u;
  }
  for (int64_t n = 0; n < d; ++n) {
    double acc = 0.0;
    int64_t base = (e * d + n) * F;
    for (int64_t f = 0; f < F; ++f) acc += elem(w_down, w_dtype, base + f) * h[f];
    y[n] = acc;
  }
}

/* Expert FFN over dispatched rows: for each listed row r (expert row_expert[r])
 * y_rows[r,:] = FFN_e(x_rows[r,:]); h_rows[r,:] (may be NULL) gets h. */
void oracle_expert_rows(int64_t d, int64_t F, int w_dtype, const void* w_gate,
                        const void* w_up, const void* w_down, int64_t n_rows,
                        const int32_t* row_expert, const double* x_rows,
                        double* y_rows, double* h_rows) {
#pragma omp parallel
  {
    double* h = (double*)malloc((size_t)F * sizeof(double));
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
      expert_row(d, F, w_dtype, w_gate, w_up, w_down, row_expert[r],
                 x_rows + r * d, y_rows + r * d, h);
      if (h_rows) memcpy(h_rows + r * F, h, (size_t)F * sizeof(double));
    }
    free(h);
  }
}

/* --------------------------------------------------------------- combine -- */

/* Reading R7 over dispatched rows, for each token t:
 * out[t,:] = s * sum_{j: idx<N} gate[t,j] * y_perm[slot_row[t,j], :]
 *              + sum_{j: idx>=N} gate[t,j] * x[t,:]                         */
void oracle_combine(int64_t T, int64_t d, int64_t N, int64_t k, double s,
                    const double* x, const double* y_perm, const int32_t* idx,
                    const double* gate, const int32_t* slot_row, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t i = 0; i < d; ++i) {
      double routed = 0.0, ident = 0.0;
      for (int64_t j = 0; j < k; ++j) {
        int64_t sl = t * k + j;
        if (idx[sl] < N)
          routed += gate[sl] * y_perm[(int64_t)slot_row[sl] * d + i];
        else
          ident += gate[sl] * x[t * d + i];
      }
      out[t * d + i] = s * routed + ident;
    }
  }
}

/* ---------------------------------------------------------- whole layer -- */

/* The layer's definition applied token by token, with no dispatch at all:
 * route the token, then evaluate its selected experts directly.
 * tokens[n_tok]: which tokens to evaluate (out row n is token tokens[n]).
 * force_idx [T,k] or NULL: when given, use this selection instead of the top-k
 * (gates are still the softmax of this token's own raw logits over it).
 * idx_out, gate_out [n_tok, k] may be NULL. */
void oracle_layer(int64_t n_tok, const int32_t* tokens, int64_t T, int64_t d,
                  int64_t N, int64_t Z, int64_t k, int64_t F, double s,
                  int act_dtype, const void* x, const float* w_r,
                  const float* bias, const void* w_gate, const void* w_up,
                  const void* w_down, const int32_t* force_idx, double* out,
                  int32_t* idx_out, double* gate_out) {
  const int64_t E = N + Z;
  (void)T;
#pragma omp parallel
  {
    double* xt = (double*)malloc((size_t)d * sizeof(double));
    double* logit = (double*)malloc((size_t)E * sizeof(double));
    double* y = (double*)malloc((size_t)d * sizeof(double));
    double* h = (double*)malloc((size_t)F * sizeof(double));
    int32_t* sel = (int32_t*)malloc((size_t)k * sizeof(int32_t));
    double* g = (double*)malloc((size_t)k * sizeof(double));
    unsigned char* taken = (unsigned char*)malloc((size_t)E);
#pragma omp for schedule(dynamic, 1)
    for (int64_t n = 0; n < n_tok; ++n) {
      int64_t t = tokens[n];
      for (int64_t i = 0; i < d; ++i) xt[i] = elem(x, act_dtype, t * d + i);
      for (int64_t e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int64_t i = 0; i < d; ++i) acc += xt[i] * (double)w_r[e * d + i];
        logit[e] = acc;
      }
      if (force_idx) {
        for (int64_t j = 0; j < k; ++j) sel[j] = force_idx[t * k + j];
        oracle_gates_of(1, E, k, logit, sel, g);
      } else {
        select_token(E, k, logit, bias, sel, g, NULL, taken);
      }
      double* o = out + n * d;
      for (int64_t i = 0; i < d; ++i) o[i] = 0.0;
      /* routed part, scaled by s */
      for (int64_t j = 0; j < k; ++j) {
        if (sel[j] >= N) continue;
        expert_row(d, F, act_dtype, w_gate, w_up, w_down, sel[j], xt, y, h);
        for (int64_t i = 0; i < d; ++i) o[i] += s * g[j] * y[i];
      }
      /* identity part of zero experts, unscaled */
      for (int64_t j = 0; j < k; ++j) {
        if (sel[j] < N) continue;
        for (int64_t i = 0; i < d; ++i) o[i] += g[j] * xt[i];
      }
      if (idx_out)
        for (int64_t j = 0; j < k; ++j) idx_out[n * k + j] = sel[j];
      if (gate_out)
        for (int64_t j = 0; j < k; ++j) gate_out[n * k + j] = g[j];
    }
    free(xt);
    free(logit);
    free(y);
    free(h);
    free(sel);
    free(g);
    free(taken);
  }
}

/* ------------------------------------------------- router bias controller -- */

/* PID update of the zero experts' router bias (reading R13). "Meituan
 * lancerer LongCat-2.0" (snilld.dk), "MoE i praksis og prisen for
 * fleksibilitet", says a PID controller adjusts the router bias so that the
 * activation stays in the wanted range, and gives no gains, set-point or
 * controlled variable. Here the controlled value is the
 * share of routing slots that went to routed experts,
 *   share = sum_{e<N} counts[e] / (T k),
 * the error is err = share - target, and
 *   u = kp err + ki (I + err) + kd (err - prev)       (I: running sum of err)
 * clamped to [-max_step, max_step], is added to every zero expert's bias: a
 * share above target raises the zero experts' keys, so more slots go to them.
 * state = {I, prev}; both are updated (I += err, prev = err). Routed experts'
 * biases are left alone. The new bias is rounded to fp32 once. */
void oracle_pid_update(int64_t T, int64_t k, int64_t N, int64_t E,
                       const int32_t* counts, float* bias, double* state,
                       double target, double kp, double ki, double kd,
                       double max_step) {
  int64_t routed = 0;
  for (int64_t e = 0; e < N; ++e) routed += counts[e];
  const double share = (double)routed / (double)(T * k);
  const double err = share - target;
  const double integral = state[0] + err;
  double u = kp * err + ki * integral + kd * (err - state[1]);
  if (u > max_step) u = max_step;
  if (u < -max_step) u = -max_step;
  for (int64_t e = N; e < E; ++e) bias[e] = (float)((double)bias[e] + u);
  state[0] = integral;
  state[1] = err;
}
