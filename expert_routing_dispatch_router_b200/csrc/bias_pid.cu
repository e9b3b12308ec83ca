// PID controller on the router bias of the zero experts.
//
// "Meituan lancerer LongCat-2.0" (snilld.dk), "MoE i praksis og prisen for
// fleksibilitet": a PID controller adjusts the router bias so that the number
// of activated parameters stays in the wanted range. Activation here is the
// share of routing slots that went to routed experts (each such slot runs
// one expert FFN; a zero-expert slot runs none). With counts from the last
// layer call,
//   share = sum_{e<N} counts[e] / (T k),  err = share - target,
//   u = kp err + ki (I + err) + kd (err - prev),  clamped to +-max_step,
// every zero expert's bias gets +u (a share above target raises the zero
// experts' keys), and the state {I, prev} becomes {I + err, err}. The pages
// give no gains or set-point; they are parameters.
//
// One block; the double arithmetic uses explicit round-to-nearest operations
// (no fused multiply-add), so the update is exactly reproducible.
#include "moe_internal.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256)
    bias_pid_kernel(const int32_t* __restrict__ counts, float* __restrict__ bias,
                    double* __restrict__ state, int N, int E, int64_t slots, double target,
                    double kp, double ki, double kd, double max_step) {
  __shared__ long long part[256];
  __shared__ double u_s;
  griddep_wait();
  griddep_launch_dependents();
  long long c = 0;
  for (int e = threadIdx.x; e < N; e += blockDim.x) c += counts[e];
  part[threadIdx.x] = c;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double share = __ddiv_rn((double)part[0], (double)slots);
    const double err = __dadd_rn(share, -target);
    const double integral = __dadd_rn(state[0], err);
    double u = __dadd_rn(__dadd_rn(__dmul_rn(kp, err), __dmul_rn(ki, integral)),
                         __dmul_rn(kd, __dadd_rn(err, -state[1])));
    if (u > max_step) u = max_step;
    if (u < -max_step) u = -max_step;
    state[0] = integral;
    state[1] = err;
    u_s = u;
  }
  __syncthreads();
  const double u = u_s;
  for (int e = N + threadIdx.x; e < E; e += blockDim.x)
    bias[e] = __double2float_rn(__dadd_rn((double)bias[e], u));
}

}  // namespace

cudaError_t launch_bias_pid(const Shape& sh, const int32_t* counts, float* bias,
                            double* state, double target, double kp, double ki,
                            double kd, double max_step, cudaStream_t st) {
  return launch_pdl(bias_pid_kernel, dim3(1), dim3(256), 0, st, counts, bias, state,
                    (int)sh.N, (int)sh.E, sh.T * sh.k, target, kp, ki, kd, max_step);
}

}  // namespace moe
