// Upstream gradient of a policy-gradient token loss from the fresh logprobs
// ("align architecture v2: proposal", section 5.4 A, "Why the in-chunk form
// works for this loss"): the logit gradient of the objective is a per-token
// coefficient times (softmax - onehot), and that coefficient is a function of
// the new logprob, the behaviour logprob and the advantage alone. This kernel
// forms g_t = dL/dlogprob_t (L = -J) for sts_backward:
//
//   CISPO            g_t = -scale * A_t * min(r_t, 1 + eps_high)
//   clipped          g_t = -scale * A_t * r_t, or 0 where the clip binds
//                    (r_t > 1 + eps_high with A_t >= 0, r_t < 1 - eps_low with
//                    A_t < 0)
//
// with r_t = exp(logprob_t - old_logprob_t) evaluated in float64. A row whose
// logprob is not finite (-inf: the replayed token is outside the support;
// NaN: an invalid row), or whose old logprob or advantage is not finite,
// gets 0, and so does a row with scale * A_t == 0. r_t may overflow to +inf
// (logprob_t - old_logprob_t > ~709.8): CISPO's weight is then 1 + eps_high,
// the clipped surrogate is clipped for A_t >= 0 and gives an infinite
// gradient for A_t < 0 (the objective is unbounded there).
#include <cmath>

#include "sts_internal.h"

namespace sts {
namespace {

__global__ void policy_grad_kernel(int64_t T, const float* __restrict__ logprob,
                                   const float* __restrict__ old_logprob,
                                   const float* __restrict__ advantage, int objective,
                                   double eps_low, double eps_high, double scale,
                                   float* __restrict__ grad) {
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < T;
       t += (int64_t)gridDim.x * blockDim.x) {
    const float lp = logprob[t], old = old_logprob[t], adv = advantage[t];
    double g = 0.0;
    if (isfinite(lp) && isfinite(old) && isfinite(adv) && scale * (double)adv != 0.0) {
      const double a = (double)adv;
      const double r = exp((double)lp - (double)old);
      if (objective == STS_PG_CISPO) {
        g = -scale * a * fmin(r, 1.0 + eps_high);
      } else {
        const bool clipped = a >= 0.0 ? r > 1.0 + eps_high : r < 1.0 - eps_low;
        g = clipped ? 0.0 : -scale * a * r;
      }
    }
    grad[t] = (float)g;
  }
}

}  // namespace
}  // namespace sts

using namespace sts;

extern "C" sts_status sts_policy_grad(int64_t T, const float* logprob, const float* old_logprob,
                                      const float* advantage, int objective, float eps_low,
                                      float eps_high, float scale, float* grad_logprob,
                                      sts_stream_t stream) {
  if (T < 0) return STS_ERR_SHAPE;
  if (objective != STS_PG_CISPO && objective != STS_PG_CLIPPED) return STS_ERR_SHAPE;
  if (!(eps_low >= 0.f) || !(eps_high >= 0.f) || !std::isfinite(eps_low) ||
      !std::isfinite(eps_high) || !std::isfinite(scale))
    return STS_ERR_SHAPE;
  if (T == 0) return STS_OK;
  if (!logprob || !old_logprob || !advantage || !grad_logprob) return STS_ERR_NULL;
  const int threads = 256;
  const int64_t want = (T + threads - 1) / threads;
  const int blocks = (int)(want < 4096 ? want : 4096);
  policy_grad_kernel<<<blocks, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      T, logprob, old_logprob, advantage, objective, (double)eps_low, (double)eps_high,
      (double)scale, grad_logprob);
  return cudaGetLastError() == cudaSuccess ? STS_OK : STS_ERR_CUDA;
}
