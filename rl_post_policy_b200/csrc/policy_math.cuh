// Per-token PPO-clipped policy term with the k3 KL penalty, and its derivative
// with respect to the policy log-prob ("Geometric-AI Kernels" model card,
// sections "BNPO Loss" and "GRPO Loss"):
//   ratio = exp(lp - old), clipped = clip(ratio, lo, hi)
//   literal form   : term = -A * min(ratio, clipped); d/dlp = -A*ratio if ratio <= hi else 0
//   two-sided form : term = -min(A*ratio, A*clipped); d/dlp = -A*ratio if A*ratio <= A*clipped else 0
//   kl = exp(e) - e - 1 with e = ref - lp (evaluated as expm1(e) - e); d kl/dlp = -expm1(e)
// Ties at ratio == hi let the gradient through.
#pragma once

namespace pl {

// FAST selects the hardware exponential (__expf) for both exponentials: a few
// instructions instead of a few dozen, with a relative error of a few fp32 ulps,
// far inside every tolerance of the path; the memory-bound loss kernel needs it
// to stay under its per-token instruction budget at full HBM bandwidth.
template <bool HAS_KL, bool TWO_SIDED, bool FAST = false>
__device__ __forceinline__ void token_math(float lp, float old, float ref, float A, float lo, float hi,
                                           float beta, float& term, float& dterm) {
  const float ratio = FAST ? __expf(lp - old) : expf(lp - old);
  const float clipped = fminf(fmaxf(ratio, lo), hi);
  if (!TWO_SIDED) {
    term = -A * fminf(ratio, clipped);
    dterm = ratio <= hi ? -A * ratio : 0.0f;
  } else {
    const float ur = A * ratio, uc = A * clipped;
    term = -fminf(ur, uc);
    dterm = ur <= uc ? -A * ratio : 0.0f;
  }
  if (HAS_KL) {
    const float e = ref - lp;
    const float em1 = FAST ? __expf(e) - 1.0f : expm1f(e);
    term += beta * (em1 - e);
    dterm -= beta * em1;
  }
}

}  // namespace pl
