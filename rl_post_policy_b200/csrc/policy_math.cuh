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

// ---------------------------------------------------------------------------
// Two tokens at a time with the packed fp32 instructions of sm_100 (one
// instruction computes both lanes of a float2), for the bandwidth-bound loss
// kernel.  Same arithmetic as token_math<..., FAST=true>, with one exact
// simplification of the literal form: min(r, clip(r, lo, hi)) == min(r, hi)
// for lo <= hi (if r >= lo the clip is min(r, hi); if r < lo it is lo and
// min(r, lo) = r = min(r, hi)), in floating point as well.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <bool HAS_KL, bool TWO_SIDED>
__device__ __forceinline__ void token_math2(float2 lp, float2 old, float2 ref, float A, float lo, float hi,
                                            float beta, float2& term, float2& dterm) {
  constexpr float kLog2e = 1.4426950408889634f;
  const float2 m1 = make_float2(-1.0f, -1.0f);
  const float2 nA = make_float2(-A, -A);
  const float2 d = __ffma2_rn(old, m1, lp);                          // lp - old
  const float2 t = __fmul2_rn(d, make_float2(kLog2e, kLog2e));
  const float2 r = make_float2(ex2_approx(t.x), ex2_approx(t.y));    // ratio
  const float2 nAr = __fmul2_rn(r, nA);                              // -A * ratio
  if (!TWO_SIDED) {
    term = __fmul2_rn(make_float2(fminf(r.x, hi), fminf(r.y, hi)), nA);
    dterm = make_float2(r.x <= hi ? nAr.x : 0.0f, r.y <= hi ? nAr.y : 0.0f);
  } else {
    const float2 c = make_float2(fminf(fmaxf(r.x, lo), hi), fminf(fmaxf(r.y, lo), hi));
    const float2 Aa = make_float2(A, A);
    const float2 ur = __fmul2_rn(r, Aa), uc = __fmul2_rn(c, Aa);
    term = make_float2(-fminf(ur.x, uc.x), -fminf(ur.y, uc.y));
    dterm = make_float2(ur.x <= uc.x ? nAr.x : 0.0f, ur.y <= uc.y ? nAr.y : 0.0f);
  }
  if (HAS_KL) {
    const float2 e = __ffma2_rn(lp, m1, ref);                        // ref - lp
    const float2 te = __fmul2_rn(e, make_float2(kLog2e, kLog2e));
    const float2 em1 = __fadd2_rn(make_float2(ex2_approx(te.x), ex2_approx(te.y)), m1);
    const float2 kl = __ffma2_rn(e, m1, em1);                        // expm1(e) - e
    term = __ffma2_rn(make_float2(beta, beta), kl, term);
    dterm = __ffma2_rn(make_float2(-beta, -beta), em1, dterm);
  }
}

}  // namespace pl
