// Loss kernel for small batches (up to kSmallMaxTokens tokens and
// kSmallMaxRows sequences): the same per-token arithmetic as the cooperative
// kernel ("Geometric-AI Kernels" model card, "BNPO Loss" and "GRPO Loss"),
// without its grid barrier.
//
// A small batch's mask is at most 64 KB, so every block counts all of it
// itself -- the global valid-token count and, for GRPO, every sequence's count
// in shared memory -- and then scales its own tokens' gradients at once.  The
// blocks never wait on one another: an ordinary launch, no cooperative launch
// and no grid barrier, which is most of a small call's time in the
// cooperative kernel.  A block of 256 threads covers 2048 tokens at bf16/fp16
// (1024 at fp32, 256 on the scalar path), so a small batch still spreads over
// several SMs; each thread's operands are loaded before the mask is counted,
// so the two latencies overlap.  One block writes the loss itself; with
// several, the last to finish sums the
// per-block fp64 partials in block order (deterministic for a given grid),
// writes the loss and the counts, and returns its counter to zero.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "policy_math.cuh"

namespace pl {
namespace {

constexpr int kSmallThreads = 256;
constexpr int kSmallVecs = 1;  // 16-byte vectors per thread: 8 tokens at bf16/fp16, 4 at fp32

__device__ __forceinline__ float tf(float x) { return x; }
__device__ __forceinline__ float tf(__half x) { return __half2float(x); }
__device__ __forceinline__ float tf(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T ft(float x);
template <> __device__ __forceinline__ float ft<float>(float x) { return x; }
template <> __device__ __forceinline__ __half ft<__half>(float x) { return __float2half_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 ft<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Number of nonzero bytes of a 32-bit word (a byte is nonzero iff, after
// adding 0x7F to its low 7 bits, its high bit or its own high bit is set).
__device__ __forceinline__ unsigned nonzero_bytes32(unsigned w) {
  return __popc((((w & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | w) & 0x80808080u);
}

// Sequence index of token t (t < 2^32 here): one multiply-high with the
// constants LossArgs carries (seq_divider).
__device__ __forceinline__ int64_t seq_of(const LossArgs& a, int64_t t) {
  if (a.div32) {
    const unsigned n = (unsigned)t;
    const unsigned q = __umulhi(a.seq_magic, n);
    return (int64_t)((q + ((n - q) >> a.seq_sh1)) >> a.seq_sh2);
  }
  return t / a.seq;
}

template <typename T>
__device__ __forceinline__ float adv_of(const LossArgs& a, int64_t r) {
  if (a.adv_lp_dtype) return tf(reinterpret_cast<const T*>(a.adv)[r]);
  return reinterpret_cast<const float*>(a.adv)[r];
}

template <typename T, bool VEC>
constexpr int64_t small_tokens_per_block() {
  return (int64_t)kSmallThreads * kSmallVecs * (VEC ? (int64_t)(16 / sizeof(T)) : 1);
}

template <typename T, bool HAS_KL, bool HAS_GRAD, bool TWO_SIDED, bool VEC>
__global__ void __launch_bounds__(kSmallThreads) loss_small_kernel(LossArgs a) {
  constexpr int VW = VEC ? (int)(16 / sizeof(T)) : 1;
  constexpr int64_t kTok = small_tokens_per_block<T, VEC>();
  __shared__ unsigned s_rows[kSmallMaxRows];
  __shared__ unsigned s_total;
  __shared__ double s_red[kSmallThreads / 32];
  __shared__ int s_last;

  unsigned* done = reinterpret_cast<unsigned*>(a.ws + 8);
  double* partial = reinterpret_cast<double*>(a.ws + a.partial_offset);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t n = a.n, seq = a.seq;
  const bool rows = a.need_rows != 0;
  const T* lp = reinterpret_cast<const T*>(a.lp);
  const T* od = reinterpret_cast<const T*>(a.old);
  const T* rf = reinterpret_cast<const T*>(a.ref);
  T* gr = reinterpret_cast<T*>(a.grad);
  const int64_t t0 = (int64_t)blockIdx.x * kTok;
  const int64_t t1 = min(n, t0 + kTok);

  // This thread's log-probs and mask bytes do not depend on the counts: their
  // loads go out first, so their latency overlaps the mask count below.
  uint4 ul[kSmallVecs], uo[kSmallVecs], ur[kSmallVecs];
  uint2 um[kSmallVecs];
  if (VEC) {
#pragma unroll
    for (int v = 0; v < kSmallVecs; ++v) {
      const int64_t t = t0 + ((int64_t)v * kSmallThreads + tid) * VW;
      if (t + VW <= t1) {
        ul[v] = __ldg(reinterpret_cast<const uint4*>(lp + t));
        uo[v] = __ldg(reinterpret_cast<const uint4*>(od + t));
        ur[v] = HAS_KL ? __ldg(reinterpret_cast<const uint4*>(rf + t)) : make_uint4(0, 0, 0, 0);
        um[v] = VW == 8 ? __ldg(reinterpret_cast<const uint2*>(a.mask + t))
                        : make_uint2(__ldg(reinterpret_cast<const unsigned*>(a.mask + t)), 0u);
      }
    }
  }

  for (int r = tid; r < kSmallMaxRows; r += kSmallThreads) s_rows[r] = 0u;
  if (tid == 0) s_total = 0u;
  __syncthreads();

  // ---- every block counts the whole mask ----
  unsigned my = 0;
  if (VEC) {
    // 16 mask bytes per load; a word inside one sequence adds to it at once
    const int64_t nw = n / 16;
    const uint4* m16 = reinterpret_cast<const uint4*>(a.mask);
    for (int64_t w = tid; w < nw; w += kSmallThreads) {
      const uint4 u = __ldg(m16 + w);
      const unsigned c = nonzero_bytes32(u.x) + nonzero_bytes32(u.y) + nonzero_bytes32(u.z) + nonzero_bytes32(u.w);
      my += c;
      if (rows && c) {
        const int64_t t = w * 16;
        const int64_t ra = seq_of(a, t), rb = seq_of(a, t + 15);
        if (ra == rb) {
          atomicAdd(&s_rows[ra], c);
        } else {
          const uint8_t* b = a.mask + t;
          for (int j = 0; j < 16; ++j)
            if (b[j]) atomicAdd(&s_rows[seq_of(a, t + j)], 1u);
        }
      }
    }
    for (int64_t t = nw * 16 + tid; t < n; t += kSmallThreads)
      if (a.mask[t]) {
        ++my;
        if (rows) atomicAdd(&s_rows[seq_of(a, t)], 1u);
      }
  } else {
    for (int64_t t = tid; t < n; t += kSmallThreads)
      if (a.mask[t]) {
        ++my;
        if (rows) atomicAdd(&s_rows[seq_of(a, t)], 1u);
      }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) my += __shfl_xor_sync(0xffffffffu, my, o);
  if (lane == 0 && my) atomicAdd(&s_total, my);
  __syncthreads();
  const unsigned total = s_total;
  const float inv_total = (float)(1.0 / (double)(total > 0u ? total : 1u));

  // ---- this block's tokens: loss terms and the scaled gradient ----
  const float lo = a.lo, hi = a.hi, beta = a.beta;
  auto scale_of = [&](int64_t r) {
    return a.grpo ? (float)(1.0 / ((double)a.bs * (double)(s_rows[r] > 0u ? s_rows[r] : 1u))) : inv_total;
  };
  float acc = 0.0f;
#pragma unroll
  for (int v = 0; v < kSmallVecs; ++v) {
    const int64_t t = t0 + ((int64_t)v * kSmallThreads + tid) * VW;
    if (t >= t1) continue;
    if (VEC && t + VW <= t1) {
      const T* el = reinterpret_cast<const T*>(&ul[v]);
      const T* eo = reinterpret_cast<const T*>(&uo[v]);
      const T* er = reinterpret_cast<const T*>(&ur[v]);
      const uint8_t* em = reinterpret_cast<const uint8_t*>(&um[v]);
      uint4 ug;
      T* eg = reinterpret_cast<T*>(&ug);
      int64_t r = seq_of(a, t);
      if ((t - r * seq) + VW <= seq) {
        // the vector lies in one sequence: two tokens per packed instruction
        const float A = adv_of<T>(a, r), sc = scale_of(r);
#pragma unroll
        for (int k = 0; k < VW / 2; ++k) {
          float2 term, dterm;
          token_math2<HAS_KL, TWO_SIDED>(make_float2(tf(el[2 * k]), tf(el[2 * k + 1])),
                                         make_float2(tf(eo[2 * k]), tf(eo[2 * k + 1])),
                                         HAS_KL ? make_float2(tf(er[2 * k]), tf(er[2 * k + 1])) : make_float2(0.f, 0.f),
                                         A, lo, hi, beta, term, dterm);
          const float s0 = em[2 * k] ? sc : 0.0f, s1 = em[2 * k + 1] ? sc : 0.0f;
          acc += term.x * s0 + term.y * s1;
          eg[2 * k] = ft<T>(dterm.x * s0);
          eg[2 * k + 1] = ft<T>(dterm.y * s1);
        }
      } else {
        int64_t next = (r + 1) * seq;
        float A = adv_of<T>(a, r), sc = scale_of(r);
#pragma unroll
        for (int j = 0; j < VW; ++j) {
          if (t + j == next) {
            ++r;
            next += seq;
            A = adv_of<T>(a, r);
            sc = scale_of(r);
          }
          float term, dterm;
          token_math<HAS_KL, TWO_SIDED, true>(tf(el[j]), tf(eo[j]), HAS_KL ? tf(er[j]) : 0.0f, A, lo, hi, beta,
                                              term, dterm);
          const bool valid = em[j] != 0;
          acc += valid ? term * sc : 0.0f;
          eg[j] = ft<T>(valid ? dterm * sc : 0.0f);
        }
      }
      if (HAS_GRAD) *reinterpret_cast<uint4*>(gr + t) = ug;
    } else {
      // scalar operands, or the ragged end of the batch
      for (int64_t u = t; u < min(t1, t + VW); ++u) {
        const int64_t r = seq_of(a, u);
        const float sc = scale_of(r);
        float term, dterm;
        token_math<HAS_KL, TWO_SIDED, true>(tf(lp[u]), tf(od[u]), HAS_KL ? tf(rf[u]) : 0.0f, adv_of<T>(a, r), lo,
                                            hi, beta, term, dterm);
        const bool valid = a.mask[u] != 0;
        acc += valid ? term * sc : 0.0f;
        if (HAS_GRAD) gr[u] = ft<T>(valid ? dterm * sc : 0.0f);
      }
    }
  }

  // ---- block partial; one block writes the loss, or the last of several sums the partials in order ----
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) s_red[warp] = (double)acc;
  __syncthreads();
  if (gridDim.x == 1) {
    if (tid == 0) {
      double s = 0.0;
      for (int w = 0; w < kSmallThreads / 32; ++w) s += s_red[w];
      *a.loss_out = (float)s;
      if (a.n_valid_out) *a.n_valid_out = (int64_t)total;
    }
  } else {
    if (tid == 0) {
      double s = 0.0;
      for (int w = 0; w < kSmallThreads / 32; ++w) s += s_red[w];
      partial[blockIdx.x] = s;
      __threadfence();
      s_last = atomicAdd(done, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (warp == 0) {
      double ps = 0.0;
      for (unsigned b = lane; b < gridDim.x; b += 32) ps += __ldcg(&partial[b]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      if (lane == 0) {
        *a.loss_out = (float)ps;
        if (a.n_valid_out) *a.n_valid_out = (int64_t)total;
        *done = 0u;
      }
    }
  }
  if (a.row_valid_out)
    for (int64_t r = tid; r < a.bs; r += kSmallThreads) a.row_valid_out[r] = (int64_t)s_rows[r];
}

template <typename T, bool HAS_KL, bool HAS_GRAD, bool TWO_SIDED, bool VEC>
cudaError_t launch_small_t(const LossArgs& a, cudaStream_t stream) {
  constexpr int64_t kTok = small_tokens_per_block<T, VEC>();
  const int64_t blocks = a.n > 0 ? (a.n + kTok - 1) / kTok : 1;
  launch_begin(1, stream);
  loss_small_kernel<T, HAS_KL, HAS_GRAD, TWO_SIDED, VEC><<<(unsigned)blocks, kSmallThreads, 0, stream>>>(a);
  launch_end(1, stream);
  return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_small_t(const LossArgs& a, bool kl, bool g, bool two, bool vec, cudaStream_t s) {
#define PL_SMALL_CASE(KL, G, TW, VE) \
  if (kl == KL && g == G && two == TW && vec == VE) return launch_small_t<T, KL, G, TW, VE>(a, s);
  PL_SMALL_CASE(true, true, false, true)
  PL_SMALL_CASE(true, true, false, false)
  PL_SMALL_CASE(true, true, true, true)
  PL_SMALL_CASE(true, true, true, false)
  PL_SMALL_CASE(true, false, false, true)
  PL_SMALL_CASE(true, false, false, false)
  PL_SMALL_CASE(true, false, true, true)
  PL_SMALL_CASE(true, false, true, false)
  PL_SMALL_CASE(false, true, false, true)
  PL_SMALL_CASE(false, true, false, false)
  PL_SMALL_CASE(false, true, true, true)
  PL_SMALL_CASE(false, true, true, false)
  PL_SMALL_CASE(false, false, false, true)
  PL_SMALL_CASE(false, false, false, false)
  PL_SMALL_CASE(false, false, true, true)
  PL_SMALL_CASE(false, false, true, false)
#undef PL_SMALL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

bool loss_small_eligible(int64_t bs, int64_t n) {
  // at most 64 blocks even on the scalar path (1024 threads x 2 tokens each)
  return n > 0 && n <= kSmallMaxTokens && bs <= kSmallMaxRows;
}

cudaError_t launch_loss_small(const LossArgs& a, DType dt, bool has_kl, bool has_grad, bool two_sided, bool vec,
                              cudaStream_t stream) {
  switch (dt) {
    case DType::F32: return dispatch_small_t<float>(a, has_kl, has_grad, two_sided, vec, stream);
    case DType::F16: return dispatch_small_t<__half>(a, has_kl, has_grad, two_sided, vec, stream);
    case DType::BF16: return dispatch_small_t<__nv_bfloat16>(a, has_kl, has_grad, two_sided, vec, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace pl
