// Single-launch BNPO/GRPO loss kernel (forward + optional backward).
//
// Per token ("Geometric-AI Kernels" model card, "BNPO Loss"):
//   ratio = exp(lp - old), clipped = clip(ratio, lo, hi), per_token = -A*min(ratio, clipped),
//   kl = exp(ref - lp) - (ref - lp) - 1   (here expm1(e) - e, e = ref - lp)
// Reductions: BNPO divides by the global valid-token count ("BNPO Loss"), GRPO by
// each sequence's count and then by bs ("GRPO Loss").  The counts are taken on the
// device with integer atomics (no host mask.sum()), as the card's "BNPO Loss"
// section describes; the KL branch is compiled out when beta == 0.
//
// One cooperative launch, three phases:
//   A. every block counts the mask over its contiguous token range (global and
//      per-sequence counts, exact u64 atomics);
//   -- bounded grid barrier (gives up after kWaitLimitNs and raises the error flag);
//   B. 16-byte vector loads of the log-probs, per-token math in fp32, the scaled
//      gradient written in the log-prob dtype, and a per-block partial loss;
//   C. the last block to finish sums the partials in block order (fp64, so the
//      result is deterministic), writes the loss and counts, and returns the
//      workspace counters to zero.
// Batches of up to 65536 tokens take the barrier-free kernel of loss_small.cu
// instead, with the same per-token arithmetic (policy_math.cuh).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "policy_math.cuh"

namespace pl {
namespace {

constexpr int kThreads = 512;
constexpr int kSmemRows = 64;
constexpr size_t kMaskBitsBytes = 64 * 1024;  // one byte per vector: up to 512K tokens per block (bf16)

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// 16-byte vector <-> VW floats.
template <typename T, int VW>
__device__ __forceinline__ void load16(const T* p, float (&v)[VW]) {
  static_assert(VW * sizeof(T) == 16, "16-byte vectors");
  uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
  for (int j = 0; j < VW; ++j) v[j] = to_f(e[j]);
}

// 16-byte vector of log-probs -> VW/2 float2 pairs (bf16: one shift or mask per element).
__device__ __forceinline__ void load16_pairs(const __nv_bfloat16* p, float2 (&v)[4]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const unsigned w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) v[k] = make_float2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xFFFF0000u));
}
__device__ __forceinline__ void load16_pairs(const __half* p, float2 (&v)[4]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const unsigned w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) v[k] = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
}
__device__ __forceinline__ void load16_pairs(const float* p, float2 (&v)[2]) {
  const float4 u = __ldg(reinterpret_cast<const float4*>(p));
  v[0] = make_float2(u.x, u.y);
  v[1] = make_float2(u.z, u.w);
}

__device__ __forceinline__ uint4 ld16_raw(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ void unpack16_pairs(const uint4& u, const __nv_bfloat16*, float2 (&v)[4]) {
  const unsigned w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) v[k] = make_float2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xFFFF0000u));
}
__device__ __forceinline__ void unpack16_pairs(const uint4& u, const __half*, float2 (&v)[4]) {
  const unsigned w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) v[k] = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
}
__device__ __forceinline__ void unpack16_pairs(const uint4& u, const float*, float2 (&v)[2]) {
  v[0] = make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
  v[1] = make_float2(__uint_as_float(u.z), __uint_as_float(u.w));
}

__device__ __forceinline__ void store16_pairs(__nv_bfloat16* p, const float2 (&g)[4]) {
  uint4 u;
  unsigned* w = reinterpret_cast<unsigned*>(&u);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(g[k].x, g[k].y);
    w[k] = *reinterpret_cast<const unsigned*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store16_pairs(__half* p, const float2 (&g)[4]) {
  uint4 u;
  unsigned* w = reinterpret_cast<unsigned*>(&u);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __half2 h = __floats2half2_rn(g[k].x, g[k].y);
    w[k] = *reinterpret_cast<const unsigned*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store16_pairs(float* p, const float2 (&g)[2]) {
  *reinterpret_cast<float4*>(p) = make_float4(g[0].x, g[0].y, g[1].x, g[1].y);
}

template <typename T, int VW>
__device__ __forceinline__ void store16(T* p, const float (&v)[VW]) {
  uint4 u;
  T* e = reinterpret_cast<T*>(&u);
#pragma unroll
  for (int j = 0; j < VW; ++j) e[j] = from_f<T>(v[j]);
  *reinterpret_cast<uint4*>(p) = u;
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Row (sequence) index of token t: one multiply-high when n < 2^32 (see seq_divider).
__device__ __forceinline__ int64_t row_of(const LossArgs& a, int64_t t) {
  if (a.div32) {
    const unsigned n = (unsigned)t;
    const unsigned q = __umulhi(a.seq_magic, n);
    return (int64_t)((q + ((n - q) >> a.seq_sh1)) >> a.seq_sh2);
  }
  return t / a.seq;
}


template <typename T>
__device__ __forceinline__ float load_adv(const LossArgs& a, int64_t r) {
  if (a.adv_lp_dtype) return to_f(reinterpret_cast<const T*>(a.adv)[r]);
  return reinterpret_cast<const float*>(a.adv)[r];
}

template <typename T, bool HAS_KL, bool HAS_GRAD, bool TWO_SIDED, bool VEC>
__global__ void __launch_bounds__(kThreads, 2) loss_kernel(LossArgs a) {
  constexpr int VW = VEC ? (int)(16 / sizeof(T)) : 1;
  // Phase A leaves the block's mask in shared memory as one bit per token (one
  // byte per vector of VW tokens), so phase B does not read it from HBM again.
  extern __shared__ uint8_t s_maskbits[];
  __shared__ unsigned long long s_rows[kSmemRows];
  __shared__ double s_red[kThreads / 32];
  __shared__ unsigned long long s_cnt[kThreads / 32];
  __shared__ int s_flag;

  unsigned* err = reinterpret_cast<unsigned*>(a.ws);
  unsigned* arrive = reinterpret_cast<unsigned*>(a.ws + 4);
  unsigned* done = reinterpret_cast<unsigned*>(a.ws + 8);
  unsigned long long* nvalid = reinterpret_cast<unsigned long long*>(a.ws + 16);
  unsigned long long* rowcnt = reinterpret_cast<unsigned long long*>(a.ws + kWsHeader);
  double* partial = reinterpret_cast<double*>(a.ws + a.partial_offset);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t n = a.n, seq = a.seq;
  const int64_t t0 = min(n, (int64_t)blockIdx.x * a.chunk);
  const int64_t t1 = min(n, t0 + a.chunk);
  const bool any = t1 > t0;
  const int64_t r0 = any ? t0 / seq : 0;
  const int64_t r1 = any ? (t1 - 1) / seq : -1;
  const bool rows_in_smem = a.need_rows && any && (r1 - r0 + 1) <= kSmemRows;

  if (tid < kSmemRows) s_rows[tid] = 0;
  if (tid == 0) s_flag = 0;
  __syncthreads();

  // ---------------- phase A: valid-token counts ----------------
  // Each thread reads 16 mask bytes per load, four independent loads at a time
  // (64 KB in flight per SM), keeps a run (row, count) that it flushes when its
  // row changes, and -- on the vector path -- leaves the block's mask in shared
  // memory as one bit per token (one byte per VW-token vector) for phase B.
  const bool bits_in_smem = VEC && a.mask_bits_smem;
  unsigned long long my_total = 0;
  const uint8_t* mk = a.mask;
  int64_t run_row = -1;
  unsigned run_cnt = 0;
  auto flush = [&](int64_t r, unsigned c) {
    my_total += c;
    if (a.need_rows && c) {
      if (rows_in_smem) atomicAdd(&s_rows[r - r0], (unsigned long long)c);
      else atomicAdd(&rowcnt[r], (unsigned long long)c);
    }
  };
  auto count_one = [&](int64_t r, unsigned c) {
    if (r != run_row) {
      flush(run_row, run_cnt);
      run_row = r;
      run_cnt = 0;
    }
    run_cnt += c;
  };
  // 16 mask bytes starting at token t (t - t0 a multiple of 16): counts, and bits into shared memory.
  auto mask16 = [&](int64_t t, const uint4 u) {
    const unsigned w[4] = {u.x, u.y, u.z, u.w};
    unsigned h[4], nib[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      h[q] = (((w[q] & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | w[q]) & 0x80808080u;   // high bit of each nonzero byte
      nib[q] = ((h[q] >> 7) | (h[q] >> 14) | (h[q] >> 21) | (h[q] >> 28)) & 0xFu;
    }
    if (bits_in_smem) {
      const int64_t vi = (t - t0) / VW;
      if constexpr (VW == 8) {
        s_maskbits[vi] = (uint8_t)(nib[0] | (nib[1] << 4));
        s_maskbits[vi + 1] = (uint8_t)(nib[2] | (nib[3] << 4));
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) s_maskbits[vi + q] = (uint8_t)nib[q];
      }
    }
    const int64_t r = row_of(a, t);
    if ((t - r * seq) + 16 <= seq) {
      count_one(r, __popc(h[0]) + __popc(h[1]) + __popc(h[2]) + __popc(h[3]));
    } else {
      int64_t rr = r, boundary = (r + 1) * seq;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (t + j == boundary) { ++rr; boundary += seq; }
        count_one(rr, (nib[j >> 2] >> (j & 3)) & 1u);
      }
    }
  };
  constexpr int kU = 4;
  for (int64_t base = t0 + (int64_t)tid * 16; base < t1; base += (int64_t)kThreads * 16 * kU) {
    uint4 u[kU];
#pragma unroll
    for (int k = 0; k < kU; ++k) {
      const int64_t t = base + (int64_t)k * kThreads * 16;
      if (VEC && t + 16 <= t1) u[k] = __ldg(reinterpret_cast<const uint4*>(mk + t));
    }
#pragma unroll
    for (int k = 0; k < kU; ++k) {
      const int64_t t = base + (int64_t)k * kThreads * 16;
      if (t >= t1) break;
      if (VEC && t + 16 <= t1) {
        mask16(t, u[k]);
      } else {
        // ragged tail of the last block, or unaligned operands: byte by byte
        const int64_t te = min(t1, t + 16);
        int64_t rr = row_of(a, t), boundary = (rr + 1) * seq;
        unsigned vbits = 0;
        for (int64_t v = t; v < te; ++v) {
          if (v == boundary) { ++rr; boundary += seq; }
          const unsigned m = mk[v] != 0;
          count_one(rr, m);
          vbits |= m << ((v - t0) % VW);
          if (bits_in_smem && ((v - t0) % VW == VW - 1 || v == te - 1)) {
            s_maskbits[(v - t0) / VW] = (uint8_t)vbits;
            vbits = 0;
          }
        }
      }
    }
  }
  // phase B's first two vectors of each thread toward L2 while the grid gathers
  // at the barrier (measured 0.7% faster at 2^27 tokens)
  if (VEC) {
    const T* lpp = reinterpret_cast<const T*>(a.lp);
    const T* odp = reinterpret_cast<const T*>(a.old);
    const T* rfp = reinterpret_cast<const T*>(a.ref);
#pragma unroll
    for (int d = 0; d < 2; ++d) {
      const int64_t tp = t0 + ((int64_t)tid + (int64_t)d * kThreads) * VW;
      if (tp + VW <= t1) {
        prefetch_l2(lpp + tp);
        prefetch_l2(odp + tp);
        if (HAS_KL) prefetch_l2(rfp + tp);
      }
    }
  }
  flush(run_row, run_cnt);
  // block total of valid tokens -> one global atomic
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) my_total += __shfl_xor_sync(0xffffffffu, my_total, o);
  if (lane == 0) s_cnt[warp] = my_total;
  __syncthreads();
  if (tid == 0) {
    unsigned long long s = 0;
    for (int w = 0; w < kThreads / 32; ++w) s += s_cnt[w];
    if (s) atomicAdd(nvalid, s);
  }
  if (rows_in_smem && tid < (int)(r1 - r0 + 1) && s_rows[tid]) atomicAdd(&rowcnt[r0 + tid], s_rows[tid]);

  // ---------------- bounded grid barrier ----------------
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    atomicAdd(arrive, 1u);
    const unsigned long long start = globaltimer_ns();
    while (ld_acquire_u32(arrive) < gridDim.x + a.extra_arrivals) {
      if (globaltimer_ns() - start > a.wait_ns) {
        atomicOr(err, kDevErrTimeout);
        s_flag = 1;
        break;
      }
      __nanosleep(100);
    }
    __threadfence();
  }
  __syncthreads();

  // ---------------- phase B: per-token loss and gradient ----------------
  float acc = 0.0f;
  float2 acc2 = make_float2(0.0f, 0.0f);
  if (!s_flag && any) {
    const unsigned long long total = __ldcg(nvalid);
    const float inv_total = (float)(1.0 / (double)(total > 0 ? total : 1));
    const T* lp = reinterpret_cast<const T*>(a.lp);
    const T* od = reinterpret_cast<const T*>(a.old);
    const T* rf = reinterpret_cast<const T*>(a.ref);
    T* gr = reinterpret_cast<T*>(a.grad);
    const float lo = a.lo, hi = a.hi, beta = a.beta;
    int64_t cur_row = -1;
    float A = 0.0f, scale = 0.0f;
    auto row_state = [&](int64_t r) {
      if (r != cur_row) {
        cur_row = r;
        A = load_adv<T>(a, r);
        if (a.grpo) {
          const unsigned long long c = __ldcg(&rowcnt[r]);
          scale = (float)(1.0 / ((double)a.bs * (double)(c > 0 ? c : 1)));
        } else {
          scale = inv_total;
        }
      }
    };
    auto scalar_span = [&](int64_t t, int64_t te) {
      // unaligned operands, or the ragged tail of the last block
      for (int64_t u = t; u < te; ++u) {
        row_state(row_of(a, u));
        float term, dterm;
        token_math<HAS_KL, TWO_SIDED, true>(to_f(lp[u]), to_f(od[u]), HAS_KL ? to_f(rf[u]) : 0.0f, A, lo,
                                            hi, beta, term, dterm);
        const bool valid = a.mask[u] != 0;
        acc += valid ? term * scale : 0.0f;
        if (HAS_GRAD) gr[u] = from_f<T>(valid ? dterm * scale : 0.0f);
      }
    };
    uint4 cu_l = make_uint4(0u, 0u, 0u, 0u), cu_o = cu_l, cu_r = cu_l;
    if constexpr (VEC) {
      const int64_t tf = t0 + (int64_t)tid * VW;
      if (tf + VW <= t1) {
        cu_l = ld16_raw(lp + tf);
        cu_o = ld16_raw(od + tf);
        if (HAS_KL) cu_r = ld16_raw(rf + tf);
      }
    }
    for (int64_t t = t0 + (int64_t)tid * VW; t < t1; t += (int64_t)kThreads * VW) {
      if constexpr (VEC) {
        if (t + VW > t1) {
          scalar_span(t, t1);
          continue;
        }
        constexpr int NP = VW / 2;
        // this thread's next vector: its loads in flight while this one is computed,
        // and the one after it toward L2
        const int64_t tn = t + (int64_t)kThreads * VW;
        uint4 nx_l = cu_l, nx_o = cu_o, nx_r = cu_r;
        if (tn + VW <= t1) {
          nx_l = ld16_raw(lp + tn);
          nx_o = ld16_raw(od + tn);
          if (HAS_KL) nx_r = ld16_raw(rf + tn);
          const int64_t tnn = tn + (int64_t)kThreads * VW;
          if (tnn + VW <= t1) {
            prefetch_l2(lp + tnn);
            prefetch_l2(od + tnn);
            if (HAS_KL) prefetch_l2(rf + tnn);
          }
        }
        float2 pl[NP], po[NP], pr[NP], pg[NP];
        unpack16_pairs(cu_l, lp, pl);
        unpack16_pairs(cu_o, od, po);
        if (HAS_KL) unpack16_pairs(cu_r, rf, pr);
        cu_l = nx_l;
        cu_o = nx_o;
        cu_r = nx_r;
        unsigned bits;
        if (bits_in_smem) {
          bits = s_maskbits[(t - t0) / VW];
        } else {
          bits = 0;
          if constexpr (VW == 8) {
            const uint2 u = __ldg(reinterpret_cast<const uint2*>(a.mask + t));
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              bits |= (((u.x >> (8 * j)) & 0xFFu) != 0u) << j;
              bits |= (((u.y >> (8 * j)) & 0xFFu) != 0u) << (j + 4);
            }
          } else {
            const unsigned u = __ldg(reinterpret_cast<const unsigned*>(a.mask + t));
#pragma unroll
            for (int j = 0; j < 4; ++j) bits |= (((u >> (8 * j)) & 0xFFu) != 0u) << j;
          }
        }
        int64_t r = row_of(a, t);
        if ((t - r * seq) + VW <= seq) {
          // the whole vector lies in one sequence: two tokens per packed instruction
          row_state(r);
#pragma unroll
          for (int k = 0; k < NP; ++k) {
            float2 term, dterm;
            token_math2<HAS_KL, TWO_SIDED>(pl[k], po[k], HAS_KL ? pr[k] : make_float2(0.0f, 0.0f), A, lo, hi,
                                           beta, term, dterm);
            const float2 sc = make_float2(((bits >> (2 * k)) & 1u) ? scale : 0.0f,
                                          ((bits >> (2 * k + 1)) & 1u) ? scale : 0.0f);
            acc2 = __ffma2_rn(term, sc, acc2);
            pg[k] = __fmul2_rn(dterm, sc);
          }
        } else {
          int64_t boundary = (r + 1) * seq;
#pragma unroll
          for (int j = 0; j < VW; ++j) {
            if (t + j == boundary) { ++r; boundary += seq; }
            row_state(r);
            const float l = (j & 1) ? pl[j >> 1].y : pl[j >> 1].x;
            const float o = (j & 1) ? po[j >> 1].y : po[j >> 1].x;
            const float f = HAS_KL ? ((j & 1) ? pr[j >> 1].y : pr[j >> 1].x) : 0.0f;
            float term, dterm;
            token_math<HAS_KL, TWO_SIDED, true>(l, o, f, A, lo, hi, beta, term, dterm);
            const bool valid = (bits >> j) & 1u;
            acc += valid ? term * scale : 0.0f;
            const float gv = valid ? dterm * scale : 0.0f;
            if (j & 1) pg[j >> 1].y = gv; else pg[j >> 1].x = gv;
          }
        }
        if (HAS_GRAD) store16_pairs(gr + t, pg);
      } else {
        scalar_span(t, t + 1);
      }
    }
  }

  // block partial (warp shuffle in fp32, then fp64 across warps)
  acc += acc2.x + acc2.y;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) s_red[warp] = (double)acc;
  __syncthreads();

  // ---------------- phase C: last-block finalize ----------------
  if (tid == 0) {
    double s = 0.0;
    for (int w = 0; w < kThreads / 32; ++w) s += s_red[w];
    partial[blockIdx.x] = s;
    __threadfence();
    const unsigned prev = atomicAdd(done, 1u);
    s_flag = (prev == gridDim.x - 1) ? 2 : 0;
  }
  __syncthreads();
  if (s_flag == 2) {
    __threadfence();
    // Fixed-order fp64 sum of the block partials: thread i takes partials i,
    // i+512, ... in order, then a fixed shuffle tree and warp order -- the same
    // result on every run for a given grid.
    double ps = 0.0;
    for (unsigned b = tid; b < gridDim.x; b += kThreads) ps += __ldcg(&partial[b]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
    if (lane == 0) s_red[warp] = ps;
    __syncthreads();
    if (tid == 0) {
      double sum = 0.0;
      for (int w = 0; w < kThreads / 32; ++w) sum += s_red[w];
      *a.loss_out = (float)sum;
      if (a.n_valid_out) *a.n_valid_out = (int64_t)__ldcg(nvalid);
      *nvalid = 0ull;
      *arrive = 0u;
      *done = 0u;
    }
    for (int64_t r = tid; r < a.bs; r += kThreads) {
      if (a.row_valid_out) a.row_valid_out[r] = (int64_t)__ldcg(&rowcnt[r]);
      rowcnt[r] = 0ull;
    }
  }
}

template <typename T, bool HAS_KL, bool HAS_GRAD, bool TWO_SIDED, bool VEC>
cudaError_t launch_t(const LossArgs& a0, cudaStream_t stream) {
  auto kern = loss_kernel<T, HAS_KL, HAS_GRAD, TWO_SIDED, VEC>;
  const size_t dyn = VEC ? kMaskBitsBytes : 0;
  static int per_sm_dev[kMaxDevices] = {};  // resident blocks per SM, per device (0: not yet known)
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  int per_sm;
  {
    std::lock_guard<std::mutex> lock(setup_mutex());
    if (per_sm_dev[dev] == 0) {
      cudaError_t e = cudaSuccess;
      if (dyn > 48 * 1024)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
      int n = 0;
      if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, dyn);
      if (e != cudaSuccess) return e;
      per_sm_dev[dev] = n < 1 ? 1 : n;
    }
    per_sm = per_sm_dev[dev];
  }
  DevInfo di;
  cudaError_t e = dev_info(&di);
  if (e != cudaSuccess) return e;
  LossArgs a = a0;
  // Enough blocks to cover the tokens with a few vector iterations per thread,
  // never more than can be co-resident (the grid barrier needs all of them).
  constexpr int64_t kMinTokensPerBlock = 4096;
  int64_t want = (a.n + kMinTokensPerBlock - 1) / kMinTokensPerBlock;
  int64_t cap = (int64_t)per_sm * di.sm_count;
  if (cap > kLossMaxBlocks) cap = kLossMaxBlocks;
  int64_t grid = want < 1 ? 1 : (want > cap ? cap : want);
  int64_t chunk = (a.n + grid - 1) / grid;
  chunk = (chunk + 63) / 64 * 64;
  if (chunk < 64) chunk = 64;
  grid = a.n > 0 ? (a.n + chunk - 1) / chunk : 1;
  a.chunk = chunk;
  constexpr int VWh = VEC ? (int)(16 / sizeof(T)) : 1;
  a.mask_bits_smem = VEC && (chunk / VWh) <= (int64_t)kMaskBitsBytes;
  a.wait_ns = debug_knobs().wait_ns;
  a.extra_arrivals = debug_knobs().extra_arrivals;
  void* args[] = {&a};
  launch_begin(1, stream);
  e = cudaLaunchCooperativeKernel((const void*)kern, dim3((unsigned)grid), dim3(kThreads), args, dyn, stream);
  launch_end(1, stream);
  return e;
}

template <typename T>
cudaError_t dispatch_t(const LossArgs& a, bool kl, bool g, bool two, bool vec, cudaStream_t s) {
#define PL_LOSS_CASE(KL, G, TW, VE) \
  if (kl == KL && g == G && two == TW && vec == VE) return launch_t<T, KL, G, TW, VE>(a, s);
  PL_LOSS_CASE(true, true, false, true)
  PL_LOSS_CASE(true, true, false, false)
  PL_LOSS_CASE(true, true, true, true)
  PL_LOSS_CASE(true, true, true, false)
  PL_LOSS_CASE(true, false, false, true)
  PL_LOSS_CASE(true, false, false, false)
  PL_LOSS_CASE(true, false, true, true)
  PL_LOSS_CASE(true, false, true, false)
  PL_LOSS_CASE(false, true, false, true)
  PL_LOSS_CASE(false, true, false, false)
  PL_LOSS_CASE(false, true, true, true)
  PL_LOSS_CASE(false, true, true, false)
  PL_LOSS_CASE(false, false, false, true)
  PL_LOSS_CASE(false, false, false, false)
  PL_LOSS_CASE(false, false, true, true)
  PL_LOSS_CASE(false, false, true, false)
#undef PL_LOSS_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_loss(const LossArgs& a, DType dt, bool has_kl, bool has_grad, bool two_sided,
                        bool vec, cudaStream_t stream) {
  switch (dt) {
    case DType::F32: return dispatch_t<float>(a, has_kl, has_grad, two_sided, vec, stream);
    case DType::F16: return dispatch_t<__half>(a, has_kl, has_grad, two_sided, vec, stream);
    case DType::BF16: return dispatch_t<__nv_bfloat16>(a, has_kl, has_grad, two_sided, vec, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace pl
