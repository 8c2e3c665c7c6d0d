// Reverse-KL self-distillation kernel (forward, optionally fused with the
// gradient with respect to the student logits).
//
// "Geometric-AI Kernels" model card, section "Reverse KL":
//   p = softmax(student row), q = softmax(teacher row),
//   kl_r = sum_v p_v (log p_v - log q_v),  loss = sum_r mask_r kl_r / n_valid,
//   grad_v = mask_r / n_valid * p_v (log p_v - log q_v - kl_r).
// The card's forward reads every logit row once with an online normalisation;
// this kernel does the same.  n_valid is clamped to >= 1 (the card leaves the
// all-masked batch as inf/NaN).
//
// Per row, with s the student logits and t the teacher logits, pass 1 keeps
//   ms = max s, zs = sum e^(s - ms), a = sum e^(s - ms) (s - t),
//   mt = max t, zt = sum e^(t - mt)
// (rescaled whenever a running maximum grows).  Then
//   E_p[s - t] = a / zs,   lse_s - lse_t = (ms - mt) + ln(zs / zt),
//   kl = E_p[s - t] - (lse_s - lse_t),
// and the gradient needs only E_p[s - t]:
//   log p_v - log q_v - kl = (s_v - t_v) - E_p[s - t],
//   grad_v = scale * p_v * ((s_v - t_v) - E_p[s - t]),  scale = [mask_r] / max(n_valid, 1).
//
// Layout: a row is split across a thread-block cluster of `cl` CTAs (1..8);
// CTA k of the cluster owns columns [k*slice, (k+1)*slice).  Each CTA reduces
// its slice's statistics (warp shuffles, then warps in order), the cluster
// merges the CTAs' statistics in rank order through distributed shared memory,
// and pass 2 re-reads the CTA's slice (mostly an L2 hit: the host picks `cl`
// so that the slices of all resident CTAs fit in about 1.25 x L2) and writes
// the gradient.
// Pass 1 reads with an L2 evict-last policy and pass 2 with evict-first (the
// gradient is stored evict-first too), so the slice stays in L2 between its
// two reads and leaves it after the second.
// Rows are dealt to the clusters by kind: the k-th valid row goes to cluster
// k mod ncl, and the j-th masked row to cluster (n_valid + j) mod ncl, so every
// cluster reads within one row of the same number of valid rows, whatever the
// mask (a plain round-robin over all rows left some clusters with several more
// valid rows than others).  Fully masked rows are not read at all (their
// gradient slice is written as zeros).  Every CTA counts the mask itself, so
// the scale is known before any gradient is written, without a grid barrier.
// The loss is summed per cluster in row order (fp64) and the last cluster to
// finish adds the cluster partials in cluster order: the result is
// deterministic for a given mask and grid.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace pl {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxCluster = 8;
constexpr int kMaxClusters = 1024;
constexpr float kL2E = 1.4426950408889634f;   // log2(e)

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Element type traits: scalar decode/encode and 16-byte vectors as float pairs.
template <typename T> struct Elt;
template <> struct Elt<__nv_bfloat16> {
  static constexpr int kPairs = 4;   // 8 elements per 16 bytes
  __device__ static float get(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  __device__ static void put(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
  __device__ static float2 pair(unsigned w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  }
  __device__ static unsigned pack(float2 g) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(g.x, g.y);
    return *reinterpret_cast<const unsigned*>(&h);
  }
};
template <> struct Elt<__half> {
  static constexpr int kPairs = 4;
  __device__ static float get(const __half* p) { return __half2float(*p); }
  __device__ static void put(__half* p, float x) { *p = __float2half_rn(x); }
  __device__ static float2 pair(unsigned w) { return __half22float2(*reinterpret_cast<const __half2*>(&w)); }
  __device__ static unsigned pack(float2 g) {
    const __half2 h = __floats2half2_rn(g.x, g.y);
    return *reinterpret_cast<const unsigned*>(&h);
  }
};
template <> struct Elt<float> {
  static constexpr int kPairs = 2;   // 4 elements per 16 bytes
  __device__ static float get(const float* p) { return *p; }
  __device__ static void put(float* p, float x) { *p = x; }
};

// 16-byte vector -> pairs.
template <typename T>
__device__ __forceinline__ void unpack(const uint4& u, float2 (&v)[Elt<T>::kPairs]) {
  if constexpr (sizeof(T) == 4) {
    v[0] = make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
    v[1] = make_float2(__uint_as_float(u.z), __uint_as_float(u.w));
  } else {
    v[0] = Elt<T>::pair(u.x);
    v[1] = Elt<T>::pair(u.y);
    v[2] = Elt<T>::pair(u.z);
    v[3] = Elt<T>::pair(u.w);
  }
}
template <typename T>
__device__ __forceinline__ uint4 pack(const float2 (&g)[Elt<T>::kPairs]) {
  if constexpr (sizeof(T) == 4) {
    return make_uint4(__float_as_uint(g[0].x), __float_as_uint(g[0].y), __float_as_uint(g[1].x),
                      __float_as_uint(g[1].y));
  } else {
    return make_uint4(Elt<T>::pack(g[0]), Elt<T>::pack(g[1]), Elt<T>::pack(g[2]), Elt<T>::pack(g[3]));
  }
}

// Packed pairs of a 16-bit type, for exact maxima without decoding.
template <typename T> struct T2Of { using type = unsigned; };
template <> struct T2Of<__nv_bfloat16> { using type = __nv_bfloat162; };
template <> struct T2Of<__half> { using type = __half2; };
template <typename T> __device__ __forceinline__ typename T2Of<T>::type as_t2(unsigned w) {
  return *reinterpret_cast<const typename T2Of<T>::type*>(&w);
}
__device__ __forceinline__ float2 to_f2(__nv_bfloat162 h) { return __bfloat1622float2(h); }
__device__ __forceinline__ float2 to_f2(__half2 h) { return __half22float2(h); }

__device__ __forceinline__ int64_t imin(int64_t x, int64_t y) { return x < y ? x : y; }



__device__ __forceinline__ unsigned long long policy_evict_last() {
  unsigned long long p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ unsigned long long policy_evict_first() {
  unsigned long long p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint4 ld16_hint(const void* p, unsigned long long pol) {
  uint4 u;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "l"(p), "l"(pol));
  return u;
}
__device__ __forceinline__ void st16_hint(void* p, uint4 u, unsigned long long pol) {
  asm volatile("st.global.L1::no_allocate.L2::cache_hint.v4.b32 [%0], {%1,%2,%3,%4}, %5;"
               :: "l"(p), "r"(u.x), "r"(u.y), "r"(u.z), "r"(u.w), "l"(pol) : "memory");
}
__device__ __forceinline__ void prefetch_l2_last(const void* p) {
  asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p));
}

// Running statistics of one row (or of part of it).
struct Stats {
  float ms, zs, a, mt, zt;
};

__device__ __forceinline__ float rescale(float m_old, float m_new) {
  return m_old == m_new ? 1.0f : ex2((m_old - m_new) * kL2E);
}

// Merge of two partial statistics.  Plain multiplies and adds (no contraction),
// so merge(x, y) and merge(y, x) agree bit for bit.
__device__ __forceinline__ Stats merge(const Stats& x, const Stats& y) {
  Stats r;
  r.ms = fmaxf(x.ms, y.ms);
  const float fx = rescale(x.ms, r.ms), fy = rescale(y.ms, r.ms);
  r.zs = __fadd_rn(__fmul_rn(x.zs, fx), __fmul_rn(y.zs, fy));
  r.a = __fadd_rn(__fmul_rn(x.a, fx), __fmul_rn(y.a, fy));
  r.mt = fmaxf(x.mt, y.mt);
  const float gx = rescale(x.mt, r.mt), gy = rescale(y.mt, r.mt);
  r.zt = __fadd_rn(__fmul_rn(x.zt, gx), __fmul_rn(y.zt, gy));
  return r;
}

__device__ __forceinline__ Stats shfl_down(const Stats& x, int d) {
  Stats r;
  r.ms = __shfl_down_sync(0xffffffffu, x.ms, d);
  r.zs = __shfl_down_sync(0xffffffffu, x.zs, d);
  r.a = __shfl_down_sync(0xffffffffu, x.a, d);
  r.mt = __shfl_down_sync(0xffffffffu, x.mt, d);
  r.zt = __shfl_down_sync(0xffffffffu, x.zt, d);
  return r;
}

// Per-thread accumulator: scalar maxima, pairwise sums (two lanes of packed math).
struct Acc {
  float ms = -INFINITY, mt = -INFINITY;
  float2 zs = make_float2(0.f, 0.f), a = make_float2(0.f, 0.f), zt = make_float2(0.f, 0.f);

  __device__ __forceinline__ void raise_max(float bs, float bt) {
    if (bs > ms) {
      const float f = ex2((ms - bs) * kL2E);
      zs = __fmul2_rn(zs, make_float2(f, f));
      a = __fmul2_rn(a, make_float2(f, f));
      ms = bs;
    }
    if (bt > mt) {
      const float f = ex2((mt - bt) * kL2E);
      zt = __fmul2_rn(zt, make_float2(f, f));
      mt = bt;
    }
  }
  // Adds one pair of (student, teacher) values; the maxima already cover them.
  __device__ __forceinline__ void add(float2 s, float2 t, float2 nmsl, float2 nmtl) {
    const float2 l2e = make_float2(kL2E, kL2E);
    const float2 xs = __ffma2_rn(s, l2e, nmsl);
    const float2 xt = __ffma2_rn(t, l2e, nmtl);
    const float2 es = make_float2(ex2(xs.x), ex2(xs.y));
    const float2 et = make_float2(ex2(xt.x), ex2(xt.y));
    zs = __fadd2_rn(zs, es);
    zt = __fadd2_rn(zt, et);
    a = __ffma2_rn(es, __ffma2_rn(t, make_float2(-1.f, -1.f), s), a);
  }
  __device__ __forceinline__ void add_scalar(float s, float t) {
    raise_max(s, t);
    const float es = ex2((s - ms) * kL2E), et = ex2((t - mt) * kL2E);
    zs.x += es;
    zt.x += et;
    a.x = fmaf(es, s - t, a.x);
  }
  __device__ __forceinline__ Stats stats() const {
    return Stats{ms, zs.x + zs.y, a.x + a.y, mt, zt.x + zt.y};
  }
};

struct RklArgs {
  const void* s;
  const void* t;
  const uint8_t* mask;
  void* grad;
  float* loss_out;
  float* kl_rows;
  int64_t* n_valid_out;
  unsigned char* ws;
  int64_t N, V;
  int64_t slice;   // columns per CTA (multiple of 8)
  int cl;          // CTAs per cluster
  int vec;         // 16-byte vector path (s, t and grad share their address mod 16)
  // register-resident gradient form only
  unsigned long long wait_ns;  // bound of every wait
  unsigned extra_tx;           // test-only: extra bytes each slot's load expects (0 in normal use)
};

__device__ __forceinline__ unsigned cluster_rank() {
  unsigned r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ unsigned cluster_id() {
  unsigned r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ unsigned cluster_count() {
  unsigned r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster(const float* local, unsigned rank) {
  unsigned addr = static_cast<unsigned>(__cvta_generic_to_shared(local)), remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(addr), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// Number of nonzero bytes of a 32-bit word.
__device__ __forceinline__ int nonzero_bytes(unsigned w) {
  return __popc((((w & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | w) & 0x80808080u);
}

// Elements of [0, n) before the first 16-byte boundary of p (all of them when !vec).
template <typename T>
__device__ __forceinline__ int head_elems(const T* p, int n, bool vec) {
  if (!vec) return n;
  const int h = (int)((16 - (reinterpret_cast<uintptr_t>(p) & 15)) & 15) / (int)sizeof(T);
  return h < n ? h : n;
}

template <typename T, bool GRAD>
__global__ void __launch_bounds__(kThreads, 2) reverse_kl_kernel(RklArgs a) {
  constexpr int kP = Elt<T>::kPairs;
  constexpr int kE = 2 * kP;            // elements per 16-byte vector
  constexpr int kU = 2;                 // vectors per tensor in flight per thread
  using T2 = typename T2Of<T>::type;
  __shared__ Stats warp_stats[kWarps];
  __shared__ float xch[2][5];           // this CTA's statistics for the cluster, by row parity
  __shared__ float row_stats[5];
  __shared__ unsigned long long s_count;
  __shared__ double s_part;             // kl summed over this cluster's valid rows (rank 0)
  __shared__ int s_wcnt[3][kWarps];     // per-warp valid, masked and dealt-here row counts
  __shared__ int s_rows[kThreads];      // this cluster's rows of the current block (offsets)

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned crank = cluster_rank(), cid = cluster_id(), ncl = cluster_count();

  // ---- valid rows (every CTA counts the whole mask) ----
  if (tid == 0) {
    s_count = 0;
    s_part = 0.0;
  }
  __syncthreads();
  int64_t n_valid = a.N;
  if (a.mask) {
    const uint8_t* m = a.mask;
    const int64_t head = imin(a.N, (int64_t)((16 - (reinterpret_cast<uintptr_t>(m) & 15)) & 15));
    const int64_t nv16 = (a.N - head) / 16;
    unsigned long long c = 0;
    for (int64_t i = tid; i < head; i += kThreads) c += m[i] != 0;
    const uint4* m16 = reinterpret_cast<const uint4*>(m + head);
    for (int64_t i = tid; i < nv16; i += kThreads) {
      const uint4 u = __ldg(m16 + i);
      c += nonzero_bytes(u.x) + nonzero_bytes(u.y) + nonzero_bytes(u.z) + nonzero_bytes(u.w);
    }
    for (int64_t i = head + nv16 * 16 + tid; i < a.N; i += kThreads) c += m[i] != 0;
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) c += __shfl_down_sync(0xffffffffu, c, d);
    if (lane == 0 && c) atomicAdd(&s_count, c);
    __syncthreads();
    n_valid = (int64_t)s_count;
  }
  const float log2_scale = -log2f((float)(n_valid > 1 ? n_valid : 1));

  const int64_t v0 = imin(a.V, (int64_t)crank * a.slice);
  const int64_t v1 = imin(a.V, v0 + a.slice);
  const int n = (int)(v1 - v0);   // the host keeps V < 2^31
  int parity = 0;

  // Rows are taken in blocks of kThreads: every CTA of the cluster classifies
  // the block's rows and lists, in row order, the ones dealt to this cluster.
  int64_t vseen = 0, mseen = 0;   // valid and masked rows before the block
  const unsigned below = (1u << lane) - 1u;
  for (int64_t base = 0; base < a.N; base += kThreads) {
    const int64_t rr = base + tid;
    const bool in = rr < a.N;
    const bool valid = in && (!a.mask || a.mask[rr] != 0);
    const unsigned bv = __ballot_sync(0xffffffffu, valid), bm = __ballot_sync(0xffffffffu, in && !valid);
    if (lane == 0) {
      s_wcnt[0][warp] = __popc(bv);
      s_wcnt[1][warp] = __popc(bm);
    }
    __syncthreads();
    int pv = __popc(bv & below), pm = __popc(bm & below), tv = 0, tm = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int x = s_wcnt[0][w], y = s_wcnt[1][w];
      if (w < warp) {
        pv += x;
        pm += y;
      }
      tv += x;
      tm += y;
    }
    const bool mine = valid ? (vseen + pv) % (int64_t)ncl == (int64_t)cid
                            : (in && (n_valid + mseen + pm) % (int64_t)ncl == (int64_t)cid);
    const unsigned bk = __ballot_sync(0xffffffffu, mine);
    if (lane == 0) s_wcnt[2][warp] = __popc(bk);
    __syncthreads();
    int pk = __popc(bk & below), nk = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int x = s_wcnt[2][w];
      if (w < warp) pk += x;
      nk += x;
    }
    if (mine) s_rows[pk] = tid;
    vseen += tv;
    mseen += tm;
    __syncthreads();

    for (int q = 0; q < nk; ++q) {
      const int64_t r = base + s_rows[q];
      const T* srow = static_cast<const T*>(a.s) + r * a.V + v0;
      const T* trow = static_cast<const T*>(a.t) + r * a.V + v0;
      T* grow = GRAD ? static_cast<T*>(a.grad) + r * a.V + v0 : nullptr;
      const int head = head_elems(srow, n, a.vec != 0);
      const int nvec = (n - head) / kE;
      const int tail0 = head + nvec * kE;
      const T* sv = srow + head;
      const T* tv = trow + head;

      if (a.mask && a.mask[r] == 0) {
        if (GRAD) {
          for (int i = tid; i < head; i += kThreads) Elt<T>::put(grow + i, 0.0f);
          uint4* gv = reinterpret_cast<uint4*>(grow + head);
          for (int i = tid; i < nvec; i += kThreads) gv[i] = make_uint4(0, 0, 0, 0);
          for (int i = tail0 + tid; i < n; i += kThreads) Elt<T>::put(grow + i, 0.0f);
        }
        if (a.kl_rows && crank == 0 && tid == 0) a.kl_rows[r] = 0.0f;
        continue;
      }

      // ---- pass 1: online statistics over the slice ----
      Acc acc;
      const unsigned long long pl_last = policy_evict_last();
      for (int i = tid; i < head; i += kThreads) acc.add_scalar(Elt<T>::get(srow + i), Elt<T>::get(trow + i));
      for (int i = tail0 + tid; i < n; i += kThreads) acc.add_scalar(Elt<T>::get(srow + i), Elt<T>::get(trow + i));
      int i = tid;
      for (; i + (kU - 1) * kThreads < nvec; i += kU * kThreads) {
        uint4 us[kU], ut[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          us[u] = ld16_hint(sv + (i + u * kThreads) * kE, pl_last);
          ut[u] = ld16_hint(tv + (i + u * kThreads) * kE, pl_last);
        }
        // the next block's vectors into L2, each one that exists (a partial last block too)
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int j = i + (kU + u) * kThreads;
          if (j < nvec) {
            prefetch_l2_last(sv + j * kE);
            prefetch_l2_last(tv + j * kE);
          }
        }
        float bs, bt;
        if constexpr (sizeof(T) == 2) {
          // maxima of the packed 16-bit values (exact); each element is decoded once, below
          T2 ms2 = as_t2<T>(us[0].x), mt2 = as_t2<T>(ut[0].x);
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            if (u) {
              ms2 = __hmax2(ms2, as_t2<T>(us[u].x));
              mt2 = __hmax2(mt2, as_t2<T>(ut[u].x));
            }
            ms2 = __hmax2(__hmax2(ms2, as_t2<T>(us[u].y)), __hmax2(as_t2<T>(us[u].z), as_t2<T>(us[u].w)));
            mt2 = __hmax2(__hmax2(mt2, as_t2<T>(ut[u].y)), __hmax2(as_t2<T>(ut[u].z), as_t2<T>(ut[u].w)));
          }
          const float2 fs = to_f2(ms2), ft = to_f2(mt2);
          bs = fmaxf(fs.x, fs.y);
          bt = fmaxf(ft.x, ft.y);
        } else {
          bs = -INFINITY;
          bt = -INFINITY;
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            float2 ps[kP], pt[kP];
            unpack<T>(us[u], ps);
            unpack<T>(ut[u], pt);
#pragma unroll
            for (int k = 0; k < kP; ++k) {
              bs = fmaxf(bs, fmaxf(ps[k].x, ps[k].y));
              bt = fmaxf(bt, fmaxf(pt[k].x, pt[k].y));
            }
          }
        }
        acc.raise_max(bs, bt);
        const float2 nmsl = make_float2(-acc.ms * kL2E, -acc.ms * kL2E);
        const float2 nmtl = make_float2(-acc.mt * kL2E, -acc.mt * kL2E);
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          float2 ps[kP], pt[kP];
          unpack<T>(us[u], ps);
          unpack<T>(ut[u], pt);
#pragma unroll
          for (int k = 0; k < kP; ++k) acc.add(ps[k], pt[k], nmsl, nmtl);
        }
      }
      for (; i < nvec; i += kThreads) {
        float2 ps[kP], pt[kP];
        unpack<T>(ld16_hint(sv + i * kE, pl_last), ps);
        unpack<T>(ld16_hint(tv + i * kE, pl_last), pt);
        float bs = -INFINITY, bt = -INFINITY;
#pragma unroll
        for (int k = 0; k < kP; ++k) {
          bs = fmaxf(bs, fmaxf(ps[k].x, ps[k].y));
          bt = fmaxf(bt, fmaxf(pt[k].x, pt[k].y));
        }
        acc.raise_max(bs, bt);
        const float2 nmsl = make_float2(-acc.ms * kL2E, -acc.ms * kL2E);
        const float2 nmtl = make_float2(-acc.mt * kL2E, -acc.mt * kL2E);
#pragma unroll
        for (int k = 0; k < kP; ++k) acc.add(ps[k], pt[k], nmsl, nmtl);
      }

      // ---- reduce: warp, then warps in order, then CTAs of the cluster in rank order ----
      Stats st = acc.stats();
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) {
        const Stats o = shfl_down(st, d);
        st = merge(st, o);
      }
      if (lane == 0) warp_stats[warp] = st;
      __syncthreads();
      if (warp == 0) {
        st = lane < kWarps ? warp_stats[lane] : Stats{-INFINITY, 0.f, 0.f, -INFINITY, 0.f};
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) {
          const Stats o = shfl_down(st, d);
          st = merge(st, o);
        }
        if (lane == 0) {
          xch[parity][0] = st.ms;
          xch[parity][1] = st.zs;
          xch[parity][2] = st.a;
          xch[parity][3] = st.mt;
          xch[parity][4] = st.zt;
        }
      }
      if (a.cl > 1) {
        cluster_sync();
        if (warp == 0) {
          Stats o{-INFINITY, 0.f, 0.f, -INFINITY, 0.f};
          if (lane < a.cl) {
            o.ms = ld_cluster(&xch[parity][0], lane);
            o.zs = ld_cluster(&xch[parity][1], lane);
            o.a = ld_cluster(&xch[parity][2], lane);
            o.mt = ld_cluster(&xch[parity][3], lane);
            o.zt = ld_cluster(&xch[parity][4], lane);
          }
          // rank order 0, 1, ..., cl-1
          st = Stats{__shfl_sync(0xffffffffu, o.ms, 0), __shfl_sync(0xffffffffu, o.zs, 0),
                     __shfl_sync(0xffffffffu, o.a, 0), __shfl_sync(0xffffffffu, o.mt, 0),
                     __shfl_sync(0xffffffffu, o.zt, 0)};
          for (int k = 1; k < a.cl; ++k) {
            const Stats q{__shfl_sync(0xffffffffu, o.ms, k), __shfl_sync(0xffffffffu, o.zs, k),
                          __shfl_sync(0xffffffffu, o.a, k), __shfl_sync(0xffffffffu, o.mt, k),
                          __shfl_sync(0xffffffffu, o.zt, k)};
            st = merge(st, q);
          }
        }
        parity ^= 1;
      }
      if (tid == 0) {
        row_stats[0] = st.ms;
        row_stats[1] = st.zs;
        row_stats[2] = st.a;
        row_stats[3] = st.mt;
        row_stats[4] = st.zt;
      }
      __syncthreads();
      const float ms = row_stats[0], zs = row_stats[1], am = row_stats[2], mt = row_stats[3], zt = row_stats[4];
      const float ep = am / zs;                                // E_p[s - t]
      const float kl = ep - ((ms - mt) + logf(zs / zt));       // minus (lse_s - lse_t)
      if (crank == 0 && tid == 0) {
        s_part += (double)kl;
        if (a.kl_rows) a.kl_rows[r] = kl;
      }

      // ---- pass 2: grad_v = scale * p_v * ((s_v - t_v) - E_p[s - t]) ----
      if (GRAD) {
        // scale * p_v = 2^(s_v log2e - (ms log2e + log2 zs) + log2 scale)
        const float off = -(ms * kL2E + log2f(zs)) + log2_scale;
        for (int j = tid; j < head; j += kThreads) {
          const float s = Elt<T>::get(srow + j), t = Elt<T>::get(trow + j);
          Elt<T>::put(grow + j, ex2(fmaf(s, kL2E, off)) * ((s - t) - ep));
        }
        for (int j = tail0 + tid; j < n; j += kThreads) {
          const float s = Elt<T>::get(srow + j), t = Elt<T>::get(trow + j);
          Elt<T>::put(grow + j, ex2(fmaf(s, kL2E, off)) * ((s - t) - ep));
        }
        // Vectors in blocks of kU * kThreads, last block first: pass 1 streamed the
        // slice forwards, so its most recently read part is the likeliest L2 hit.
        uint4* gv = reinterpret_cast<uint4*>(grow + head);
        const unsigned long long pl_first = policy_evict_first();
        const float2 l2e = make_float2(kL2E, kL2E), off2 = make_float2(off, off), nep = make_float2(-ep, -ep);
        const int nblk = (nvec + kU * kThreads - 1) / (kU * kThreads);
        for (int b = nblk - 1; b >= 0; --b) {
          const int j0 = b * kU * kThreads + tid;
          uint4 us[kU], ut[kU];
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int j = j0 + u * kThreads;
            if (j < nvec) {
              us[u] = ld16_hint(sv + j * kE, pl_first);
              ut[u] = ld16_hint(tv + j * kE, pl_first);
            }
          }
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int j = j0 + u * kThreads;
            if (j < nvec) {
              float2 ps[kP], pt[kP], g[kP];
              unpack<T>(us[u], ps);
              unpack<T>(ut[u], pt);
#pragma unroll
              for (int k = 0; k < kP; ++k) {
                const float2 x = __ffma2_rn(ps[k], l2e, off2);
                const float2 p = make_float2(ex2(x.x), ex2(x.y));
                const float2 w = __fadd2_rn(__ffma2_rn(pt[k], make_float2(-1.f, -1.f), ps[k]), nep);
                g[k] = __fmul2_rn(p, w);
              }
              st16_hint(gv + j, pack<T>(g), pl_first);
            }
          }
        }
      }
      // The statistics buffers are rewritten by the next row.
      __syncthreads();
    }
  }
  // Peers may still read this CTA's exchange slots.
  if (a.cl > 1) cluster_sync();

  // ---- loss: cluster partials, summed in cluster order by the last cluster ----
  if (crank == 0 && warp == 0) {
    double* partials = reinterpret_cast<double*>(a.ws + kWsHeader);
    unsigned* done = reinterpret_cast<unsigned*>(a.ws + 8);
    unsigned prev = 0;
    if (lane == 0) {
      partials[cid] = s_part;
      __threadfence();
      prev = atomicAdd(done, 1u);
    }
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev == ncl - 1) {
      __threadfence();
      double sum = 0.0;
      for (unsigned j = lane; j < ncl; j += 32) sum += *reinterpret_cast<volatile double*>(partials + j);
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) sum += __shfl_down_sync(0xffffffffu, sum, d);
      if (lane == 0) {
        *a.loss_out = (float)(sum / (double)(n_valid > 1 ? n_valid : 1));
        if (a.n_valid_out) *a.n_valid_out = n_valid;
        *done = 0u;
      }
    }
  }
}

// ---------------------------------------------------------------- register-resident gradient form
// The forward + gradient call for 16-bit logits whose rows are 16-byte
// aligned.  A row's slice is read from HBM once: 1-D bulk copies bring it into
// shared-memory slots of 8 KB per tensor, pass 1 moves each slot into the
// registers of the 512 compute threads (one 16-byte vector of each tensor per
// thread and slot) while it accumulates the statistics, and releases the slot
// at once, so a producer warp fetches the next row's slice while this row is
// reduced, merged across the cluster and turned into its gradient.  Pass 2
// reads nothing from memory: the gradient comes from the registers.  The
// cluster merge exchanges the CTAs' statistics through distributed shared
// memory with release/acquire mbarrier arrivals (every wait bounded), in rank
// order as in reverse_kl_kernel.
constexpr int kResThreads = 512;             // compute threads
constexpr int kResWarps = kResThreads / 32;
constexpr int kResBlock = kResThreads + 32;  // + one producer warp
constexpr int kResSlots = 8;                 // slots per CTA slice
constexpr int kResSlotBytes = 8192;          // per tensor and slot: 512 threads x 16 bytes

__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kResThreads) : "memory"); }
__device__ __forceinline__ uint4 ld_shared16(uint32_t saddr) {
  uint4 u;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "r"(saddr));
  return u;
}
__device__ __forceinline__ void st_cluster_f32(uint32_t cluster_addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_addr), "f"(v) : "memory");
}
// Bounded wait on a barrier other CTAs of the cluster arrive on (acquire at cluster scope).
__device__ __forceinline__ bool xwait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                      unsigned long long limit) {
  if (sm100::mbar_try_wait_cluster(bar, parity)) return true;
  const unsigned long long t0 = sm100::globaltimer();
  while (!*abort) {
    if (sm100::mbar_try_wait_cluster(bar, parity)) return true;
    if (sm100::globaltimer() - t0 > limit) {
      *abort = 1;
      return false;
    }
  }
  return false;
}

template <typename T>
__global__ void __launch_bounds__(kResBlock, 1) reverse_kl_resident_kernel(RklArgs a) {
  static_assert(sizeof(T) == 2, "16-bit logits");
  constexpr int kP = Elt<T>::kPairs;
  constexpr int kE = 2 * kP;                      // elements per 16-byte vector
  constexpr int kSub = kResSlotBytes / (int)sizeof(T);
  extern __shared__ __align__(128) unsigned char ring[];   // [slot][tensor][kResSlotBytes]
  __shared__ uint64_t full[kResSlots], empty[kResSlots], xbar[2];
  __shared__ Stats warp_stats[kResWarps];
  __shared__ float xch[2][kMaxCluster][5];        // every CTA's statistics, by row parity
  __shared__ unsigned long long s_count;
  __shared__ double s_part;
  __shared__ int s_abort;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned crank = cluster_rank(), cid = cluster_id(), ncl = cluster_count();
  const int cl = a.cl;
  if (tid == 0) {
    s_count = 0;
    s_part = 0.0;
    s_abort = 0;
    for (int j = 0; j < kResSlots; ++j) {
      sm100::mbar_init(&full[j], 1);
      sm100::mbar_init(&empty[j], kResWarps);   // one arrival per compute warp
    }
    sm100::mbar_init(&xbar[0], cl);
    sm100::mbar_init(&xbar[1], cl);
    sm100::fence_barrier_init();
  }
  __syncthreads();
  cluster_sync();   // every CTA's barriers exist before any remote arrival

  // ---- valid rows (every CTA counts the whole mask) ----
  int64_t n_valid = a.N;
  if (a.mask) {
    if (tid < kResThreads) {
      const uint8_t* m = a.mask;
      const int64_t head = imin(a.N, (int64_t)((16 - (reinterpret_cast<uintptr_t>(m) & 15)) & 15));
      const int64_t nv16 = (a.N - head) / 16;
      unsigned long long c = 0;
      for (int64_t i = tid; i < head; i += kResThreads) c += m[i] != 0;
      const uint4* m16 = reinterpret_cast<const uint4*>(m + head);
      for (int64_t i = tid; i < nv16; i += kResThreads) {
        const uint4 u = __ldg(m16 + i);
        c += nonzero_bytes(u.x) + nonzero_bytes(u.y) + nonzero_bytes(u.z) + nonzero_bytes(u.w);
      }
      for (int64_t i = head + nv16 * 16 + tid; i < a.N; i += kResThreads) c += m[i] != 0;
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) c += __shfl_down_sync(0xffffffffu, c, d);
      if (lane == 0 && c) atomicAdd(&s_count, c);
    }
    __syncthreads();
    n_valid = (int64_t)s_count;
  }
  const float log2_scale = -log2f((float)(n_valid > 1 ? n_valid : 1));

  const int64_t v0 = imin(a.V, (int64_t)crank * a.slice);
  const int64_t v1 = imin(a.V, v0 + a.slice);
  const int n = (int)(v1 - v0);                   // multiple of 8 (the host checks V and slice)
  const int nslot = (n + kSub - 1) / kSub;        // <= kResSlots (the host picks the cluster size)
  volatile int* abort = &s_abort;

  if (warp == kResWarps) {
    // ---------------- producer: the slices of this cluster's valid rows, in row order ----------------
    if (lane == 0) {
      const unsigned long long pol = policy_evict_first();
      uint32_t eph = 0;
      for (int64_t r = cid; r < a.N && !*abort; r += ncl) {
        if (a.mask && a.mask[r] == 0) continue;
        const T* srow = static_cast<const T*>(a.s) + r * a.V + v0;
        const T* trow = static_cast<const T*>(a.t) + r * a.V + v0;
        for (int j = 0; j < nslot; ++j) {
          // the consumers have moved this slot's previous row into registers
          if (!sm100::mbar_wait(&empty[j], ((eph >> j) & 1u) ^ 1u, abort, a.wait_ns)) break;
          eph ^= 1u << j;
          const uint32_t bytes = (uint32_t)min(kSub, n - j * kSub) * (uint32_t)sizeof(T);
          unsigned char* dst = ring + (size_t)j * 2 * kResSlotBytes;
          sm100::mbar_arrive_expect_tx(&full[j], 2 * bytes + a.extra_tx);
          sm100::bulk_load_1d(dst, srow + j * kSub, bytes, &full[j], pol);
          sm100::bulk_load_1d(dst + kResSlotBytes, trow + j * kSub, bytes, &full[j], pol);
        }
      }
      if (*abort) {
        // leave time for copies already issued to land before shared memory is released
        const unsigned long long t0 = sm100::globaltimer();
        while (sm100::globaltimer() - t0 < 100000ull) __nanosleep(1000);
      }
    }
  } else {
    // ---------------- compute threads ----------------
    uint32_t fph = 0, xph = 0;
    int parity = 0;
    uint4 sr[kResSlots], tr[kResSlots];
    const uint32_t ring_u32 = sm100::smem_u32(ring);
    const unsigned long long pl_first = policy_evict_first();
    for (int64_t r = cid; r < a.N; r += ncl) {
      T* grow = static_cast<T*>(a.grad) + r * a.V + v0;
      if (a.mask && a.mask[r] == 0) {
        // a masked row is not read; its gradient slice is zero
#pragma unroll
        for (int j = 0; j < kResSlots; ++j) {
          const int nv = j < nslot ? min(kSub, n - j * kSub) / kE : 0;
          if (tid < nv) st16_hint(reinterpret_cast<uint4*>(grow + j * kSub) + tid, make_uint4(0, 0, 0, 0), pl_first);
        }
        if (a.kl_rows && crank == 0 && tid == 0) a.kl_rows[r] = 0.0f;
        continue;
      }

      // ---- pass 1: each slot into registers, online statistics ----
      Acc acc;
#pragma unroll
      for (int j = 0; j < kResSlots; ++j) {
        if (j < nslot) {
          const int nv = min(kSub, n - j * kSub) / kE;
          const bool ok = !*abort && sm100::mbar_wait(&full[j], (fph >> j) & 1u, abort, a.wait_ns);
          fph ^= 1u << j;
          if (ok && tid < nv) {
            const uint32_t base = ring_u32 + (uint32_t)(j * 2 * kResSlotBytes) + (uint32_t)tid * 16u;
            sr[j] = ld_shared16(base);
            tr[j] = ld_shared16(base + kResSlotBytes);
          }
          __syncwarp();
          if (lane == 0) sm100::mbar_arrive(&empty[j]);   // the warp is done with the slot
          if (ok && tid < nv) {
            float2 ps[kP], pt[kP];
            unpack<T>(sr[j], ps);
            unpack<T>(tr[j], pt);
            float bs = -INFINITY, bt = -INFINITY;
#pragma unroll
            for (int k = 0; k < kP; ++k) {
              bs = fmaxf(bs, fmaxf(ps[k].x, ps[k].y));
              bt = fmaxf(bt, fmaxf(pt[k].x, pt[k].y));
            }
            acc.raise_max(bs, bt);
            const float2 nmsl = make_float2(-acc.ms * kL2E, -acc.ms * kL2E);
            const float2 nmtl = make_float2(-acc.mt * kL2E, -acc.mt * kL2E);
#pragma unroll
            for (int k = 0; k < kP; ++k) acc.add(ps[k], pt[k], nmsl, nmtl);
          }
        }
      }

      // ---- reduce: warp, then warps in order, then every CTA of the cluster in rank order ----
      Stats st = acc.stats();
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) st = merge(st, shfl_down(st, d));
      if (lane == 0) warp_stats[warp] = st;
      consumers_sync();
      if (warp == 0) {
        st = lane < kResWarps ? warp_stats[lane] : Stats{-INFINITY, 0.f, 0.f, -INFINITY, 0.f};
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) st = merge(st, shfl_down(st, d));
        // lane k < cl writes this CTA's statistics into slot [parity][crank] of CTA k
        // of the cluster and arrives on its exchange barrier (release at cluster scope)
        const float v[5] = {__shfl_sync(0xffffffffu, st.ms, 0), __shfl_sync(0xffffffffu, st.zs, 0),
                            __shfl_sync(0xffffffffu, st.a, 0), __shfl_sync(0xffffffffu, st.mt, 0),
                            __shfl_sync(0xffffffffu, st.zt, 0)};
        if (lane < cl) {
          const uint32_t dst = sm100::mapa_shared(sm100::smem_u32(&xch[parity][crank][0]), (uint32_t)lane);
#pragma unroll
          for (int q = 0; q < 5; ++q) st_cluster_f32(dst + 4u * q, v[q]);
          sm100::mbar_arrive_cluster(sm100::mapa_shared(sm100::smem_u32(&xbar[parity]), (uint32_t)lane));
        }
      }
      // every CTA's statistics for this row have arrived
      xwait(&xbar[parity], (xph >> parity) & 1u, abort, a.wait_ns);
      xph ^= 1u << parity;
      Stats rs{xch[parity][0][0], xch[parity][0][1], xch[parity][0][2], xch[parity][0][3], xch[parity][0][4]};
      for (int k = 1; k < cl; ++k)
        rs = merge(rs, Stats{xch[parity][k][0], xch[parity][k][1], xch[parity][k][2], xch[parity][k][3],
                             xch[parity][k][4]});
      parity ^= 1;
      const float ep = rs.a / rs.zs;                                      // E_p[s - t]
      const float kl = ep - ((rs.ms - rs.mt) + logf(rs.zs / rs.zt));      // minus (lse_s - lse_t)
      if (crank == 0 && tid == 0) {
        s_part += (double)kl;
        if (a.kl_rows) a.kl_rows[r] = kl;
      }

      // ---- pass 2: grad_v = scale * p_v * ((s_v - t_v) - E_p[s - t]) from the registers ----
      const float off = -(rs.ms * kL2E + log2f(rs.zs)) + log2_scale;
      const float2 l2e = make_float2(kL2E, kL2E), off2 = make_float2(off, off), nep = make_float2(-ep, -ep);
#pragma unroll
      for (int j = 0; j < kResSlots; ++j) {
        const int nv = j < nslot ? min(kSub, n - j * kSub) / kE : 0;
        if (tid < nv) {
          float2 ps[kP], pt[kP], g[kP];
          unpack<T>(sr[j], ps);
          unpack<T>(tr[j], pt);
#pragma unroll
          for (int k = 0; k < kP; ++k) {
            const float2 x = __ffma2_rn(ps[k], l2e, off2);
            const float2 p = make_float2(ex2(x.x), ex2(x.y));
            const float2 w = __fadd2_rn(__ffma2_rn(pt[k], make_float2(-1.f, -1.f), ps[k]), nep);
            g[k] = __fmul2_rn(p, w);
          }
          st16_hint(reinterpret_cast<uint4*>(grow + j * kSub) + tid, pack<T>(g), pl_first);
        }
      }
    }
  }
  __syncthreads();
  cluster_sync();   // no CTA leaves while a peer may still write into its exchange slots

  // ---- loss: cluster partials, summed in cluster order by the last cluster ----
  if (crank == 0 && warp == 0) {
    double* partials = reinterpret_cast<double*>(a.ws + kWsHeader);
    unsigned* done = reinterpret_cast<unsigned*>(a.ws + 8);
    unsigned prev = 0;
    if (lane == 0) {
      partials[cid] = s_part;
      __threadfence();
      prev = atomicAdd(done, 1u);
    }
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev == ncl - 1) {
      __threadfence();
      double sum = 0.0;
      for (unsigned j = lane; j < ncl; j += 32) sum += *reinterpret_cast<volatile double*>(partials + j);
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) sum += __shfl_down_sync(0xffffffffu, sum, d);
      if (lane == 0) {
        *a.loss_out = (float)(sum / (double)(n_valid > 1 ? n_valid : 1));
        if (a.n_valid_out) *a.n_valid_out = n_valid;
        *done = 0u;
      }
    }
  }
  if (tid == 0 && *abort) atomicOr(reinterpret_cast<unsigned*>(a.ws), kDevErrTimeout);
}

template <typename T>
size_t resident_smem(int nslot) { return (size_t)nslot * 2 * kResSlotBytes; }

template <typename T>
cudaError_t launch_resident_t(const RklArgs& a, unsigned nclusters, int nslot, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)a.cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(nclusters * (unsigned)a.cl);
  cfg.blockDim = dim3(kResBlock);
  cfg.dynamicSmemBytes = resident_smem<T>(nslot);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, reverse_kl_resident_kernel<T>, a);
}

// Resident clusters of the register-resident kernel at `cl` CTAs with `nslot` slots.
template <typename T>
int max_resident_clusters_t(int cl, int nslot) {
  static std::mutex mu;
  static int cache[16][4][kResSlots + 1] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return 0;
  const int ci = cl == 1 ? 0 : cl == 2 ? 1 : cl == 4 ? 2 : 3;
  std::lock_guard<std::mutex> lk(mu);
  int& slot = cache[dev][ci][nslot];
  if (slot == 0) {
    const size_t smem = resident_smem<T>(nslot);
    if (cudaFuncSetAttribute(reverse_kl_resident_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(kResSlots * 2 * kResSlotBytes)) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)cl * 64);
    cfg.blockDim = dim3(kResBlock);
    cfg.dynamicSmemBytes = smem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nc = 0;
    if (cudaOccupancyMaxActiveClusters(&nc, reverse_kl_resident_kernel<T>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    slot = nc > 0 ? nc : -1;
  }
  return slot > 0 ? slot : 0;
}

template <typename T, bool GRAD>
cudaError_t launch_t(const RklArgs& a, unsigned nclusters, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)a.cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(nclusters * (unsigned)a.cl);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, reverse_kl_kernel<T, GRAD>, a);
}

template <typename T, bool GRAD>
int max_clusters_t(int cl) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)cl * 64);
  cfg.blockDim = dim3(kThreads);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, reverse_kl_kernel<T, GRAD>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

// Resident clusters per (dtype, grad, cluster size), per device.
int max_clusters(DType dt, bool grad, int cl) {
  static std::mutex mu;
  static int cache[16][3][2][4] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return 0;
  const int ci = cl == 1 ? 0 : cl == 2 ? 1 : cl == 4 ? 2 : 3;
  std::lock_guard<std::mutex> lk(mu);
  int& slot = cache[dev][(int)dt][grad ? 1 : 0][ci];
  if (slot == 0) {
    int v = 0;
    switch ((int)dt * 2 + (grad ? 1 : 0)) {
      case 0: v = max_clusters_t<float, false>(cl); break;
      case 1: v = max_clusters_t<float, true>(cl); break;
      case 2: v = max_clusters_t<__half, false>(cl); break;
      case 3: v = max_clusters_t<__half, true>(cl); break;
      case 4: v = max_clusters_t<__nv_bfloat16, false>(cl); break;
      default: v = max_clusters_t<__nv_bfloat16, true>(cl); break;
    }
    slot = v;
  }
  return slot;
}

}  // namespace

size_t reverse_kl_ws_bytes() { return kWsHeader + (size_t)kMaxClusters * 8; }

}  // namespace pl

using namespace pl;

extern "C" size_t pl_reverse_kl_workspace_bytes(int64_t N, int64_t V) {
  (void)N;
  (void)V;
  return reverse_kl_ws_bytes();
}

extern "C" pl_status pl_reverse_kl(const void* student, const void* teacher, const uint8_t* mask, int64_t N,
                                   int64_t V, uint32_t mode, float* loss_out, void* grad_out,
                                   float* kl_rows_out, int64_t* n_valid_out, void* workspace, size_t ws_bytes,
                                   pl_stream_t stream) {
  if (!loss_out || N < 0 || V < 1 || V > INT32_MAX || (N > 0 && (!student || !teacher))) return PL_ERR_ARG;
  if (mode & ~PL_DTYPE_MASK) return PL_ERR_ARG;
  const uint32_t d = (mode & PL_DTYPE_MASK) >> 4;
  if (d > 2) return PL_ERR_DTYPE;
  const DType dt = static_cast<DType>(d);
  const size_t esz = dtype_size(dt);
  const uintptr_t ps = reinterpret_cast<uintptr_t>(student), pt = reinterpret_cast<uintptr_t>(teacher),
                  pg = reinterpret_cast<uintptr_t>(grad_out);
  if ((ps | pt | pg) % esz) return PL_ERR_ALIGN;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255)) return PL_ERR_ALIGN;
  if (workspace && ws_bytes < reverse_kl_ws_bytes()) return PL_ERR_WORKSPACE;
  pl_status st = check_arch();
  if (st != PL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* ws = workspace;
  if (!ws && (st = own_workspace(s, reverse_kl_ws_bytes(), &ws, true)) != PL_OK) return st;

  DevInfo di;
  if (dev_info(&di) != cudaSuccess) return PL_ERR_CUDA;

  // The register-resident form for the gradient of 16-bit logits whose rows
  // start on 16-byte boundaries (the smallest cluster whose slices fit the
  // shared-memory slots), on request: measured at the card's shape it was
  // slower than the streaming kernel (517 against 336 us).
  const int path = debug_knobs().rkl_path;
  if (grad_out && dt != DType::F32 && V % 8 == 0 && ((ps | pt | pg) & 15) == 0 && path == 2) {
    constexpr int64_t kSub = kResSlotBytes / 2;
    int rc_cl = 0, nslot = 0, mc = 0;
    const int forced_cl = debug_knobs().rkl_cluster;
    for (int c = forced_cl ? forced_cl : 1; c <= kMaxCluster; c *= 2) {
      const int64_t sl = ((V + c - 1) / c + 7) / 8 * 8;
      const int ns = (int)((sl + kSub - 1) / kSub);
      if (ns <= kResSlots) {
        mc = dt == DType::BF16 ? max_resident_clusters_t<__nv_bfloat16>(c, ns)
                               : max_resident_clusters_t<__half>(c, ns);
        if (mc > 0) {
          rc_cl = c;
          nslot = ns;
          break;
        }
      }
      if (forced_cl) break;
    }
    if (rc_cl > 0) {
      RklArgs a{};
      a.s = student;
      a.t = teacher;
      a.mask = mask;
      a.grad = grad_out;
      a.loss_out = loss_out;
      a.kl_rows = kl_rows_out;
      a.n_valid_out = n_valid_out;
      a.ws = static_cast<unsigned char*>(ws);
      a.N = N;
      a.V = V;
      a.slice = ((V + rc_cl - 1) / rc_cl + 7) / 8 * 8;
      a.cl = rc_cl;
      a.vec = 1;
      a.wait_ns = debug_knobs().wait_ns;
      a.extra_tx = debug_knobs().extra_tx;
      const int64_t want = N > 0 ? N : 1;
      const unsigned ncl = (unsigned)std::min<int64_t>(std::min<int64_t>(want, mc), kMaxClusters);
      launch_begin(2, s);
      const cudaError_t e = dt == DType::BF16 ? launch_resident_t<__nv_bfloat16>(a, ncl, nslot, s)
                                              : launch_resident_t<__half>(a, ncl, nslot, s);
      launch_end(2, s);
      return e == cudaSuccess ? PL_OK : PL_ERR_CUDA;
    }
  }
  int l2 = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess)
    return PL_ERR_CUDA;
  const bool grad = grad_out != nullptr;

  // Cluster size: the smallest that (a) keeps the re-read slices of all
  // resident CTAs within 1.25 x L2 (gradient only) and (b) gives every
  // resident CTA a row slice.  Pass 2 walks its slice backwards, most recently
  // read first, so slices a little beyond L2 still mostly hit; a smaller
  // cluster saves merges (measured: 2-3% faster at 1.1-1.2 x L2 than the next
  // larger cluster within L2).
  int cl = 1, resident = 0;
  int64_t slice = 0;
  const int forced = debug_knobs().rkl_cluster;
  for (int c = forced ? forced : 1; c <= kMaxCluster; c *= 2) {
    const int mc = max_clusters(dt, grad, c);
    if (mc <= 0) continue;
    cl = c;
    resident = mc;
    slice = ((V + c - 1) / c + 7) / 8 * 8;
    const double inflight = (double)mc * c * (double)slice * 2.0 * (double)esz;
    const bool fits = !grad || inflight <= 1.25 * (double)l2;
    const bool fills = N * c >= (int64_t)mc * c;
    if (forced || (fits && fills)) break;
  }
  if (resident <= 0) return PL_ERR_CUDA;
  const int64_t want = N > 0 ? N : 1;
  const unsigned ncl = (unsigned)std::min<int64_t>(std::min<int64_t>(want, resident), kMaxClusters);

  RklArgs a{};
  a.s = student;
  a.t = teacher;
  a.mask = mask;
  a.grad = grad_out;
  a.loss_out = loss_out;
  a.kl_rows = kl_rows_out;
  a.n_valid_out = n_valid_out;
  a.ws = static_cast<unsigned char*>(ws);
  a.N = N;
  a.V = V;
  a.slice = slice;
  a.cl = cl;
  a.vec = ((ps & 15) == (pt & 15)) && (!grad || (pg & 15) == (ps & 15));

  launch_begin(2, s);
  cudaError_t e;
  switch ((int)dt * 2 + (grad ? 1 : 0)) {
    case 0: e = launch_t<float, false>(a, ncl, s); break;
    case 1: e = launch_t<float, true>(a, ncl, s); break;
    case 2: e = launch_t<__half, false>(a, ncl, s); break;
    case 3: e = launch_t<__half, true>(a, ncl, s); break;
    case 4: e = launch_t<__nv_bfloat16, false>(a, ncl, s); break;
    default: e = launch_t<__nv_bfloat16, true>(a, ncl, s); break;
  }
  launch_end(2, s);
  return e == cudaSuccess ? PL_OK : PL_ERR_CUDA;
}
