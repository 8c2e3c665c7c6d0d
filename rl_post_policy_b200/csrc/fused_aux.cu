// Memory-bound kernels of the fused linear path (everything except the GEMMs).
//
//   count_kernel    -- exact per-sequence and global valid-token counts (mask != 0),
//                      needed before any gradient can be scaled ("Geometric-AI
//                      Kernels" model card: the denominators are computed on the GPU).
//   combine_kernel  -- per row: logsumexp from the per-tile (max, sum exp) partials
//                      of the GEMM epilogue, logp = z[target] - lse for the policy
//                      and the reference model, then the clipped-ratio loss with
//                      the KL term, g = dLoss/dlogp and the chunk's loss partials.
//   dlogits_kernel  -- in place over the chunk's logits workspace:
//                      dz = g * (onehot(target) - exp(z - lse)) * 2^e, stored in the
//                      model dtype (2^e keeps fp16 dz in range; bf16 chunks paired
//                      into one dW job take e = 0), and the column sums of dz (the bias gradient),
//                      stored / accumulated in fp32 / converted like dW.
//   finalize_kernel -- fixed-order sum of every chunk's loss partials.
//   convert_kernel  -- the fp32 dW accumulator of a multi-chunk call, rounded
//                      once to the model dtype after the last chunk's add.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fused.h"
#include "gemm.h"
#include "policy_math.cuh"
#include "sm100.cuh"

namespace pl {
namespace {

__device__ __forceinline__ float cvt(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float cvt(__half x) { return __half2float(x); }
template <typename T> __device__ __forceinline__ T to_t(float x);
template <> __device__ __forceinline__ __nv_bfloat16 to_t<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
template <> __device__ __forceinline__ __half to_t<__half>(float x) { return __float2half_rn(x); }
template <typename T> __device__ __forceinline__ float2 unpack2(uint32_t u);
template <> __device__ __forceinline__ float2 unpack2<__nv_bfloat16>(uint32_t u) {
  // a bf16 is the high half of the fp32 with the same value
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
template <> __device__ __forceinline__ float2 unpack2<__half>(uint32_t u) {
  __half2 h;
  *reinterpret_cast<uint32_t*>(&h) = u;
  return __half22float2(h);
}
template <typename T> __device__ __forceinline__ uint32_t pack_t(float a, float b);
template <> __device__ __forceinline__ uint32_t pack_t<__nv_bfloat16>(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
template <> __device__ __forceinline__ uint32_t pack_t<__half>(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// ---------------------------------------------------------------- counts
__global__ void count_kernel(const uint8_t* __restrict__ mask, int64_t bs, int64_t T,
                             unsigned char* ws, int nchunks, const FusedOffsets off) {
  unsigned* done = reinterpret_cast<unsigned*>(ws + 8);
  unsigned long long* nvalid = reinterpret_cast<unsigned long long*>(ws + 16);
  unsigned long long* rowcnt = reinterpret_cast<unsigned long long*>(ws + off.row_cnt);
  unsigned* gmax = reinterpret_cast<unsigned*>(ws + off.gmax);
  __shared__ unsigned long long s_cnt[8];
  __shared__ int s_last;
  const int64_t b = blockIdx.x;
  if (b == 0)
    for (int c = threadIdx.x; c < nchunks; c += blockDim.x) gmax[c] = 0u;
  unsigned long long c = 0;
  const uint8_t* m = mask + b * T;
  for (int64_t t = threadIdx.x; t < T; t += blockDim.x) c += m[t] != 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) s_cnt[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long s = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += s_cnt[w];
    rowcnt[b] = s;
    __threadfence();
    s_last = atomicAdd(done, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (s_last && threadIdx.x == 0) {
    __threadfence();
    unsigned long long s = 0;
    for (int64_t r = 0; r < bs; ++r) s += __ldcg(&rowcnt[r]);
    *nvalid = s;
    *done = 0u;
  }
}

// ---------------------------------------------------------------- combine
template <bool HAS_KL, bool TWO_SIDED>
__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a) {
  __shared__ double s_part[8];
  __shared__ float s_gmax[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t i = (int64_t)blockIdx.x * 8 + warp;  // row within the chunk
  float contrib = 0.0f, gabs = 0.0f;
  if (i < a.rows) {
    const int64_t g = a.row0 + i;
    const unsigned char* ws = a.ws;
    const float2* part = reinterpret_cast<const float2*>(ws + a.off.part) + i * a.nparts;
    const float* zt = reinterpret_cast<const float*>(ws + a.off.zt);
    // logsumexp over the vocabulary tiles: lse = M + log(sum_j s_j exp(m_j - M))
    float M = -INFINITY;
    for (int j = lane; j < a.nparts; j += 32) M = fmaxf(M, part[j].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float S = 0.0f;
    for (int j = lane; j < a.nparts; j += 32) S += part[j].y * expf(part[j].x - M);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
    const float lse = M + logf(S);
    float ref_lp = 0.0f;
    if (HAS_KL) {
      const float2* pr = reinterpret_cast<const float2*>(ws + a.off.part_ref) + i * a.nparts;
      float Mr = -INFINITY;
      for (int j = lane; j < a.nparts; j += 32) Mr = fmaxf(Mr, pr[j].x);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) Mr = fmaxf(Mr, __shfl_xor_sync(0xffffffffu, Mr, o));
      float Sr = 0.0f;
      for (int j = lane; j < a.nparts; j += 32) Sr += pr[j].y * expf(pr[j].x - Mr);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) Sr += __shfl_xor_sync(0xffffffffu, Sr, o);
      const float* ztr = reinterpret_cast<const float*>(ws + a.off.zt_ref);
      ref_lp = ztr[i] - (Mr + logf(Sr));
    }
    if (lane == 0) {
      const int64_t tgt = a.targets[g];
      const bool tvalid = tgt >= 0 && tgt < a.V;
      if (!tvalid) atomicOr(reinterpret_cast<unsigned*>(a.ws), kDevErrTarget);
      const float logp = tvalid ? zt[i] - lse : __int_as_float(0x7fc00000);
      const int64_t b = g / a.T;
      const bool valid = tvalid && a.mask[g] != 0;
      const float A = a.adv_lp_dtype ? (a.bf16 ? cvt(reinterpret_cast<const __nv_bfloat16*>(a.adv)[b])
                                               : cvt(reinterpret_cast<const __half*>(a.adv)[b]))
                                     : reinterpret_cast<const float*>(a.adv)[b];
      float scale;
      if (a.grpo) {
        const unsigned long long c = reinterpret_cast<const unsigned long long*>(ws + a.off.row_cnt)[b];
        scale = (float)(1.0 / ((double)a.bs * (double)(c > 0 ? c : 1)));
      } else {
        const unsigned long long c = *reinterpret_cast<const unsigned long long*>(ws + 16);
        scale = (float)(1.0 / (double)(c > 0 ? c : 1));
      }
      float term = 0.0f, dterm = 0.0f;
      if (valid)
        token_math<HAS_KL, TWO_SIDED>(logp, a.old_lp[g], ref_lp, A, a.lo, a.hi, a.beta, term, dterm);
      const float gv = valid ? dterm * scale * a.g_scale : 0.0f;
      contrib = valid ? term * scale : 0.0f;
      gabs = fabsf(gv);
      reinterpret_cast<float*>(a.ws + a.off.g)[i] = gv;
      reinterpret_cast<float*>(a.ws + a.off.lse)[i] = lse;
      if (a.logp_out) a.logp_out[g] = logp;
      if (HAS_KL && a.ref_logp_out) a.ref_logp_out[g] = tvalid ? ref_lp : __int_as_float(0x7fc00000);
    }
  }
  if (lane == 0) {
    s_part[warp] = (double)contrib;
    s_gmax[warp] = gabs;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    float gm = 0.0f;
    for (int w = 0; w < 8; ++w) {
      s += s_part[w];
      gm = fmaxf(gm, s_gmax[w]);
    }
    reinterpret_cast<double*>(a.ws + a.off.loss_part)[(int64_t)a.chunk * a.part_stride + blockIdx.x] = s;
    if (gm > 0.0f) atomicMax(reinterpret_cast<unsigned*>(a.ws + a.off.gmax) + a.chunk, __float_as_uint(gm));
  }
}

// ---------------------------------------------------------------- combine (selective log-prob form)
// One warp per row: lse from the vocabulary-tile partials, logp = z[target] - lse,
// and g_i = grad_logp[i] supplied by the caller (the backward of the selective
// log-prob, "Add SM100 CuTe DSL GRPO fast path": the fused-linear selective-logprob
// autograd path receives the upstream gradient of the log-probs).
__global__ void __launch_bounds__(256) combine_ext_kernel(CombineArgs a) {
  __shared__ float s_gmax[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t i = (int64_t)blockIdx.x * 8 + warp;
  float gabs = 0.0f;
  if (i < a.rows) {
    const int64_t g = a.row0 + i;
    const float2* part = reinterpret_cast<const float2*>(a.ws + a.off.part) + i * a.nparts;
    float M = -INFINITY;
    for (int j = lane; j < a.nparts; j += 32) M = fmaxf(M, part[j].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float S = 0.0f;
    for (int j = lane; j < a.nparts; j += 32) S += part[j].y * expf(part[j].x - M);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
    if (lane == 0) {
      const float lse = M + logf(S);
      const int64_t tgt = a.targets[g];
      const bool tvalid = tgt >= 0 && tgt < a.V;
      if (!tvalid) atomicOr(reinterpret_cast<unsigned*>(a.ws), kDevErrTarget);
      const float zt = reinterpret_cast<const float*>(a.ws + a.off.zt)[i];
      const float gv = (tvalid && a.grad_logp) ? a.grad_logp[g] * a.g_scale : 0.0f;
      gabs = fabsf(gv);
      reinterpret_cast<float*>(a.ws + a.off.g)[i] = gv;
      reinterpret_cast<float*>(a.ws + a.off.lse)[i] = lse;
      if (a.logp_out) a.logp_out[g] = tvalid ? zt - lse : __int_as_float(0x7fc00000);
    }
  }
  if (lane == 0) s_gmax[warp] = gabs;
  __syncthreads();
  if (threadIdx.x == 0) {
    float gm = 0.0f;
    for (int w = 0; w < 8; ++w) gm = fmaxf(gm, s_gmax[w]);
    if (gm > 0.0f) atomicMax(reinterpret_cast<unsigned*>(a.ws + a.off.gmax) + a.chunk, __float_as_uint(gm));
  }
}

__global__ void clear_gmax_kernel(unsigned char* ws, int nchunks, FusedOffsets off) {
  unsigned* gmax = reinterpret_cast<unsigned*>(ws + off.gmax);
  for (int c = threadIdx.x; c < nchunks; c += blockDim.x) gmax[c] = 0u;
}

// ---------------------------------------------------------------- dlogits
// Block = 256 threads = 8 warps over one 256-column strip (blockIdx.x) and one
// group of rows (blockIdx.y).  The group's rows stream through shared memory in
// tiles of 32 rows x 256 columns (16 KB of 16-bit logits): one thread issues the
// TMA loads of a kDlStages-deep ring up front, every thread turns its part of a
// landed tile into dz in place (lane l: columns [8l, 8l+8); warp w: rows w,
// w+8, w+16, w+24), and the tile goes back to the same global rows by TMA
// store, after which its slot takes the tile kDlStages further on.  The copies
// need no registers, so a block keeps up to 64 KB of loads in flight.  Rows
// past the chunk and columns past V are zero-filled on load and dropped on
// store.  The bias gradient: each block writes its strip's column sums for its
// row group; the strip's last block to finish adds the row groups in order
// (deterministic) and stores / accumulates them.
constexpr int kDlStages = 4;

template <typename T>
__global__ void __launch_bounds__(256, 3) dlogits_kernel(const __grid_constant__ DlogitsArgs a) {
  extern __shared__ __align__(128) uint8_t dl_ring[];  // kDlStages tiles of kDlTileBytes
  __shared__ uint64_t full[kDlStages];
  __shared__ float s_col[8][256];
  __shared__ int s_last;
  __shared__ int s_abort;
  const unsigned char* ws = a.ws;
  const float* row_lse = reinterpret_cast<const float*>(ws + a.off.lse);
  const float* row_g = reinterpret_cast<const float*>(ws + a.off.g);
  // power-of-two scale 2^e keeping max|dz| * 2^e <= 2^14 (fp16 range), exact to undo
  const float gm = __uint_as_float(reinterpret_cast<const unsigned*>(ws + a.off.gmax)[a.chunk]);
  int e = 0;
  if (gm > 0.0f && !a.unit_scale) {
    e = 14 - (int)ceilf(log2f(gm));
    e = max(-100, min(100, e));
  }
  const float sc = ldexpf(1.0f, e);
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
    reinterpret_cast<float*>(a.ws + a.off.inv_scale)[a.chunk] = ldexpf(1.0f, -e);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t col = (int64_t)blockIdx.x * 256 + lane * 8;
  const int32_t x0 = (int32_t)(blockIdx.x * 256);
  const int64_t r_begin = (int64_t)blockIdx.y * a.rg_rows;
  const int64_t r_end = min(a.rows, r_begin + a.rg_rows);
  const int ntiles = (int)((r_end - r_begin + kDlTileRows - 1) / kDlTileRows);
  const uint32_t ring = sm100::smem_u32(dl_ring);
  if (threadIdx.x == 0) {
    for (int st = 0; st < kDlStages; ++st) sm100::mbar_init(&full[st], 1);
    s_abort = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  int issued = 0;  // tiles whose load thread 0 has issued
  if (threadIdx.x == 0) {
    for (; issued < ntiles && issued < kDlStages; ++issued) {
      sm100::mbar_arrive_expect_tx(&full[issued], kDlTileBytes);
      sm100::tma_load_2d(dl_ring + issued * kDlTileBytes, &a.tmap, &full[issued], x0,
                         (int32_t)(r_begin + (int64_t)issued * kDlTileRows));
    }
  }
  float2 csum2[4];  // column sums of dz * 2^e (scaled back, exactly, at the end)
#pragma unroll
  for (int h = 0; h < 4; ++h) csum2[h] = make_float2(0.0f, 0.0f);
  constexpr float kLog2e = 1.4426950408889634f;
  // Per-row inputs of a tile (g, lse, target), loaded one tile ahead so that
  // their latency hides behind the previous tile's work.
  float gi[4], lsei[4];
  int ti[4];
  auto row_inputs = [&](int kt, float (&g4)[4], float (&l4)[4], int (&t4)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t i = r_begin + (int64_t)kt * kDlTileRows + warp + 8 * j;
      g4[j] = 0.0f; l4[j] = 0.0f; t4[j] = -1;
      if (i < r_end) {
        g4[j] = __ldg(row_g + i);
        l4[j] = __ldg(row_lse + i) * kLog2e;
        const int64_t tg = __ldg(a.targets + a.row0 + i);
        t4[j] = (tg >= 0 && tg < a.V) ? (int)tg : -1;
      }
    }
  };
  if (ntiles > 0) row_inputs(0, gi, lsei, ti);
  int k = 0;
  for (; k < ntiles; ++k) {
    const int slot = k % kDlStages;
    bool rv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) rv[j] = r_begin + (int64_t)k * kDlTileRows + warp + 8 * j < r_end;
    float gn[4], ln[4];
    int tn[4];
    if (k + 1 < ntiles) row_inputs(k + 1, gn, ln, tn);
    if (sm100::mbar_wait(&full[slot], (uint32_t)(k / kDlStages) & 1u, &s_abort, a.wait_ns)) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (!rv[j]) continue;
        uint4* p = reinterpret_cast<uint4*>(dl_ring + slot * kDlTileBytes + (warp + 8 * j) * 512 + lane * 16);
        const uint4 raw = *p;
        // dz * 2^e = -(g * 2^e) * p_v, plus g * 2^e at the target column; two
        // columns per packed fp32 instruction
        const float gs = gi[j] * sc;
        const float2 nl2 = make_float2(-lsei[j], -lsei[j]);
        const float2 ngs2 = make_float2(-gs, -gs);
        const float2 l2e2 = make_float2(kLog2e, kLog2e);
        const uint32_t r32[4] = {raw.x, raw.y, raw.z, raw.w};
        float2 ds[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float2 x = __ffma2_rn(unpack2<T>(r32[h]), l2e2, nl2);
          ds[h] = __fmul2_rn(make_float2(ex2_approx(x.x), ex2_approx(x.y)), ngs2);
        }
        const int rel = ti[j] - (int)col;  // the target's column within this thread's 8, if any
        if ((unsigned)rel < 8u) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            if (rel == 2 * h) ds[h].x += gs;
            if (rel == 2 * h + 1) ds[h].y += gs;
          }
        }
        uint4 w;
        uint32_t* w32 = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          csum2[h] = __fadd2_rn(csum2[h], ds[h]);
          w32[h] = pack_t<T>(ds[h].x, ds[h].y);
        }
        *p = w;
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      gi[j] = gn[j];
      lsei[j] = ln[j];
      ti[j] = tn[j];
    }
    sm100::fence_proxy_async_smem();  // the tile's generic writes before the TMA store reads them
    __syncthreads();
    if (s_abort) break;
    if (threadIdx.x == 0) {
      sm100::tma_store_2d(&a.tmap, ring + slot * kDlTileBytes, x0, (int32_t)(r_begin + (int64_t)k * kDlTileRows));
      sm100::bulk_commit_group();
      if (issued < ntiles) {
        // the slot is refilled once the store has read it out
        sm100::bulk_wait_group_read<0>();
        sm100::mbar_arrive_expect_tx(&full[slot], kDlTileBytes);
        sm100::tma_load_2d(dl_ring + slot * kDlTileBytes, &a.tmap, &full[slot], x0,
                           (int32_t)(r_begin + (int64_t)issued * kDlTileRows));
        ++issued;
      }
    }
  }
  if (threadIdx.x == 0) {
    sm100::bulk_wait_group_all();
    if (s_abort) {
      // let the loads already issued land (bounded) before the block's shared memory goes away
      volatile int no_abort = 0;
      for (int t = k; t < issued; ++t)
        sm100::mbar_wait(&full[t % kDlStages], (uint32_t)(t / kDlStages) & 1u, &no_abort, a.wait_ns);
      atomicOr(reinterpret_cast<unsigned*>(a.ws), kDevErrTimeout);
    }
  }
  if (s_abort) return;
  if (a.dbias_mode == kAccNone) return;
  const float inv_sc = ldexpf(1.0f, -e);
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    s_col[warp][lane * 8 + 2 * h] = csum2[h].x * inv_sc;
    s_col[warp][lane * 8 + 2 * h + 1] = csum2[h].y * inv_sc;
  }
  __syncthreads();
  const int64_t v = (int64_t)blockIdx.x * 256 + threadIdx.x;
  float s = 0.0f;
#pragma unroll
  for (int w = 0; w < 8; ++w) s += s_col[w][threadIdx.x];
  if (a.n_rg > 1) {
    // this row group's column sums; the strip's last block adds the groups in order
    if (v < a.V) a.db_part[(int64_t)blockIdx.y * a.V + v] = s;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(a.db_cnt + blockIdx.x, 1u) == (unsigned)a.n_rg - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    s = 0.0f;
    if (v < a.V)
      for (int r = 0; r < a.n_rg; ++r) s += __ldcg(a.db_part + (int64_t)r * a.V + v);
    if (threadIdx.x == 0) a.db_cnt[blockIdx.x] = 0u;
  }
  if (v < a.V) {
    float* acc = a.dbias_acc;
    T* out = reinterpret_cast<T*>(a.dbias);
    switch (a.dbias_mode) {
      case kAccStoreModel: out[v] = to_t<T>(s); break;
      case kAccStoreF32: acc[v] = s; break;
      case kAccAddF32: acc[v] += s; break;
      case kAccAddConvert: out[v] = to_t<T>(acc[v] + s); break;
      default: break;
    }
  }
}

// ---------------------------------------------------------------- finalize
__global__ void finalize_kernel(const unsigned char* ws, FusedOffsets off, int nchunks, int part_stride,
                                int nblocks_last, float* loss, int64_t* n_valid_out) {
  if (threadIdx.x != 0) return;
  const double* part = reinterpret_cast<const double*>(ws + off.loss_part);
  double s = 0.0;
  for (int c = 0; c < nchunks; ++c) {
    const int nb = c == nchunks - 1 ? nblocks_last : part_stride;
    for (int b = 0; b < nb; ++b) s += part[(int64_t)c * part_stride + b];
  }
  *loss = (float)s;
  if (n_valid_out) *n_valid_out = (int64_t) * reinterpret_cast<const unsigned long long*>(ws + 16);
}

}  // namespace

cudaError_t launch_count(const uint8_t* mask, int64_t bs, int64_t T, unsigned char* ws, int nchunks,
                         const FusedOffsets& off, cudaStream_t s) {
  if (bs <= 0) return cudaSuccess;
  { launch_begin(2, s); count_kernel<<<(unsigned)bs, 256, 0, s>>>(mask, bs, T, ws, nchunks, off); launch_end(2, s); }
  return cudaGetLastError();
}

cudaError_t launch_combine(const CombineArgs& a, bool has_kl, bool two_sided, cudaStream_t s) {
  const unsigned grid = (unsigned)((a.rows + 7) / 8);
  if (grid == 0) return cudaSuccess;
  if (has_kl) {
    if (two_sided) { launch_begin(2, s); combine_kernel<true, true><<<grid, 256, 0, s>>>(a); launch_end(2, s); }
    else { launch_begin(2, s); combine_kernel<true, false><<<grid, 256, 0, s>>>(a); launch_end(2, s); }
  } else {
    if (two_sided) { launch_begin(2, s); combine_kernel<false, true><<<grid, 256, 0, s>>>(a); launch_end(2, s); }
    else { launch_begin(2, s); combine_kernel<false, false><<<grid, 256, 0, s>>>(a); launch_end(2, s); }
  }
  return cudaGetLastError();
}

cudaError_t launch_combine_ext(const CombineArgs& a, cudaStream_t s) {
  const unsigned grid = (unsigned)((a.rows + 7) / 8);
  if (grid == 0) return cudaSuccess;
  { launch_begin(2, s); combine_ext_kernel<<<grid, 256, 0, s>>>(a); launch_end(2, s); }
  return cudaGetLastError();
}

cudaError_t launch_clear_gmax(unsigned char* ws, int nchunks, const FusedOffsets& off, cudaStream_t s) {
  { launch_begin(2, s); clear_gmax_kernel<<<1, 256, 0, s>>>(ws, nchunks, off); launch_end(2, s); }
  return cudaGetLastError();
}

cudaError_t launch_dlogits(const DlogitsArgs& a0, DType dt, cudaStream_t s) {
  if (a0.rows <= 0) return cudaSuccess;
  DlogitsArgs a = a0;
  // row groups of >= 128 rows (whole 32-row tiles), at most kDlMaxRowGroups
  int64_t rg = (a.rows + kDlMaxRowGroups - 1) / kDlMaxRowGroups;
  rg = rg < 128 ? 128 : (rg + kDlTileRows - 1) / kDlTileRows * kDlTileRows;
  a.rg_rows = rg;
  a.n_rg = (int)((a.rows + rg - 1) / rg);
  a.wait_ns = debug_knobs().wait_ns;
  // the chunk's [rows, V] logits, {256, 32} boxes, rows ld elements apart
  if (!make_tmap_2d(&a.tmap, a.logits, dt, (uint64_t)a.V, (uint64_t)a.rows, (uint64_t)a.ld * 2, 256,
                    kDlTileRows, false))
    return cudaErrorInvalidValue;
  const dim3 grid((unsigned)((a.V + 255) / 256), (unsigned)a.n_rg);
  const size_t smem = (size_t)kDlStages * kDlTileBytes;
  static bool attr_set[kMaxDevices][2] = {};
  const int ti = dt == DType::BF16 ? 0 : 1;
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(setup_mutex());
    if (!attr_set[dev][ti]) {
      const cudaError_t e = dt == DType::BF16
          ? cudaFuncSetAttribute(dlogits_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
          : cudaFuncSetAttribute(dlogits_kernel<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      attr_set[dev][ti] = true;
    }
  }
  if (dt == DType::BF16) {
    { launch_begin(2, s); dlogits_kernel<__nv_bfloat16><<<grid, 256, smem, s>>>(a); launch_end(2, s); }
  } else {
    { launch_begin(2, s); dlogits_kernel<__half><<<grid, 256, smem, s>>>(a); launch_end(2, s); }
  }
  return cudaGetLastError();
}

namespace {
// out[i] = round(acc[i]) for n = 8 * n8 elements; 8 per thread per step (two
// 16-byte loads that bypass L1 and are marked read-once, one 16-byte store).
template <typename T>
__global__ void __launch_bounds__(256) convert_kernel(const float4* __restrict__ acc, uint4* __restrict__ out,
                                                      int64_t n8) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const float4 a = __ldcs(acc + 2 * i), b = __ldcs(acc + 2 * i + 1);
    uint4 o;
    o.x = pack_t<T>(a.x, a.y);
    o.y = pack_t<T>(a.z, a.w);
    o.z = pack_t<T>(b.x, b.y);
    o.w = pack_t<T>(b.z, b.w);
    out[i] = o;
  }
}
// The same for an output that is not 16-byte aligned (element stores).
template <typename T>
__global__ void __launch_bounds__(256) convert_kernel_unaligned(const float* __restrict__ acc, T* __restrict__ out,
                                                                int64_t n) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) out[i] = to_t<T>(acc[i]);
}
}  // namespace

cudaError_t launch_convert(const float* acc, void* out, int64_t n, DType dt, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  if (n % 8) return cudaErrorInvalidValue;
  DevInfo di;
  cudaError_t e = dev_info(&di);
  if (e != cudaSuccess) return e;
  const int64_t n8 = n / 8;
  int64_t blocks = (n8 + 255) / 256;
  const int64_t cap = (int64_t)di.sm_count * 8;  // 8 resident blocks of 256 threads per SM
  if (blocks > cap) blocks = cap;
  const unsigned g = (unsigned)blocks;
  if ((reinterpret_cast<uintptr_t>(out) & 15) || (reinterpret_cast<uintptr_t>(acc) & 15)) {
    if (dt == DType::BF16) {
      launch_begin(2, s);
      convert_kernel_unaligned<__nv_bfloat16><<<g, 256, 0, s>>>(acc, static_cast<__nv_bfloat16*>(out), n);
      launch_end(2, s);
    } else {
      launch_begin(2, s);
      convert_kernel_unaligned<__half><<<g, 256, 0, s>>>(acc, static_cast<__half*>(out), n);
      launch_end(2, s);
    }
    return cudaGetLastError();
  }
  const float4* a = reinterpret_cast<const float4*>(acc);
  uint4* o = reinterpret_cast<uint4*>(out);
  if (dt == DType::BF16) {
    { launch_begin(2, s); convert_kernel<__nv_bfloat16><<<g, 256, 0, s>>>(a, o, n8); launch_end(2, s); }
  } else {
    { launch_begin(2, s); convert_kernel<__half><<<g, 256, 0, s>>>(a, o, n8); launch_end(2, s); }
  }
  return cudaGetLastError();
}

cudaError_t launch_finalize(const unsigned char* ws, const FusedOffsets& off, int nchunks, int part_stride,
                            int nblocks_last, float* loss, int64_t* n_valid_out, cudaStream_t s) {
  { launch_begin(2, s); finalize_kernel<<<1, 32, 0, s>>>(ws, off, nchunks, part_stride, nblocks_last, loss, n_valid_out); launch_end(2, s); }
  return cudaGetLastError();
}

}  // namespace pl
