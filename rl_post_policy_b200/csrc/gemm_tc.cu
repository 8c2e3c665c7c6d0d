// Persistent tcgen05 GEMM for sm_100a with the epilogues of the fused path.
//
// CTAs run in pairs (clusters of two, one CTA per SM); a pair owns a 256 x 256
// or 256 x 512 output tile (NH = 1 or 2 N=256 MMAs per K step, picked per
// launch by pick_tile_width) and the grid holds as many pairs as can be
// resident, each walking its share of the tiles of up to two GEMM problems.
// Per CTA:
//   warp 0    one lane issues TMA tile loads (128-byte swizzle, no multicast)
//             of this CTA's 128 rows of A and its half of the tile's columns of
//             B into the operand ring (6 stages of 32 KB at NH = 1, 4 of 48 KB
//             at NH = 2); the pair leader's mbarrier counts both CTAs' bytes;
//   warp 1    allocates 512 tensor-memory columns (two alternating 128 x 256
//             fp32 accumulators at NH = 1, one 128 x 512 at NH = 2,
//             cta_group::2); in the leader one lane issues
//             tcgen05.mma.cta_group::2 (M=256, N=256, K=16), which reads the A
//             and B halves from both CTAs' shared memory and writes each CTA's
//             128 accumulator rows into its own tensor memory, and commits each
//             stage back to both producers and each tile to both epilogues;
//   warps 2.. the epilogue, EW = 8 warps (or 4): one accumulator row per thread
//             (tcgen05.ld 32x32b), 32 columns at a time, two warps per 32-lane
//             quarter of tensor memory splitting each 256-column group; it
//             overlaps the next tile's mainloop (second accumulator at NH = 1,
//             the drained half at NH = 2); both CTAs release the accumulator on
//             the leader's barrier.
// Splitting B across the pair halves each SM's shared-memory operand traffic
// compared with one CTA computing a 128 x 256 tile alone.
// Operands may be K-major or MN-major (the backward GEMMs read the logits
// workspace and the weights transposed without copying them).
//
// Epilogues ("Add SM100 CuTe DSL GRPO fast path", Liger-Kernel PR #1363,
// "Summary": full logits are never materialised beyond a bounded workspace):
//   kEpiLse   -- per (row, 128-column half of a 256-column vocabulary tile):
//                running max and sum of exp(z - max) over the valid columns,
//                the target logit when the row's target falls in it, optional
//                bias add, and the logits stored in the model dtype by TMA;
//   kEpiStore -- acc * scale stored in the model dtype (dX, one-chunk dW) or
//                fp32 (dW accumulated across chunks: a TMA store, then TMA adds),
//                through shared-memory boxes and TMA, or per-thread stores for
//                outputs that are not 16-byte aligned.
//
// Every wait is bounded (GemmParams::wait_ns); when one runs out the CTA sets a
// shared abort flag, every role drains out, the leader waits (bounded) for its
// issued MMAs, tensor memory is released and the sticky device error flag is
// raised.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "gemm.h"
#include "sm100.cuh"

namespace pl {
namespace {

using namespace sm100;

constexpr uint32_t kABytes = kBM * kBK * 2;             // 16 KB: this CTA's 128 rows of A
constexpr uint32_t kBBytes = kBNh * kBK * 2;            // 16 KB: this CTA's 128 rows of B per MMA
constexpr uint32_t kTmemCols = 512;
constexpr int kQSlots = 4;   // dynamic queue: tile ids in flight between the roles
// Epilogue staging for the TMA output paths: 8 boxes of 4 KB (32 rows x 128
// bytes), one per epilogue warp (8 warps) or two (4 warps).
constexpr uint32_t kOutBoxBytes = kOutBoxM * kOutBoxN * 4;
constexpr uint32_t kOutStageBytes = 8 * kOutBoxBytes;

// Pair tile kPairM x (kBN * NH).  NH = 1: one N=256 MMA per K=16 step, two
// accumulators alternating between tiles (the epilogue of tile t overlaps the
// mainloop of t+1), 6 stages of 32 KB.  NH = 2: two N=256 MMAs per step share
// the A stage (25% fewer operand bytes per flop and half the barrier round
// trips), one 512-column accumulator, 4 stages of 48 KB.
template <int NH>
struct TileCfg {
  static constexpr int kTileN = kBN * NH;
  static constexpr int kStages = NH == 1 ? 6 : 4;
  static constexpr uint32_t kStageBytes = kABytes + NH * kBBytes;
  // [alignment slack][operand ring][barriers, padded to 1 KB][output staging].
  // Launches without a TMA output path leave the staging off the allocation,
  // which keeps 32 KB more of the SM's unified L1 / shared memory as L1.
  static constexpr size_t kSmemBase = 1024 + kStages * kStageBytes + 1024;
  static constexpr size_t kSmem = kSmemBase + kOutStageBytes;
  static_assert(kSmem <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
};

__device__ __forceinline__ float cvt_in(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float cvt_in(__half x) { return __half2float(x); }

template <typename T> __device__ __forceinline__ uint32_t pack2(float a, float b);
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <> __device__ __forceinline__ uint32_t pack2<__half>(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <typename T> __device__ __forceinline__ T cvt_out(float x);
template <> __device__ __forceinline__ __nv_bfloat16 cvt_out<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
template <> __device__ __forceinline__ __half cvt_out<__half>(float x) { return __float2half_rn(x); }

template <typename T> struct AbFormat;
template <> struct AbFormat<__half> { static constexpr uint32_t v = 0; };
template <> struct AbFormat<__nv_bfloat16> { static constexpr uint32_t v = 1; };

struct TileCoord {
  int job, mb, nb;
  int kb, nk;  // first k-step and number of k-steps of this tile (all of K unless the job is split)
  int half;    // -1: the whole pair tile; 0 or 1: only its columns [256 * half, 256 * half + 256)
};

// Tile `tile` of the launch: its job, row block, column block and K range.  A
// split job lists all tiles of its first K half, then all of the second.
__device__ __forceinline__ TileCoord tile_coord(const GemmParams& p, int tile) {
  TileCoord c;
  c.job = 0;
#pragma unroll
  for (int q = 1; q < kMaxJobs; ++q)
    if (q < p.njobs && tile >= p.jobs[q].tile_begin) c.job = q;
  const GemmJob& j = p.jobs[c.job];
  int local = tile - j.tile_begin;
  c.kb = 0;
  c.nk = j.k_steps;
  c.half = -1;
  if (j.tail > 0) {
    const int base = j.tiles_m * j.tiles_n - j.tail;
    if (local >= base) {
      const int hh = local - base;
      local = base + (hh >> 1);
      c.half = hh & 1;
    }
  }
  if (j.k_split > 1) {
    const int per = j.tiles_m * j.tiles_n;
    const int ks = local / per;
    local -= ks * per;
    c.kb = ks * j.k_per;
    c.nk = min(j.k_per, j.k_steps - c.kb);
  }
  if (j.n_inner) {
    c.mb = local / j.tiles_n;
    c.nb = local - c.mb * j.tiles_n;
  } else {
    c.nb = local / j.tiles_m;
    c.mb = local - c.nb * j.tiles_m;
  }
  return c;
}

}  // namespace

// Global tile id of the i-th tile of `pair`, or -1 once the pair is done.
__host__ __device__ int pair_tile(const GemmParams& p, int pair, int npairs, int i) {
  if (p.sched == 0) {
    const int t = pair + i * npairs;
    return t < p.total_tiles ? t : -1;
  }
  const int T0 = p.jobs[1].tile_begin;
  int k = i;
  if (pair < T0) {
    if (k == 0) return pair;
    k -= 1;
  }
  const int cnt = (pair < T0 ? p.na : p.nb) + (pair < p.rem ? 1 : 0);
  if (k >= cnt) return -1;
  const int lo = pair < T0 ? pair : T0;
  const int hi = pair > T0 ? pair - T0 : 0;
  const int rm = pair < p.rem ? pair : p.rem;
  return T0 + lo * p.na + hi * p.nb + rm + k;
}

__host__ __device__ int queue_tile(const GemmParams& p, int q) {
  if (p.q_w < 0) return q;
  const int t_lead = p.jobs[p.q_f0].tile_begin;
  if (q < t_lead) return q;
  const long long qq = q - t_lead;
  const long long tw_begin = p.jobs[p.q_w].tile_begin;
  const long long tf = tw_begin - t_lead;
  const long long r = (long long)p.total_tiles - t_lead;
  const long long f0 = qq * tf / r, f1 = (qq + 1) * tf / r;
  if (f1 > f0) return (int)(t_lead + f0);   // the f0-th tile of jobs [q_f0, q_w)
  return (int)(tw_begin + (qq - f0));       // the (qq - f0)-th tile of job q_w
}

namespace {

// Stores 32 consecutive values (or the first `nvalid`) of one row.
template <typename T>
__device__ __forceinline__ void store_row32(T* dst, const float (&v)[32], int nvalid) {
  if (nvalid >= 32 && ((reinterpret_cast<uintptr_t>(dst) & 15) == 0)) {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 u;
      u.x = pack2<T>(v[8 * q + 0], v[8 * q + 1]);
      u.y = pack2<T>(v[8 * q + 2], v[8 * q + 3]);
      u.z = pack2<T>(v[8 * q + 4], v[8 * q + 5]);
      u.w = pack2<T>(v[8 * q + 6], v[8 * q + 7]);
      d4[q] = u;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < nvalid) dst[j] = cvt_out<T>(v[j]);
  }
}

__device__ __forceinline__ void store_row32_f32(float* dst, const float (&v)[32], int nvalid) {
  if (nvalid >= 32 && ((reinterpret_cast<uintptr_t>(dst) & 15) == 0)) {
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int q = 0; q < 8; ++q) d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < nvalid) dst[j] = v[j];
  }
}

__device__ __forceinline__ void add_row32_f32(const float* src, float (&v)[32], int nvalid) {
  if (nvalid >= 32 && ((reinterpret_cast<uintptr_t>(src) & 15) == 0)) {
    const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 a = s4[q];
      v[4 * q] += a.x;
      v[4 * q + 1] += a.y;
      v[4 * q + 2] += a.z;
      v[4 * q + 3] += a.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < nvalid) v[j] += src[j];
  }
}

// v[q] = v[q] * sc + src[q] over the first nvalid of 32 columns (v[q] * sc past
// them); src is read once, with streaming loads.
__device__ __forceinline__ void scale_add_row32(const float* src, float (&v)[32], float sc, int nvalid) {
  if (nvalid >= 32 && ((reinterpret_cast<uintptr_t>(src) & 15) == 0)) {
    const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 a = __ldcs(s4 + q);
      v[4 * q] = v[4 * q] * sc + a.x;
      v[4 * q + 1] = v[4 * q + 1] * sc + a.y;
      v[4 * q + 2] = v[4 * q + 2] * sc + a.z;
      v[4 * q + 3] = v[4 * q + 3] * sc + a.w;
    }
  } else {
#pragma unroll
    for (int q = 0; q < 32; ++q) v[q] = q < nvalid ? v[q] * sc + __ldcs(src + q) : v[q] * sc;
  }
}

// 2^x with the hardware approximation (flushes subnormal results to zero);
// the epilogue only takes it of values <= 0, whose results lie in (0, 1].
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The bias of up to 64 consecutive columns (the first nvalid) added to v.
template <typename T>
__device__ __forceinline__ void add_bias64(const T* bias, float (&v)[64], int nvalid) {
  if (nvalid >= 64 && ((reinterpret_cast<uintptr_t>(bias) & 15) == 0)) {
    const uint4* b4 = reinterpret_cast<const uint4*>(bias);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint4 u = __ldg(b4 + q);
      const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
      for (int k = 0; k < 8; ++k) v[8 * q + k] += cvt_in(e[k]);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 64; ++k)
      if (k < nvalid) v[k] += cvt_in(bias[k]);
  }
}

template <typename T>
__device__ __forceinline__ void add_bias32(const T* bias, float (&v)[32], int nvalid) {
  if (nvalid >= 32 && ((reinterpret_cast<uintptr_t>(bias) & 15) == 0)) {
    const uint4* b4 = reinterpret_cast<const uint4*>(bias);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 u = __ldg(b4 + q);
      const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[8 * q + j] += cvt_in(e[j]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < nvalid) v[j] += cvt_in(bias[j]);
  }
}

template <typename T, int NH, int EW>
__global__ void __launch_bounds__(gemm_threads(EW), 1) gemm_kernel(const __grid_constant__ GemmParams p) {
  static_assert(EW == 4 || EW == 8, "4 or 8 epilogue warps");
  // readers of a dynamic-queue slot: the peer's producer, the MMA issuer and
  // every epilogue warp of both CTAs
  constexpr int kQReaders = 2 + 2 * EW;
  using Cfg = TileCfg<NH>;
  constexpr int kStages = Cfg::kStages;
  constexpr uint32_t kStageBytes = Cfg::kStageBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint8_t* out_stage = smem + kStages * kStageBytes + 1024;  // 1024-byte aligned; only with a TMA output
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  // dynamic queue (GemmParams::dyn): a ring of claimed tile ids, published by the
  // leader's producer into both CTAs, each slot released by every role that reads it
  uint64_t* qfull = done + 1;
  uint64_t* qempty = qfull + kQSlots;
  int* qring_raw = reinterpret_cast<int*>(qempty + kQSlots);
  volatile int* qring = qring_raw;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qring_raw + kQSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: pair leader (issues the MMAs), 1: peer
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * EW * 32);  // both CTAs' epilogue threads release the leader's accumulator
    }
    mbar_init(done, 1);
    for (int q = 0; q < kQSlots; ++q) {
      mbar_init(&qfull[q], 1);                // the leader producer's arrival
      mbar_init(&qempty[q], kQReaders);       // (leader only) every reader of the slot
    }
    *abort_flag = 0;
    fence_barrier_init();
    for (int q = 0; q < p.njobs; ++q) {
      prefetch_tmap(&p.maps[p.jobs[q].a_map]);
      prefetch_tmap(&p.maps[p.jobs[q].b_map]);
      if (p.jobs[q].k_seg > 0) {
        prefetch_tmap(&p.maps[p.jobs[q].a_map2]);
        prefetch_tmap(&p.maps[p.jobs[q].b_map2]);
      }
      if (p.jobs[q].out_path != kOutDirect) prefetch_tmap(&p.maps[p.jobs[q].out_map]);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const unsigned long long lim = p.wait_ns;

  // ---- dynamic queue: entry `it` of this pair's tile sequence ----
  // Readers wait for the leader producer's publication (acquire at cluster
  // scope), take the id, and release the slot on the leader's barrier.
  // Returns the tile (or -1: no more), or -2 when a wait ran out.
  auto q_read = [&](int it) -> int {
    const int slot = it % kQSlots;
    const uint32_t par = (uint32_t)(it / kQSlots) & 1u;
    if (!mbar_wait_cluster(&qfull[slot], par, abort_flag, lim)) return -2;
    return qring[slot];
  };
  auto q_release = [&](int it) {
    mbar_arrive_cluster(mapa_shared(smem_u32(&qempty[it % kQSlots]), 0));
  };
  // The leader producer: claim the next queue entry and publish its tile id in
  // both CTAs once every reader has released the slot's previous entry.
  auto q_claim = [&](int it) -> int {
    const int slot = it % kQSlots;
    const uint32_t par = (uint32_t)(it / kQSlots) & 1u;
    const unsigned q = atomicAdd(p.ctr, 1u);
    const int tile = q < (unsigned)p.total_tiles ? queue_tile(p, (int)q) : -1;
    if (!mbar_wait_cluster(&qempty[slot], par ^ 1u, abort_flag, lim)) return -2;
    qring[slot] = tile;
    st_cluster_s32(mapa_shared(smem_u32(&qring_raw[slot]), 1), tile);
    mbar_arrive(&qfull[slot]);
    mbar_arrive_cluster(mapa_shared(smem_u32(&qfull[slot]), 1));
    return tile;
  };

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs; completions counted by the leader) ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int it = 0; !*abort_flag; ++it) {
        int tile;
        if (p.dyn) {
          if (leader) {
            tile = q_claim(it);
          } else {
            tile = q_read(it);
            if (tile != -2) q_release(it);
          }
        } else {
          tile = pair_tile(p, pair, npairs, it);
        }
        if (tile < 0) break;
        const TileCoord tc = tile_coord(p, tile);
        const GemmJob& j = p.jobs[tc.job];
        const int m0 = tc.mb * kPairM + (int)rank * kBM;
        const int nt0 = tc.nb * Cfg::kTileN + (int)rank * kBNh;
        // a half tile loads one B half (its columns) into the stage's first B slot
        const int nb_loads = tc.half < 0 ? NH : 1;
        const uint32_t stage_tx = 2 * (kABytes + (uint32_t)nb_loads * kBBytes) + p.extra_tx;
        for (int k = 0; k < tc.nk; ++k) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, lim)) break;
          if (leader) mbar_arrive_expect_tx(&full[stage], stage_tx);
          const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
          uint8_t* a_dst = ring + stage * kStageBytes;
          uint8_t* b_dst = a_dst + kABytes;
          // the job's second K segment (if any) through its own maps, K from 0
          const int kg = tc.kb + k;
          const bool seg2 = j.k_seg > 0 && kg >= j.k_seg;
          const CUtensorMap* amap = &p.maps[seg2 ? j.a_map2 : j.a_map];
          const CUtensorMap* bmap = &p.maps[seg2 ? j.b_map2 : j.b_map];
          const int k0 = (seg2 ? kg - j.k_seg : kg) * kBK;
          if (!j.a_mn) {
            tma_load_2d_pair(a_dst, amap, bar, k0, m0);
          } else {
            tma_load_2d_pair(a_dst, amap, bar, m0, k0);
            tma_load_2d_pair(a_dst + 8192, amap, bar, m0 + 64, k0);
          }
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            if (h >= nb_loads) break;
            // MMA h needs columns [h*kBN, (h+1)*kBN) of the tile; this CTA holds kBNh of them
            const int n0 = nt0 + (tc.half < 0 ? h : tc.half) * kBN;
            uint8_t* bh = b_dst + h * kBBytes;
            if (!j.b_mn) {
              tma_load_2d_pair(bh, bmap, bar, k0, n0);
            } else {
              tma_load_2d_pair(bh, bmap, bar, n0, k0);
              tma_load_2d_pair(bh + 8192, bmap, bar, n0 + 64, k0);
            }
          }
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*abort_flag) {
        // Leave time for copies already issued to land before shared memory is released.
        const unsigned long long t0 = globaltimer();
        while (globaltimer() - t0 < 100000ull) __nanosleep(1000);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader CTA only) ----------------
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      const uint32_t ring_addr = smem_u32(ring);
      // The K=16 MMAs of one stage into accumulator half h (column offset d_col);
      // k counts the tile's own k-steps, so its first step overwrites the accumulator.
      auto issue = [&](int st, int k, const GemmJob& j, uint32_t idesc, int h, uint32_t d_col) {
        const uint32_t a_addr = ring_addr + st * kStageBytes;
        const uint32_t b_addr = a_addr + kABytes + h * kBBytes;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = j.a_mn ? smem_desc(a_addr + kk * 2048, 8192, 1024)
                                     : smem_desc(a_addr + kk * 32, 16, 1024);
          const uint64_t bd = j.b_mn ? smem_desc(b_addr + kk * 2048, 8192, 1024)
                                     : smem_desc(b_addr + kk * 32, 16, 1024);
          mma_f16_ss_pair(tmem_base + d_col, ad, bd, idesc, (k | kk) != 0 ? 1u : 0u);
        }
      };
      for (int it = 0; !*abort_flag; ++it) {
        int tile;
        if (p.dyn) {
          tile = q_read(it);
          if (tile != -2) q_release(it);
        } else {
          tile = pair_tile(p, pair, npairs, it);
        }
        if (tile < 0) break;
        const TileCoord tc = tile_coord(p, tile);
        const GemmJob& j = p.jobs[tc.job];
        const uint32_t idesc = instr_desc_f16(AbFormat<T>::v, j.a_mn, j.b_mn, kPairM, kBN);
        bool ok = true;
        if constexpr (NH == 1) {
          if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, lim)) break;
          tc_fence_after();
          for (int k = 0; k < tc.nk; ++k) {
            if (!mbar_wait(&full[stage], phase, abort_flag, lim)) { ok = false; break; }
            tc_fence_after();
            issue(stage, k, j, idesc, 0, acc * kBN);
            mma_commit_pair(&empty[stage], 0x3);
            if (++stage == kStages) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (!ok) break;
          mma_commit_pair(&tfull[acc], 0x3);
          if (++acc == 2) {
            acc = 0;
            acc_phase ^= 1;
          }
        } else if (tc.half >= 0) {
          // A half tile: its one 256-column MMA per stage goes into accumulator
          // half 0 (the epilogue drains only that half and releases half 1 at
          // once, which keeps both halves' barrier phases in step with the tiles).
          if (!mbar_wait(&tempty[0], acc_phase ^ 1, abort_flag, lim)) break;
          tc_fence_after();
          for (int k = 0; k < tc.nk; ++k) {
            if (!mbar_wait(&full[stage], phase, abort_flag, lim)) { ok = false; break; }
            tc_fence_after();
            issue(stage, k, j, idesc, 0, 0);
            mma_commit_pair(&empty[stage], 0x3);
            if (++stage == kStages) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (!ok) break;
          mma_commit_pair(&tfull[0], 0x3);
          acc_phase ^= 1;
        } else {
          // One 512-column accumulator, drained by the epilogue in two halves
          // (tempty[0], tempty[1]).  Half 0 of this tile starts once the
          // previous tile's half 0 is drained; a stage whose half-1 MMAs cannot
          // be issued yet (half 1 still draining) is held back, uncommitted, and
          // flushed in k order as soon as half 1 is free (or when every stage
          // is held).  Each half still accumulates in k order.
          if (!mbar_wait(&tempty[0], acc_phase ^ 1, abort_flag, lim)) break;
          tc_fence_after();
          bool h1 = mbar_try_wait(&tempty[1], acc_phase ^ 1);
          if (h1) tc_fence_after();
          int held = 0, held_stage = 0, held_k = 0;
          auto flush = [&]() {
            for (int q = 0; q < held; ++q) {
              const int st = (held_stage + q) % kStages;
              issue(st, held_k + q, j, idesc, 1, kBN);
              mma_commit_pair(&empty[st], 0x3);
            }
            held = 0;
          };
          for (int k = 0; k < tc.nk; ++k) {
            if (!mbar_wait(&full[stage], phase, abort_flag, lim)) { ok = false; break; }
            tc_fence_after();
            issue(stage, k, j, idesc, 0, 0);
            if (!h1 && mbar_try_wait(&tempty[1], acc_phase ^ 1)) {
              tc_fence_after();
              h1 = true;
            }
            if (h1) {
              flush();
              issue(stage, k, j, idesc, 1, kBN);
              mma_commit_pair(&empty[stage], 0x3);
            } else {
              if (held == 0) {
                held_stage = stage;
                held_k = k;
              }
              ++held;
              if (held == kStages) {
                if (!mbar_wait(&tempty[1], acc_phase ^ 1, abort_flag, lim)) { ok = false; break; }
                tc_fence_after();
                h1 = true;
                flush();
              }
            }
            if (++stage == kStages) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (ok && held) {
            if (!mbar_wait(&tempty[1], acc_phase ^ 1, abort_flag, lim)) ok = false;
            else {
              tc_fence_after();
              flush();
            }
          }
          if (!ok) break;
          mma_commit_pair(&tfull[0], 0x3);
          acc_phase ^= 1;
        }
      }
      // Every MMA this thread issued has completed before tensor memory is released.
      mma_commit_pair(done, 0x1);
      volatile int no_abort = 0;
      mbar_wait(done, 0, &no_abort, lim);
    }
  } else {
    // ---------------- epilogue (warps 2 .. EW+1, both CTAs) ----------------
    // A warp may only read the tensor-memory quarter warp % 4.  With 8 warps,
    // warps 2-5 take columns [0, 128) of every 256-column group and warps 6-9
    // columns [128, 256); with 4, each warp takes the whole group.
    constexpr int kCG = EW / 4;    // column groups
    constexpr int kBoxes = 8 / EW;  // staging boxes per warp
    const int quarter = warp & 3;  // tensor-memory lanes [32*quarter, 32*quarter+32)
    const int colgrp = (warp - 2) / 4;
    const int c_lo = colgrp * (kBN / 32 / kCG);  // first 32-column slice
    const int c_hi = c_lo + kBN / 32 / kCG;
    const int r_local = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    constexpr float kLog2e = 1.4426950408889634f;
    // this warp's two staging boxes for the TMA output paths
    const uint32_t box0 = smem_u32(out_stage) + (uint32_t)((warp - 2) * kBoxes) * kOutBoxBytes;
    int sbuf = 0;
    for (int it = 0;; ++it) {
      int tile;
      if (p.dyn) {
        tile = q_read(it);
        __syncwarp();
        if (lane == 0 && tile != -2) q_release(it);
      } else {
        tile = pair_tile(p, pair, npairs, it);
      }
      if (tile < 0) break;
      const TileCoord tc = tile_coord(p, tile);
      const GemmJob& j = p.jobs[tc.job];
      const int m0 = tc.mb * kPairM + (int)rank * kBM;
      const int row = m0 + r_local;
      const bool row_ok = row < j.M;
      // the row's target id, loaded while the tile's accumulator is still being computed
      const int64_t tgt = (j.epi == kEpiLse && row_ok) ? __ldg(j.targets + row) : (int64_t)-1;
      if (!mbar_wait(&tfull[NH == 1 ? acc : 0], acc_phase, abort_flag, lim)) break;
      tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < NH; ++h) {
        // 256-column group h of the tile: TMEM columns [col_base, col_base + 256);
        // a half tile has one group, its columns in accumulator half 0
        const int colh = tc.half < 0 ? h : tc.half;
        const int n0 = (tc.half >= 0 && h > 0) ? j.N : tc.nb * Cfg::kTileN + colh * kBN;
        const int grp = tc.nb * NH + colh;  // index of this 256-column group along N
        const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (NH == 1 ? acc : h) * kBN;
        // hands the group's accumulator columns back to the issuer (once per group)
        bool released = false;
        auto release = [&]() {
          if (released) return;
          released = true;
          tc_fence_before();
          mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&tempty[NH == 1 ? acc : h]), 0));
        };
        if (n0 >= j.N) {
          // past the end of N: zeros only, nothing to store
        } else if (j.epi == kEpiLse) {
          const T* bias = reinterpret_cast<const T*>(j.bias);
          T* logits = reinterpret_cast<T*>(j.logits);
          // logits through shared memory and TMA stores (see the kEpiStore
          // path below), 64 columns per box, or per-thread stores
          const bool tma_logits = logits && j.out_path == kOutTmaStore;
          const int y = m0 + quarter * 32;
          const int64_t tgt_rel = tgt >= 0 ? tgt - (int64_t)n0 : (int64_t)-1;
          float m_run = -INFINITY, s_run = 0.0f, ztv = 0.0f;
          bool got = false;
  #pragma unroll 1
          for (int c = c_lo; c < c_hi; c += 2) {
            uint32_t w[32];
            // the box's 64 columns in one tensor-memory load
            float v[64];
            tmem_ld_32x32b_x64(taddr + c * 32, v);
            const int col0 = n0 + c * 32;
            const int nv0 = min(32, j.N - col0), nv1 = min(32, j.N - col0 - 32);
            if (nv0 > 0) {
              if (bias) add_bias64<T>(bias + col0, v, nv0 + (nv1 > 0 ? nv1 : 0));
              if (j.logit_scale != 1.0f) {
  #pragma unroll
                for (int q = 0; q < 64; ++q) v[q] *= j.logit_scale;
              }
            }
            if (nv1 == 32) {
              // 64 full columns: the maximum by a tree and the sum of exponentials in
              // four independent packed accumulators (short dependency chains), with
              // one rescale of the running sum
              float t[16];
  #pragma unroll
              for (int i = 0; i < 16; ++i)
                t[i] = fmaxf(fmaxf(v[2 * i], v[2 * i + 1]), fmaxf(v[32 + 2 * i], v[33 + 2 * i]));
  #pragma unroll
              for (int i = 0; i < 8; ++i) t[i] = fmaxf(t[i], t[i + 8]);
  #pragma unroll
              for (int i = 0; i < 4; ++i) t[i] = fmaxf(t[i], t[i + 4]);
              const float m_new = fmaxf(m_run, fmaxf(fmaxf(t[0], t[1]), fmaxf(t[2], t[3])));
              const float2 nmb = make_float2(-m_new * kLog2e, -m_new * kLog2e);
              const float2 l2e = make_float2(kLog2e, kLog2e);
              float2 sacc[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                                make_float2(0.0f, 0.0f)};
  #pragma unroll
              for (int q = 0; q < 64; q += 2) {
                const float2 x = __ffma2_rn(make_float2(v[q], v[q + 1]), l2e, nmb);
                sacc[(q >> 1) & 3] = __fadd2_rn(sacc[(q >> 1) & 3], make_float2(ex2_approx(x.x), ex2_approx(x.y)));
              }
              const float2 s01 = __fadd2_rn(sacc[0], sacc[1]), s23 = __fadd2_rn(sacc[2], sacc[3]);
              const float2 s4 = __fadd2_rn(s01, s23);
              s_run = s_run * ex2_approx(fmaf(m_run, kLog2e, nmb.x)) + (s4.x + s4.y);
              m_run = m_new;
            } else {
              // a ragged end of N: each 32-column slice with its own column predicates
  #pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int nvalid = h ? nv1 : nv0;
                if (nvalid <= 0) continue;
                float cmax = -INFINITY;
  #pragma unroll
                for (int q = 0; q < 32; ++q)
                  if (q < nvalid) cmax = fmaxf(cmax, v[32 * h + q]);
                const float m_new = fmaxf(m_run, cmax);
                const float mb = m_new * kLog2e;
                float s = 0.0f;
  #pragma unroll
                for (int q = 0; q < 32; ++q)
                  if (q < nvalid) s += ex2_approx(fmaf(v[32 * h + q], kLog2e, -mb));
                s_run = s_run * ex2_approx(fmaf(m_run, kLog2e, -mb)) + s;
                m_run = m_new;
              }
            }
            // the target logit, if this box holds the row's target column
            const int64_t rel = tgt_rel - c * 32;
            if (rel >= 0 && rel < 64 && rel < (int64_t)(nv0 + (nv1 > 0 ? nv1 : 0))) {
  #pragma unroll
              for (int q = 0; q < 64; ++q)
                if (q == (int)rel) ztv = v[q];
              got = true;
            }
            if (logits && !tma_logits && row_ok) {
              if (nv0 > 0) {
                float u[32];
  #pragma unroll
                for (int q = 0; q < 32; ++q) u[q] = v[q];
                store_row32<T>(logits + (int64_t)row * j.logits_ld + col0, u, nv0);
              }
              if (nv1 > 0) {
                float u[32];
  #pragma unroll
                for (int q = 0; q < 32; ++q) u[q] = v[32 + q];
                store_row32<T>(logits + (int64_t)row * j.logits_ld + col0 + 32, u, nv1);
              }
            }
            if (tma_logits) {
  #pragma unroll
              for (int q = 0; q < 32; ++q) w[q] = pack2<T>(v[2 * q], v[2 * q + 1]);
            }
            if (tma_logits && n0 + c * 32 < j.N && y < j.M) {
              // the box's previous contents have been read out by the TMA unit
              if (lane == 0) bulk_wait_group_read<kBoxes - 1>();
              __syncwarp();
              const uint32_t box = box0 + (uint32_t)sbuf * kOutBoxBytes;
              const uint32_t my_row = box + (uint32_t)lane * 128u;
  #pragma unroll
              for (int q = 0; q < 8; ++q)
                st_shared_v4(my_row + ((uint32_t)(q ^ (lane & 7)) << 4), w[4 * q], w[4 * q + 1], w[4 * q + 2],
                             w[4 * q + 3]);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&p.maps[j.out_map], box, n0 + c * 32, y);
                bulk_commit_group();
              }
              if (kBoxes > 1) sbuf ^= 1;
            }
          }
          if (row_ok) {
            // one partial per row, 256-column group and column group; (-inf, 0)
            // for a column group wholly past N
            j.part[(int64_t)row * j.part_ld + grp * kEpiColGroups + colgrp] = make_float2(m_run, s_run);
            if (kCG == 1) j.part[(int64_t)row * j.part_ld + grp * kEpiColGroups + 1] = make_float2(-INFINITY, 0.0f);
            if (got) j.zt[row] = ztv;
          }
        } else if (j.out_path != kOutDirect) {
          // The result through shared memory and the TMA unit.  Each warp
          // stages its 32 rows in one 4 KB box of 128-byte rows (32 fp32 or 64
          // 16-bit columns) with the 128-byte swizzle: 16-byte chunk q of row r
          // sits at chunk q ^ (r % 8), so a warp's 16-byte stores hit every
          // bank once per 8 lanes.  Lane 0 then issues the box's store (or fp32
          // add), which the TMA unit writes as whole 128-byte lines.  Rows and
          // columns past the output's extent are dropped by the TMA unit.
          const float sc = j.scale ? __ldg(j.scale) : 1.0f;
          const CUtensorMap* omap = &p.maps[j.out_map];
          const int y = m0 + quarter * 32;
          const int step = j.out_f32 ? 1 : 2;  // 32-column TMEM slices per box
          // one staged box of packed words: columns [col0, col0 + 128 bytes)
          auto store_box = [&](const uint32_t (&w)[32], int col0) {
            if (col0 >= j.N || y >= j.M) return;
            // the box's previous contents have been read out by the TMA unit
            if (lane == 0) bulk_wait_group_read<kBoxes - 1>();
            __syncwarp();
            const uint32_t box = box0 + (uint32_t)sbuf * kOutBoxBytes;
            const uint32_t my_row = box + (uint32_t)lane * 128u;
  #pragma unroll
            for (int q = 0; q < 8; ++q)
              st_shared_v4(my_row + ((uint32_t)(q ^ (lane & 7)) << 4), w[4 * q], w[4 * q + 1], w[4 * q + 2],
                           w[4 * q + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (j.out_path == kOutTmaReduce) tma_reduce_add_2d(omap, box, col0, y);
              else tma_store_2d(omap, box, col0, y);
              bulk_commit_group();
            }
            if (kBoxes > 1) sbuf ^= 1;
          };
          if (kCG == 2 && !j.acc_in && !j.out_f32) {
            // 8 warps, a 16-bit output: this warp's 128 columns of the group come into
            // registers first (scaled and packed, 16 columns per tensor-memory load) and
            // the accumulator half goes back to the issuer before any of them is staged,
            // so the next tile's MMAs into it overlap the stores (the issuer waited for
            // the staging of each half before)
            uint32_t w[2][32];
  #pragma unroll
            for (int b = 0; b < 8; ++b) {
              float v[16];
              tmem_ld_32x32b_x16(taddr + (uint32_t)(c_lo * 32 + b * 16), v);
  #pragma unroll
              for (int q = 0; q < 8; ++q) w[b >> 2][(b & 3) * 8 + q] = pack2<T>(v[2 * q] * sc, v[2 * q + 1] * sc);
            }
            release();
  #pragma unroll
            for (int b = 0; b < 2; ++b) store_box(w[b], n0 + (c_lo + 2 * b) * 32);
          } else {
  #pragma unroll 1
            for (int c = c_lo; c < c_hi; c += step) {
              uint32_t w[32];
              float v[32];
              tmem_ld_32x32b_x32(taddr + c * 32, v);
              if (j.out_f32) {
  #pragma unroll
                for (int q = 0; q < 32; ++q) w[q] = __float_as_uint(v[q] * sc);
              } else if (j.acc_in) {
                // the fp32 accumulator of the earlier chunks added to this tile, then
                // rounded once to the model dtype (the last chunk of a multi-chunk dW)
                const float* arow = j.acc_in + (int64_t)(row_ok ? row : 0) * j.out_ld;
                const int colA = n0 + c * 32;
                float sa = row_ok ? 1.0f : 0.0f;  // rows past M: no load, dropped by the TMA store
                if (row_ok) scale_add_row32(arow + colA, v, sc, min(32, j.N - colA));
                else sa = sc;
  #pragma unroll
                for (int q = 0; q < 16; ++q) w[q] = pack2<T>(v[2 * q] * sa, v[2 * q + 1] * sa);
                tmem_ld_32x32b_x32(taddr + (c + 1) * 32, v);
                if (row_ok) scale_add_row32(arow + colA + 32, v, sc, min(32, j.N - colA - 32));
  #pragma unroll
                for (int q = 0; q < 16; ++q) w[16 + q] = pack2<T>(v[2 * q] * sa, v[2 * q + 1] * sa);
              } else {
  #pragma unroll
                for (int q = 0; q < 16; ++q) w[q] = pack2<T>(v[2 * q] * sc, v[2 * q + 1] * sc);
                tmem_ld_32x32b_x32(taddr + (c + 1) * 32, v);
  #pragma unroll
                for (int q = 0; q < 16; ++q) w[16 + q] = pack2<T>(v[2 * q] * sc, v[2 * q + 1] * sc);
              }
              store_box(w, n0 + c * 32);
            }
          }
        } else {
          const float sc = j.scale ? __ldg(j.scale) : 1.0f;
  #pragma unroll 1
          for (int c = c_lo; c < c_hi; ++c) {
            float v[32];
            tmem_ld_32x32b_x32(taddr + c * 32, v);
            const int col0 = n0 + c * 32;
            const int nvalid = min(32, j.N - col0);
            if (!row_ok || nvalid <= 0) continue;
  #pragma unroll
            for (int q = 0; q < 32; ++q) v[q] *= sc;
            const int64_t off = (int64_t)row * j.out_ld + col0;
            if (j.acc_in) add_row32_f32(j.acc_in + off, v, nvalid);
            if (j.out_f32) store_row32_f32(reinterpret_cast<float*>(j.out) + off, v, nvalid);
            else store_row32<T>(reinterpret_cast<T*>(j.out) + off, v, nvalid);
          }
        }
        release();
      }  // groups
      if (NH == 1) {
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      } else {
        acc_phase ^= 1;
      }
    }
    // every TMA store / add this warp issued has been performed before exit
    if (lane == 0) bulk_wait_group_all();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no remote arrival or pair MMA is still aimed at either CTA
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.err, kDevErrTimeout);
  if (p.dyn && threadIdx.x == 0) {
    // the last CTA to finish returns the queue counter to zero for the next launch
    // (every claim of this CTA's pair precedes its arrival here)
    __threadfence();
    if (atomicAdd(p.ctr_done, 1u) == gridDim.x - 1) {
      *reinterpret_cast<volatile unsigned*>(p.ctr) = 0u;
      *reinterpret_cast<volatile unsigned*>(p.ctr_done) = 0u;
      __threadfence();
    }
  }
}

}  // namespace

void gemm_finalize_jobs(GemmParams* p) {
  int begin = 0;
  const int tile_n = kBN * (p->nh == 2 ? 2 : 1);
  for (int i = 0; i < p->njobs; ++i) {
    GemmJob& j = p->jobs[i];
    j.tiles_m = (j.M + kPairM - 1) / kPairM;
    j.tiles_n = (j.N + tile_n - 1) / tile_n;
    j.k_steps = (j.K + kBK - 1) / kBK;
    // a split needs a k-step for each half (an empty half would store an unwritten accumulator)
    j.k_split = (j.k_split == 2 && j.k_steps >= 2) ? 2 : 1;
    j.k_per = (j.k_steps + j.k_split - 1) / j.k_split;
    j.tile_begin = begin;
    begin += job_tiles(j);
  }
  p->total_tiles = begin;
}

// Cost of a launch in k-step units (one K=64 step of one N=256 MMA group).
// Each tile also pays a fixed kTileOverhead for its accumulator hand-off and
// pipeline turn; fitted to the backward launch of a 1024-row chunk (V=128256,
// H=4096), whose 16-k-step dW tiles ran about 18% slower at 256 wide than at
// 512 wide.
constexpr double kTileOverhead = 8.0;

namespace {
// k-steps of one tile of job j (of one K half for a split job)
long tile_ksteps(const GemmJob& j) { return j.k_split > 1 ? j.k_per : j.k_steps; }
}  // namespace

// Chooses the tile schedule for `P` pairs (see GemmParams::sched).  Tile costs
// are k-steps x width plus the per-tile overhead.
void balance_schedule(GemmParams* p, int P) {
  p->sched = 0;
  p->na = p->nb = p->rem = 0;
  if (p->njobs != 2) return;
  const GemmJob& j0 = p->jobs[0];
  const GemmJob& j1 = p->jobs[1];
  const long T0 = job_tiles(j0), T1 = job_tiles(j1);
  const double w = p->nh == 2 ? 2.0 : 1.0;
  const double c0 = tile_ksteps(j0) * w + kTileOverhead, c1 = (tile_ksteps(j1) > 0 ? tile_ksteps(j1) : 1) * w + kTileOverhead;
  if (T0 > P || c0 < 4 * c1 || T1 == 0) return;  // equal-cost tiles: round-robin is balanced
  const double ideal = (T0 * c0 + T1 * c1) / P;
  long nb = (long)(ideal / c1);
  long na = (long)((ideal - c0) / c1);
  if (na < 0) na = 0;
  auto total = [&] { return T0 * na + (P - T0) * nb; };
  while (total() > T1) {
    if (P - T0 > 0 && nb > 0 && (na == 0 || nb * c1 >= c0 + na * c1)) --nb;
    else if (na > 0) --na;
    else --nb;
  }
  while (T1 - total() >= P) {
    if (P - T0 > 0) ++nb;
    else ++na;
  }
  p->sched = 1;
  p->na = (int)na;
  p->nb = (int)nb;
  p->rem = (int)(T1 - total());
}

// Estimated launch length on P pairs with pair tiles nh MMAs wide: the busiest
// pair's load, in k-step units, under the schedule balance_schedule picks.
double launch_estimate(GemmParams p, int nh, int P) {
  p.nh = nh;
  gemm_finalize_jobs(&p);
  balance_schedule(&p, P);
  const long T0 = job_tiles(p.jobs[0]);
  const long T1 = p.njobs > 1 ? job_tiles(p.jobs[1]) : 0;
  const double c0 = tile_ksteps(p.jobs[0]) * (double)nh + kTileOverhead;
  const double c1 = p.njobs > 1 ? tile_ksteps(p.jobs[1]) * (double)nh + kTileOverhead : 0.0;
  double worst = 0.0;
  for (long q = 0; q < P; ++q) {
    long n0, n1;
    if (p.sched == 1) {
      n0 = q < T0 ? 1 : 0;
      n1 = (q < T0 ? p.na : p.nb) + (q < p.rem ? 1 : 0);
    } else {
      const long ntot = q < T0 + T1 ? (T0 + T1 - 1 - q) / P + 1 : 0;
      n0 = q < T0 ? (T0 - 1 - q) / P + 1 : 0;
      n1 = ntot - n0;
    }
    const double load = n0 * c0 + n1 * c1;
    if (load > worst) worst = load;
  }
  return worst;
}

// 256 x 512 tiles move 25% fewer operand bytes per flop, halve the barrier
// round trips and the tile count; measured on this kernel they run the same
// k-step work about 10% faster when the launch stays balanced.  They need every
// problem to be at least 512 wide.
constexpr double kWideSpeed = 0.9;

int pick_tile_width(const GemmParams& p, int P) {
  if (P <= 0) return 1;
  for (int i = 0; i < p.njobs; ++i)
    if (p.jobs[i].N < 2 * kBN) return 1;
  return kWideSpeed * launch_estimate(p, 2, P) < launch_estimate(p, 1, P) ? 2 : 1;
}

// Measured on the fused backward launch (1024-row chunk and whole 8192-row
// batch, V=128256, H=4096), the split was no faster: 5-10% slower at 1024 rows
// and within 1% at 8192, although the schedule estimate promised 3-6%.  So it
// runs only when a test or a measurement asks for it (debug knob 2).
constexpr double kSplitGain = 0.98;

int gemm_choose_k_split(GemmParams* p, int job, int P) {
  const int knob = debug_knobs().gemm_split == 0 ? 1 : debug_knobs().gemm_split;
  double best = 0.0;
  int best_split = 1, best_nh = 1;
  for (int split = 1; split <= 2; ++split) {
    if ((knob == 1 && split == 2) || (knob == 2 && split == 1)) continue;
    GemmParams q = *p;
    q.jobs[job].k_split = split;
    const int nh = debug_knobs().gemm_nh ? debug_knobs().gemm_nh : pick_tile_width(q, P);
    const double e = launch_estimate(q, nh, P) * (nh == 2 ? kWideSpeed : 1.0);
    if (split == 1 || knob == 2 || e < kSplitGain * best) {
      best = e;
      best_split = split;
      best_nh = nh;
    }
  }
  p->jobs[job].k_split = best_split;
  p->nh = best_nh;
  gemm_finalize_jobs(p);
  return p->jobs[job].k_split;
}

namespace {

template <typename T, int NH, int EW>
cudaError_t launch_t(const GemmParams& p, cudaStream_t stream) {
  constexpr size_t kGemmSmem = TileCfg<NH>::kSmem;
  static int max_pairs_dev[kMaxDevices] = {};  // resident CTA pairs, per device
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(gemm_threads(EW));
  cfg.dynamicSmemBytes = kGemmSmem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int max_pairs;
  {
    std::lock_guard<std::mutex> lock(setup_mutex());
    if (max_pairs_dev[dev] == 0) {  // one CTA per SM with or without the output staging
      cudaError_t e = cudaFuncSetAttribute(gemm_kernel<T, NH, EW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)kGemmSmem);
      if (e != cudaSuccess) return e;
      DevInfo di;
      if ((e = dev_info(&di)) != cudaSuccess) return e;
      cfg.gridDim = dim3(di.sm_count & ~1);
      int n = 0;
      e = cudaOccupancyMaxActiveClusters(&n, gemm_kernel<T, NH, EW>, &cfg);
      if (e != cudaSuccess) return e;
      max_pairs_dev[dev] = n > 0 ? n : 1;
    }
    max_pairs = max_pairs_dev[dev];
  }
  bool tma_out = false;
  for (int i = 0; i < p.njobs; ++i) tma_out = tma_out || p.jobs[i].out_path != kOutDirect;
  if (!tma_out) cfg.dynamicSmemBytes = TileCfg<NH>::kSmemBase;
  const int pairs = p.total_tiles < max_pairs ? p.total_tiles : max_pairs;
  cfg.gridDim = dim3(2 * pairs);
  GemmParams q = p;
  balance_schedule(&q, pairs);
  if (NH == 2 && q.sched == 0 && !q.dyn && debug_knobs().gemm_tail != 1) {
    // a round-robin launch's last partial wave in 256-wide halves
    GemmJob& last = q.jobs[q.njobs - 1];
    const int tail = tail_halves(q.total_tiles, pairs);
    if (tail > 0 && last.k_split < 2 && last.tiles_m * last.tiles_n >= tail) {
      last.tail = tail;
      gemm_finalize_jobs(&q);
    }
  }
  launch_begin(0, stream);
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_kernel<T, NH, EW>, q);
  launch_end(0, stream);
  return e;
}
}  // namespace

cudaError_t launch_gemm(const GemmParams& p0, DType dt, cudaStream_t stream) {
  GemmParams p = p0;
  p.wait_ns = debug_knobs().wait_ns;
  p.extra_tx = debug_knobs().extra_tx;
  // Tile width: 256 x 512 pair tiles (nh = 2) unless a problem is narrower than
  // 512 or the wider tiles would unbalance the launch (see pick_tile_width).
  int nh = 1;
  if (debug_knobs().gemm_nh) {
    nh = debug_knobs().gemm_nh;
  } else if (p.nh == 1 || p.nh == 2) {
    nh = p.nh;  // chosen by the caller (gemm_choose_k_split)
  } else {
    DevInfo di;
    if (dev_info(&di) == cudaSuccess) nh = pick_tile_width(p, di.sm_count / 2);
  }
  p.nh = nh;
  gemm_finalize_jobs(&p);
  if (p.total_tiles <= 0) return cudaSuccess;
  // fp32 TMA outputs (chunked dW accumulation, the debug hook) move 32-column
  // boxes: 4 epilogue warps with two boxes each drain them faster than 8 with one.
  // A split job's fp32 output is small next to its K (two adds per output element
  // over thousands of k-steps) and does not count.
  // A launch that also holds logits tiles (a chunk's backward merged with the
  // next chunk's forward) keeps 8 warps for their logsumexp epilogue.
  bool f32_tma = false, lse = false;
  for (int i = 0; i < p.njobs; ++i) {
    f32_tma = f32_tma || (p.jobs[i].out_path != kOutDirect && p.jobs[i].out_f32 && p.jobs[i].k_split < 2);
    lse = lse || p.jobs[i].epi == kEpiLse;
  }
  if (lse && debug_knobs().gemm_merge != 2) f32_tma = false;
  if (dt == DType::BF16) {
    if (f32_tma) return nh == 2 ? launch_t<__nv_bfloat16, 2, 4>(p, stream) : launch_t<__nv_bfloat16, 1, 4>(p, stream);
    return nh == 2 ? launch_t<__nv_bfloat16, 2, 8>(p, stream) : launch_t<__nv_bfloat16, 1, 8>(p, stream);
  }
  if (dt == DType::F16) {
    if (f32_tma) return nh == 2 ? launch_t<__half, 2, 4>(p, stream) : launch_t<__half, 1, 4>(p, stream);
    return nh == 2 ? launch_t<__half, 2, 8>(p, stream) : launch_t<__half, 1, 8>(p, stream);
  }
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------- tensor maps
namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}
}  // namespace

bool make_tmap_2d(CUtensorMap* map, const void* base, DType dt, uint64_t inner, uint64_t outer,
                  uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (pitch_bytes & 15)) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType t = dt == DType::BF16  ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                : dt == DType::F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUresult r = fn(map, t, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace pl
