// Host-visible description of one launch of the persistent tcgen05 GEMM.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "internal.h"

namespace pl {

constexpr int kBM = 128;       // tile rows (tensor-memory lanes)
constexpr int kBN = 256;       // tile columns (tensor-memory columns per accumulator)
constexpr int kBK = 64;        // K per pipeline stage (one 128-byte swizzle row)
constexpr int kStages = 4;
constexpr int kGemmThreads = 192;  // warp 0: TMA, warp 1: MMA, warps 2-5: epilogue

enum EpiKind : int {
  kEpiLse = 0,    // logits tile -> per-row (max, sum exp) + target logit (+ store logits)
  kEpiStore = 1,  // acc * scale (+ fp32 acc_in) -> out (model dtype or fp32)
};

// One GEMM problem D[M,N] = sum_k A(m,k) B(n,k), tiled kBM x kBN.
//   A(m,k): K-major means A[m*lda + k]; MN-major means A[k*lda + m] (likewise B).
struct GemmJob {
  int a_map, b_map;        // tensor-map indices in GemmParams::maps
  int a_mn, b_mn;          // 0 = K-major, 1 = MN-major
  int M, N, K;
  int tiles_m, tiles_n, k_steps;
  int n_inner;             // 1: consecutive tiles walk N first (share the A rows)
  int tile_begin;          // first global tile index of this job
  int epi;
  // kEpiLse
  const void* bias;        // [N] model dtype or null
  const int64_t* targets;  // [M] (rows of this job)
  float2* part;            // [M, part_ld] (max, sum exp) per (row, N tile)
  int part_ld;
  float* zt;               // [M] target logit
  void* logits;            // [M, logits_ld] model dtype or null
  int64_t logits_ld;
  // kEpiStore
  void* out;
  int out_f32;
  const float* acc_in;     // [M, out_ld] fp32 added before the store, or null
  int64_t out_ld;
  const float* scale;      // device scalar multiplier, or null for 1
};

struct __align__(64) GemmParams {
  CUtensorMap maps[4];
  GemmJob jobs[2];
  int njobs;
  int total_tiles;
  unsigned* err;
  unsigned long long wait_ns;
  unsigned extra_tx;       // test-only: extra bytes each stage expects (0 in normal use)
};

// Encodes a 2-D tensor map over a row-major [outer, inner] array of 16-bit
// elements with a row pitch of `pitch_bytes`, box {box_inner, box_outer},
// 128-byte swizzle, zero fill outside the extent.
bool make_tmap_2d(CUtensorMap* map, const void* base, DType dt, uint64_t inner, uint64_t outer,
                  uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer);

// Fills tiles_m/tiles_n/k_steps/tile_begin of each job and total_tiles.
void gemm_finalize_jobs(GemmParams* p);

cudaError_t launch_gemm(const GemmParams& p, DType dt, cudaStream_t stream);

}  // namespace pl
