// Host-visible description of one launch of the persistent tcgen05 GEMM.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "internal.h"

namespace pl {

// A CTA pair (a cluster of two CTAs on two SMs) owns one kPairM x (NH * kBN)
// output tile (NH = 1 or 2 N=256 MMAs per K step): each CTA holds kBM rows of A,
// NH * kBNh rows of B and kBM x (NH * kBN) fp32 accumulators in its tensor
// memory; the pair leader issues the M=256 MMAs.
constexpr int kBM = 128;       // rows per CTA (tensor-memory lanes)
constexpr int kPairM = 256;    // rows per CTA pair (the MMA's M)
constexpr int kBN = 256;       // tile columns (tensor-memory columns per accumulator)
constexpr int kBNh = 128;      // B rows (N) held by each CTA of the pair
constexpr int kBK = 64;        // K per pipeline stage (one 128-byte swizzle row)
// Warp 0: TMA producer; warp 1: MMA issuer; then EW epilogue warps, EW = 8
// (two per 32-lane quarter of tensor memory, splitting each 256-column group in
// column halves) or 4 (one per quarter, two staging boxes each: launches with an
// fp32 TMA output, whose 32-column boxes are too small to leave one box per warp).
constexpr int kEpiColGroups = 2;   // LSE partials per row and 256-column group
__host__ __device__ constexpr int gemm_threads(int ew) { return 64 + 32 * ew; }

enum EpiKind : int {
  kEpiLse = 0,    // logits tile -> per-row (max, sum exp) + target logit (+ store logits)
  kEpiStore = 1,  // acc * scale (+ fp32 acc_in) -> out (model dtype or fp32)
};

// How a kEpiStore job writes its result.
enum OutPath : int {
  kOutDirect = 0,     // per-thread row stores (and acc_in loads) from registers
  kOutTmaStore = 1,   // staged in shared memory, TMA tile store through maps[out_map]
  kOutTmaReduce = 2,  // fp32 only: staged, TMA element-wise add into maps[out_map]
};

// Output tensor maps for the kOutTma* paths cover [M, N] (row pitch out_ld)
// with boxes of kOutBoxM rows x 128 bytes -- kOutBoxN fp32 or kOutBoxN16
// 16-bit columns -- and the 128-byte swizzle: one box is one epilogue warp's
// 32 rows.  N * element size must be a multiple of 16 bytes.
constexpr int kOutBoxN = 32;
constexpr int kOutBoxN16 = 64;
constexpr int kOutBoxM = 32;

// One GEMM problem D[M,N] = sum_k A(m,k) B(n,k), tiled kPairM x kBN.
//   A(m,k): K-major means A[m*lda + k]; MN-major means A[k*lda + m] (likewise B).
struct GemmJob {
  int a_map, b_map;        // tensor-map indices in GemmParams::maps
  int a_mn, b_mn;          // 0 = K-major, 1 = MN-major
  int M, N, K;
  int tiles_m, tiles_n, k_steps;
  // K split: 1, or 2 -- every output tile is then computed as two tiles, one per
  // half of the k-steps, and each adds its fp32 result into `out` through the TMA
  // unit (out_path kOutTmaReduce, out_f32, onto a zeroed buffer; with exactly two
  // addends onto zero the sum does not depend on their order).  Halving the
  // length of a problem's longest tiles lets the schedule balance a launch whose
  // long tiles would otherwise finish last.
  int k_split;
  int k_per;               // k-steps per split (set by gemm_finalize_jobs)
  // 512-wide launches: the job's last `tail` tiles each run as two 256-wide
  // tiles (columns [0, 256) and [256, 512) of the pair tile), listed after its
  // other tiles, so that a round-robin launch's last partial wave is spread over
  // twice as many pairs (set by launch_gemm; 0 = none).
  int tail;
  int n_inner;             // 1: consecutive tiles walk N first (share the A rows)
  // Two K segments: k-steps [0, k_seg) read A and B through a_map / b_map, and
  // k-steps [k_seg, k_steps) through a_map2 / b_map2, counting K from 0 again
  // (two row chunks of the fused path contributing to dW through one job: their
  // dlogits sit in different workspace slots).  k_seg = 0: one segment.
  int k_seg;
  int a_map2, b_map2;
  int tile_begin;          // first global tile index of this job
  int epi;
  // kEpiLse
  const void* bias;        // [N] model dtype or null
  const int64_t* targets;  // [M] (rows of this job)
  float2* part;            // [M, part_ld] (max, sum exp) per row and 128-column half of each
                           // 256-column group: entry grp * kEpiColGroups + column group
  int part_ld;
  float* zt;               // [M] target logit
  void* logits;            // [M, logits_ld] model dtype or null
  int64_t logits_ld;
  float logit_scale;       // 1 / temperature, applied after the bias (1 for temperature 1)
  // kEpiStore
  void* out;
  int out_f32;
  int out_path;            // OutPath; kOutTma* need out_map
  int out_map;             // tensor-map index of `out` for the kOutTma* paths
  const float* acc_in;     // [M, out_ld] fp32 added before the store, or null (16-bit outputs
                           // of kOutDirect and kOutTmaStore)
  int64_t out_ld;
  const float* scale;      // device scalar multiplier, or null for 1
};

constexpr int kMaxJobs = 4;
constexpr int kMaxMaps = 14;

struct __align__(64) GemmParams {
  CUtensorMap maps[kMaxMaps];
  GemmJob jobs[kMaxJobs];
  int njobs;
  int total_tiles;
  // Dynamic tile queue (dyn = 1): the pairs claim tiles from a global counter
  // (*ctr, zero before the launch; the last CTA to finish sets it and *ctr_done
  // back to zero) in queue order: the tiles of jobs [0, q_f0) first, then the
  // tiles of jobs [q_f0, q_w) interleaved evenly with those of job q_w (q_w < 0:
  // no interleaving, every tile in job order).  Used for launches whose jobs
  // differ in tile cost and in memory traffic: long tiles first, and
  // memory-heavy tiles spread over the launch next to compute-heavy ones.
  int dyn, q_f0, q_w;
  unsigned* ctr;
  unsigned* ctr_done;
  // Tile schedule (set by launch_gemm).  0: pair p takes tiles p, p+P, p+2P ...
  // 1: two jobs of very different tile cost -- pair p < T0 takes job-0 tile p,
  //    then every pair takes a contiguous run of job-1 tiles, `na` (p < T0) or
  //    `nb` long plus one for the first `rem` pairs, so that all pairs carry
  //    about the same number of k-steps.
  int sched, na, nb, rem;
  int nh;                  // N=256 MMAs per K step (1 or 2): tiles are kPairM x (nh * kBN)
  unsigned* err;
  unsigned long long wait_ns;
  unsigned extra_tx;       // test-only: extra bytes each stage expects (0 in normal use)
};

// Tensor-map boxes: K-major operands load {kBK, kBM} (A) or {kBK, kBNh} (B)
// boxes; MN-major operands load {64, kBK} boxes, two per 128 rows/columns.
// Encodes a 2-D tensor map over a row-major [outer, inner] array of `dt`
// elements (16-bit, or fp32 for the kOutTma* outputs) with a row pitch of
// `pitch_bytes`, box {box_inner, box_outer}, zero fill outside the extent, and
// the 128-byte swizzle (box rows of at most 128 bytes) or none (box rows of
// up to 256 elements, laid out densely in shared memory).
bool make_tmap_2d(CUtensorMap* map, const void* base, DType dt, uint64_t inner, uint64_t outer,
                  uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128 = true);

// Fills tiles_m/tiles_n/k_steps/k_per/tile_begin of each job and total_tiles, for
// tiles nh * kBN wide.  launch_gemm picks nh (unless p->nh is set) and calls it again.
void gemm_finalize_jobs(GemmParams* p);

// Tiles of a job (output tiles times its K split, plus one for each tail tile run in halves).
inline int job_tiles(const GemmJob& j) {
  return j.tiles_m * j.tiles_n * (j.k_split > 1 ? j.k_split : 1) + (j.tail > 0 ? j.tail : 0);
}

// Tiles of a round-robin launch of T equal 512-wide tiles on P pairs to run in
// halves: the last partial wave's R = T mod P tiles when R <= P / 2 (their 2R
// halves then take half a tile's time on 2R pairs instead of a whole one on R),
// else none.
inline int tail_halves(int T, int P) {
  if (P <= 1 || T <= P) return 0;
  const int r = T % P;
  return (r > 0 && 2 * r <= P) ? r : 0;
}

cudaError_t launch_gemm(const GemmParams& p, DType dt, cudaStream_t stream);

// The tile width launch_gemm uses on P pairs (1: 256 wide, 2: 512 wide) unless
// a test forces one or p.nh is set, from the jobs' M, N, K and K splits.
double launch_estimate(GemmParams p, int nh, int P);
int pick_tile_width(const GemmParams& p, int P);

// Decides whether job `job` of a two-problem launch is computed in two K halves
// (see GemmJob::k_split) and with which tile width, on P pairs: sets
// p->jobs[job].k_split and p->nh.  A debug knob can force the split on or off.
// Returns the chosen k_split.
int gemm_choose_k_split(GemmParams* p, int job, int P);

// Tile schedule (host side of what the kernel runs): balance_schedule fills
// sched/na/nb/rem for P pairs; pair_tile gives the i-th tile of a pair or -1.
void balance_schedule(GemmParams* p, int P);
__host__ __device__ int pair_tile(const GemmParams& p, int pair, int npairs, int i);
// Global tile id of the q-th entry of the dynamic queue (see GemmParams::dyn).
__host__ __device__ int queue_tile(const GemmParams& p, int q);

}  // namespace pl
