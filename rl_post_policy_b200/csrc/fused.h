// Workspace layout and kernel arguments of the fused linear path.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "internal.h"

namespace pl {

// Byte offsets of the regions of a fused-path workspace (after the common
// 256-byte header).  Every region starts on a 1024-byte boundary.
struct FusedOffsets {
  int64_t row_cnt;    // u64 [bs]           valid tokens per sequence
  int64_t loss_part;  // f64 [nchunks, part_stride]  per-block loss partials
  int64_t gmax;       // u32 [nchunks]       max |g| of the chunk (float bits)
  int64_t inv_scale;  // f32 [nchunks]       2^-e undoing the dlogits scale
  int64_t lse;        // f32 [C]             policy logsumexp of the chunk's rows
  int64_t g;          // f32 [C]             dLoss/dlogp of the chunk's rows
  int64_t zt;         // f32 [C]             policy target logit
  int64_t zt_ref;     // f32 [C]             reference target logit
  int64_t part;       // float2 [C, ntv]     policy (max, sum exp) per vocab tile
  int64_t part_ref;   // float2 [C, ntv]     reference ditto
  int64_t logits;     // T [C, ld]           logits, then dlogits (if a gradient is wanted)
  int64_t dw_acc;     // f32 [V, H]          dW accumulator (multi-chunk only)
  int64_t dx_acc;     // f32 [C, H]          the chunk's dX when the backward splits its K (zeroed per chunk)
  int64_t db_acc;     // f32 [V]             dbias accumulator (multi-chunk only)
  int64_t db_part;    // f32 [kDlMaxRowGroups, V]  dbias column sums per dlogits row group
  int64_t db_cnt;     // u32 [ceil(V/256)]   finished row groups per 256-column strip (self-resetting)
  int64_t total;
};

// How a chunk's weight/bias gradient contribution is written.
enum AccMode : int {
  kAccNone = 0,
  kAccStoreModel = 1,  // only chunk: store in the model dtype
  kAccStoreF32 = 2,    // first of several: store fp32 (the accumulator is born here)
  kAccAddF32 = 3,      // middle: fp32 read-modify-write
  kAccAddConvert = 4,  // last: fp32 accumulator + this chunk -> model dtype
};

struct CombineArgs {
  unsigned char* ws;
  FusedOffsets off;
  const int64_t* targets;
  const float* old_lp;
  const void* adv;
  const uint8_t* mask;
  float* logp_out;
  float* ref_logp_out;
  int64_t row0, rows, bs, T, V;
  int nparts;         // (max, sum exp) partials per row
  int chunk, part_stride;
  float lo, hi, beta;
  int grpo, adv_lp_dtype, bf16;
  const float* grad_logp;   // selective log-prob form: external dLoss/dlogp [N]
  float g_scale;            // 1 / temperature: dLoss/dlogp -> gradient of the raw logits
};

// The dlogits pass splits a chunk's rows into at most this many groups.
constexpr int kDlMaxRowGroups = 4;

// dlogits tiles: 32 rows x 256 columns of 16-bit logits.
constexpr int kDlTileRows = 32;
constexpr uint32_t kDlTileBytes = kDlTileRows * 256 * 2;

struct DlogitsArgs {
  CUtensorMap tmap;   // the chunk's logits, set by launch_dlogits
  unsigned char* ws;
  FusedOffsets off;
  const int64_t* targets;
  void* logits;
  int64_t ld;
  int64_t row0, rows, V;
  int chunk;
  int unit_scale;     // 1: dz is stored unscaled (2^0), whatever max|g| is (bf16 chunks whose
                      // dW contributions share one GEMM job and so one epilogue scale)
  int dbias_mode;
  float* dbias_acc;
  void* dbias;
  float* db_part;     // row-group column sums (when a bias gradient is wanted)
  unsigned* db_cnt;
  int64_t rg_rows;    // set by launch_dlogits
  int n_rg;
  unsigned long long wait_ns;  // bound of each wait for a tile (set by launch_dlogits)
};

cudaError_t launch_count(const uint8_t* mask, int64_t bs, int64_t T, unsigned char* ws, int nchunks,
                         const FusedOffsets& off, cudaStream_t s);
cudaError_t launch_combine(const CombineArgs& a, bool has_kl, bool two_sided, cudaStream_t s);
cudaError_t launch_dlogits(const DlogitsArgs& a, DType dt, cudaStream_t s);
// Selective log-prob form: lse and logp per row, g_i = grad_logp[i] (0 when null).
cudaError_t launch_combine_ext(const CombineArgs& a, cudaStream_t s);
// Zeroes the per-chunk max|g| slots (the count kernel does it in the loss form).
cudaError_t launch_clear_gmax(unsigned char* ws, int nchunks, const FusedOffsets& off, cudaStream_t s);
// out[0..n) = acc[0..n) rounded to the model dtype (n a multiple of 8; 16-byte
// vectors when both pointers are 16-byte aligned, element stores otherwise).
cudaError_t launch_convert(const float* acc, void* out, int64_t n, DType dt, cudaStream_t s);
cudaError_t launch_finalize(const unsigned char* ws, const FusedOffsets& off, int nchunks, int part_stride,
                            int nblocks_last, float* loss, int64_t* n_valid_out, cudaStream_t s);

}  // namespace pl
