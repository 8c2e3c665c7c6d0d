// Internal declarations shared by the host-side sources of libpl.so.
#pragma once

#include <cstddef>
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "../../include/pl.h"

namespace pl {

// Element type of log-probs / model tensors (the mode's dtype field).
enum class DType : int { F32 = 0, F16 = 1, BF16 = 2 };

inline size_t dtype_size(DType d) { return d == DType::F32 ? 4 : 2; }

// Sticky device error bits, stored in the first word of every workspace.
constexpr unsigned kDevErrTimeout = 1u;
constexpr unsigned kDevErrTarget = 2u;

// Every workspace starts with this 256-byte header:
//   +0  u32 error flag (sticky, cleared by pl_device_status)
//   +4  u32 grid-barrier arrival counter
//   +8  u32 finished-block counter
//   +16 u64 global valid-token count
//   +32 u32 GEMM tile-queue counter, +36 u32 its finished-CTA counter (fused path;
//       both return to zero at the end of every launch that uses them)
constexpr size_t kWsHeader = 256;
constexpr size_t kWsGemmQueue = 32;

// Bound on every device-side wait, in nanoseconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// Loss-kernel workspace: header, u64 row counts [bs], f64 block partials.
constexpr int kLossMaxBlocks = 4096;
inline size_t loss_partial_offset(int64_t bs) {
  size_t off = kWsHeader + (size_t)(bs > 0 ? bs : 0) * 8;
  return (off + 255) & ~(size_t)255;
}
inline size_t loss_ws_bytes(int64_t bs) { return loss_partial_offset(bs) + (size_t)kLossMaxBlocks * 8; }

struct LossArgs {
  const void* lp;
  const void* old;
  const void* ref;
  const void* adv;
  const uint8_t* mask;
  void* grad;
  float* loss_out;
  int64_t* n_valid_out;
  int64_t* row_valid_out;
  unsigned char* ws;
  int64_t bs, seq, n;
  int64_t chunk;        // tokens per block, multiple of 64
  float lo, hi, beta;
  int grpo;
  int adv_lp_dtype;
  int need_rows;
  int64_t partial_offset;  // byte offset of the f64 block partials inside ws
  unsigned long long wait_ns;
  unsigned extra_arrivals;
  // Division by seq with a multiply (used when n < 2^32): see seq_divider().
  unsigned seq_magic, seq_sh1, seq_sh2;
  int div32;
  int mask_bits_smem;   // phase A keeps the block's mask bits in shared memory
};

// Constants of unsigned 32-bit division by an invariant d >= 1 with one
// multiply-high, after Granlund & Montgomery, "Division by invariant integers
// using multiplication" (PLDI 1994), section 4:
//   l = ceil(log2 d), m = floor(2^32 (2^l - d) / d) + 1,
//   q = (t + ((n - t) >> min(l,1))) >> max(l-1,0) with t = mulhi(m, n).
inline void seq_divider(uint64_t d, unsigned* magic, unsigned* sh1, unsigned* sh2) {
  unsigned l = 0;
  while ((1ull << l) < d) ++l;
  *magic = (unsigned)(((1ull << 32) * ((1ull << l) - d)) / d + 1);
  *sh1 = l < 1 ? l : 1;
  *sh2 = l > 0 ? l - 1 : 0;
}

// Argument checks shared by the loss entry points (no device call); sets *dt.
pl_status validate_loss(const void* lp, const void* old, const void* ref, const void* adv,
                        const uint8_t* mask, int64_t bs, int64_t seq, float eps_lo, float eps_hi,
                        float beta, uint32_t mode, float* loss_out, DType* dt);

// Fills LossArgs and launches the loss kernel on `ws` (a zero-initialised
// loss workspace of at least loss_ws_bytes(bs) bytes).
pl_status run_loss(const void* lp, const void* old, const void* ref, const void* adv,
                   const uint8_t* mask, int64_t bs, int64_t seq, float eps_lo, float eps_hi,
                   float beta, uint32_t mode, DType dt, float* loss_out, void* grad_out,
                   int64_t* n_valid_out, int64_t* row_valid_out, void* ws, cudaStream_t stream);

// Launches the single-pass loss kernel; returns a CUDA error code.
// Small batches (n <= kSmallMaxTokens tokens, bs <= kSmallMaxRows) can take a
// kernel without the grid barrier, in which every block counts the whole mask.
constexpr int64_t kSmallMaxTokens = 65536;
constexpr int kSmallMaxRows = 1024;
bool loss_small_eligible(int64_t bs, int64_t n);
cudaError_t launch_loss_small(const LossArgs& a, DType dt, bool has_kl, bool has_grad, bool two_sided, bool vec,
                              cudaStream_t stream);
cudaError_t launch_loss(const LossArgs& a, DType dt, bool has_kl, bool has_grad, bool two_sided,
                        bool vec, cudaStream_t stream);

// Test-only knobs (set through pl_debug_set_wait): the bound on device waits
// and two ways to make a bounded wait run out on purpose -- extra grid-barrier
// arrivals the loss kernel waits for, and extra bytes a GEMM pipeline stage
// expects from its TMA loads.  Defaults: kWaitLimitNs, 0, 0.
struct DebugKnobs {
  unsigned long long wait_ns = kWaitLimitNs;
  unsigned extra_arrivals = 0;
  unsigned extra_tx = 0;
  int rkl_cluster = 0;   // reverse-KL CTAs per cluster (1, 2, 4 or 8; 0 = the host's choice)
  int gemm_nh = 0;       // GEMM tile width in N=256 MMAs (1 or 2; 0 = the host's choice)
  int loss_path = 0;     // loss kernel: 0 = the host's choice, 1 = small-batch kernel when eligible,
                         // 2 = the cooperative kernel
  int rkl_path = 0;      // reverse KL with a gradient: 0 = the host's choice (the streaming kernel),
                         // 1 = the streaming kernel, 2 = the register-resident kernel where it applies
  int gemm_merge = 0;    // fused path with several chunks: 0 = chunk c's backward and chunk c+1's
                         // forward share a launch (8 epilogue warps), 1 = separate launches,
                         // 2 = shared launches with 4 epilogue warps
  int gemm_tail = 0;     // 512-wide round-robin launches: 0 = the last partial wave's tiles run as
                         // 256-wide halves where that shortens the launch, 1 = never
  int dw_finish = 0;     // several chunks: 0 = the host's choice (1), 1 = fp32 add, then a separate
                         // rounding kernel, 2 = the last chunk's dW epilogue adds the fp32
                         // accumulator and stores the model dtype
  int gemm_split = 0;    // K split of the backward launch's dX problem: 0 = the host's choice,
                         // 1 = never, 2 = always (when it has at least two k-steps)
  int dw_pair = 0;       // several bf16 chunks with shared launches: 0 = the host's choice (2),
                         // 1 = one dW contribution per chunk, 2 = one per pair of chunks (K = 2 C)
};
DebugKnobs& debug_knobs();

// Launch bookkeeping: every kernel launch of the library is bracketed by
// launch_begin/launch_end (kind: 0 GEMM, 1 loss kernel, 2 other).  Counts
// launches; records CUDA events on `stream` while timing is enabled.
void launch_begin(int kind, cudaStream_t stream);
void launch_end(int kind, cudaStream_t stream);

// Device properties cached per device.
struct DevInfo {
  int sm_count = 0;
  int cc_major = 0, cc_minor = 0;
  size_t smem_optin = 0;
};
cudaError_t dev_info(DevInfo* out);

// Host-side caches of per-kernel launch setup (shared-memory attributes,
// occupancy) are kept per device, under one mutex, for processes that drive
// several GPUs or call from several threads.
constexpr int kMaxDevices = 64;
int current_device();  // the current device's index, or -1
std::mutex& setup_mutex();

// PL_OK when the current device is compute capability 10.0.
pl_status check_arch();

// Library-owned, zero-initialised scratch of at least `need` bytes for the
// current device and `stream` (created or grown when `create`; growing
// synchronises the stream).  *out is NULL when none exists and !create.
pl_status own_workspace(cudaStream_t stream, size_t need, void** out, bool create);

// Bytes of a reverse-KL workspace (header + per-cluster loss partials).
size_t reverse_kl_ws_bytes();

}  // namespace pl
