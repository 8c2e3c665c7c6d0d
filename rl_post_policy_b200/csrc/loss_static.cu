// pl_loss_static: the loss-only kernel with its scratch memory held in a fixed
// array inside this library's device image, for callers that cannot allocate
// device memory on their own path.
//
// The scratch (counters, per-sequence counts, per-block partial sums) lives in
// `g_loss_scratch` below: kStaticScratchBytes bytes, enough for bs up to
// kStaticMaxBs.  Every GPU that loads libpl.so holds this array until the
// process exits.  Host code cannot use the array's name as a device address,
// so the first call on each device looks the address up with
// cudaGetSymbolAddress (with that device current) and caches it, keyed by the
// device and its current context; that first call should therefore come before
// any stream capture.  A device reset (cudaDeviceReset) gives the device a new
// context in which the module is loaded again, so the next call after it looks
// the address up again rather than reusing the old one.  All calls share the
// one array: calls whose work overlaps on the GPU race with each other, so
// issue them on one stream (or otherwise order them).
#include <cuda.h>

#include <mutex>

#include "internal.h"

namespace pl {
namespace {

constexpr int64_t kStaticMaxBs = 4096;
constexpr size_t kStaticPartialOffset = ((kWsHeader + kStaticMaxBs * 8) + 255) & ~(size_t)255;
constexpr size_t kStaticScratchBytes = kStaticPartialOffset + (size_t)kLossMaxBlocks * 8;

static __device__ __align__(256) unsigned char g_loss_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};
CUcontext g_ctx[kMaxDevices] = {};

// The current context through the driver entry point the runtime hands out
// (the library does not link the driver library itself).
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  }
  return fn;
}

// Device address of g_loss_scratch on the current device, looked up once per
// device and context.
pl_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return PL_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PL_ERR_CUDA;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  CUcontext ctx = nullptr;
  if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS) return PL_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!ctx || !g_addr[dev] || g_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_loss_scratch) != cudaSuccess || !p) return PL_ERR_CUDA;
    // the lookup makes the device's primary context current if nothing had yet
    if (!ctx && (get_ctx(&ctx) != CUDA_SUCCESS || !ctx)) return PL_ERR_CUDA;
    g_addr[dev] = p;
    g_ctx[dev] = ctx;
  }
  *out = g_addr[dev];
  return PL_OK;
}

}  // namespace
}  // namespace pl

using namespace pl;

extern "C" pl_status pl_loss_static(const void* policy_lp, const void* old_lp, const void* ref_lp,
                                    const void* adv, const uint8_t* mask, int64_t bs, int64_t seq,
                                    float eps_lo, float eps_hi, float beta, uint32_t mode,
                                    float* loss_out, void* grad_out, int64_t* n_valid_out,
                                    int64_t* row_valid_out, uint32_t* status_out,
                                    pl_stream_t stream) {
  DType dt;
  pl_status st = validate_loss(policy_lp, old_lp, ref_lp, adv, mask, bs, seq, eps_lo, eps_hi, beta, mode,
                               loss_out, &dt);
  if (st != PL_OK) return st;
  if (bs > kStaticMaxBs || loss_ws_bytes(bs) > kStaticScratchBytes) return PL_ERR_WORKSPACE;
  if ((st = check_arch()) != PL_OK) return st;
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != PL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* base = static_cast<unsigned char*>(scratch);
  // The array keeps the previous call's contents: zero the counters and the
  // per-sequence counts this call will accumulate into (the error word at
  // offset 0 is left alone; it is handed to status_out below).
  if (cudaMemsetAsync(base + 4, 0, kWsHeader - 4 + (size_t)(bs > 0 ? bs : 0) * 8, s) != cudaSuccess)
    return PL_ERR_CUDA;
  st = run_loss(policy_lp, old_lp, ref_lp, adv, mask, bs, seq, eps_lo, eps_hi, beta, mode, dt, loss_out,
                grad_out, n_valid_out, row_valid_out, scratch, s);
  if (st != PL_OK) return st;
  if (status_out) {
    if (cudaMemcpyAsync(status_out, base, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
        cudaMemsetAsync(base, 0, sizeof(uint32_t), s) != cudaSuccess)
      return PL_ERR_CUDA;
  }
  return PL_OK;
}
