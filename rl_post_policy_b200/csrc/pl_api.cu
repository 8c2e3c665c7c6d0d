// C ABI entry points of libpl.so: argument validation, scratch management,
// status reporting, and the launch of the loss-only kernel.  The fused linear
// path's host driver lives in fused_api.cu.
#include <cmath>
#include <map>
#include <mutex>
#include <utility>

#include "internal.h"

namespace pl {

cudaError_t dev_info(DevInfo* out) {
  static std::mutex mu;
  static std::map<int, DevInfo> cache;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) { *out = it->second; return cudaSuccess; }
  DevInfo di;
  int v = 0;
  if ((e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  di.sm_count = v;
  if ((e = cudaDeviceGetAttribute(&v, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return e;
  di.cc_major = v;
  if ((e = cudaDeviceGetAttribute(&v, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) return e;
  di.cc_minor = v;
  if ((e = cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  di.smem_optin = (size_t)v;
  cache[dev] = di;
  *out = di;
  return cudaSuccess;
}

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

std::mutex& setup_mutex() {
  static std::mutex mu;
  return mu;
}

pl_status check_arch() {
  DevInfo di;
  if (dev_info(&di) != cudaSuccess) return PL_ERR_CUDA;
  if (di.cc_major != 10 || di.cc_minor != 0) return PL_ERR_ARCH;
  return PL_OK;
}

namespace {
// Library-owned scratch, one per (device, stream).
struct OwnWs {
  void* ptr = nullptr;
  size_t bytes = 0;
};
std::mutex g_ws_mu;
std::map<std::pair<int, cudaStream_t>, OwnWs> g_ws;
}  // namespace

pl_status own_workspace(cudaStream_t stream, size_t need, void** out, bool create) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return PL_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_ws_mu);
  OwnWs& w = g_ws[{dev, stream}];
  if (w.bytes >= need && w.ptr) { *out = w.ptr; return PL_OK; }
  if (!create) { *out = w.ptr; return PL_OK; }
  if (w.ptr) {
    // Growing: the old buffer may still be read by work queued on `stream`.
    if (cudaStreamSynchronize(stream) != cudaSuccess) return PL_ERR_CUDA;
    cudaFree(w.ptr);
    w.ptr = nullptr;
    w.bytes = 0;
  }
  size_t bytes = need < (1u << 20) ? (1u << 20) : need;
  void* p = nullptr;
  if (cudaMalloc(&p, bytes) != cudaSuccess) return PL_ERR_CUDA;
  if (cudaMemset(p, 0, bytes) != cudaSuccess) { cudaFree(p); return PL_ERR_CUDA; }
  w.ptr = p;
  w.bytes = bytes;
  *out = p;
  return PL_OK;
}

namespace {

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

bool finite_nonneg(float x) { return std::isfinite(x) && x >= 0.0f; }

constexpr uint32_t kLossModeBits = PL_REDUCTION_MASK | PL_DTYPE_MASK | PL_ADV_LP_DTYPE | PL_CLIP_TWO_SIDED;

}  // namespace

// Host-side validation shared by the loss entry points (no device call).
pl_status validate_loss(const void* lp, const void* old, const void* ref, const void* adv,
                        const uint8_t* mask, int64_t bs, int64_t seq, float eps_lo, float eps_hi,
                        float beta, uint32_t mode, float* loss_out, DType* dt) {
  if (bs < 0 || seq < 0 || !loss_out) return PL_ERR_ARG;
  if (seq > 0 && bs > INT64_MAX / seq) return PL_ERR_ARG;
  if (mode & ~kLossModeBits) return PL_ERR_ARG;
  if ((mode & PL_REDUCTION_MASK) > PL_GRPO) return PL_ERR_ARG;
  const uint32_t d = (mode & PL_DTYPE_MASK) >> 4;
  if (d > 2) return PL_ERR_DTYPE;
  *dt = (DType)d;
  if (!finite_nonneg(eps_lo) || !finite_nonneg(eps_hi) || !finite_nonneg(beta)) return PL_ERR_ARG;
  if (eps_lo > 1.0f) return PL_ERR_ARG;
  const int64_t n = bs * seq;
  if (n > 0 && (!lp || !old || !adv || !mask)) return PL_ERR_ARG;
  if (n > 0 && beta != 0.0f && !ref) return PL_ERR_ARG;
  return PL_OK;
}

pl_status run_loss(const void* lp, const void* old, const void* ref, const void* adv,
                   const uint8_t* mask, int64_t bs, int64_t seq, float eps_lo, float eps_hi,
                   float beta, uint32_t mode, DType dt, float* loss_out, void* grad_out,
                   int64_t* n_valid_out, int64_t* row_valid_out, void* ws, cudaStream_t stream) {
  LossArgs a{};
  a.lp = lp;
  a.old = old;
  a.ref = ref;
  a.adv = adv;
  a.mask = mask;
  a.grad = grad_out;
  a.loss_out = loss_out;
  a.n_valid_out = n_valid_out;
  a.row_valid_out = row_valid_out;
  a.ws = static_cast<unsigned char*>(ws);
  a.bs = bs;
  a.seq = seq;
  a.n = bs * seq;
  a.lo = 1.0f - eps_lo;
  a.hi = 1.0f + eps_hi;
  a.beta = beta;
  a.grpo = (mode & PL_REDUCTION_MASK) == PL_GRPO;
  a.adv_lp_dtype = (mode & PL_ADV_LP_DTYPE) != 0;
  a.need_rows = a.grpo || row_valid_out != nullptr;
  a.partial_offset = (int64_t)loss_partial_offset(bs);
  a.div32 = seq > 0 && a.n < (1ll << 32) && seq < (1ll << 32);
  if (a.div32) seq_divider((uint64_t)seq, &a.seq_magic, &a.seq_sh1, &a.seq_sh2);
  const bool has_kl = beta != 0.0f;
  const bool has_grad = grad_out != nullptr;
  const bool vec = aligned(lp, 16) && aligned(old, 16) && (!has_kl || aligned(ref, 16)) &&
                   (!has_grad || aligned(grad_out, 16)) && aligned(mask, 16);
  // Small batches skip the cooperative launch and its grid barrier, unless a
  // test forces the cooperative kernel or makes its barrier wait run out.
  const DebugKnobs& k = debug_knobs();
  const bool small = loss_small_eligible(bs, a.n) && k.loss_path != 2 && k.extra_arrivals == 0;
  cudaError_t e = small ? launch_loss_small(a, dt, has_kl, has_grad, (mode & PL_CLIP_TWO_SIDED) != 0, vec, stream)
                        : launch_loss(a, dt, has_kl, has_grad, (mode & PL_CLIP_TWO_SIDED) != 0, vec, stream);
  return e == cudaSuccess ? PL_OK : PL_ERR_CUDA;
}

}  // namespace pl

using namespace pl;

extern "C" {

pl_status pl_init(int64_t max_bs, pl_stream_t stream) {
  if (max_bs < 0) return PL_ERR_ARG;
  pl_status st = check_arch();
  if (st != PL_OK) return st;
  void* ws = nullptr;
  const size_t need = std::max(loss_ws_bytes(max_bs), reverse_kl_ws_bytes());
  return own_workspace(reinterpret_cast<cudaStream_t>(stream), need, &ws, true);
}

pl_status pl_loss(const void* policy_lp, const void* old_lp, const void* ref_lp, const void* adv,
                  const uint8_t* mask, int64_t bs, int64_t seq, float eps_lo, float eps_hi,
                  float beta, uint32_t mode, float* loss_out, void* grad_out, pl_stream_t stream) {
  DType dt;
  pl_status st = validate_loss(policy_lp, old_lp, ref_lp, adv, mask, bs, seq, eps_lo, eps_hi, beta,
                               mode, loss_out, &dt);
  if (st != PL_OK) return st;
  if ((st = check_arch()) != PL_OK) return st;
  void* ws = nullptr;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = own_workspace(s, loss_ws_bytes(bs), &ws, true)) != PL_OK) return st;
  return run_loss(policy_lp, old_lp, ref_lp, adv, mask, bs, seq, eps_lo, eps_hi, beta, mode, dt,
                  loss_out, grad_out, nullptr, nullptr, ws, s);
}

pl_status pl_loss_ex(const void* policy_lp, const void* old_lp, const void* ref_lp, const void* adv,
                     const uint8_t* mask, int64_t bs, int64_t seq, float eps_lo, float eps_hi,
                     float beta, uint32_t mode, float* loss_out, void* grad_out,
                     int64_t* n_valid_out, int64_t* row_valid_out, void* workspace,
                     size_t ws_bytes, pl_stream_t stream) {
  DType dt;
  pl_status st = validate_loss(policy_lp, old_lp, ref_lp, adv, mask, bs, seq, eps_lo, eps_hi, beta,
                               mode, loss_out, &dt);
  if (st != PL_OK) return st;
  if (!workspace || ws_bytes < loss_ws_bytes(bs) || !aligned(workspace, 256)) return PL_ERR_WORKSPACE;
  if ((st = check_arch()) != PL_OK) return st;
  return run_loss(policy_lp, old_lp, ref_lp, adv, mask, bs, seq, eps_lo, eps_hi, beta, mode, dt,
                  loss_out, grad_out, n_valid_out, row_valid_out, workspace,
                  reinterpret_cast<cudaStream_t>(stream));
}

size_t pl_loss_workspace_bytes(int64_t bs, int64_t seq) {
  (void)seq;
  return loss_ws_bytes(bs < 0 ? 0 : bs);
}

pl_status pl_device_status(const void* workspace, pl_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* ws = const_cast<void*>(workspace);
  if (!ws) {
    pl_status st = own_workspace(s, 0, &ws, false);
    if (st != PL_OK) return st;
    if (!ws) return PL_OK;  // pl_loss never ran on this (device, stream)
  }
  if (cudaStreamSynchronize(s) != cudaSuccess) return PL_ERR_CUDA;
  unsigned flag = 0;
  if (cudaMemcpy(&flag, ws, sizeof(flag), cudaMemcpyDeviceToHost) != cudaSuccess) return PL_ERR_CUDA;
  if (flag == 0) return PL_OK;
  if (cudaMemset(ws, 0, sizeof(flag)) != cudaSuccess) return PL_ERR_CUDA;
  if (flag & kDevErrTimeout) return PL_ERR_DEVICE_TIMEOUT;
  return PL_ERR_BAD_TARGET;
}

const char* pl_status_string(pl_status status) {
  switch (status) {
    case PL_OK: return "PL_OK";
    case PL_ERR_ARG: return "PL_ERR_ARG: invalid argument";
    case PL_ERR_DTYPE: return "PL_ERR_DTYPE: unsupported dtype";
    case PL_ERR_ALIGN: return "PL_ERR_ALIGN: row pitch not a multiple of 16 bytes";
    case PL_ERR_WORKSPACE: return "PL_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case PL_ERR_ARCH: return "PL_ERR_ARCH: device is not compute capability 10.0";
    case PL_ERR_CUDA: return "PL_ERR_CUDA: CUDA runtime error";
    case PL_ERR_DEVICE_TIMEOUT: return "PL_ERR_DEVICE_TIMEOUT: a bounded device wait ran out";
    case PL_ERR_BAD_TARGET: return "PL_ERR_BAD_TARGET: target id outside [0, V)";
  }
  return "unknown pl_status";
}

int pl_version(void) { return 100; }

}  // extern "C"
