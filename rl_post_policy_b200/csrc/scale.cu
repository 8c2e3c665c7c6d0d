// pl_scale: x *= *scale in place (device scalar, so no host synchronisation).
// Used by the autograd wrappers to apply the incoming gradient of a scalar loss
// to the gradient the fused forward+backward kernel already produced.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"

namespace pl {
namespace {

template <typename T>
__global__ void scale_kernel(T* x, int64_t n, const float* scale) {
  const float s = __ldg(scale);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    if constexpr (sizeof(T) == 4) {
      x[i] = x[i] * s;
    } else if constexpr (std::is_same<T, __half>::value) {
      x[i] = __float2half_rn(__half2float(x[i]) * s);
    } else {
      x[i] = __float2bfloat16_rn(__bfloat162float(x[i]) * s);
    }
  }
}

__global__ void count_ratio_kernel(const int64_t* local, const int64_t* global_, float* out) {
  const int64_t l = *local, g = *global_;
  out[0] = (float)((double)(l > 1 ? l : 1) / (double)(g > 1 ? g : 1));
}

}  // namespace
}  // namespace pl

using namespace pl;

extern "C" pl_status pl_scale(void* x, int64_t n, uint32_t mode, const float* scale, pl_stream_t stream) {
  if (n < 0 || (n > 0 && (!x || !scale))) return PL_ERR_ARG;
  if (mode & ~PL_DTYPE_MASK) return PL_ERR_ARG;
  const uint32_t d = (mode & PL_DTYPE_MASK) >> 4;
  if (d > 2) return PL_ERR_DTYPE;
  if (n == 0) return PL_OK;
  pl_status st = check_arch();
  if (st != PL_OK) return st;
  DevInfo di;
  if (dev_info(&di) != cudaSuccess) return PL_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t want = (n + 255) / 256;
  const unsigned grid = (unsigned)(want < (int64_t)di.sm_count * 8 ? want : (int64_t)di.sm_count * 8);
  launch_begin(2, s);
  if (d == 0) scale_kernel<float><<<grid, 256, 0, s>>>(static_cast<float*>(x), n, scale);
  else if (d == 1) scale_kernel<__half><<<grid, 256, 0, s>>>(static_cast<__half*>(x), n, scale);
  else scale_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<__nv_bfloat16*>(x), n, scale);
  launch_end(2, s);
  return cudaGetLastError() == cudaSuccess ? PL_OK : PL_ERR_CUDA;
}

extern "C" pl_status pl_count_ratio(const int64_t* local, const int64_t* global_, float* factor_out,
                                    pl_stream_t stream) {
  if (!local || !global_ || !factor_out) return PL_ERR_ARG;
  pl_status st = check_arch();
  if (st != PL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  launch_begin(2, s);
  count_ratio_kernel<<<1, 1, 0, s>>>(local, global_, factor_out);
  launch_end(2, s);
  return cudaGetLastError() == cudaSuccess ? PL_OK : PL_ERR_CUDA;
}
