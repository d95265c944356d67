// Self-check of the attention kernel's polynomial exponential: the same
// device function (exp2_poly2, sm100_ptx.cuh), applied to caller data, so a
// test can compare it with 2^x computed on the host.
#include <cuda_runtime.h>

#include "sm100_ptx.cuh"
#include "wmkv.h"
#include "wmkv_internal.h"

namespace {

__global__ void exp2_poly_kernel(const float2* __restrict__ x, float2* __restrict__ y, int64_t n2) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n2) return;
  const float2 v = x[i];
  float lo, hi;
  wmkv::f2_split(wmkv::exp2_poly2(wmkv::f2_make(v.x, v.y)), lo, hi);
  y[i] = make_float2(lo, hi);
}

}  // namespace

extern "C" int wm_selftest_exp2(const float* x, float* y, int64_t n, wm_stream_t stream) {
  if (!x || !y || n < 2 || (n & 1) || (reinterpret_cast<uintptr_t>(x) & 7) ||
      (reinterpret_cast<uintptr_t>(y) & 7) || n / 2 / 256 >= (int64_t(1) << 31))
    return WM_ERR_INVALID_ARG;
  const int64_t n2 = n / 2;
  exp2_poly_kernel<<<static_cast<unsigned>((n2 + 255) / 256), 256, 0,
                     reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const float2*>(x), reinterpret_cast<float2*>(y), n2);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? WM_OK : wmkv::note_cuda_error(e);
}
