// Dense FP8 attention for callers that cannot allocate device memory.
//
// wm_attend_dense_fp8 widens the E4M3 keys and values into bf16 scratch that
// the caller passes in.  Some callers cannot provide it: a plug-in or
// extension that is handed only the tensors of one call and has no allocator
// of its own, a host framework whose memory pool owns every device
// allocation and refuses allocations made behind its back, or a serving
// process that must not grow its device footprint (or take the
// synchronisation cudaMalloc and cudaFree can imply) once it is running.
// wm_attend_dense_fp8_static does the same work with the scratch in a fixed
// device array that belongs to this library.
//
// The array is a file-scope __device__ variable: every GPU that loads this
// library holds WM_FP8_STATIC_SCRATCH_BYTES of it until the process exits.
// In host code the array's name is only a host-side stand-in, not a device
// address, so this file asks the runtime for the array's device address once
// per device, with that device current, and hands that address to the
// kernels.
#include <cuda_runtime.h>

#include <mutex>

#include "wmkv.h"
#include "wmkv_internal.h"

namespace {

constexpr int64_t kStaticScratchBytes = WM_FP8_STATIC_SCRATCH_BYTES;

static __device__ __align__(256) uint8_t g_fp8_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_fp8_scratch on the current device, looked up the first
// time each device asks (with that device current); nullptr, with the CUDA
// error in *err, if the lookup failed.
uint8_t* static_scratch(cudaError_t* err) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *err = e != cudaSuccess ? e : cudaErrorInvalidDevice;
    return nullptr;
  }
  static std::once_flag once[kMaxDevices];
  static uint8_t* addr[kMaxDevices];
  static cudaError_t result[kMaxDevices];
  std::call_once(once[dev], [dev] {
    void* p = nullptr;
    result[dev] = cudaGetSymbolAddress(&p, g_fp8_scratch);
    addr[dev] = result[dev] == cudaSuccess ? static_cast<uint8_t*>(p) : nullptr;
  });
  *err = result[dev];
  return addr[dev];
}

}  // namespace

extern "C" {

int wm_attend_dense_fp8_static(const void* Q, const void* K8, const void* V8, const float* k_scale,
                               const float* v_scale, void* O, int64_t Lq, int64_t Lk, int heads,
                               int d, int* dev_status, wm_stream_t stream) {
  const int64_t need = wm_attend_dense_fp8_scratch_bytes(Lk, heads, d);
  if (need > kStaticScratchBytes) return WM_ERR_INVALID_ARG;
  cudaError_t e = cudaSuccess;
  uint8_t* scratch = static_scratch(&e);
  if (!scratch) return wmkv::note_cuda_error(e);
  // every byte the attention reads is written by the widening first, so the
  // previous call's contents need no clearing
  return wm_attend_dense_fp8(Q, K8, V8, k_scale, v_scale, O, Lq, Lk, heads, d, scratch,
                             kStaticScratchBytes, dev_status, stream);
}

}  // extern "C"
