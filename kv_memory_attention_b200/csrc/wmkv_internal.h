// Internal declarations shared by the library's translation units.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include <utility>

namespace wmkv {

// Launch `kernel` on `stream` with programmatic stream serialization: the
// kernel may start while its predecessor finishes; every kernel of this
// library executes griddepcontrol.wait before its first global memory access,
// so stream order is preserved for all data.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
#ifndef WMKV_NO_PDL
  cfg.numAttrs = 1;
#else
  cfg.numAttrs = 0;
#endif
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Device-side error word values (written by kernels, read by the host).
constexpr int DEV_OK = 0;
constexpr int DEV_TIMEOUT = 1;

// Dense flash attention over keys [0, lk): see attend_sm100.cu.
// Q/O: [lq, heads, d]; K/V: rows [0, lk) of arrays whose rows are `heads*d`
// bf16 values.  Returns a cudaError_t from encoding/launching.
cudaError_t launch_attend(const void* q, const void* k, const void* v, void* o, int64_t lq,
                          int64_t lk, int heads, int d, int* status, cudaStream_t stream);

// Copy `n16` 16-byte chunks of a and b (two independent arrays) in one launch.
cudaError_t launch_copy_pair(const void* a_src, const void* b_src, void* a_dst, void* b_dst,
                             int64_t n16, cudaStream_t stream);

// RAW -> SUM eviction in every block of one allocation.
//   base: the allocation; block b's K buffer at base + b*block_stride_bytes,
//   its V buffer at + tensor_stride_bytes.  Copies `n16` chunks from
//   src_off_bytes to dst_off_bytes inside each of the 2*blocks buffers.
cudaError_t launch_evict(void* base, int blocks, int64_t block_stride_bytes,
                         int64_t tensor_stride_bytes, int64_t src_off_bytes,
                         int64_t dst_off_bytes, int64_t n16, cudaStream_t stream);

}  // namespace wmkv
