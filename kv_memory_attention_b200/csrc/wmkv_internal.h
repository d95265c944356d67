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

// A run of keys: rows [0, rows) of K and V arrays whose rows are `heads*d`
// bf16 values.
struct KVSegment {
  const void* k;
  const void* v;
  int64_t rows;
};
// A record copy the attention launch performs on the side (K and V, n16
// 16-byte units each).
struct RecordCopy {
  const void* k_src;
  const void* v_src;
  void* k_dst;
  void* v_dst;
  int64_t n16;
};

// Dense flash attention of Q [lq, heads, d] over the keys of 1..3 segments
// (softmax over all of them together), O [lq, heads, d]: see attend_sm100.cu.
// `copy` (may be null) is performed by the same launch; only supported where
// attend_copies_in_kernel(d).  Returns a cudaError_t from encoding/launching.
// Bound on each wait inside an attention launch, in SM cycles (about 2 s at
// the 1.965 GHz maximum clock).
constexpr unsigned long long DEFAULT_WAIT_LIMIT_CYCLES = 4000000000ull;

// k_scale / v_scale (device, one float per head, may be null): the keys and
// values are the stored numbers times their head's scale (FP8 buffers).
//
// part (device, part_ctas x 128 x (d + 2) floats, may be null): scratch that
// lets a launch of more than one wave of CTAs split the query tiles of its
// last, partial wave by key range (a second, combine launch follows); null
// keeps one CTA per (query tile, head).
cudaError_t launch_attend(const void* q, void* o, int64_t lq, const KVSegment* segs, int nseg,
                          int heads, int d, int* status, const RecordCopy* copy,
                          unsigned long long wait_limit, const float* k_scale,
                          const float* v_scale, float* part, int part_ctas, cudaStream_t stream);
bool attend_copies_in_kernel(int d);

// Keeps the CUDA error's text for wm_last_cuda_error; returns WM_ERR_CUDA.
int note_cuda_error(cudaError_t e);

// SM count of the current device (queried once per device).
int device_sm_count();

// FP8 (E4M3) buffers.  Quantise `elems` bf16 values of K and of V ([rows,
// heads, d], elems a multiple of 8) into codes with one scale per head
// (device arrays of `heads` floats): code = E4M3(x / scale), round to nearest
// even, saturate to +-448.
cudaError_t launch_quantize_pair(const void* k_src, const void* v_src, void* k_dst, void* v_dst,
                                 int64_t elems, int heads, int d, const float* k_scale,
                                 const float* v_scale, cudaStream_t stream);
// Both in one pass over `elems` values of K and of V: values [slot_lo,
// slot_hi) come from the bf16 record (quantised into k_codes/v_codes there),
// the rest from the codes already stored; all are widened into k_out/v_out.
// elems, slot_lo and slot_hi are multiples of 8.
cudaError_t launch_store_widen_pair(const void* k_rec, const void* v_rec, void* k_codes, void* v_codes,
                                    void* k_out, void* v_out, int64_t elems, int64_t slot_lo,
                                    int64_t slot_hi, int heads, int d, const float* k_scale,
                                    const float* v_scale, cudaStream_t stream);
// Widen `elems` E4M3 codes of K and of V (elems a multiple of 16) to the
// bfloat16 values they hold (exact).
cudaError_t launch_widen_pair(const void* k_codes, const void* v_codes, void* k_out, void* v_out,
                              int64_t elems, cudaStream_t stream);

// Copy `n16` 16-byte chunks of a and b (two independent arrays) in one launch.
cudaError_t launch_copy_pair(const void* a_src, const void* b_src, void* a_dst, void* b_dst,
                             int64_t n16, cudaStream_t stream);

// Rotation of adjacent dimension pairs (at most 64 per head row).
struct SinkTable {
  float c[64];
  float s[64];
  unsigned long long mask;  // bit i: pair i turns
};
// Z0 key rotation in every block: rows [0, rows) of the K buffer at
// base + b*block_stride_bytes.
cudaError_t launch_rotate_z0(void* base, int blocks, int64_t block_stride_bytes, int64_t rows,
                             int heads, int d, const SinkTable& tab, cudaStream_t stream);

// RAW -> SUM eviction in every block of one allocation.
//   base: the allocation; block b's K buffer at base + b*block_stride_bytes,
//   its V buffer at + tensor_stride_bytes.  Copies `n16` chunks from
//   src_off_bytes to dst_off_bytes inside each of the 2*blocks buffers.
cudaError_t launch_evict(void* base, int blocks, int64_t block_stride_bytes,
                         int64_t tensor_stride_bytes, int64_t src_off_bytes,
                         int64_t dst_off_bytes, int64_t n16, cudaStream_t stream);

}  // namespace wmkv
