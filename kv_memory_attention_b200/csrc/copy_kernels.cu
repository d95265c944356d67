// Record write and RAW -> SUM eviction: HBM-bound bit copies.
//
// Model card "GTA world model: weights and inference code", section "One
// buffer, no mask": every pass stores the current frame's record in its slot;
// a frame that drops out of the raw window keeps only its X summary rows (K
// and V), moved from its RAW slot into SUM.  The page counts this small
// per-block row copy as the whole price of long-term memory.
//
// Both are contiguous copies in the token-major buffer layout, moved as
// 16-byte vectors with several independent loads in flight per thread and a
// grid sized to the SM count.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "sm100_ptx.cuh"
#include "wmkv_internal.h"

namespace wmkv {

namespace {

constexpr int COPY_THREADS = 256;
constexpr int UNROLL = 4;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void copy_span(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                          int64_t n, int64_t first, int64_t stride) {
  for (int64_t i = first; i < n; i += stride * UNROLL) {
    uint4 r[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t idx = i + u * stride;
      if (idx < n) r[u] = ld_stream(src + idx);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t idx = i + u * stride;
      if (idx < n) dst[idx] = r[u];
    }
  }
}

// blockIdx.y selects array a (0) or b (1).
__global__ void __launch_bounds__(COPY_THREADS) copy_pair_kernel(const uint4* __restrict__ a_src,
                                                                 const uint4* __restrict__ b_src,
                                                                 uint4* __restrict__ a_dst,
                                                                 uint4* __restrict__ b_dst,
                                                                 int64_t n) {
  pdl_launch_dependents();
  pdl_wait_prior();
  const uint4* src = blockIdx.y ? b_src : a_src;
  uint4* dst = blockIdx.y ? b_dst : a_dst;
  const int64_t stride = int64_t(gridDim.x) * COPY_THREADS;
  copy_span(src, dst, n, int64_t(blockIdx.x) * COPY_THREADS + threadIdx.x, stride);
}

// blockIdx.y = 2*block + tensor (0 = K, 1 = V).
__global__ void __launch_bounds__(COPY_THREADS) evict_kernel(uint8_t* base, int64_t block_stride,
                                                             int64_t tensor_stride, int64_t src_off,
                                                             int64_t dst_off, int64_t n) {
  pdl_launch_dependents();
  pdl_wait_prior();
  uint8_t* buf = base + int64_t(blockIdx.y >> 1) * block_stride + int64_t(blockIdx.y & 1) * tensor_stride;
  const uint4* src = reinterpret_cast<const uint4*>(buf + src_off);
  uint4* dst = reinterpret_cast<uint4*>(buf + dst_off);
  const int64_t stride = int64_t(gridDim.x) * COPY_THREADS;
  copy_span(src, dst, n, int64_t(blockIdx.x) * COPY_THREADS + threadIdx.x, stride);
}

// Start image keys moved forward in time (model card "GTA world model:
// weights and inference code", section "Running for a long time: the start
// image follows the window"): RoPE keys are rotations, so multiplying a stored
// key by one more rotation moves it forward; only the keys of the start
// image (Z0 rows of every block's K buffer) change, in place.
// Adjacent dimension pairs (2i, 2i+1) of each head turn by (c_i, s_i) as
// complex numbers, in float32 with every product and sum rounded separately
// (no fused multiply-add), then to bf16; pairs whose bit in `mask` is clear
// are left untouched.  One thread per 16-byte vector (4 pairs).
__global__ void __launch_bounds__(COPY_THREADS) rotate_z0_kernel(uint8_t* base, int64_t block_stride,
                                                                 int64_t vec_per_block,
                                                                 int vec_per_row_head,
                                                                 SinkTable tab) {
  pdl_launch_dependents();
  pdl_wait_prior();
  const int64_t i = int64_t(blockIdx.x) * COPY_THREADS + threadIdx.x;
  if (i >= vec_per_block) return;
  uint4* v = reinterpret_cast<uint4*>(base + int64_t(blockIdx.y) * block_stride) + i;
  const int pair0 = static_cast<int>(i % vec_per_row_head) * 4;
  uint4 x = *v;
  uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int pr = pair0 + k;
    if (!((tab.mask >> pr) & 1ull)) continue;
    const float a = __uint_as_float(w[k] << 16);
    const float b = __uint_as_float(w[k] & 0xFFFF0000u);
    const float c = tab.c[pr], s = tab.s[pr];
    const float na = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
    const float nb = __fadd_rn(__fmul_rn(a, s), __fmul_rn(b, c));
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(na));
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(nb));
    w[k] = lo | (hi << 16);
  }
  *v = make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace

// SM count of the current device (queried once per device, thread-safe).
int device_sm_count() {
  constexpr int MAX_DEVICES = 64;
  static std::once_flag once[MAX_DEVICES];
  static int count[MAX_DEVICES];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return 148;
  std::call_once(once[dev], [dev] {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    count[dev] = n;
  });
  return count[dev];
}

namespace {

unsigned grid_x_for(int64_t n16, int parallel_arrays) {
  // enough CTAs for every vector to be touched once with UNROLL in flight,
  // capped at a few waves of the SM count across all arrays
  const int64_t per_cta = int64_t(COPY_THREADS) * UNROLL;
  int64_t want = (n16 + per_cta - 1) / per_cta;
  const int64_t cap = (int64_t(device_sm_count()) * 8 + parallel_arrays - 1) / parallel_arrays;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  return static_cast<unsigned>(want);
}

}  // namespace

cudaError_t launch_copy_pair(const void* a_src, const void* b_src, void* a_dst, void* b_dst,
                             int64_t n16, cudaStream_t stream) {
  if (n16 <= 0) return cudaSuccess;
  dim3 grid(grid_x_for(n16, 2), 2);
  return launch_pdl(copy_pair_kernel, grid, dim3(COPY_THREADS), 0, stream,
                    static_cast<const uint4*>(a_src), static_cast<const uint4*>(b_src),
                    static_cast<uint4*>(a_dst), static_cast<uint4*>(b_dst), n16);
}

cudaError_t launch_rotate_z0(void* base, int blocks, int64_t block_stride_bytes, int64_t rows,
                             int heads, int d, const SinkTable& tab, cudaStream_t stream) {
  const int64_t vec_per_row_head = d / 8;
  const int64_t vec_per_block = rows * heads * vec_per_row_head;
  if (vec_per_block <= 0 || blocks <= 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>((vec_per_block + COPY_THREADS - 1) / COPY_THREADS),
            static_cast<unsigned>(blocks));
  return launch_pdl(rotate_z0_kernel, grid, dim3(COPY_THREADS), 0, stream,
                    static_cast<uint8_t*>(base), block_stride_bytes, vec_per_block,
                    static_cast<int>(vec_per_row_head), tab);
}

cudaError_t launch_evict(void* base, int blocks, int64_t block_stride_bytes,
                         int64_t tensor_stride_bytes, int64_t src_off_bytes, int64_t dst_off_bytes,
                         int64_t n16, cudaStream_t stream) {
  if (n16 <= 0 || blocks <= 0) return cudaSuccess;
  dim3 grid(grid_x_for(n16, 2 * blocks), static_cast<unsigned>(2 * blocks));
  return launch_pdl(evict_kernel, grid, dim3(COPY_THREADS), 0, stream, static_cast<uint8_t*>(base),
                    block_stride_bytes, tensor_stride_bytes, src_off_bytes, dst_off_bytes, n16);
}

}  // namespace wmkv
