// FP8 (E4M3) frame memory: quantisation of a record into its slot, and the
// widening of the stored codes into bfloat16 for the attention kernel.
//
// The buffer format follows the page of another system ("commaai/worldmodel-4B",
// README: its checkpoint keeps FP8 KV caches); the page names no scaling, so
// this library reads it as OCP FP8 E4M3 codes with one float32 scale per
// (block, head) for K and one for V: code = E4M3(x / scale), rounded to
// nearest even and saturated to +-448; the value a code stands for is
// code * scale.
//
// The attention reads the codes widened to bfloat16.  Every E4M3 value is a
// bfloat16 value (4 significant bits, exponents 2^-9 .. 2^8), so the widening
// is exact; the scales are applied by the attention kernel in float32 (K's to
// the softmax scale, V's to the output normalisation), so no rounding enters
// between the stored code and the arithmetic of the attention.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sm100_ptx.cuh"
#include "wmkv_internal.h"

namespace wmkv {

namespace {

constexpr int THREADS = 256;

// Two floats -> two E4M3 codes (round to nearest even, saturate to +-448,
// NaN -> NaN); `lo` lands in the low byte.
__device__ __forceinline__ uint16_t e4m3x2_from_f32(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two E4M3 codes (low byte first) -> their values as bfloat16x2 (exact: the
// conversion to half precision is exact, and so is half -> float -> bfloat16
// for values with 4 significant bits).
__device__ __forceinline__ uint32_t bf16x2_from_e4m3x2(uint16_t c) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  float lo, hi;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(h2));
  return pack_bf16x2(lo, hi);
}

// blockIdx.y selects K (0) or V (1).  Element group g holds elements
// [8g, 8g + 8) of a [rows, heads, d] array; d is a multiple of 8, so a group
// belongs to one head: (8g / d) mod heads.
__global__ void __launch_bounds__(THREADS) quantize_pair_kernel(
    const uint4* __restrict__ k_src, const uint4* __restrict__ v_src, uint2* __restrict__ k_dst,
    uint2* __restrict__ v_dst, int64_t n8, int heads, int d, const float* __restrict__ k_scale,
    const float* __restrict__ v_scale) {
  pdl_launch_dependents();
  pdl_wait_prior();
  const uint4* src = blockIdx.y ? v_src : k_src;
  uint2* dst = blockIdx.y ? v_dst : k_dst;
  const float* scale = blockIdx.y ? v_scale : k_scale;
  const int groups_per_head = d / 8;
  const int64_t stride = int64_t(gridDim.x) * THREADS;
  for (int64_t g = int64_t(blockIdx.x) * THREADS + threadIdx.x; g < n8; g += stride) {
    const float s = scale[(g / groups_per_head) % heads];
    const uint4 x = src[g];
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t out[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      uint16_t c[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint32_t pair = w[2 * i + j];
        const float a = __fdiv_rn(__uint_as_float(pair << 16), s);
        const float b = __fdiv_rn(__uint_as_float(pair & 0xFFFF0000u), s);
        c[j] = e4m3x2_from_f32(a, b);
      }
      out[i] = uint32_t(c[0]) | (uint32_t(c[1]) << 16);
    }
    dst[g] = make_uint2(out[0], out[1]);
  }
}

// blockIdx.y selects K (0) or V (1): 16 codes per thread and step.
__global__ void __launch_bounds__(THREADS) widen_pair_kernel(const uint4* __restrict__ k_codes,
                                                             const uint4* __restrict__ v_codes,
                                                             uint4* __restrict__ k_out,
                                                             uint4* __restrict__ v_out, int64_t n16) {
  pdl_launch_dependents();
  pdl_wait_prior();
  const uint4* src = blockIdx.y ? v_codes : k_codes;
  uint4* dst = blockIdx.y ? v_out : k_out;
  const int64_t stride = int64_t(gridDim.x) * THREADS;
  for (int64_t i = int64_t(blockIdx.x) * THREADS + threadIdx.x; i < n16; i += stride) {
    const uint4 c = src[i];
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    uint32_t o[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      o[2 * k] = bf16x2_from_e4m3x2(static_cast<uint16_t>(w[k] & 0xFFFFu));
      o[2 * k + 1] = bf16x2_from_e4m3x2(static_cast<uint16_t>(w[k] >> 16));
    }
    dst[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// The record write and the widening of one block's prefix in one pass
// (wm_write_attend on an FP8 memory).  Units of 8 values over [0, end) rows of
// K (blockIdx.y = 0) or V (1): units in [slot_lo, slot_hi) come from the
// caller's bf16 record -- quantised, stored as codes in the slot, and widened
// from those codes -- the others are widened from the codes in the buffer.
__global__ void __launch_bounds__(THREADS) store_widen_pair_kernel(
    const uint4* __restrict__ k_rec, const uint4* __restrict__ v_rec, uint2* __restrict__ k_codes,
    uint2* __restrict__ v_codes, uint4* __restrict__ k_out, uint4* __restrict__ v_out, int64_t n8,
    int64_t slot_lo, int64_t slot_hi, int heads, int d, const float* __restrict__ k_scale,
    const float* __restrict__ v_scale) {
  pdl_launch_dependents();
  pdl_wait_prior();
  const uint4* rec = blockIdx.y ? v_rec : k_rec;
  uint2* codes = blockIdx.y ? v_codes : k_codes;
  uint4* out = blockIdx.y ? v_out : k_out;
  const float* scale = blockIdx.y ? v_scale : k_scale;
  const int groups_per_head = d / 8;
  const int64_t stride = int64_t(gridDim.x) * THREADS;
  for (int64_t g = int64_t(blockIdx.x) * THREADS + threadIdx.x; g < n8; g += stride) {
    uint2 c;
    if (g >= slot_lo && g < slot_hi) {
      const float s = scale[(g / groups_per_head) % heads];
      const uint4 x = rec[g - slot_lo];
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
      uint32_t q[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        uint16_t h[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint32_t pair = w[2 * i + j];
          h[j] = e4m3x2_from_f32(__fdiv_rn(__uint_as_float(pair << 16), s),
                                 __fdiv_rn(__uint_as_float(pair & 0xFFFF0000u), s));
        }
        q[i] = uint32_t(h[0]) | (uint32_t(h[1]) << 16);
      }
      c = make_uint2(q[0], q[1]);
      codes[g] = c;
    } else {
      c = codes[g];
    }
    out[g] = make_uint4(bf16x2_from_e4m3x2(static_cast<uint16_t>(c.x & 0xFFFFu)),
                        bf16x2_from_e4m3x2(static_cast<uint16_t>(c.x >> 16)),
                        bf16x2_from_e4m3x2(static_cast<uint16_t>(c.y & 0xFFFFu)),
                        bf16x2_from_e4m3x2(static_cast<uint16_t>(c.y >> 16)));
  }
}

unsigned grid_for(int64_t units, int sms) {
  int64_t want = (units + THREADS - 1) / THREADS;
  const int64_t cap = int64_t(sms) * 8;
  if (want > cap) want = cap;
  return static_cast<unsigned>(want < 1 ? 1 : want);
}

}  // namespace

cudaError_t launch_quantize_pair(const void* k_src, const void* v_src, void* k_dst, void* v_dst,
                                 int64_t elems, int heads, int d, const float* k_scale,
                                 const float* v_scale, cudaStream_t stream) {
  if (elems <= 0) return cudaSuccess;
  if (elems % 8 != 0 || d % 8 != 0) return cudaErrorInvalidValue;
  const int64_t n8 = elems / 8;
  dim3 grid(grid_for(n8, device_sm_count()), 2);
  return launch_pdl(quantize_pair_kernel, grid, dim3(THREADS), 0, stream,
                    static_cast<const uint4*>(k_src), static_cast<const uint4*>(v_src),
                    static_cast<uint2*>(k_dst), static_cast<uint2*>(v_dst), n8, heads, d, k_scale,
                    v_scale);
}

cudaError_t launch_store_widen_pair(const void* k_rec, const void* v_rec, void* k_codes, void* v_codes,
                                    void* k_out, void* v_out, int64_t elems, int64_t slot_lo,
                                    int64_t slot_hi, int heads, int d, const float* k_scale,
                                    const float* v_scale, cudaStream_t stream) {
  if (elems <= 0) return cudaSuccess;
  if (elems % 8 || slot_lo % 8 || slot_hi % 8 || d % 8 || slot_lo < 0 || slot_hi < slot_lo ||
      slot_hi > elems)
    return cudaErrorInvalidValue;
  const int64_t n8 = elems / 8;
  dim3 grid(grid_for(n8, device_sm_count()), 2);
  return launch_pdl(store_widen_pair_kernel, grid, dim3(THREADS), 0, stream,
                    static_cast<const uint4*>(k_rec), static_cast<const uint4*>(v_rec),
                    static_cast<uint2*>(k_codes), static_cast<uint2*>(v_codes),
                    static_cast<uint4*>(k_out), static_cast<uint4*>(v_out), n8, slot_lo / 8,
                    slot_hi / 8, heads, d, k_scale, v_scale);
}

cudaError_t launch_widen_pair(const void* k_codes, const void* v_codes, void* k_out, void* v_out,
                              int64_t elems, cudaStream_t stream) {
  if (elems <= 0) return cudaSuccess;
  if (elems % 16 != 0) return cudaErrorInvalidValue;
  const int64_t n16 = elems / 16;
  dim3 grid(grid_for(n16, device_sm_count()), 2);
  return launch_pdl(widen_pair_kernel, grid, dim3(THREADS), 0, stream,
                    static_cast<const uint4*>(k_codes), static_cast<const uint4*>(v_codes),
                    static_cast<uint4*>(k_out), static_cast<uint4*>(v_out), n16);
}

}  // namespace wmkv
