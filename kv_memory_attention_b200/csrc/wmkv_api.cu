// C ABI of the frame memory: the host state machine (slot arithmetic, the
// filled prefix, call-order checks) and the launches behind it.
//
// Layout and rotation follow the model card "GTA world model: weights and
// inference code": section "A frame is a record" (R = H*W raw + X summary
// rows), "What a frame attends to" (Z0 whole, the last Y frames whole, older
// in-window frames as summaries) and "One buffer, no mask" (one buffer per
// block, | Z0 | RAW (Y+1) | SUM (W-Y) x X |, read = buffer[0:end], and the
// worked example: frame 31 over frame 28's RAW slot, frame 28's summary over
// frame 6's).  Frame t >= 1 uses RAW slot (t-1) mod (Y+1) and frame f's
// summary SUM slot (f-1) mod (W-Y): with this base the filled rows stay a
// contiguous prefix while the buffer fills.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <new>
#include <vector>

#include "wmkv.h"
#include "wmkv_internal.h"

struct wm_kvbuf {
  int device = 0;
  int blocks = 0, heads = 0, d = 0, grid_h = 0, grid_w = 0, X = 0, Y = 0, W = 0;
  int64_t HW = 0, R = 0, C = 0;
  int kv_format = WM_KV_BF16;
  int64_t row_bytes = 0;     // heads * d * (2 for bf16, 1 for E4M3 codes)
  int64_t tensor_bytes = 0;  // C * row_bytes (one K or V buffer)
  int64_t block_bytes = 0;   // 2 * tensor_bytes
  uint8_t* buf = nullptr;
  int* status = nullptr;     // device error word
  // E4M3 buffers: per (block, head) scales on the device (K for all blocks,
  // then V), and the bf16 widening of one block's filled prefix (K, then V)
  float* scales = nullptr;
  uint8_t* widened = nullptr;
  int64_t t = -1;            // current frame
  std::vector<int64_t> written;  // per block: frame of the latest write_record
  // streaming sink (start image keys follow the window)
  bool sink = false;
  std::vector<double> theta;   // per dimension pair, radians per frame (0: not temporal)
  int gap_trigger = 5, gap_target = 1;
  int64_t z0_pos = 0;          // temporal position of the start image
  unsigned long long wait_limit = wmkv::DEFAULT_WAIT_LIMIT_CYCLES;  // attention launches
  // scratch for attention launches that split their last wave's query tiles
  // by key range: part_ctas x 128 x (d + 2) floats (part_ctas = SM count)
  float* part = nullptr;
  int part_ctas = 0;
};

namespace {

thread_local char g_last_cuda[256] = "";

int cuda_fail(cudaError_t e) {
  std::snprintf(g_last_cuda, sizeof(g_last_cuda), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return WM_ERR_CUDA;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t capacity(int64_t hw, int64_t X, int64_t Y, int64_t W) {
  return (hw + X) * (Y + 2) + X * (W - Y);
}

int64_t end_at(int64_t hw, int64_t X, int64_t Y, int64_t W, int64_t t) {
  if (t < 0) return -1;
  const int64_t R = hw + X;
  const int64_t n_raw = t < Y + 1 ? t : Y + 1;
  int64_t n_sum = t - Y - 1;
  if (n_sum < 0) n_sum = 0;
  if (n_sum > W - Y) n_sum = W - Y;
  return R * (1 + n_raw) + X * n_sum;
}

int raw_slot(int64_t Y, int64_t t) { return t < 1 ? -1 : static_cast<int>((t - 1) % (Y + 1)); }

int sum_slot(int64_t Y, int64_t W, int64_t f) {
  return (f < 1 || W <= Y) ? -1 : static_cast<int>((f - 1) % (W - Y));
}

void sink_table(const wm_kvbuf* h, int64_t shift, wmkv::SinkTable* tab) {
  *tab = {};
  for (int i = 0; i < h->d / 2; ++i) {
    const double a = h->theta[i] * static_cast<double>(shift);
    tab->c[i] = static_cast<float>(std::cos(a));
    tab->s[i] = static_cast<float>(std::sin(a));
    if (h->theta[i] != 0.0) tab->mask |= 1ull << i;
  }
}

int64_t record_row(int64_t hw, int64_t X, int64_t Y, int64_t t) {
  if (t < 0) return -1;
  if (t == 0) return 0;
  return (hw + X) * (1 + raw_slot(Y, t));
}

}  // namespace

namespace wmkv {
// Records a CUDA error for wm_last_cuda_error and returns WM_ERR_CUDA (for
// entry points defined in other files).
int note_cuda_error(cudaError_t e) { return cuda_fail(e); }
}  // namespace wmkv

extern "C" {

static int kvbuf_create(wm_kvbuf** out, int blocks, int heads, int d, int grid_h, int grid_w, int X,
                        int Y, int W, int kv_format, const float* k_scale, const float* v_scale) {
  if (!out) return WM_ERR_INVALID_ARG;
  *out = nullptr;
  if (blocks < 1 || heads < 1 || heads > 65535 || grid_h < 1 || grid_w < 1 || X < 1 || Y < 0 ||
      W < Y)
    return WM_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return WM_ERR_UNSUPPORTED;
  const int elem_bytes = kv_format == WM_KV_E4M3 ? 1 : 2;
  if (kv_format == WM_KV_E4M3) {
    if (!k_scale || !v_scale) return WM_ERR_INVALID_ARG;
    for (int64_t i = 0; i < int64_t(blocks) * heads; ++i)
      if (!(k_scale[i] > 0.f) || !(v_scale[i] > 0.f) || !std::isfinite(k_scale[i]) ||
          !std::isfinite(v_scale[i]))
        return WM_ERR_INVALID_ARG;
  }
  const int64_t hw = int64_t(grid_h) * grid_w;
  const int64_t C = capacity(hw, X, Y, W);
  const int64_t row_bytes = int64_t(heads) * d * elem_bytes;
  // rows are addressed with 32-bit TMA coordinates
  if (C >= (int64_t(1) << 31) || hw + X >= (int64_t(1) << 31)) return WM_ERR_INVALID_ARG;
  const int64_t tensor_bytes = C * row_bytes;
  if (tensor_bytes / row_bytes != C || tensor_bytes > (int64_t(1) << 46) / (2 * int64_t(blocks)))
    return WM_ERR_INVALID_ARG;

  wm_kvbuf* h = new (std::nothrow) wm_kvbuf;
  if (!h) return WM_ERR_OOM;
  h->blocks = blocks;
  h->heads = heads;
  h->d = d;
  h->grid_h = grid_h;
  h->grid_w = grid_w;
  h->X = X;
  h->Y = Y;
  h->W = W;
  h->HW = hw;
  h->R = hw + X;
  h->C = C;
  h->kv_format = kv_format;
  h->row_bytes = row_bytes;
  h->tensor_bytes = tensor_bytes;
  h->block_bytes = 2 * tensor_bytes;
  h->written.assign(blocks, -1);

  auto fail = [h](cudaError_t e) -> int {
    cudaFree(h->buf);
    cudaFree(h->status);
    cudaFree(h->scales);
    cudaFree(h->widened);
    cudaFree(h->part);
    delete h;
    if (e == cudaErrorMemoryAllocation) {
      cudaGetLastError();
      return WM_ERR_OOM;
    }
    return cuda_fail(e);
  };
  cudaError_t e = cudaGetDevice(&h->device);
  if (e != cudaSuccess) return fail(e);
  const size_t total = size_t(h->block_bytes) * size_t(blocks);
  e = cudaMalloc(&h->buf, total);
  if (e == cudaSuccess) e = cudaMalloc(&h->status, sizeof(int));
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->part_ctas, cudaDevAttrMultiProcessorCount, h->device);
  if (e == cudaSuccess)
    e = cudaMalloc(&h->part, size_t(h->part_ctas) * 128 * (d + 2) * sizeof(float));

  if (e == cudaSuccess && kv_format == WM_KV_E4M3) {
    const size_t ns = size_t(blocks) * heads;
    e = cudaMalloc(&h->scales, 2 * ns * sizeof(float));
    if (e == cudaSuccess) e = cudaMemcpy(h->scales, k_scale, ns * sizeof(float), cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
      e = cudaMemcpy(h->scales + ns, v_scale, ns * sizeof(float), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMalloc(&h->widened, size_t(2) * C * heads * d * 2);
  }
  if (e == cudaSuccess) e = cudaMemset(h->buf, 0, total);
  if (e == cudaSuccess) e = cudaMemset(h->status, 0, sizeof(int));
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail(e);
  *out = h;
  return WM_OK;
}

int wm_kvbuf_create(wm_kvbuf** out, int blocks, int heads, int d, int grid_h, int grid_w, int X,
                    int Y, int W) {
  return kvbuf_create(out, blocks, heads, d, grid_h, grid_w, X, Y, W, WM_KV_BF16, nullptr, nullptr);
}

int wm_kvbuf_create_fp8(wm_kvbuf** out, int blocks, int heads, int d, int grid_h, int grid_w,
                        int X, int Y, int W, const float* k_scale, const float* v_scale) {
  return kvbuf_create(out, blocks, heads, d, grid_h, grid_w, X, Y, W, WM_KV_E4M3, k_scale, v_scale);
}

int wm_kv_format(const wm_kvbuf* h) { return h ? h->kv_format : WM_ERR_INVALID_ARG; }

int wm_kvbuf_destroy(wm_kvbuf* h) {
  if (!h) return WM_ERR_INVALID_ARG;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaSetDevice(h->device);
  cudaError_t e = cudaDeviceSynchronize();
  cudaFree(h->buf);
  cudaFree(h->status);
  cudaFree(h->scales);
  cudaFree(h->widened);
  cudaFree(h->part);
  cudaSetDevice(dev);
  delete h;
  return e == cudaSuccess ? WM_OK : cuda_fail(e);
}

// The handle's buffers live on the device that was current at creation; its
// kernels must be launched there (another device would read memory it does
// not own).
static bool on_handle_device(const wm_kvbuf* h) {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess && dev == h->device;
}

int wm_advance(wm_kvbuf* h, int64_t t, wm_stream_t stream) {
  if (!h) return WM_ERR_INVALID_ARG;
  if (t != h->t + 1 || !on_handle_device(h)) return WM_ERR_STATE;
  const int64_t f = t - h->Y - 1;  // frame leaving the raw window
  if (f >= 1 && h->W > h->Y) {
    const int64_t src_row = h->R * (1 + raw_slot(h->Y, f)) + h->HW;
    const int64_t dst_row = h->R * (h->Y + 2) + int64_t(h->X) * sum_slot(h->Y, h->W, f);
    const int64_t n16 = int64_t(h->X) * h->row_bytes / 16;
    cudaError_t e = wmkv::launch_evict(h->buf, h->blocks, h->block_bytes, h->tensor_bytes,
                                       src_row * h->row_bytes, dst_row * h->row_bytes, n16,
                                       reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (h->sink && t >= 1) {
    const int64_t oldest = t - h->W > 1 ? t - h->W : 1;  // oldest frame in memory
    const int64_t gap = oldest - h->z0_pos;
    if (gap >= h->gap_trigger) {
      const int64_t shift = gap - h->gap_target;
      wmkv::SinkTable tab;
      sink_table(h, shift, &tab);
      cudaError_t e = wmkv::launch_rotate_z0(h->buf, h->blocks, h->block_bytes, h->R, h->heads,
                                             h->d, tab, reinterpret_cast<cudaStream_t>(stream));
      if (e != cudaSuccess) return cuda_fail(e);
      h->z0_pos += shift;
    }
  }
  h->t = t;
  return WM_OK;
}

int wm_set_sink(wm_kvbuf* h, const float* theta, int n_pairs, int gap_trigger, int gap_target) {
  if (!h || !theta || n_pairs != h->d / 2 || gap_target < 0 || gap_trigger <= gap_target)
    return WM_ERR_INVALID_ARG;
  if (h->kv_format != WM_KV_BF16) return WM_ERR_UNSUPPORTED;
  if (h->t >= 0) return WM_ERR_STATE;
  h->theta.assign(theta, theta + n_pairs);
  h->gap_trigger = gap_trigger;
  h->gap_target = gap_target;
  h->z0_pos = 0;
  h->sink = true;
  return WM_OK;
}

int64_t wm_sink_position(const wm_kvbuf* h) { return h ? h->z0_pos : -1; }

int wm_sink_cos_sin(const wm_kvbuf* h, int64_t shift, float* c, float* s) {
  if (!h || !h->sink || !c || !s) return WM_ERR_INVALID_ARG;
  wmkv::SinkTable tab;
  sink_table(h, shift, &tab);
  for (int i = 0; i < h->d / 2; ++i) {
    c[i] = tab.c[i];
    s[i] = tab.s[i];
  }
  return WM_OK;
}

// Scales of block b (device): K's heads, V's heads.
static const float* block_k_scale(const wm_kvbuf* h, int b) { return h->scales + int64_t(b) * h->heads; }
static const float* block_v_scale(const wm_kvbuf* h, int b) {
  return h->scales + (int64_t(h->blocks) + b) * h->heads;
}

// Store a bf16 record [R, heads, d] into rows starting at row0 of block b.
static cudaError_t store_record(wm_kvbuf* h, int block, int64_t row0, const void* K, const void* V,
                                cudaStream_t s) {
  uint8_t* kdst = h->buf + int64_t(block) * h->block_bytes + row0 * h->row_bytes;
  uint8_t* vdst = kdst + h->tensor_bytes;
  if (h->kv_format == WM_KV_E4M3)
    return wmkv::launch_quantize_pair(K, V, kdst, vdst, h->R * h->heads * h->d, h->heads, h->d,
                                      block_k_scale(h, block), block_v_scale(h, block), s);
  return wmkv::launch_copy_pair(K, V, kdst, vdst, h->R * h->row_bytes / 16, s);
}

// Attention of Q over buffer[0:end] of block b; an E4M3 buffer is first
// widened into the handle's bf16 scratch and attended with its scales.
static cudaError_t attend_prefix(wm_kvbuf* h, int block, const void* Q, void* O, cudaStream_t s) {
  const int64_t end = end_at(h->HW, h->X, h->Y, h->W, h->t);
  const uint8_t* kbuf = h->buf + int64_t(block) * h->block_bytes;
  const uint8_t* vbuf = kbuf + h->tensor_bytes;
  if (h->kv_format == WM_KV_E4M3) {
    uint8_t* wk = h->widened;
    uint8_t* wv = h->widened + h->C * h->heads * h->d * 2;
    cudaError_t e = wmkv::launch_widen_pair(kbuf, vbuf, wk, wv, end * h->heads * h->d, s);
    if (e != cudaSuccess) return e;
    const wmkv::KVSegment seg = {wk, wv, end};
    return wmkv::launch_attend(Q, O, h->R, &seg, 1, h->heads, h->d, h->status, nullptr, h->wait_limit,
                               block_k_scale(h, block), block_v_scale(h, block), h->part,
                               h->part_ctas, s);
  }
  const wmkv::KVSegment seg = {kbuf, vbuf, end};
  return wmkv::launch_attend(Q, O, h->R, &seg, 1, h->heads, h->d, h->status, nullptr, h->wait_limit,
                             nullptr, nullptr, h->part, h->part_ctas, s);
}

int wm_write_record(wm_kvbuf* h, int block, int64_t t, const void* K, const void* V,
                    wm_stream_t stream) {
  if (!h || block < 0 || block >= h->blocks || !aligned16(K) || !aligned16(V))
    return WM_ERR_INVALID_ARG;
  if (h->t < 0 || t != h->t || !on_handle_device(h)) return WM_ERR_STATE;
  const int64_t row0 = record_row(h->HW, h->X, h->Y, t);
  cudaError_t e = store_record(h, block, row0, K, V, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  h->written[block] = t;
  return WM_OK;
}

int wm_attend(wm_kvbuf* h, int block, const void* Q, void* O, wm_stream_t stream) {
  if (!h || block < 0 || block >= h->blocks || !aligned16(Q) || !aligned16(O))
    return WM_ERR_INVALID_ARG;
  if (h->t < 0 || h->written[block] != h->t || !on_handle_device(h)) return WM_ERR_STATE;
  cudaError_t e = attend_prefix(h, block, Q, O, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return WM_OK;
}

int wm_set_wait_limit(wm_kvbuf* h, uint64_t cycles) {
  if (!h) return WM_ERR_INVALID_ARG;
  h->wait_limit = cycles;
  return WM_OK;
}

int wm_write_attend(wm_kvbuf* h, int block, int64_t t, const void* Q, const void* K,
                    const void* V, void* O, wm_stream_t stream) {
  if (!h || block < 0 || block >= h->blocks || !aligned16(Q) || !aligned16(K) || !aligned16(V) ||
      !aligned16(O))
    return WM_ERR_INVALID_ARG;
  if (h->t < 0 || t != h->t || !on_handle_device(h)) return WM_ERR_STATE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t row0 = record_row(h->HW, h->X, h->Y, t);
  uint8_t* kbuf = h->buf + int64_t(block) * h->block_bytes;
  uint8_t* vbuf = kbuf + h->tensor_bytes;
  uint8_t* kslot = kbuf + row0 * h->row_bytes;
  uint8_t* vslot = vbuf + row0 * h->row_bytes;
  const int64_t n16 = h->R * h->row_bytes / 16;
  const int64_t end = end_at(h->HW, h->X, h->Y, h->W, t);
  cudaError_t e;
  if (h->kv_format == WM_KV_E4M3) {
    // the attention must see the stored (quantised) record: one pass stores
    // the record's codes in the slot and widens the whole prefix (the record
    // from its own codes), then the attention reads the widened prefix
    h->written[block] = -1;
    const int64_t per_row = int64_t(h->heads) * h->d;
    uint8_t* wk = h->widened;
    uint8_t* wv = h->widened + h->C * per_row * 2;
    e = wmkv::launch_store_widen_pair(K, V, kbuf, vbuf, wk, wv, end * per_row, row0 * per_row,
                                      (row0 + h->R) * per_row, h->heads, h->d,
                                      block_k_scale(h, block), block_v_scale(h, block), s);
    const wmkv::KVSegment seg = {wk, wv, end};
    if (e == cudaSuccess)
      e = wmkv::launch_attend(Q, O, h->R, &seg, 1, h->heads, h->d, h->status, nullptr, h->wait_limit,
                              block_k_scale(h, block), block_v_scale(h, block), h->part,
                              h->part_ctas, s);
  } else if (wmkv::attend_copies_in_kernel(h->d)) {
    // keys: buffer rows before the slot, buffer rows after it, and the record
    // itself from the caller (the slot is being written by the same launch)
    wmkv::KVSegment segs[3];
    int nseg = 0;
    if (row0 > 0) segs[nseg++] = {kbuf, vbuf, row0};
    const int64_t after = row0 + h->R;
    if (end > after)
      segs[nseg++] = {kbuf + after * h->row_bytes, vbuf + after * h->row_bytes, end - after};
    segs[nseg++] = {K, V, h->R};
    const wmkv::RecordCopy cp = {K, V, kslot, vslot, n16};
    e = wmkv::launch_attend(Q, O, h->R, segs, nseg, h->heads, h->d, h->status, &cp, h->wait_limit,
                            nullptr, nullptr, h->part, h->part_ctas, s);
  } else {
    e = wmkv::launch_copy_pair(K, V, kslot, vslot, n16, s);
    const wmkv::KVSegment seg = {kbuf, vbuf, end};
    if (e == cudaSuccess)
      e = wmkv::launch_attend(Q, O, h->R, &seg, 1, h->heads, h->d, h->status, nullptr,
                              h->wait_limit, nullptr, nullptr, h->part, h->part_ctas, s);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  h->written[block] = t;
  return WM_OK;
}

int64_t wm_end(const wm_kvbuf* h) { return h ? end_at(h->HW, h->X, h->Y, h->W, h->t) : -1; }
int64_t wm_capacity(const wm_kvbuf* h) { return h ? h->C : -1; }
int64_t wm_current_frame(const wm_kvbuf* h) { return h ? h->t : -1; }
int wm_raw_slot(const wm_kvbuf* h, int64_t t) { return h ? raw_slot(h->Y, t) : -1; }
int wm_sum_slot(const wm_kvbuf* h, int64_t f) { return h ? sum_slot(h->Y, h->W, f) : -1; }

int wm_kv_ptrs(const wm_kvbuf* h, int block, void** K, void** V) {
  if (!h || block < 0 || block >= h->blocks || !K || !V) return WM_ERR_INVALID_ARG;
  *K = h->buf + int64_t(block) * h->block_bytes;
  *V = h->buf + int64_t(block) * h->block_bytes + h->tensor_bytes;
  return WM_OK;
}

int wm_sync_status(wm_kvbuf* h) {
  if (!h) return WM_ERR_INVALID_ARG;
  // on the handle's device; the caller's current device is restored
  int prev = 0;
  cudaError_t e = cudaGetDevice(&prev);
  if (e == cudaSuccess && prev != h->device) e = cudaSetDevice(h->device);
  if (e != cudaSuccess) return cuda_fail(e);
  int flag = 0;
  e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&flag, h->status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && flag != wmkv::DEV_OK) e = cudaMemset(h->status, 0, sizeof(int));
  if (prev != h->device) cudaSetDevice(prev);
  if (e != cudaSuccess) return cuda_fail(e);
  return flag != wmkv::DEV_OK ? WM_ERR_TIMEOUT : WM_OK;
}

const char* wm_strerror(int code) {
  switch (code) {
    case WM_OK: return "ok";
    case WM_ERR_INVALID_ARG: return "invalid argument";
    case WM_ERR_STATE: return "call out of order";
    case WM_ERR_UNSUPPORTED: return "unsupported shape";
    case WM_ERR_OOM: return "device allocation failed";
    case WM_ERR_CUDA: return "CUDA error";
    case WM_ERR_TIMEOUT: return "kernel gave up a bounded wait";
    default: return "unknown error";
  }
}

const char* wm_last_cuda_error(void) { return g_last_cuda; }

int64_t wm_layout_capacity(int grid_h, int grid_w, int X, int Y, int W) {
  if (grid_h < 1 || grid_w < 1 || X < 1 || Y < 0 || W < Y) return -1;
  return capacity(int64_t(grid_h) * grid_w, X, Y, W);
}

int64_t wm_layout_end(int grid_h, int grid_w, int X, int Y, int W, int64_t t) {
  if (grid_h < 1 || grid_w < 1 || X < 1 || Y < 0 || W < Y) return -1;
  return end_at(int64_t(grid_h) * grid_w, X, Y, W, t);
}

int wm_layout_raw_slot(int Y, int64_t t) { return Y < 0 ? -1 : raw_slot(Y, t); }

int wm_layout_sum_slot(int Y, int W, int64_t f) {
  return (Y < 0 || W < Y) ? -1 : sum_slot(Y, W, f);
}

int64_t wm_layout_record_row(int grid_h, int grid_w, int X, int Y, int64_t t) {
  if (grid_h < 1 || grid_w < 1 || X < 1 || Y < 0) return -1;
  return record_row(int64_t(grid_h) * grid_w, X, Y, t);
}

int wm_attend_dense(const void* Q, const void* K, const void* V, void* O, int64_t Lq, int64_t Lk,
                    int heads, int d, int* dev_status, wm_stream_t stream) {
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || Lq < 1 || Lk < 1 ||
      heads < 1 || Lq >= (int64_t(1) << 31) || Lk >= (int64_t(1) << 31))
    return WM_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return WM_ERR_UNSUPPORTED;
  if ((Lq + 127) / 128 > 0x7FFFFFFF || heads > 65535) return WM_ERR_INVALID_ARG;
  const wmkv::KVSegment seg = {K, V, Lk};
  cudaError_t e = wmkv::launch_attend(Q, O, Lq, &seg, 1, heads, d, dev_status, nullptr,
                                      wmkv::DEFAULT_WAIT_LIMIT_CYCLES, nullptr, nullptr, nullptr, 0,
                                      reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return WM_OK;
}

int64_t wm_attend_dense_fp8_scratch_bytes(int64_t Lk, int heads, int d) {
  if (Lk < 1 || heads < 1 || (d != 64 && d != 128)) return -1;
  return 2 * Lk * heads * d * 2;
}

int wm_attend_dense_fp8(const void* Q, const void* K8, const void* V8, const float* k_scale,
                        const float* v_scale, void* O, int64_t Lq, int64_t Lk, int heads, int d,
                        void* scratch, int64_t scratch_bytes, int* dev_status, wm_stream_t stream) {
  if (!aligned16(Q) || !aligned16(K8) || !aligned16(V8) || !aligned16(O) || !aligned16(scratch) ||
      !k_scale || !v_scale || Lq < 1 || Lk < 1 || heads < 1 || heads > 65535 ||
      Lq >= (int64_t(1) << 31) || Lk >= (int64_t(1) << 31))
    return WM_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return WM_ERR_UNSUPPORTED;
  if (scratch_bytes < wm_attend_dense_fp8_scratch_bytes(Lk, heads, d)) return WM_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* wk = static_cast<uint8_t*>(scratch);
  uint8_t* wv = wk + Lk * heads * d * 2;
  cudaError_t e = wmkv::launch_widen_pair(K8, V8, wk, wv, Lk * heads * d, s);
  const wmkv::KVSegment seg = {wk, wv, Lk};
  if (e == cudaSuccess)
    e = wmkv::launch_attend(Q, O, Lq, &seg, 1, heads, d, dev_status, nullptr,
                            wmkv::DEFAULT_WAIT_LIMIT_CYCLES, k_scale, v_scale, nullptr, 0, s);
  if (e != cudaSuccess) return cuda_fail(e);
  return WM_OK;
}

}  // extern "C"
