/*
 * wmkv.h -- Summaryformer frame memory and the attention that reads it, on B200 (sm_100a).
 *
 * Source of the method: the model card "GTA world model: weights and inference
 * code" (lucidml/gta), sections "A frame is a record", "What a frame attends
 * to" and "One buffer, no mask".
 *
 * Every block of the model keeps ONE preallocated key buffer and ONE value
 * buffer, each laid out by rows as
 *
 *     | Z0: record(0) | RAW: (Y+1) rotating records | SUM: (W-Y) x X rotating summary rows |
 *
 * where a record is the frame's H*W raw tokens followed by its X summary
 * tokens (R = H*W + X rows).  A row is `heads x d` bfloat16 values, row-major
 * (token-major: element (row, h, c) sits at ((row*heads)+h)*d + c).
 * Capacity C = R*(Y+2) + X*(W-Y) rows.  Slot conventions (they reproduce the
 * page's served-shape example: frame 31 reuses frame 28's RAW slot, and frame
 * 28's summary lands in the SUM slot that held frame 6's):
 *   - frame 0 is written into Z0 and never evicted;
 *   - frame t >= 1 is written into RAW slot (t-1) mod (Y+1);
 *   - at the start of frame t >= Y+2, frame f = t-Y-1 leaves the raw window:
 *     the K and V of its X summary rows are copied into SUM slot (f-1) mod (W-Y);
 *   - attention reads buffer[0:end], the filled prefix, with no mask:
 *     end(t) = R*(1 + min(t, Y+1)) + X*min(max(t-Y-1, 0), W-Y).
 *
 * Calls are asynchronous on the given CUDA stream (wm_stream_t is the same
 * type as cudaStream_t; NULL is the legacy default stream).  Host-side
 * checks run first: a call that fails them returns an error code and
 * launches nothing.  Device pointers passed in (Q, K, V, O) are owned by the
 * caller, must be 16-byte aligned, and must stay valid until the stream
 * reaches the call; the library keeps no reference to them afterwards.
 *
 * A handle belongs to the CUDA device that was current when it was created:
 * wm_advance, wm_write_record, wm_attend and wm_write_attend return
 * WM_ERR_STATE unless that device is current (and the stream belongs to it).
 * A handle is used by one host thread at a time.  Beyond the handles, the
 * library keeps only one-time set-up done by the first call of each kind
 * (kernel attributes, the driver's tensor-map encoder), guarded for threads.
 * wm_advance, wm_write_record, wm_attend and wm_write_attend make no
 * synchronous CUDA call and allocate nothing, so once each has run once
 * outside a capture, a sequence of them can be captured into a CUDA graph;
 * the graph replays exactly the launches of that sequence, with its frame
 * numbers (the slot pattern repeats every lcm(Y+1, W-Y) frames).
 */
#ifndef WMKV_H
#define WMKV_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define WM_API __attribute__((visibility("default")))
#else
#define WM_API
#endif

typedef struct CUstream_st* wm_stream_t;
typedef struct wm_kvbuf wm_kvbuf;

/* Error codes. */
enum {
  WM_OK = 0,
  WM_ERR_INVALID_ARG = -1,  /* bad argument: range, NULL or misaligned pointer  */
  WM_ERR_STATE = -2,        /* call out of order (see each call)                 */
  WM_ERR_UNSUPPORTED = -3,  /* shape the kernels do not implement (d not 64/128) */
  WM_ERR_OOM = -4,          /* device allocation failed                          */
  WM_ERR_CUDA = -5,         /* a CUDA runtime call or launch failed              */
  WM_ERR_TIMEOUT = -6       /* a kernel gave up a bounded wait (device flag)     */
};

/* Create the memory of one session: `blocks` per-block K/V buffer pairs on the
 * current CUDA device.  Defined by the model card, section "One buffer, no
 * mask" (one preallocated buffer per block, | Z0 | RAW (Y+1) records | SUM
 * (W-Y) x X summary rows |, capacity C = R*(Y+2) + X*(W-Y) rows: 6,528 at the
 * served 24x42 grid with X = 96, Y = 2, W = 24) and section "A frame is a
 * record" (R = grid_h*grid_w raw rows followed by X summary rows).
 * Buffers are zero-filled, in one allocation of
 * blocks * 2 * C * heads * d * 2 bytes (block b's K buffer first, then its V).
 * The handle also holds a scratch of (SM count) * 128 * (d + 2) floats: an
 * attention launch of more than one wave of (query tile, head) CTAs whose
 * last wave is at most half full splits that wave's query tiles by key range
 * and merges the partial results in a second launch.  Attention calls on one
 * handle whose launches can overlap on the device (different streams with no
 * event between them) may share that scratch and must be ordered.
 * Requirements: blocks >= 1, heads >= 1, d in {64, 128}, grid_h >= 1,
 * grid_w >= 1, X >= 1, 0 <= Y <= W (W == Y gives an empty SUM region).
 * Returns WM_ERR_INVALID_ARG / WM_ERR_UNSUPPORTED before touching the device,
 * WM_ERR_OOM or WM_ERR_CUDA if allocation fails.  *out receives the handle. */
WM_API int wm_kvbuf_create(wm_kvbuf** out, int blocks, int heads, int d, int grid_h, int grid_w, int X,
                    int Y, int W);

/* Storage formats of a session's buffers (wm_kv_format). */
enum { WM_KV_BF16 = 0, WM_KV_E4M3 = 1 };

/* The same memory with K and V stored as FP8 E4M3 codes, one byte per value.
 * The page of another system ("commaai/worldmodel-4B", README) says its
 * checkpoint keeps FP8 KV caches and names no scaling; this library reads
 * that as OCP FP8 E4M3 (sign, 4 exponent bits with bias 7, 3 mantissa bits,
 * subnormals, no infinities, largest finite 448) with one float32 scale per
 * (block, head) for K and one for V: k_scale[block * heads + h], likewise
 * v_scale, host arrays of blocks * heads positive finite floats, copied.
 * wm_write_record / wm_write_attend store code = E4M3(x / scale) (float32
 * division, round to nearest even, saturated to +-448, NaN kept);
 * wm_advance moves codes; wm_attend attends over code * scale, i.e. exactly
 * the dequantised prefix (the codes are widened to bf16 in the handle's
 * scratch, 2 * C * heads * d * 2 bytes allocated here, and the scales enter
 * in float32: K's with the softmax scale, V's with the output
 * normalisation).  wm_write_attend is two launches: one stores the record's
 * codes in its slot and widens the block's prefix, one attends.
 * Calls on one E4M3 handle must be ordered on the device (one stream, or
 * events between streams): they share its scratch.  wm_set_sink returns
 * WM_ERR_UNSUPPORTED for this format.  Other arguments and errors as for
 * wm_kvbuf_create; WM_ERR_INVALID_ARG for a missing or non-positive scale. */
WM_API int wm_kvbuf_create_fp8(wm_kvbuf** out, int blocks, int heads, int d, int grid_h,
                               int grid_w, int X, int Y, int W, const float* k_scale,
                               const float* v_scale);

/* WM_KV_BF16 or WM_KV_E4M3; WM_ERR_INVALID_ARG for a NULL handle. */
WM_API int wm_kv_format(const wm_kvbuf* h);

/* Free the buffers and the handle (synchronises the device first). */
WM_API int wm_kvbuf_destroy(wm_kvbuf* h);

/* Start frame t (section "One buffer, no mask": a frame that leaves the raw
 * window keeps only its X summary rows, moved RAW -> SUM).  t must be 0, then 1, 2, ...
 * one call each, else WM_ERR_STATE.  For t >= Y+2 (and W > Y) one launch
 * copies frame t-Y-1's X summary rows of K and of V into SUM, in every block. */
WM_API int wm_advance(wm_kvbuf* h, int64_t t, wm_stream_t stream);

/* Write frame t's record of `block` ("A frame is a record"): K and V are
 * device arrays [R, heads, d] bf16 (raw rows first, then the X summary rows).
 * t must equal the frame last passed to wm_advance (else WM_ERR_STATE).
 * Frame 0 goes to Z0, frame t >= 1 to RAW slot (t-1) mod (Y+1).  May be called
 * several times per frame (denoising passes, then the clean rewrite). */
WM_API int wm_write_record(wm_kvbuf* h, int block, int64_t t, const void* K, const void* V,
                    wm_stream_t stream);

/* Dense unmasked attention of frame t's queries over buffer[0:end] of `block`
 * (model card, section "One buffer, no mask": every query of the frame being
 * generated attends to the whole filled prefix of its block's buffer, with no
 * mask, because the buffer holds exactly the keys the frame may see; section
 * "The rest of the model", Attention kernels, for the ordinary 1/sqrt(d)
 * softmax of the kernels it names):
 *   O[i,h,:] = sum_j softmax_j(Q[i,h,:] . K[j,h,:] / sqrt(d)) V[j,h,:],  j < end.
 * Q and O are device arrays [R, heads, d] bf16.  Scores, softmax and the
 * accumulation are fp32 on the tensor cores (P rounded to bf16 for P.V); O is
 * rounded to bf16.  Requires a wm_write_record(block, t) at the current t
 * (else WM_ERR_STATE). */
WM_API int wm_attend(wm_kvbuf* h, int block, const void* Q, void* O, wm_stream_t stream);

/* wm_write_record followed by wm_attend for the same block and frame, in one
 * launch where the head dimension allows (d = 64).  The two steps are the
 * model card's (sections "A frame is a record" and "One buffer, no mask");
 * doing them in one launch is this library's: the attention reads the
 * keys before and after the record's slot from the buffer and the record
 * itself from K/V (softmax attention does not depend on the order of the
 * keys), while the same launch copies K/V into the slot.  Results and buffer
 * contents are exactly those of the two separate calls.  Arguments and errors
 * as for wm_write_record and wm_attend (Q, K, V, O device [R, heads, d] bf16;
 * t must be the current frame). */
WM_API int wm_write_attend(wm_kvbuf* h, int block, int64_t t, const void* Q, const void* K,
                           const void* V, void* O, wm_stream_t stream);

/* Streaming sink (model card section "Running for a long time: the start
 * image follows the window"): the start image's keys carry temporal
 * position 0 while new frames get ever larger ids.  Let the gap be the
 * distance from that position to the oldest frame kept (max(1, t-W) during
 * frame t); when it reaches `gap_trigger` (the page: 5), wm_advance(t) rotates the
 * start image's keys (Z0 rows of K, every block) forward in place by
 * gap - gap_target frames (the page: back to a gap of 1).  Values are not
 * touched.  The page gives no rotary frequencies, so the caller passes them:
 * theta[i] (radians per frame, host array of n_pairs = d/2 floats) for the
 * adjacent dimension pair (2i, 2i+1) of every head, 0 for pairs outside the
 * temporal band.  Pair i turns as a complex number by theta[i]*shift, in
 * float32 (each product and sum rounded separately) then rounded to bf16.
 * Must be called before the first wm_advance (else WM_ERR_STATE). */
WM_API int wm_set_sink(wm_kvbuf* h, const float* theta, int n_pairs, int gap_trigger,
                       int gap_target);
/* Temporal position of the start image's keys (0 until the first rotation). */
WM_API int64_t wm_sink_position(const wm_kvbuf* h);
/* The float32 cosines and sines a rotation by `shift` frames uses (host
 * arrays of d/2 floats). */
WM_API int wm_sink_cos_sin(const wm_kvbuf* h, int64_t shift, float* c, float* s);

/* Introspection (host only, no device work). */
WM_API int64_t wm_end(const wm_kvbuf* h);                 /* end(t) at the current frame; -1 before t=0 */
WM_API int64_t wm_capacity(const wm_kvbuf* h);            /* C */
WM_API int64_t wm_current_frame(const wm_kvbuf* h);       /* last t passed to wm_advance, -1 before */
WM_API int wm_raw_slot(const wm_kvbuf* h, int64_t t);     /* (t-1) mod (Y+1) for t >= 1; -1 for t < 1 */
WM_API int wm_sum_slot(const wm_kvbuf* h, int64_t f);     /* (f-1) mod (W-Y) for f >= 1; -1 if none */
/* Device pointers of block's K and V buffers, each [C, heads, d] bf16 (E4M3
 * codes, one byte each, for a WM_KV_E4M3 handle).  Owned by the handle; valid
 * until wm_kvbuf_destroy. */
WM_API int wm_kv_ptrs(const wm_kvbuf* h, int block, void** K, void** V);

/* Synchronise the handle's device (the caller's current device is restored),
 * then read and clear the handle's device error flag:
 * WM_ERR_TIMEOUT if a kernel gave up a bounded wait since the last call,
 * WM_ERR_CUDA if the synchronisation itself failed, else WM_OK. */
WM_API int wm_sync_status(wm_kvbuf* h);

/* Bound, in SM clock cycles, on each wait inside this handle's attention
 * launches (wm_attend, wm_write_attend) for work another part of the same
 * launch produces (tensor loads, tensor-core results, softmax tiles).  The
 * default, 4e9 cycles (about 2 s at the 1.965 GHz maximum clock), is far above
 * any wait of a healthy launch.  A launch that runs out of it finishes the
 * copies and tensor-core work it started, releases its tensor memory, exits,
 * and leaves WM_ERR_TIMEOUT for wm_sync_status; its outputs, and a slot that a
 * wm_write_attend in it was writing, are then undefined until written again.
 * A smaller bound exercises that path: 0 makes the first wait that is not
 * already satisfied give up.  The page has no counterpart: this is the
 * library's guard against a launch that would otherwise never end.
 * Returns WM_ERR_INVALID_ARG for a NULL handle. */
WM_API int wm_set_wait_limit(wm_kvbuf* h, uint64_t cycles);

/* Static description of an error code. */
WM_API const char* wm_strerror(int code);
/* Text of the last CUDA error seen by this thread in a wm_* call ("" if none). */
WM_API const char* wm_last_cuda_error(void);

/* Self-check of the polynomial 2^x the attention kernel evaluates on the FMA
 * pipe for 3 of every 8 exponentials (head dimension 64): y[i] = that
 * polynomial's 2^x[i], for device float arrays of n (even, >= 2) values,
 * 8-byte aligned.  The page has no counterpart; the call exists so that a
 * test can bound the approximation's error on the device (relative error at
 * most 1.7e-3 for x in [-125, 127]; x below -125 gives 2^-125).
 * WM_ERR_INVALID_ARG for NULL, misaligned or odd-sized arrays. */
WM_API int wm_selftest_exp2(const float* x, float* y, int64_t n, wm_stream_t stream);

/* Pure layout arithmetic (no handle, no device) used by tests and tools. */
WM_API int64_t wm_layout_capacity(int grid_h, int grid_w, int X, int Y, int W);
WM_API int64_t wm_layout_end(int grid_h, int grid_w, int X, int Y, int W, int64_t t);
WM_API int wm_layout_raw_slot(int Y, int64_t t);
WM_API int wm_layout_sum_slot(int Y, int W, int64_t f);
/* First row of frame t's record (Z0 for t = 0, its RAW slot otherwise). */
WM_API int64_t wm_layout_record_row(int grid_h, int grid_w, int X, int Y, int64_t t);

/* Dense attention with no frame memory.  The model card (section "One
 * buffer, no mask") contrasts the 6,528 keys of the served buffer with the
 * 26,208 the same span would need at full resolution; this call runs that
 * full-resolution comparison point:
 *   O[i,h,:] = sum_j softmax_j(Q[i,h,:] . K[j,h,:] / sqrt(d)) V[j,h,:],  j < Lk,
 * Q/O device [Lq, heads, d], K/V device [Lk, heads, d], all bf16, same
 * kernel and numerics as wm_attend.  Lq >= 1, Lk >= 1, d in {64, 128}.
 * Beyond the page's statement of the operation, the call takes a stream and
 * `dev_status`, an optional device int (NULL to skip) that the kernel sets
 * to 1 if it gives up a bounded wait (about 2 s); it is not touched
 * otherwise, so the caller zeroes it beforehand and reads it after the
 * stream has reached the launch.
 * Returns WM_ERR_INVALID_ARG for an empty Q or K (Lq < 1 or Lk < 1), a
 * pointer that is not 16-byte aligned or more than 65535 heads,
 * WM_ERR_UNSUPPORTED for another head dimension, WM_ERR_CUDA if the launch
 * fails; nothing is launched in those cases. */
WM_API int wm_attend_dense(const void* Q, const void* K, const void* V, void* O, int64_t Lq, int64_t Lk,
                    int heads, int d, int* dev_status, wm_stream_t stream);

/* Dense attention over caller-owned FP8 E4M3 keys and values: the
 * full-resolution comparison point of wm_attend_dense for FP8 buffers.
 *   O[i,h,:] = sum_j softmax_j(Q[i,h,:] . Kd[j,h,:] / sqrt(d)) Vd[j,h,:],  j < Lk,
 * with Kd = code_value(K8) * k_scale[h] and Vd = code_value(V8) * v_scale[h]
 * (the E4M3 reading of wm_kvbuf_create_fp8).  Q/O device [Lq, heads, d] bf16;
 * K8/V8 device [Lk, heads, d] E4M3 codes; k_scale/v_scale device arrays of
 * `heads` floats.  `scratch` is caller-owned device memory of at least
 * wm_attend_dense_fp8_scratch_bytes(Lk, heads, d) bytes, 16-byte aligned,
 * where the codes are widened to bf16; it must not be in use by another call
 * until the stream has passed this one.  dev_status as for wm_attend_dense.
 * Returns WM_ERR_INVALID_ARG for a NULL or misaligned pointer, an empty Q or
 * K, more than 65535 heads or a scratch too small, WM_ERR_UNSUPPORTED for a
 * head dimension other than 64 or 128, WM_ERR_CUDA if a launch fails. */
WM_API int wm_attend_dense_fp8(const void* Q, const void* K8, const void* V8, const float* k_scale,
                               const float* v_scale, void* O, int64_t Lq, int64_t Lk, int heads,
                               int d, void* scratch, int64_t scratch_bytes, int* dev_status,
                               wm_stream_t stream);
/* Scratch bytes wm_attend_dense_fp8 needs: 2 * Lk * heads * d * 2 (-1 for
 * arguments it rejects). */
WM_API int64_t wm_attend_dense_fp8_scratch_bytes(int64_t Lk, int heads, int d);

/* wm_attend_dense_fp8 for callers that cannot allocate device memory.  The
 * page has no counterpart: this entry point exists for callers that cannot
 * hand wm_attend_dense_fp8 a scratch buffer -- a plug-in that receives only
 * the tensors of one call and has no allocator, a host framework whose memory
 * pool owns every device allocation and refuses outside ones, a serving
 * process that must not grow its device footprint (or synchronise inside
 * cudaMalloc / cudaFree) once it runs.  It computes exactly what
 * wm_attend_dense_fp8 computes, with the same arguments minus the scratch:
 * the keys and values are widened into a fixed device array of
 * WM_FP8_STATIC_SCRATCH_BYTES (32 MiB) that this library defines and every
 * GPU that loads the library holds until the process exits.  It calls no
 * cudaMalloc, cudaFree or allocating library routine.
 *   - Limit: 2 * Lk * heads * d * 2 bytes must fit the array (Lk * heads * d
 *     at most 8,388,608, e.g. 6,528 keys x 16 heads x 64); larger calls
 *     return WM_ERR_INVALID_ARG and launch nothing.
 *   - The first call on a device looks up the array's device address with
 *     that device current (once per device); make that first call before any
 *     stream capture.
 *   - Every call shares the one array.  Each call writes the part it reads
 *     before reading it, so nothing needs clearing between calls, but calls
 *     whose work overlaps on the GPU (other streams, other threads) race:
 *     order them on one stream or with events.
 * Other arguments, requirements and errors as for wm_attend_dense_fp8. */
#define WM_FP8_STATIC_SCRATCH_BYTES (32ll << 20)
WM_API int wm_attend_dense_fp8_static(const void* Q, const void* K8, const void* V8,
                                      const float* k_scale, const float* v_scale, void* O,
                                      int64_t Lq, int64_t Lk, int heads, int d, int* dev_status,
                                      wm_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* WMKV_H */
