// Dense, unmasked softmax attention over a filled buffer prefix, for sm_100a.
//
// What it computes (model card "GTA world model: weights and inference code",
// section "One buffer, no mask": each block's queries attend to every row of
// the buffer's filled prefix, unmasked): for every head h and query row i
//     O[i,h,:] = sum_{j<lk} softmax_j(Q[i,h,:] . K[j,h,:] / sqrt(d)) V[j,h,:]
//
// Design (one CTA per 128-query tile and head, 384 threads = 3 warpgroups):
//   warp 8      TMA producer: Q tile once, then K_j / V_j tiles (128 keys) into
//               separate K and V rings (K two tiles ahead), 128-byte swizzled,
//               zero-filled past lk.
//   warp 9      owns TMEM (512 columns) and issues S_j = Q K_j^T
//               (tcgen05.mma SS: both operands K-major in smem)
//   warps 10/11 issue O_g += P_j V_j for even / odd tiles (tcgen05.mma TS: P
//               from TMEM, V MN-major in smem); three issuing warps keep the
//               tensor core fed while each waits on barriers and commits.
//               (the same for d = 128, whose two warpgroups share one O).
//   warps 0-3   softmax warpgroup 0: even key tiles, S0/P0/O0 in TMEM
//   warps 4-7   softmax warpgroup 1: odd key tiles, S1/P1/O1 in TMEM
// The control warpgroup gives registers back (setmaxnreg) so that each
// softmax thread can hold its 128 scores without spilling.  Each softmax
// thread owns one query row (= one TMEM lane).
//
// Pipeline per warpgroup g and its tile j (= g, g+2, ...):
//   wait S_full[g] -> load the S row into registers -> arrive S_free[g]
//   (for d = 64, P has its own TMEM columns, so the MMA warp can already issue
//   S_{j+2} into S_g while this tile's softmax runs) -> row max; the exponent
//   reference m moves only when the max grows by more than 2^8 (the final
//   division by l is exact either way) -> p = 2^(s*log2(e)/sqrt(d) - m) in
//   registers (MUFU, part on the FMA pipe) -> wait O_done[g] (P.V
//   of tile j-2 finished: O_g is stable and P_g is free; waiting only now
//   hides the MMA round trip behind the exponentials) -> rescale O_g if m
//   moved -> P as bf16 into TMEM -> arrive P_full[g].
// For d = 128 the two warpgroups, which attend for the same rows, share one
// O: both P.V issuers accumulate into it (2 S + 2 P + 1 O of 128, 64, 128
// columns), so P has columns of its own and S is released as soon as it is
// read, as for d = 64.  A shared O cannot be rescaled lazily, so each row's
// exponent reference is fixed: the larger of the two warpgroups' first-tile
// maxima, exchanged once.  A tile whose row max exceeds it by more than 2^64
// (the fp32 headroom of the accumulation) is computed against a clamped
// reference and the CTA flagged; before it exits, a flagged CTA recomputes
// its rows exactly in fp32 and overwrites what its epilogue wrote.
// The two warpgroups' partial results (m, l, O) are merged row by row at the
// end and stored as bf16.
//
// Every mbarrier wait is bounded (by default about 2 s); a CTA that gives up sets a shared
// abort flag, records DEV_TIMEOUT in the caller's status word, drains what it
// issued, frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "sm100_ptx.cuh"
#include "wmkv_internal.h"

namespace wmkv {

namespace {

constexpr int BM = 128;  // queries per tile
constexpr int BN = 128;  // keys per KV tile
constexpr int NUM_THREADS = 384;
// setmaxnreg split of the launch budget (NUM_THREADS x LAUNCH_REGS):
// 2 softmax warpgroups x 128 x SOFTMAX_REGS + 128 x CONTROL_REGS.
constexpr int LAUNCH_REGS = 168;
constexpr int SOFTMAX_REGS = 224;
constexpr int CONTROL_REGS = 56;
static_assert(256 * SOFTMAX_REGS + 128 * CONTROL_REGS <= NUM_THREADS * LAUNCH_REGS,
              "register split exceeds the launch budget");
// Bounded waits: each wait gives up after AttendParams::wait_limit SM cycles
// (by default about 2 s at the 1.965 GHz maximum clock, longer at lower
// clocks); the drain after a timeout waits up to 0.2 s per operation,
// whatever the limit.
constexpr uint64_t DRAIN_LIMIT_CYCLES = 400000000ull;

template <int D, bool SHARED = false>
struct Cfg {
  static constexpr int SUB = D / 64;             // 64-column (128-byte) sub-tiles per row
  static constexpr int SUB_BYTES = BN * 128;     // one sub-tile: 128 rows x 128 B
  static constexpr int TILE_BYTES = SUB * SUB_BYTES;
  // K and V rings.  A K stage is released as soon as its S MMA completes, a
  // V stage after its P.V; the producer keeps K two tiles ahead of V.
  static constexpr int NK = (D == 64) ? 5 : 3;
  static constexpr int NV = (D == 64) ? 4 : (SHARED ? 2 : 3);
  static constexpr int K_AHEAD = 2;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + TILE_BYTES;
  static constexpr int V_OFF = K_OFF + NK * TILE_BYTES;
  // staging buffer of the in-kernel record copy (d = 64 only: for d = 128 the
  // rings use the shared memory and the record is copied by its own launch)
  static constexpr bool COPY_IN_KERNEL = (D == 64);
  static constexpr int COPY_CHUNK_BYTES = 16384;  // per staging buffer (K and V chunk)
  static constexpr int COPY_STAGE_BYTES = COPY_IN_KERNEL ? 2 * COPY_CHUNK_BYTES : 0;
  static constexpr int COPY_OFF = V_OFF + NV * TILE_BYTES;
  // d = 128: the two warpgroups share one O (they attend for the same rows)
  // with one exponent reference per row, agreed on once through XCH0
  static constexpr bool SHARED_O = SHARED;
  static_assert(!SHARED || D == 128, "the shared O is the head-dimension-128 layout");
  static constexpr int XCH0_OFF = COPY_OFF + COPY_STAGE_BYTES;  // 2 x BM floats
  static constexpr int BAR_OFF = XCH0_OFF + (SHARED_O ? 2 * BM * 4 : 0);
  // barrier indices
  static constexpr int B_Q = 0;
  static constexpr int B_KFULL = 1;
  static constexpr int B_KEMPTY = B_KFULL + NK;
  static constexpr int B_VFULL = B_KEMPTY + NK;
  static constexpr int B_VEMPTY = B_VFULL + NV;
  static constexpr int B_SFULL = B_VEMPTY + NV;  // 2
  static constexpr int B_SFREE = B_SFULL + 2;    // 2
  static constexpr int B_PFULL = B_SFREE + 2;    // 2
  static constexpr int B_ODONE = B_PFULL + 2;    // 2
  static constexpr int B_OFINAL = B_ODONE + 2;
  static constexpr int B_DRAIN = B_OFINAL + 1;   // 3: one per MMA issuer
  static constexpr int B_COPY = B_DRAIN + 3;     // 2: record copy staging loads (K, V)
  static constexpr int B_OFIRST = B_COPY + 2;    // shared O: the first P.V has completed
  static constexpr int NBAR = B_OFIRST + (SHARED_O ? 1 : 0);
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;   // [0] tmem base, [1] abort
  // m[2][BM], l[2][BM] for the final merge; they reuse the Q tile, which no
  // MMA reads any more once the last P.V has completed
  static constexpr int XCH_OFF = Q_OFF;
  static constexpr int SMEM_BYTES = MISC_OFF + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;  // 1024-byte alignment slack
  // TMEM columns
  static constexpr bool P_SEP = (D == 64) || SHARED;
  // d = 64: S and P.V MMAs come from separate issuing warps (their MMAs are
  // short, so per-tile waits and commits would otherwise leave the tensor core
  // idle); d = 128: one issuing warp, which keeps S_{j+2} behind P_j.V_j in
  // issue order.
  static constexpr bool TWO_ISSUERS = P_SEP;
  static constexpr uint32_t S_COL0 = 0, S_COL1 = 128;
  static constexpr uint32_t P_COL0 = P_SEP ? 256 : S_COL0;
  static constexpr uint32_t P_COL1 = P_SEP ? 320 : S_COL1;
  static constexpr uint32_t O_COL0 = P_SEP ? 384 : 256;
  static constexpr uint32_t O_COL1 = SHARED_O ? O_COL0 : O_COL0 + D;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false, false);
  static constexpr uint32_t IDESC_O = idesc_bf16_f32(BM, D, false, true);
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory budget");
  static_assert(O_COL1 + D <= TMEM_COLS && P_COL1 + BM / 2 <= O_COL0, "TMEM budget");
  static_assert(NV % 2 == 0 || !P_SEP, "per-warpgroup P.V issuers need an even V ring");
};

// Of every 8 column pairs of a score row, this many get their exponential
// from the FMA-pipe polynomial instead of MUFU.EX2 (measured on B200: 3 is
// best for d = 64, where exponentials per FLOP are twice as frequent, against
// 2 and 4; 0 for d = 128).
template <int D>
constexpr int poly_pairs_per_8() {
  return D == 64 ? 3 : 0;
}

// log2 units: O and l are rescaled only when the row max grows by more than
// 2^8, so every exponential of a tile lies in (0, 2^8].
constexpr float RESCALE_THRESHOLD = 8.f;
// shared O (d = 128): a tile whose row max exceeds the fixed reference by more
// than this many powers of two is flagged (its exponentials would leave the
// fp32 headroom of the accumulation)
constexpr float SHARED_REF_HEADROOM = 64.f;

// Largest of the 128 scores of a row: eight independent chains of
// three-input max, then a tree.
__device__ __forceinline__ float row_max(const float (&s)[128]) {
  float mx[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) mx[c] = fmax3(s[c], s[c + 8], s[c + 16]);
#pragma unroll
  for (int c = 24; c < 120; c += 16)
#pragma unroll
    for (int i = 0; i < 8; ++i) mx[i] = fmax3(mx[i], s[c + i], s[c + 8 + i]);
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], s[120 + i]);
  return fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], fmax3(mx[5], mx[6], mx[7])));
}

// Independent partial sums of a row's exponentials (a power of two; 8
// measured slower than 4).
constexpr int ACC_CHAINS = 4;

// p = 2^(s * sl2 - m_ref) for the 128 scores of a row, packed to bf16 pairs;
// returns their sum.  POLY of every 8 column pairs take the FMA-pipe
// polynomial, the rest MUFU.EX2 (the arguments are at most RESCALE_THRESHOLD).
template <int POLY>
__device__ __forceinline__ float exp_tile(const float (&s)[128], float sl2, float m_ref,
                                          uint32_t (&pk)[64]) {
  const f2 scale2 = f2_make(sl2, sl2);
  const f2 negm2 = f2_make(-m_ref, -m_ref);
  f2 acc[ACC_CHAINS];
#pragma unroll
  for (int i = 0; i < ACC_CHAINS; ++i) acc[i] = f2_make(0.f, 0.f);
#pragma unroll
  for (int pp = 0; pp < 64; ++pp) {
    const f2 x = f2_fma(f2_make(s[2 * pp], s[2 * pp + 1]), scale2, negm2);
    f2 e;
    if ((pp % 8) >= 8 - POLY) {
      e = exp2_poly2(x);
    } else {
      float x0, x1;
      f2_split(x, x0, x1);
      e = f2_make(ex2_approx(x0), ex2_approx(x1));
    }
    acc[pp % ACC_CHAINS] = f2_add(acc[pp % ACC_CHAINS], e);
    float e0, e1;
    f2_split(e, e0, e1);
    pk[pp] = pack_bf16x2(e0, e1);
  }
#pragma unroll
  for (int w = ACC_CHAINS / 2; w >= 1; w /= 2)
#pragma unroll
    for (int i = 0; i < w; ++i) acc[i] = f2_add(acc[i], acc[i + w]);
  float a_lo, a_hi;
  f2_split(acc[0], a_lo, a_hi);
  return a_lo + a_hi;
}

// The softmax warps tell the MMA issuers that a warpgroup has read S or
// written P with one arrival per warp: the TMEM loads / stores of the whole
// warp have completed at tcgen05.wait (a warp-wide instruction), so after the
// fence and a warp sync one lane can speak for the warp (4 arrivals per
// warpgroup instead of 128).
constexpr uint32_t SOFTMAX_ARRIVALS = 4;
__device__ __forceinline__ void softmax_arrive(uint32_t bar, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

// Keys come in up to MAX_SEGS segments, each with its own K and V tensor
// maps (row extent = the segment's length, so the rows past its end are
// zero-filled).  Softmax attention does not depend on the order of the keys,
// so the fused write+attend call reads the rows before and after the current
// record's slot from the buffer and the record itself from the caller.
constexpr int MAX_SEGS = 3;

struct AttendParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k[MAX_SEGS];
  CUtensorMap tm_v[MAX_SEGS];
  __nv_bfloat16* o;
  int64_t lq;
  int seg_tiles_end[MAX_SEGS];  // cumulative number of 128-key tiles
  int seg_rows[MAX_SEGS];       // keys in each segment
  int nseg;
  int heads;
  float scale_log2;  // log2(e) / sqrt(d)
  int* status;       // may be null
  // optional copy of a record into its slot, spread over the CTAs (16-byte units)
  const uint4* copy_src[2];
  uint4* copy_dst[2];
  int64_t copy_n16;
  uint64_t wait_limit;  // SM cycles per bounded wait
  // Work of a CTA (linear id c = blockIdx.y * gridDim.x + blockIdx.x): CTAs
  // c < full_ctas own query tile c mod q_tiles of head c / q_tiles over all
  // keys; the others split the keys of the remaining query tiles, split_chunks
  // CTAs per tile, chunk_tiles key tiles each, and leave unnormalised partial
  // results in `part` (BM x D fp32 O, then BM row maxima and BM row sums per
  // CTA) for the combine launch.
  int q_tiles;
  int64_t full_ctas;
  int split_chunks;
  int chunk_tiles;
  float* part;
  // per-head factors of the stored keys and values (FP8 buffers), or null
  const float* k_scale;
  const float* v_scale;
  // the raw query and key/value segments, read only by the exact
  // recomputation of a shared-O CTA whose row maxima outgrew the fixed
  // references (d = 128)
  const __nv_bfloat16* q;
  const __nv_bfloat16* seg_k[MAX_SEGS];
  const __nv_bfloat16* seg_v[MAX_SEGS];
};

// Segment and row of key tile j, and how many of its 128 rows are keys.
struct TileLoc {
  int seg;
  int row;
  int valid;
};
__device__ __forceinline__ TileLoc tile_loc(const AttendParams& p, int j) {
  int seg = 0;
#pragma unroll
  for (int k = 0; k < MAX_SEGS - 1; ++k) seg += (k < p.nseg - 1 && j >= p.seg_tiles_end[k]) ? 1 : 0;
  const int first = seg ? p.seg_tiles_end[seg - 1] : 0;
  const int row = (j - first) * BN;
  const int left = p.seg_rows[seg] - row;
  return {seg, row, left < BN ? left : BN};
}

__device__ __forceinline__ void record_timeout(int* status) {
  if (status) atomicExch(status, DEV_TIMEOUT);
}

// MMA issue helpers, called by a whole converged warp (one elected lane
// issues).  Descriptors are built once; the start-address field (bits 0-13,
// in 16-byte units) is advanced by compile-time offsets, so the issuing warp
// spends its cycles on tcgen05.mma and not on descriptor math.
template <int D, typename C>
__device__ __forceinline__ void issue_s_warp(uint64_t dq, uint64_t dk, uint32_t d_s) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off = uint64_t(((kk / 4) * C::SUB_BYTES + (kk % 4) * 32) >> 4);
    mma_ss_elect(d_s, dq + off, dk + off, C::IDESC_S, kk > 0 ? 1u : 0u);
  }
}

template <int D, typename C>
__device__ __forceinline__ void issue_pv_warp(uint64_t dv, uint32_t p_tmem, uint32_t d_o,
                                              uint32_t accumulate) {
#pragma unroll
  for (int kk = 0; kk < BN / 16; ++kk)
    mma_ts_elect(d_o, p_tmem + kk * 8, dv + uint64_t((kk * 2048) >> 4), C::IDESC_O,
                 (accumulate | uint32_t(kk > 0)));
}

// Exact recomputation of a shared-O CTA's rows when one of its tiles had a
// row max beyond the fixed reference's headroom: fp32 online softmax, one row
// per warp at a time (all twelve warps), over the CTA's own key tiles, read
// straight from the segments; exp2f for the exponentials.  Writes what the
// epilogue wrote: the bf16 output rows, or for a key-range piece its
// unnormalised partial O, reference and sum.  Rare by construction, so
// written for clarity, not speed.
template <int D>
__device__ void exact_rows(const AttendParams& p, int q_tile, int head, int j0, int nkv,
                           float* part) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  constexpr int NW = NUM_THREADS / 32;
  constexpr int PER = D / 32;  // elements of a row per lane
  const float sl2 = p.k_scale ? p.scale_log2 * p.k_scale[head] : p.scale_log2;
  const float vs = p.v_scale ? p.v_scale[head] : 1.f;
  for (int r = warp; r < BM; r += NW) {
    const int64_t qrow = int64_t(q_tile) * BM + r;
    if (qrow >= p.lq) break;
    float q[PER], o[PER];
    const __nv_bfloat16* qp = p.q + (qrow * p.heads + head) * D + lane * PER;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      q[i] = __bfloat162float(qp[i]);
      o[i] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    for (int t = 0; t < nkv; ++t) {
      const TileLoc tl = tile_loc(p, j0 + t);
      const __nv_bfloat16* kb = p.seg_k[tl.seg];
      const __nv_bfloat16* vb = p.seg_v[tl.seg];
      for (int jj = 0; jj < tl.valid; ++jj) {
        const int64_t off = ((int64_t(tl.row) + jj) * p.heads + head) * D + lane * PER;
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) dot = fmaf(q[i], __bfloat162float(kb[off + i]), dot);
#pragma unroll
        for (int w = 16; w >= 1; w /= 2) dot += __shfl_xor_sync(0xffffffffu, dot, w);
        const float x = dot * sl2;
        const float m_new = fmaxf(m, x);
        const float corr = exp2f(m - m_new);
        const float pj = exp2f(x - m_new);
        l = l * corr + pj;
#pragma unroll
        for (int i = 0; i < PER; ++i) o[i] = fmaf(pj, __bfloat162float(vb[off + i]), o[i] * corr);
        m = m_new;
      }
    }
    if (part) {
#pragma unroll
      for (int i = 0; i < PER; ++i) part[r * D + lane * PER + i] = o[i];
      if (lane == 0) {
        part[BM * D + r] = m;
        part[BM * D + BM + r] = l;
      }
    } else {
      const float inv = vs / l;
      __nv_bfloat16* op = p.o + (qrow * p.heads + head) * D + lane * PER;
#pragma unroll
      for (int i = 0; i < PER; ++i) op[i] = __float2bfloat16_rn(o[i] * inv);
    }
  }
}

// SPLIT: the launch splits its last wave's query tiles by key range (see
// AttendParams); a launch without a split uses the instantiation that has no
// trace of it.  SHARED (d = 128): the two warpgroups accumulate into one O
// with one fixed exponent reference per row (Cfg::SHARED_O).
template <int D, bool SPLIT, bool SHARED>
__global__ void __launch_bounds__(NUM_THREADS, 1) attend_kernel(const __grid_constant__ AttendParams p) {
  using C = Cfg<D, SHARED>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + C::BAR_OFF + 8 * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* overflow_flag = reinterpret_cast<volatile int*>(misc + 2);
  float* xch_m = reinterpret_cast<float*>(smem + C::XCH_OFF);
  float* xch_l = xch_m + 2 * BM;
  float* xch0 = reinterpret_cast<float*>(smem + C::XCH0_OFF);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // this CTA's (query tile, head) and key tiles [j0, j0 + nkv)
  const int nkv_all = p.seg_tiles_end[p.nseg - 1];
  int64_t cta = 0;
  bool split = false;
  int q_tile, head, j0 = 0, nkv = nkv_all;
  if constexpr (SPLIT) {
    cta = int64_t(blockIdx.y) * gridDim.x + blockIdx.x;
    split = cta >= p.full_ctas;
    const int64_t item = split ? p.full_ctas + (cta - p.full_ctas) / p.split_chunks : cta;
    q_tile = static_cast<int>(item % p.q_tiles);
    head = static_cast<int>(item / p.q_tiles);
    if (split) {
      j0 = static_cast<int>((cta - p.full_ctas) % p.split_chunks) * p.chunk_tiles;
      nkv = p.chunk_tiles < nkv_all - j0 ? p.chunk_tiles : nkv_all - j0;
    }
  } else {
    q_tile = blockIdx.x;
    head = blockIdx.y;
  }

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_Q), 1);
    for (int s = 0; s < C::NK; ++s) {
      mbar_init(bar(C::B_KFULL + s), 1);
      mbar_init(bar(C::B_KEMPTY + s), 1);
    }
    for (int s = 0; s < C::NV; ++s) {
      mbar_init(bar(C::B_VFULL + s), 1);
      mbar_init(bar(C::B_VEMPTY + s), 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(bar(C::B_SFULL + g), 1);
      mbar_init(bar(C::B_SFREE + g), SOFTMAX_ARRIVALS);
      mbar_init(bar(C::B_PFULL + g), SOFTMAX_ARRIVALS);
      mbar_init(bar(C::B_ODONE + g), 1);
    }
    // the last P.V of each warpgroup commits once (one issuer per warpgroup
    // for d = 64; for d = 128 the single issuer commits twice)
    mbar_init(bar(C::B_OFINAL), 2);
    for (int i = 0; i < 3; ++i) mbar_init(bar(C::B_DRAIN + i), 1);
    mbar_init(bar(C::B_COPY), 1);
    mbar_init(bar(C::B_COPY + 1), 1);
    if (C::SHARED_O) mbar_init(bar(C::B_OFIRST), 1);
    misc[1] = 0;
    if (C::SHARED_O) misc[2] = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(misc), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&p.tm_q);
    for (int k = 0; k < p.nseg; ++k) {
      tma_prefetch_desc(&p.tm_k[k]);
      tma_prefetch_desc(&p.tm_v[k]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  // everything above overlaps the previous kernel in the stream; global
  // memory (Q, K, V, O, status) is touched only after this point
  pdl_wait_prior();

  // Each warpgroup re-sizes its registers at the top of its own branch (the
  // allocator gives code below a join the smaller of the two limits).
  if (warp >= 8) {
   regs_dec<CONTROL_REGS>();
   if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_expect_tx(bar(C::B_Q), C::TILE_BYTES);
      for (int s = 0; s < C::SUB; ++s)
        tma_load_3d(sbase + C::Q_OFF + s * C::SUB_BYTES, &p.tm_q, s * 64, head, q_tile * BM,
                    bar(C::B_Q));
      // This CTA's share of the record (fused write + attend), K and V chunks
      // staged through shared memory with bulk copies.  Nothing in this launch
      // reads the slot (its keys come from the caller's record), so the copy
      // overlaps the first tiles; it runs once the K/V rings have been filled,
      // where the producer would otherwise wait for a free slot.
      bool copied = !(C::COPY_IN_KERNEL && p.copy_n16 > 0);
      auto copy_record = [&]() {
        const int64_t G = int64_t(gridDim.x) * gridDim.y;
        const int64_t c = int64_t(blockIdx.y) * gridDim.x + blockIdx.x;
        const int64_t per = (p.copy_n16 + G - 1) / G;
        const int64_t lo = c * per;
        const int64_t hi = lo + per < p.copy_n16 ? lo + per : p.copy_n16;
        constexpr int64_t CH = C::COPY_CHUNK_BYTES / 16;
        uint32_t cph = 0;
        for (int64_t u = lo; u < hi && !*abort_flag; u += CH) {
          const uint32_t bytes = static_cast<uint32_t>((hi - u < CH ? hi - u : CH) * 16);
          bulk_wait_read_all();
          for (int t = 0; t < 2; ++t) {
            mbar_expect_tx(bar(C::B_COPY + t), bytes);
            bulk_load(sbase + C::COPY_OFF + t * C::COPY_CHUNK_BYTES, p.copy_src[t] + u, bytes,
                      bar(C::B_COPY + t));
          }
          int landed = 0;
          for (; landed < 2; ++landed) {
            if (!mbar_wait_bounded(bar(C::B_COPY + landed), cph, abort_flag, p.wait_limit)) break;
            bulk_store(p.copy_dst[landed] + u, sbase + C::COPY_OFF + landed * C::COPY_CHUNK_BYTES,
                       bytes);
          }
          bulk_commit();
          if (landed < 2) {
            // gave up: let the staging loads still in flight land before the
            // CTA can exit (their shared memory goes to the next CTA)
            volatile int no_abort = 0;
            for (int t = landed; t < 2; ++t)
              mbar_wait_bounded(bar(C::B_COPY + t), cph, &no_abort, DRAIN_LIMIT_CYCLES);
            break;
          }
          cph ^= 1;
        }
      };
      // K tile i and V tile i - K_AHEAD per step; each waits for its own ring slot
      int k_issued = 0, v_issued = 0;
      for (int i = 0; i < nkv + C::K_AHEAD; ++i) {
        if (!copied && (i >= C::NK || i >= nkv)) {
          copy_record();
          copied = true;
        }
        if (i < nkv) {
          const int st = i % C::NK;
          if (i >= C::NK && !mbar_wait_bounded(bar(C::B_KEMPTY + st), ((i / C::NK) - 1) & 1,
                                               abort_flag, p.wait_limit))
            break;
          const TileLoc tl = tile_loc(p, j0 + i);
          mbar_expect_tx(bar(C::B_KFULL + st), C::TILE_BYTES);
          for (int s = 0; s < C::SUB; ++s)
            tma_load_3d(sbase + C::K_OFF + st * C::TILE_BYTES + s * C::SUB_BYTES, &p.tm_k[tl.seg],
                        s * 64, head, tl.row, bar(C::B_KFULL + st));
          k_issued = i + 1;
        }
        const int jv = i - C::K_AHEAD;
        if (jv >= 0 && jv < nkv) {
          const int st = jv % C::NV;
          if (jv >= C::NV && !mbar_wait_bounded(bar(C::B_VEMPTY + st), ((jv / C::NV) - 1) & 1,
                                                abort_flag, p.wait_limit))
            break;
          const TileLoc tl = tile_loc(p, j0 + jv);
          mbar_expect_tx(bar(C::B_VFULL + st), C::TILE_BYTES);
          for (int s = 0; s < C::SUB; ++s)
            tma_load_3d(sbase + C::V_OFF + st * C::TILE_BYTES + s * C::SUB_BYTES, &p.tm_v[tl.seg],
                        s * 64, head, tl.row, bar(C::B_VFULL + st));
          v_issued = jv + 1;
        }
      }
      if (!copied) copy_record();
      bulk_wait_all();   // bulk stores complete (no-op if none were issued)
      if (*abort_flag) {
        // Let the copies this thread started land before the CTA exits.
        volatile int no_abort = 0;
        mbar_wait_bounded(bar(C::B_Q), 0, &no_abort, DRAIN_LIMIT_CYCLES);
        for (int i = k_issued - C::NK < 0 ? 0 : k_issued - C::NK; i < k_issued; ++i)
          mbar_wait_bounded(bar(C::B_KFULL + i % C::NK), (i / C::NK) & 1, &no_abort,
                            DRAIN_LIMIT_CYCLES);
        for (int i = v_issued - C::NV < 0 ? 0 : v_issued - C::NV; i < v_issued; ++i)
          mbar_wait_bounded(bar(C::B_VFULL + i % C::NV), (i / C::NV) & 1, &no_abort,
                            DRAIN_LIMIT_CYCLES);
      }
    }
  } else if (warp >= 9) {
    // ------------------------------------------------------------ MMA issuers
    // Waits on the softmax warpgroups (S_free, P_full) suspend the waiting
    // lanes (try_wait) so that the issuers do not take issue slots from the
    // softmax warps on the same SM sub-partitions; waits on TMA data that
    // normally has landed already (K_full, V_full) poll (test_wait).
    // For d = 64 three issuing warps share the tensor core: warp 9 issues
    // S = Q K^T, warps 10/11 issue O += P V, so that each one's barrier waits
    // and commits overlap with the others' MMAs; for d = 128 warp 9 issues
    // everything.  A commit tracks only the MMAs its own lane issued.
    // The issuing warps stay converged: every lane waits, the wait results are
    // made warp-uniform, and one elected lane issues each MMA and commit.
    {
      constexpr uint64_t TILE16 = C::TILE_BYTES >> 4;
      bool ok = true;
      if (!C::TWO_ISSUERS) {
        // d = 128: one warp issues everything in order; S_{j+2} follows
        // P_j.V_j in the MMA pipe, which is what lets P overwrite S_j in place
        if (warp == 9) {
          const uint64_t dq = sdesc_sw128(sbase + C::Q_OFF, 16, 1024);
          const uint64_t dk0 = sdesc_sw128(sbase + C::K_OFF, 16, 1024);
          const uint64_t dv0 = sdesc_sw128(sbase + C::V_OFF, C::SUB_BYTES, 1024);
          uint32_t k_st = 0, k_ph = 0, v_st = 0, v_ph = 0, pf_ph = 0;
          ok = __all_sync(0xffffffffu, mbar_spin_bounded(bar(C::B_Q), 0, abort_flag, p.wait_limit));
          auto do_s = [&](int g) -> bool {
            if (!__all_sync(0xffffffffu, mbar_spin_bounded(bar(C::B_KFULL + k_st), k_ph, abort_flag,
                                                           p.wait_limit)))
              return false;
            tc_fence_after();
            issue_s_warp<D, C>(dq, dk0 + k_st * TILE16, tmem + (g ? C::S_COL1 : C::S_COL0));
            tc_commit_elect(bar(C::B_SFULL + g));
            tc_commit_elect(bar(C::B_KEMPTY + k_st));
            if (++k_st == C::NK) { k_st = 0; k_ph ^= 1; }
            return true;
          };
          for (int j = 0; ok && j < 2 && j < nkv; ++j) ok = do_s(j);
          for (int j = 0; ok && j < nkv; ++j) {
            const int g = j & 1;
            if (!__all_sync(0xffffffffu,
                            mbar_wait_bounded(bar(C::B_PFULL + g), (pf_ph >> g) & 1, abort_flag,
                                              p.wait_limit) &&
                                mbar_spin_bounded(bar(C::B_VFULL + v_st), v_ph, abort_flag,
                                                  p.wait_limit))) {
              ok = false;
              break;
            }
            pf_ph ^= 1u << g;
            tc_fence_after();
            issue_pv_warp<D, C>(dv0 + v_st * TILE16, tmem + (g ? C::P_COL1 : C::P_COL0),
                             tmem + (g ? C::O_COL1 : C::O_COL0), j >= 2 ? 1u : 0u);
            tc_commit_elect(bar(C::B_ODONE + g));
            tc_commit_elect(bar(C::B_VEMPTY + v_st));
            if (++v_st == C::NV) { v_st = 0; v_ph ^= 1; }
            if (j + 2 < nkv && !(ok = do_s(g))) break;
          }
          if (ok) {
            tc_commit_elect(bar(C::B_OFINAL));
            tc_commit_elect(bar(C::B_OFINAL));
          }
        }
      } else {
      if (warp == 9) {
        const uint64_t dq = sdesc_sw128(sbase + C::Q_OFF, 16, 1024);
        const uint64_t dk0 = sdesc_sw128(sbase + C::K_OFF, 16, 1024);
        uint32_t k_st = 0, k_ph = 0;  // ring slot / phase of the next K tile
        uint32_t fr_ph = 0;           // bit g: phase of the barrier that frees S_g
        ok = __all_sync(0xffffffffu, mbar_spin_bounded(bar(C::B_Q), 0, abort_flag, p.wait_limit));
        for (int j = 0; ok && j < nkv; ++j) {
          const int g = j & 1;
          if (j >= 2) {
            // S_g is free once the warpgroup has read S_{j-2} (d = 64: P has its
            // own columns) or once P_{j-2}.V_{j-2} has completed (d = 128: P
            // overwrote S_{j-2})
            const int fb = C::P_SEP ? C::B_SFREE + g : C::B_ODONE + g;
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(fb), (fr_ph >> g) & 1, abort_flag,
                                                           p.wait_limit))) {
              ok = false;
              break;
            }
            fr_ph ^= 1u << g;
          }
          if (!__all_sync(0xffffffffu, mbar_spin_bounded(bar(C::B_KFULL + k_st), k_ph, abort_flag,
                                                         p.wait_limit))) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s_warp<D, C>(dq, dk0 + k_st * TILE16, tmem + (g ? C::S_COL1 : C::S_COL0));
          tc_commit_elect(bar(C::B_SFULL + g));
          tc_commit_elect(bar(C::B_KEMPTY + k_st));
          if (++k_st == C::NK) { k_st = 0; k_ph ^= 1; }
        }
      } else {
        // warp 10: P.V of even tiles, warp 11: odd tiles (each issuing warp
        // keeps its own V slots: the V ring has an even number of stages)
        const int g = warp - 10;
        const uint64_t dv0 = sdesc_sw128(sbase + C::V_OFF, C::SUB_BYTES, 1024);
        const uint32_t p_tm = tmem + (g ? C::P_COL1 : C::P_COL0);
        const uint32_t o_tm = tmem + (g ? C::O_COL1 : C::O_COL0);
        uint32_t pf_ph = 0;
        for (int j = g; ok && j < nkv; j += 2) {
          const int v_st = j % C::NV;
          const uint32_t v_ph = (j / C::NV) & 1;
          if (!__all_sync(0xffffffffu,
                          mbar_wait_bounded(bar(C::B_PFULL + g), pf_ph, abort_flag, p.wait_limit) &&
                              mbar_spin_bounded(bar(C::B_VFULL + v_st), v_ph, abort_flag,
                                                p.wait_limit))) {
            ok = false;
            break;
          }
          pf_ph ^= 1;
          if (C::SHARED_O && j == 1 &&
              !__all_sync(0xffffffffu, mbar_wait_bounded(bar(C::B_OFIRST), 0, abort_flag,
                                                         p.wait_limit))) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv_warp<D, C>(dv0 + v_st * TILE16, p_tm, o_tm,
                           (C::SHARED_O ? j >= 1 : j >= 2) ? 1u : 0u);
          tc_commit_elect(bar(C::B_ODONE + g));
          tc_commit_elect(bar(C::B_VEMPTY + v_st));
          if (C::SHARED_O && j == 0) tc_commit_elect(bar(C::B_OFIRST));
        }
        if (ok) tc_commit_elect(bar(C::B_OFINAL));
      }
      }
      if (!ok) {
        // let this warp's MMAs finish before TMEM is released
        volatile int no_abort = 0;
        const int db = C::B_DRAIN + (warp - 9);
        tc_commit_elect(bar(db));
        mbar_wait_bounded(bar(db), 0, &no_abort, DRAIN_LIMIT_CYCLES);
      }
    }
   }
  } else {
    regs_inc<SOFTMAX_REGS>();
    // ------------------------------------------------------------ softmax
    const int wg = warp / 4;
    const int wq = warp % 4;
    const int row = wq * 32 + lane;
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + (wg ? C::S_COL1 : C::S_COL0);
    const uint32_t p_addr = tmem + lane_off + (wg ? C::P_COL1 : C::P_COL0);
    const uint32_t o_addr = tmem + lane_off + (wg ? C::O_COL1 : C::O_COL0);
    const float sl2 = p.k_scale ? p.scale_log2 * p.k_scale[head] : p.scale_log2;
    float m_ref = -INFINITY;  // exponent reference (log2 units)
    float l_run = 0.f;
    bool ok = true;
    int n = 0;
    if (C::SHARED_O && wg >= nkv) {
      // no tile for this warpgroup: take part in the reference exchange only
      xch0[wg * BM + row] = -INFINITY;
      named_bar_sync(2, 256);
      m_ref = fmaxf(xch0[row], xch0[BM + row]);
    }
    for (int j = wg; j < nkv; j += 2, ++n) {
      ok = mbar_wait_bounded(bar(C::B_SFULL + wg), n & 1, abort_flag, p.wait_limit);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (C::SHARED_O && n == 0) {
          xch0[wg * BM + row] = -INFINITY;
          named_bar_sync(2, 256);
        }
        break;
      }
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld32_at<0>(s_addr, sr);
      tmem_ld32_at<32>(s_addr + 32, sr);
      tmem_ld32_at<64>(s_addr + 64, sr);
      tmem_ld32_at<96>(s_addr + 96, sr);
      tmem_wait_ld();
      if (C::P_SEP) {
        tc_fence_before();
        softmax_arrive(bar(C::B_SFREE + wg), lane);
      }
      float s[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
      {
        const int valid = tile_loc(p, j0 + j).valid;
        if (valid < BN) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= valid) s[c] = -INFINITY;
        }
      }
      // Exponent reference m_ref (log2 units): it moves only when the row max
      // grows by more than RESCALE_THRESHOLD (then O and l are rescaled); the
      // final division by l removes whatever reference was used.
      const float m_tile = row_max(s) * sl2;
      float alpha = 1.f;
      bool grow = false;
      float m_use;
      if constexpr (C::SHARED_O) {
        // one reference per row for both warpgroups: the larger of their first
        // tiles' maxima, fixed from then on (no rescaling of the shared O)
        if (n == 0) {
          xch0[wg * BM + row] = m_tile;
          named_bar_sync(2, 256);
          m_ref = fmaxf(xch0[row], xch0[BM + row]);
        }
        m_use = fmaxf(m_ref, m_tile - SHARED_REF_HEADROOM);
        if (m_use != m_ref) *overflow_flag = 1;
      } else {
        if (n == 0) {
          m_ref = m_tile;
        } else if (m_tile > m_ref + RESCALE_THRESHOLD) {
          alpha = ex2_approx(m_ref - m_tile);
          m_ref = m_tile;
          grow = true;
        }
        m_use = m_ref;
      }
      uint32_t pk[64];
      const float tile_sum = exp_tile<poly_pairs_per_8<D>()>(s, sl2, m_use, pk);
      // l is rescaled by alpha (1 unless the reference grew) before this tile's sum
      l_run = l_run * alpha + tile_sum;
      if (n > 0) {
        // P.V of this warpgroup's previous tile has finished: O is stable, P is free
        ok = mbar_wait_bounded(bar(C::B_ODONE + wg), (n - 1) & 1, abort_flag, p.wait_limit);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t orr[32];
            tmem_ld32(o_addr + c * 32, orr);
            tmem_wait_ld();
            const f2 a2 = f2_make(alpha, alpha);
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              f2 v = f2_make(__uint_as_float(orr[i]), __uint_as_float(orr[i + 1]));
              v = f2_mul(v, a2);
              float lo, hi;
              f2_split(v, lo, hi);
              orr[i] = __float_as_uint(lo);
              orr[i + 1] = __float_as_uint(hi);
            }
            tmem_st32(o_addr + c * 32, orr);
          }
        }
      }
      tmem_st32_at<0>(p_addr, pk);
      tmem_st32_at<32>(p_addr + 32, pk);
      tmem_wait_st();
      tc_fence_before();
      softmax_arrive(bar(C::B_PFULL + wg), lane);
    }
    // all P.V products must have landed before O is read
    if (ok) {
      ok = mbar_wait_bounded(bar(C::B_OFINAL), 0, abort_flag, p.wait_limit);
      ok = __all_sync(0xffffffffu, ok);
    }
    tc_fence_after();
    xch_m[wg * BM + row] = m_ref;
    xch_l[wg * BM + row] = l_run;
    named_bar_sync(1, 256);
    if (ok && !*abort_flag && split) {
      // unnormalised partial result of this key range: O = O_0 a_0 + O_1 a_1
      // with the row's reference mf, and l = l_0 a_0 + l_1 a_1
      const float m0 = xch_m[row], m1 = xch_m[BM + row];
      const float l0 = xch_l[row], l1 = xch_l[BM + row];
      const float mf = fmaxf(m0, m1);
      const float a0 = ex2_approx(m0 - mf);
      const float a1 = nkv > 1 ? ex2_approx(m1 - mf) : 0.f;
      const bool has1 = !C::SHARED_O && nkv > 1;
      float* part = p.part + (cta - p.full_ctas) * int64_t(BM * (D + 2));
      const uint32_t o0 = tmem + lane_off + C::O_COL0;
      const uint32_t o1 = tmem + lane_off + C::O_COL1;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        const int col = wg * (D / 2) + c * 32;
        uint32_t r0[32], r1[32];
        tmem_ld32(o0 + col, r0);
        if (has1) tmem_ld32(o1 + col, r1);
        tmem_wait_ld();
        float4* dst = reinterpret_cast<float4*>(part + row * D + col);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float x[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            x[k] = __uint_as_float(r0[4 * i + k]) * a0;
            if (has1) x[k] = fmaf(__uint_as_float(r1[4 * i + k]), a1, x[k]);
          }
          dst[i] = make_float4(x[0], x[1], x[2], x[3]);
        }
      }
      if (wg == 0) {
        part[BM * D + row] = mf;
        part[BM * D + BM + row] = l0 * a0 + l1 * a1;
      }
    } else if (ok && !*abort_flag) {
      const float m0 = xch_m[row], m1 = xch_m[BM + row];
      const float l0 = xch_l[row], l1 = xch_l[BM + row];
      const float mf = fmaxf(m0, m1);
      const float a0 = ex2_approx(m0 - mf);
      const float a1 = ex2_approx(m1 - mf);
      const float inv = (p.v_scale ? p.v_scale[head] : 1.f) / (l0 * a0 + l1 * a1);
      const float c0 = a0 * inv, c1 = a1 * inv;
      const bool has1 = !C::SHARED_O && nkv > 1;
      const int64_t qrow = int64_t(q_tile) * BM + row;
      __nv_bfloat16* orow = p.o + (qrow * p.heads + head) * D;
      const uint32_t o0 = tmem + lane_off + C::O_COL0;
      const uint32_t o1 = tmem + lane_off + C::O_COL1;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        const int col = wg * (D / 2) + c * 32;
        uint32_t r0[32], r1[32];
        tmem_ld32(o0 + col, r0);
        if (has1) tmem_ld32(o1 + col, r1);
        tmem_wait_ld();
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0 = __uint_as_float(r0[2 * i]) * c0;
          float x1 = __uint_as_float(r0[2 * i + 1]) * c0;
          if (has1) {
            x0 = fmaf(__uint_as_float(r1[2 * i]), c1, x0);
            x1 = fmaf(__uint_as_float(r1[2 * i + 1]), c1, x1);
          }
          packed[i] = pack_bf16x2(x0, x1);
        }
        if (qrow < p.lq) {
          uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) record_timeout(p.status);
  if constexpr (C::SHARED_O) {
    if (*overflow_flag && !*abort_flag)
      exact_rows<D>(p, q_tile, head, j0, nkv,
                    split ? p.part + (cta - p.full_ctas) * int64_t(BM * (D + 2)) : nullptr);
  }
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Merge of a split query tile's partial results: per row, M = max_k m_k and
//   O = v_scale * sum_k 2^(m_k - M) O_k / sum_k 2^(m_k - M) l_k,
// rounded to bf16.  One thread per (row, group of 8 columns): blockIdx.x is
// the split tile (item full_ctas + blockIdx.x), blockIdx.y a slice of rows.
constexpr int COMBINE_THREADS = 256;
template <int D>
__global__ void __launch_bounds__(COMBINE_THREADS) combine_kernel(const float* __restrict__ part,
                                                                  int64_t full_ctas, int q_tiles,
                                                                  int split_chunks, int64_t lq,
                                                                  int heads,
                                                                  const float* __restrict__ v_scale,
                                                                  __nv_bfloat16* __restrict__ o) {
  pdl_launch_dependents();
  pdl_wait_prior();
  constexpr int CG = D / 8;
  constexpr int64_t PART = int64_t(BM) * (D + 2);
  const int idx = blockIdx.y * COMBINE_THREADS + threadIdx.x;
  const int row = idx / CG, cg = idx % CG;
  const int64_t item = full_ctas + blockIdx.x;
  const int q_tile = static_cast<int>(item % q_tiles);
  const int head = static_cast<int>(item / q_tiles);
  const int64_t qrow = int64_t(q_tile) * BM + row;
  if (row >= BM || qrow >= lq) return;
  const float* base = part + int64_t(blockIdx.x) * split_chunks * PART;
  float m = -INFINITY;
#pragma unroll 4
  for (int k = 0; k < split_chunks; ++k) m = fmaxf(m, base[k * PART + BM * D + row]);
  float l = 0.f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int k = 0; k < split_chunks; ++k) {
    const float* ps = base + k * PART;
    const float w = exp2f(ps[BM * D + row] - m);
    l = fmaf(w, ps[BM * D + BM + row], l);
    const float4 a = reinterpret_cast<const float4*>(ps + row * D + cg * 8)[0];
    const float4 b = reinterpret_cast<const float4*>(ps + row * D + cg * 8)[1];
    acc[0] = fmaf(w, a.x, acc[0]); acc[1] = fmaf(w, a.y, acc[1]);
    acc[2] = fmaf(w, a.z, acc[2]); acc[3] = fmaf(w, a.w, acc[3]);
    acc[4] = fmaf(w, b.x, acc[4]); acc[5] = fmaf(w, b.y, acc[5]);
    acc[6] = fmaf(w, b.z, acc[6]); acc[7] = fmaf(w, b.w, acc[7]);
  }
  const float sc = (v_scale ? v_scale[head] : 1.f) / l;
  uint32_t pk[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) pk[i] = pack_bf16x2(acc[2 * i] * sc, acc[2 * i + 1] * sc);
  *reinterpret_cast<uint4*>(o + (qrow * heads + head) * D + cg * 8) =
      make_uint4(pk[0], pk[1], pk[2], pk[3]);
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [rows, heads, d] bf16, box = 128 rows x 1 head x 64 columns, 128-byte swizzle.
bool encode_rows_map(CUtensorMap* m, const void* base, int64_t rows, int heads, int d) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(heads), cuuint64_t(rows)};
  cuuint64_t strides[2] = {cuuint64_t(d) * 2, cuuint64_t(heads) * d * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr int MAX_DEVICES = 64;

// Kernel attributes belong to a device: they are set once on each device used,
// for each instantiation.  setmaxnreg.inc waits until registers are free, so
// the launch must carry exactly the budget the register split assumes, or the
// kernel is not launched.
template <int D, bool SHARED>
cudaError_t launch_d(const AttendParams& prm, dim3 grid, cudaStream_t stream) {
  using C = Cfg<D, SHARED>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES)
    return cudaErrorInvalidDevice;
  const int64_t split_tiles = (int64_t(grid.x) * grid.y - prm.full_ctas) / prm.split_chunks;
  const bool split = split_tiles > 0;
  static std::once_flag once[2][MAX_DEVICES];
  static cudaError_t attr_err[2][MAX_DEVICES];
  auto prepare = [dev](auto kernel, int which) {
    std::call_once(once[which][dev], [kernel, which, dev] {
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           C::SMEM_ALLOC);
      cudaFuncAttributes fa;
      if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, kernel);
      if (e == cudaSuccess && fa.numRegs != LAUNCH_REGS) e = cudaErrorInvalidConfiguration;
      attr_err[which][dev] = e;
    });
    return attr_err[which][dev];
  };
  cudaError_t e = split ? prepare(attend_kernel<D, true, SHARED>, 1)
                        : prepare(attend_kernel<D, false, SHARED>, 0);
  if (e != cudaSuccess) return e;
  e = split ? launch_pdl(attend_kernel<D, true, SHARED>, grid, dim3(NUM_THREADS), C::SMEM_ALLOC,
                         stream, prm)
            : launch_pdl(attend_kernel<D, false, SHARED>, grid, dim3(NUM_THREADS), C::SMEM_ALLOC,
                         stream, prm);
  if (e == cudaSuccess && split)
    e = launch_pdl(combine_kernel<D>,
                   dim3(static_cast<unsigned>(split_tiles),
                        static_cast<unsigned>((BM * (D / 8) + COMBINE_THREADS - 1) / COMBINE_THREADS)),
                   dim3(COMBINE_THREADS), 0, stream,
                   static_cast<const float*>(prm.part), prm.full_ctas, prm.q_tiles, prm.split_chunks,
                   prm.lq, prm.heads, prm.v_scale, prm.o);
  return e;
}

}  // namespace

bool attend_copies_in_kernel(int d) { return Cfg<64>::COPY_IN_KERNEL && d == 64; }

cudaError_t launch_attend(const void* q, void* o, int64_t lq, const KVSegment* segs, int nseg,
                          int heads, int d, int* status, const RecordCopy* copy,
                          unsigned long long wait_limit, const float* k_scale,
                          const float* v_scale, float* part, int part_ctas, cudaStream_t stream) {
  if (nseg < 1 || nseg > MAX_SEGS) return cudaErrorInvalidValue;
  AttendParams prm = {};
  if (!encode_rows_map(&prm.tm_q, q, lq, heads, d)) return cudaErrorInvalidValue;
  int tiles = 0;
  for (int k = 0; k < nseg; ++k) {
    if (segs[k].rows < 1 || segs[k].rows >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
    if (!encode_rows_map(&prm.tm_k[k], segs[k].k, segs[k].rows, heads, d) ||
        !encode_rows_map(&prm.tm_v[k], segs[k].v, segs[k].rows, heads, d))
      return cudaErrorInvalidValue;
    tiles += static_cast<int>((segs[k].rows + BN - 1) / BN);
    prm.seg_tiles_end[k] = tiles;
    prm.seg_rows[k] = static_cast<int>(segs[k].rows);
    prm.seg_k[k] = static_cast<const __nv_bfloat16*>(segs[k].k);
    prm.seg_v[k] = static_cast<const __nv_bfloat16*>(segs[k].v);
  }
  prm.nseg = nseg;
  prm.q = static_cast<const __nv_bfloat16*>(q);
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lq = lq;
  prm.heads = heads;
  prm.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  prm.status = status;
  prm.wait_limit = wait_limit;
  prm.k_scale = k_scale;
  prm.v_scale = v_scale;
  if (copy && copy->n16 > 0) {
    if (!attend_copies_in_kernel(d)) return cudaErrorInvalidValue;
    prm.copy_src[0] = static_cast<const uint4*>(copy->k_src);
    prm.copy_src[1] = static_cast<const uint4*>(copy->v_src);
    prm.copy_dst[0] = static_cast<uint4*>(copy->k_dst);
    prm.copy_dst[1] = static_cast<uint4*>(copy->v_dst);
    prm.copy_n16 = copy->n16;
  }
  // One CTA per (query tile, head); when that is one or more full waves of the
  // SMs plus a remainder of at most half a wave, the remainder's query tiles
  // are split by key range over the SMs the last wave would leave idle (their
  // partial results merged by the combine launch).
  const int64_t q_tiles = (lq + BM - 1) / BM;
  const int64_t items = q_tiles * heads;
  prm.q_tiles = static_cast<int>(q_tiles);
  prm.full_ctas = items;
  prm.split_chunks = 1;
  prm.chunk_tiles = tiles;
  prm.part = part;
  dim3 grid(static_cast<unsigned>(q_tiles), static_cast<unsigned>(heads));
  const int sms = device_sm_count();
  if (part && items > sms && items <= 0x7FFFFFFF) {
    const int64_t tail = items % sms;
    int chunks = (tail > 0 && tail <= sms / 2) ? static_cast<int>(sms / tail) : 0;
    if (chunks > tiles) chunks = tiles;
    if (chunks >= 2) {
      const int per = (tiles + chunks - 1) / chunks;
      chunks = (tiles + per - 1) / per;  // every chunk non-empty
      if (chunks >= 2 && tail * chunks <= part_ctas) {
        prm.full_ctas = items - tail;
        prm.split_chunks = chunks;
        prm.chunk_tiles = per;
        grid = dim3(static_cast<unsigned>(prm.full_ctas + tail * chunks), 1);
      }
    }
  }
  if (d == 64) return launch_d<64, false>(prm, grid, stream);
  if (d == 128) return launch_d<128, true>(prm, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace wmkv
