// Dense, unmasked softmax attention over a filled buffer prefix, for sm_100a.
//
// What it computes (model card "GTA world model: weights and inference code",
// section "One buffer, no mask": one dense read of the filled prefix per
// block, no mask): for every head h and query row i
//     O[i,h,:] = sum_{j<lk} softmax_j(Q[i,h,:] . K[j,h,:] / sqrt(d)) V[j,h,:]
//
// Design (one CTA per 128-query tile and head):
//   warp 8      TMA producer: Q tile once, then K_j / V_j tiles (128 keys) into
//               an NS-stage ring, 128-byte swizzled, zero-filled past lk.
//   warp 9      owns TMEM (512 columns) and issues every tcgen05.mma:
//                 S_j = Q K_j^T          (SS: both operands K-major in smem)
//                 O_g += P_j V_j         (TS: P from TMEM, V MN-major in smem)
//   warps 0-3   softmax warpgroup 0: even KV tiles, S0/O0 in TMEM
//   warps 4-7   softmax warpgroup 1: odd KV tiles, S1/O1 in TMEM
// Each softmax thread owns one query row (= one TMEM lane).  It reads its S
// row, updates the running max m and sum l (exp2 with log2(e)/sqrt(d)
// folded into the score scale), rescales its O row in TMEM when m grew,
// writes P as bf16 over the first half of its S columns, and signals the MMA
// warp.  The two warpgroups ping-pong so that the tensor core computes one
// tile's S while the other tile's softmax runs.  At the end the two partial
// results (m0,l0,O0) and (m1,l1,O1) are merged row by row and stored as bf16.
//
// Every mbarrier wait is bounded (2 s); a CTA that gives up sets a shared
// abort flag, records DEV_TIMEOUT in the caller's status word, drains what it
// issued, frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "sm100_ptx.cuh"
#include "wmkv_internal.h"

namespace wmkv {

namespace {

constexpr int BM = 128;  // queries per tile
constexpr int BN = 128;  // keys per KV tile
constexpr int NUM_THREADS = 320;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;
constexpr uint64_t DRAIN_LIMIT_NS = 200000000ull;

template <int D>
struct Cfg {
  static constexpr int SUB = D / 64;             // 64-column (128-byte) sub-tiles per row
  static constexpr int SUB_BYTES = BN * 128;     // one sub-tile: 128 rows x 128 B
  static constexpr int TILE_BYTES = SUB * SUB_BYTES;
  static constexpr int NS = (D == 64) ? 4 : 2;   // K/V ring stages
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + TILE_BYTES;
  static constexpr int V_OFF = K_OFF + NS * TILE_BYTES;
  static constexpr int BAR_OFF = V_OFF + NS * TILE_BYTES;
  // barrier indices
  static constexpr int B_Q = 0;
  static constexpr int B_KFULL = 1;
  static constexpr int B_VFULL = B_KFULL + NS;
  static constexpr int B_EMPTY = B_VFULL + NS;
  static constexpr int B_SFULL = B_EMPTY + NS;   // 2
  static constexpr int B_PFULL = B_SFULL + 2;    // 2
  static constexpr int B_OFINAL = B_PFULL + 2;
  static constexpr int B_DRAIN = B_OFINAL + 1;
  static constexpr int NBAR = B_DRAIN + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;   // [0] tmem base, [1] abort
  static constexpr int XCH_OFF = MISC_OFF + 16;         // m[2][BM], l[2][BM]
  static constexpr int SMEM_BYTES = XCH_OFF + 4 * BM * 4;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;  // 1024-byte alignment slack
  // TMEM columns: S0, S1 (128 fp32 each), O0, O1 (D fp32 each)
  static constexpr uint32_t S0_COL = 0, S1_COL = 128, O0_COL = 256, O1_COL = 256 + D;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false, false);
  static constexpr uint32_t IDESC_O = idesc_bf16_f32(BM, D, false, true);
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory budget");
  static_assert(O1_COL + D <= TMEM_COLS, "TMEM budget");
};

struct AttendParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  __nv_bfloat16* o;
  int64_t lq;
  int64_t lk;
  int heads;
  float scale_log2;  // log2(e) / sqrt(d)
  int* status;       // may be null
};

__device__ __forceinline__ void record_timeout(int* status) {
  if (status) atomicExch(status, DEV_TIMEOUT);
}

template <int D>
__global__ void __launch_bounds__(NUM_THREADS, 1) attend_kernel(const __grid_constant__ AttendParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + C::BAR_OFF + 8 * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  float* xch_m = reinterpret_cast<float*>(smem + C::XCH_OFF);
  float* xch_l = xch_m + 2 * BM;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int q_tile = blockIdx.x;
  const int head = blockIdx.y;
  const int nkv = static_cast<int>((p.lk + BN - 1) / BN);

  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_Q), 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar(C::B_KFULL + s), 1);
      mbar_init(bar(C::B_VFULL + s), 1);
      mbar_init(bar(C::B_EMPTY + s), 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(bar(C::B_SFULL + g), 1);
      mbar_init(bar(C::B_PFULL + g), 128);
    }
    mbar_init(bar(C::B_OFINAL), 1);
    mbar_init(bar(C::B_DRAIN), 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(misc), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_expect_tx(bar(C::B_Q), C::TILE_BYTES);
      for (int s = 0; s < C::SUB; ++s)
        tma_load_3d(sbase + C::Q_OFF + s * C::SUB_BYTES, &p.tm_q, s * 64, head, q_tile * BM,
                    bar(C::B_Q));
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int st = j % C::NS;
        const int round = j / C::NS;
        if (round > 0 && !mbar_wait_bounded(bar(C::B_EMPTY + st), (round - 1) & 1, abort_flag,
                                            WAIT_LIMIT_NS))
          break;
        mbar_expect_tx(bar(C::B_KFULL + st), C::TILE_BYTES);
        for (int s = 0; s < C::SUB; ++s)
          tma_load_3d(sbase + C::K_OFF + st * C::TILE_BYTES + s * C::SUB_BYTES, &p.tm_k, s * 64,
                      head, j * BN, bar(C::B_KFULL + st));
        mbar_expect_tx(bar(C::B_VFULL + st), C::TILE_BYTES);
        for (int s = 0; s < C::SUB; ++s)
          tma_load_3d(sbase + C::V_OFF + st * C::TILE_BYTES + s * C::SUB_BYTES, &p.tm_v, s * 64,
                      head, j * BN, bar(C::B_VFULL + st));
        issued = j + 1;
      }
      if (*abort_flag) {
        // Let the copies this thread started land before the CTA exits.
        volatile int no_abort = 0;
        for (int j = issued - C::NS < 0 ? 0 : issued - C::NS; j < issued; ++j) {
          const int st = j % C::NS;
          const uint32_t par = (j / C::NS) & 1;
          mbar_wait_bounded(bar(C::B_KFULL + st), par, &no_abort, DRAIN_LIMIT_NS);
          mbar_wait_bounded(bar(C::B_VFULL + st), par, &no_abort, DRAIN_LIMIT_NS);
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait_bounded(bar(C::B_Q), 0, abort_flag, WAIT_LIMIT_NS);
      tc_fence_after();
      for (int j = 0; ok && j <= nkv; ++j) {
        if (j < nkv) {
          const int st = j % C::NS;
          const int g = j & 1;
          if (!mbar_wait_bounded(bar(C::B_KFULL + st), (j / C::NS) & 1, abort_flag, WAIT_LIMIT_NS)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_tile = sbase + C::K_OFF + st * C::TILE_BYTES;
          const uint32_t d_s = tmem + (g ? C::S1_COL : C::S0_COL);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk / 4) * C::SUB_BYTES + (kk % 4) * 32;
            const uint64_t a = sdesc_sw128(sbase + C::Q_OFF + off, 16, 1024);
            const uint64_t b = sdesc_sw128(k_tile + off, 16, 1024);
            mma_ss(d_s, a, b, C::IDESC_S, kk > 0 ? 1u : 0u);
          }
          tc_commit(bar(C::B_SFULL + g));
        }
        if (j >= 1) {
          const int jp = j - 1;
          const int gp = jp & 1;
          const int stp = jp % C::NS;
          if (!mbar_wait_bounded(bar(C::B_PFULL + gp), (jp / 2) & 1, abort_flag, WAIT_LIMIT_NS) ||
              !mbar_wait_bounded(bar(C::B_VFULL + stp), (jp / C::NS) & 1, abort_flag,
                                 WAIT_LIMIT_NS)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t v_tile = sbase + C::V_OFF + stp * C::TILE_BYTES;
          const uint32_t p_tmem = tmem + (gp ? C::S1_COL : C::S0_COL);
          const uint32_t d_o = tmem + (gp ? C::O1_COL : C::O0_COL);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t b = sdesc_sw128(v_tile + kk * 2048, C::SUB_BYTES, 1024);
            mma_ts(d_o, p_tmem + kk * 8, b, C::IDESC_O, (jp >= 2 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar(C::B_EMPTY + stp));
        }
      }
      if (ok) {
        tc_commit(bar(C::B_OFINAL));
      } else {
        volatile int no_abort = 0;
        tc_commit(bar(C::B_DRAIN));
        mbar_wait_bounded(bar(C::B_DRAIN), 0, &no_abort, DRAIN_LIMIT_NS);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int wg = warp / 4;
    const int wq = warp % 4;
    const int row = wq * 32 + lane;
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + (wg ? C::S1_COL : C::S0_COL);
    const uint32_t o_addr = tmem + lane_off + (wg ? C::O1_COL : C::O0_COL);
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.f;
    bool ok = true;
    int n = 0;
    for (int j = wg; j < nkv; j += 2, ++n) {
      ok = mbar_wait_bounded(bar(C::B_SFULL + wg), n & 1, abort_flag, WAIT_LIMIT_NS);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, sr[c]);
      tmem_wait_ld();
      float s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(sr[c][i]);
      if (j == nkv - 1) {
        const int valid = static_cast<int>(p.lk - int64_t(j) * BN);
        if (valid < BN) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= valid) s[c] = -INFINITY;
        }
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
      const float m_new = fmaxf(m_run, mx * sl2);
      const float alpha = ex2_approx(m_run - m_new);
      const float neg_m = -m_new;
      float sum = 0.f;
      uint32_t pk[2][32];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ex2_approx(fmaf(s[2 * c], sl2, neg_m));
        const float p1 = ex2_approx(fmaf(s[2 * c + 1], sl2, neg_m));
        sum += p0 + p1;
        pk[c / 32][c % 32] = pack_bf16x2(p0, p1);
      }
      l_run = l_run * alpha + sum;
      m_run = m_new;
      tmem_st32(s_addr, pk[0]);
      tmem_st32(s_addr + 32, pk[1]);
      if (n > 0 && __any_sync(0xffffffffu, alpha < 1.f)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orr[32];
          tmem_ld32(o_addr + c * 32, orr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
          tmem_st32(o_addr + c * 32, orr);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(C::B_PFULL + wg));
    }
    // all P.V products must have landed before O is read
    if (ok) {
      ok = mbar_wait_bounded(bar(C::B_OFINAL), 0, abort_flag, WAIT_LIMIT_NS);
      ok = __all_sync(0xffffffffu, ok);
    }
    tc_fence_after();
    xch_m[wg * BM + row] = m_run;
    xch_l[wg * BM + row] = l_run;
    named_bar_sync(1, 256);
    if (ok && !*abort_flag) {
      const float m0 = xch_m[row], m1 = xch_m[BM + row];
      const float l0 = xch_l[row], l1 = xch_l[BM + row];
      const float mf = fmaxf(m0, m1);
      const float a0 = ex2_approx(m0 - mf);
      const float a1 = ex2_approx(m1 - mf);
      const float inv = 1.f / (l0 * a0 + l1 * a1);
      const float c0 = a0 * inv, c1 = a1 * inv;
      const bool has1 = nkv > 1;
      const int64_t qrow = int64_t(q_tile) * BM + row;
      __nv_bfloat16* orow = p.o + (qrow * p.heads + head) * D;
      const uint32_t o0 = tmem + lane_off + C::O0_COL;
      const uint32_t o1 = tmem + lane_off + C::O1_COL;
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
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
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

template <int D>
cudaError_t launch_d(const AttendParams& prm, int64_t lq, int heads, cudaStream_t stream) {
  using C = Cfg<D>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(attend_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::SMEM_ALLOC);
  });
  if (attr_err != cudaSuccess) return attr_err;
  dim3 grid(static_cast<unsigned>((lq + BM - 1) / BM), static_cast<unsigned>(heads));
  attend_kernel<D><<<grid, NUM_THREADS, C::SMEM_ALLOC, stream>>>(prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend(const void* q, const void* k, const void* v, void* o, int64_t lq,
                          int64_t lk, int heads, int d, int* status, cudaStream_t stream) {
  AttendParams prm;
  if (!encode_rows_map(&prm.tm_q, q, lq, heads, d) || !encode_rows_map(&prm.tm_k, k, lk, heads, d) ||
      !encode_rows_map(&prm.tm_v, v, lk, heads, d))
    return cudaErrorInvalidValue;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lq = lq;
  prm.lk = lk;
  prm.heads = heads;
  prm.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  prm.status = status;
  if (d == 64) return launch_d<64>(prm, lq, heads, stream);
  if (d == 128) return launch_d<128>(prm, lq, heads, stream);
  return cudaErrorInvalidValue;
}

}  // namespace wmkv
