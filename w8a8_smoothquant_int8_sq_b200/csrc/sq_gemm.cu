// sq_gemm.cu -- int8 x int8 -> int32 GEMM on the sm_100a tensor cores with the
// SmoothQuant dequantising epilogue.
//
// Page: "w8a8_smoothquant.py -- W8A8 com SmoothQuant e alpha APRENDIVEL (V5)",
// SmoothQuantW8A8.forward: the product of the quantised activations and
// weights plus the bias, which on hardware is "INT8 x INT8 -> INT32 -> fp32":
//     acc[m][n] = sum_k Xq[m][k] * Wq[n][k]
//     Y[m][n]   = bf16( acc * x_scale[m] * w_scale[n] + bias[n] )
//
// Design (one CTA per SM, persistent over output tiles of 128 x BN):
//   warp 0      TMA producer: 128 x 128-byte K slices of Xq and BN x 128-byte
//               slices of Wq into a STAGES-deep shared-memory ring (128-byte
//               swizzle), completion counted on per-stage mbarriers.
//   warp 1      allocates 2*BN TMEM columns (two int32 accumulators) and issues
//               tcgen05.mma kind::i8 (M=128, N=BN, K=32) from one thread;
//               tcgen05.commit frees ring slots and publishes finished tiles.
//   warps 2..5  epilogue: tcgen05.ld of 32 columns at a time, fp32
//               dequantisation + bias, bf16 pack, 16-byte stores.  The two TMEM
//               accumulators let the epilogue of tile i overlap the main loop of
//               tile i+1.
// Every mbarrier wait is bounded in time; a timeout latches bit 0 of the device
// status word, the CTA drains the copies and MMAs it issued, frees its TMEM and
// returns.
#include <algorithm>
#include <cstdint>
#include <atomic>
#include <mutex>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {

__device__ unsigned int g_sq_device_status = 0u;

namespace {

constexpr int kBM = 128;         // MMA M (tile rows of Xq / Y)
constexpr int kBK = 128;         // K bytes per stage = one 128-byte swizzle row
constexpr int kUmmaK = 32;       // K per tcgen05.mma kind::i8
constexpr int kThreads = 192;    // 6 warps
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s per wait
// Build-time tuning knobs (defaults are the measured best on B200):
//   SQ_GEMM_PF     k-blocks of L2 prefetch ahead of the shared-memory ring (0: none)
//   SQ_GEMM_PF_A   1: prefetch the Xq slices too, 0: only the Wq slices
//   SQ_GEMM_ROTATE 1: start each tile's K loop at a tile-dependent k-block, so
//                  CTAs that share an operand slice do not all request the same
//                  lines at the same moment (int32 sums are exact in any order)
//   SQ_GEMM_BN     0: choose the tile width per problem, else force 128 or 256
#ifndef SQ_GEMM_PF
#define SQ_GEMM_PF 0
#endif
#ifndef SQ_GEMM_PF_A
#define SQ_GEMM_PF_A 0
#endif
#ifndef SQ_GEMM_ROTATE
#define SQ_GEMM_ROTATE 0
#endif
#ifndef SQ_GEMM_BN
#define SQ_GEMM_BN 0
#endif
#ifndef SQ_GEMM_SPLITK  // 1: split K over a CTA pair when 128 x 256 tiles fill at most half the SMs
#define SQ_GEMM_SPLITK 1
#endif
#ifndef SQ_GEMM_PAIR  // 1: 256 x 256 tiles on CTA pairs (cta_group::2) when they fill every pair
#define SQ_GEMM_PAIR 1
#endif
#ifndef SQ_GEMM_CHAINS128  // accumulator chains for 128-wide tiles (1 or 2)
#define SQ_GEMM_CHAINS128 2
#endif
constexpr int kPrefetchAhead = SQ_GEMM_PF;

// First k-block of a tile's K loop.
__device__ __forceinline__ int k_start(int m_blk, int n_blk, int nk) {
#if SQ_GEMM_ROTATE
  return static_cast<int>((static_cast<unsigned>(n_blk) * 3u + static_cast<unsigned>(m_blk) * 5u) %
                          static_cast<unsigned>(nk));
#else
  (void)m_blk;
  (void)n_blk;
  (void)nk;
  return 0;
#endif
}

// Output tile `tile` of a persistent GEMM -> (m block, n block).  Tiles run
// in groups of `group_m` m-blocks: within a group the m-blocks turn fastest
// and the group sweeps every n-block before the next group starts, so the
// tiles in flight at any moment share a few Wq slices and the group's Xq rows
// (group_m * BM * K bytes, sized to stay in L2) are fetched from DRAM once.
__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int group_m, int& m_blk, int& n_blk) {
  const int per_group = group_m * num_n;
  const int g = tile / per_group;
  const int first_m = g * group_m;
  const int gm = min(group_m, num_m - first_m);  // the last group may be narrower
  const int r = tile - g * per_group;
  m_blk = first_m + r % gm;
  n_blk = r / gm;
}

struct KParams {
  unsigned long long timeout_ns;  // limit of every mbarrier wait
  int skip_first_load;            // test hook: the producer never loads the first stage
  int M, N, K;
  int num_m_blocks, num_n_blocks, num_k_blocks;
  int group_m;                    // m-blocks per tile group (tile_coords)
  const float* x_scale;
  const float* w_scale;
  const uint16_t* bias;
  void* out;
  int vec_ok;  // 16-byte stores allowed (row pitch and base aligned)
};

template <int BN, int STAGES>
struct SmemLayout {
  static constexpr int kABytes = kBM * kBK;
  static constexpr int kBBytes = BN * kBK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kRingBytes = STAGES * kStageBytes;
  // barriers after the ring
  static constexpr int kBarOffset = kRingBytes;
  static constexpr int kNumBars = 2 * STAGES + 4 + 1;  // full, empty, tfull[2], tempty[2], drain
  // per epilogue warp: the tile's w_scale[BN] and bias[BN] (fp32)
  static constexpr int kEpiOffset = (kBarOffset + kNumBars * 8 + 15) / 16 * 16;
  static constexpr int kEpiBytes = 4 * 2 * BN * 4;
  static constexpr int kMiscOffset = kEpiOffset + kEpiBytes;
  static constexpr int kBytes = kMiscOffset + 16;
  static constexpr int kAlloc = kBytes + 1024;  // manual 1024-byte alignment
};

#ifdef SQ_TRACE
// Optional phase timestamps (build with -DSQ_TRACE): per CTA of the general
// GEMM, globaltimer at 0 past the wait for the previous kernel, 1 first stage
// consumed, 2 last MMA issued, 3 last epilogue store issued, 4 block start.
__device__ unsigned long long g_big_trace[1024][5];
#define SQ_BIG_MARK(i)                                               \
  do {                                                               \
    if (blockIdx.x < 1024) g_big_trace[blockIdx.x][i] = globaltimer_ns(); \
  } while (0)
#else
#define SQ_BIG_MARK(i) \
  do {                 \
  } while (0)
#endif

__device__ __forceinline__ void flag_timeout(volatile int* abort_flag) {
  *abort_flag = 1;
  atomicOr(&g_sq_device_status, 1u);
}

template <int BN, int STAGES, int EPI, int CHAINS>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const KParams p) {
  using L = SmemLayout<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOffset);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOffset + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Two accumulator buffers (epilogue of one tile overlaps the next tile's
  // main loop), each split into CHAINS int32 accumulators that alternate
  // between consecutive MMAs of a k-block so that they do not wait on each
  // other's accumulation; the epilogue adds the chains (exact).
  constexpr uint32_t kTmemCols = 2 * CHAINS * BN;
  static_assert(kTmemCols <= 512, "TMEM holds 512 columns");

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);  // one arrive per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (threadIdx.x == 0) SQ_BIG_MARK(4);
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x == 0) SQ_BIG_MARK(0);

  const int num_tiles = p.num_m_blocks * p.num_n_blocks;
  const int nk = p.num_k_blocks;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued[STAGES];
      uint32_t issued_phase[STAGES];
#pragma unroll
      for (int i = 0; i < STAGES; ++i) issued[i] = 0, issued_phase[i] = 0;
      bool ok = true;
      // L2 prefetch runs kPrefetchAhead k-blocks ahead of the shared-memory
      // ring along this CTA's (tile, k-block) sequence, so the ring's loads hit
      // L2 instead of waiting on DRAM.
      const int my_tiles = (num_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                           static_cast<int>(gridDim.x);
      const int64_t total = static_cast<int64_t>(my_tiles) * nk;
      int64_t pf = 0;
      auto prefetch_upto = [&](int64_t limit) {
        for (; pf < limit && pf < total; ++pf) {
          const int t = static_cast<int>(blockIdx.x) + static_cast<int>(pf / nk) * static_cast<int>(gridDim.x);
          int mb, nb;
          tile_coords(t, p.num_m_blocks, p.num_n_blocks, p.group_m, mb, nb);
          int k = static_cast<int>(pf % nk) + k_start(mb, nb, nk);
          if (k >= nk) k -= nk;
          if (SQ_GEMM_PF_A) tma_prefetch_l2_2d(&tmA, k * kBK, mb * kBM);
          tma_prefetch_l2_2d(&tmB, k * kBK, nb * BN);
        }
      };
      if (kPrefetchAhead > 0) prefetch_upto(kPrefetchAhead);
      int64_t seq = 0;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        int m_blk, n_blk;
        tile_coords(tile, p.num_m_blocks, p.num_n_blocks, p.group_m, m_blk, n_blk);
        const int k0 = k_start(m_blk, n_blk, nk);
        for (int kb = 0; kb < nk; ++kb, ++seq) {
          if (kPrefetchAhead > 0) prefetch_upto(seq + 1 + kPrefetchAhead);
          if (p.skip_first_load && seq == 0) {  // test hook: this stage never fills
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
            continue;
          }
          int kk = kb + k0;
          if (kk >= nk) kk -= nk;
          if (*abort_flag || !mbar_wait_bounded(&empty[stage], phase ^ 1u, p.timeout_ns)) {
            if (!*abort_flag) flag_timeout(abort_flag);
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * L::kStageBytes;
          uint8_t* sb = sa + L::kABytes;
          mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
          tma_load_2d(sa, &tmA, kk * kBK, m_blk * kBM, &full[stage]);
          tma_load_2d(sb, &tmB, kk * kBK, n_blk * BN, &full[stage]);
          issued[stage] = 1;
          issued_phase[stage] = phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // drain: every copy this thread issued must land before the CTA exits
#pragma unroll
        for (int i = 0; i < STAGES; ++i)
          if (issued[i]) (void)mbar_wait_bounded(&full[i], issued_phase[i], p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kBM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (*abort_flag || !mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, p.timeout_ns)) {
          if (!*abort_flag) flag_timeout(abort_flag);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * CHAINS * BN);
        for (int kb = 0; kb < nk; ++kb) {
          if (*abort_flag || !mbar_wait_bounded(&full[stage], phase, p.timeout_ns)) {
            if (!*abort_flag) flag_timeout(abort_flag);
            ok = false;
            break;
          }
          tc_fence_after();
          if (it == 0 && kb == 0) SQ_BIG_MARK(1);
          const uint32_t sa = smem_u32(smem + stage * L::kStageBytes);
          const uint32_t sb = sa + L::kABytes;
          const uint64_t adesc = smem_desc_k_sw128(sa);
          const uint64_t bdesc = smem_desc_k_sw128(sb);
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            // advance the start address by kk * 32 bytes (encoded >> 4) inside the swizzle atom
            mma_i8(d_tmem + static_cast<uint32_t>((kk % CHAINS) * BN), adesc + static_cast<uint64_t>(kk * 2),
                   bdesc + static_cast<uint64_t>(kk * 2), idesc, (kb != 0 || kk >= CHAINS) ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        SQ_BIG_MARK(2);
        mma_commit(&tfull[acc]);
      }
      // drain: wait until every MMA this thread issued has completed
      mma_commit(drain);
      (void)mbar_wait_bounded(drain, 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter + 32) for this warp
    // this warp's copy of the tile's w_scale and bias, staged before the
    // accumulator is ready so that no global load sits between TMEM and the stores
    float* ep_ws = reinterpret_cast<float*>(smem + L::kEpiOffset) + (warp - 2) * (2 * BN);
    float* ep_b = ep_ws + BN;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      int m_blk, n_blk;
      tile_coords(tile, p.num_m_blocks, p.num_n_blocks, p.group_m, m_blk, n_blk);
      const int row = m_blk * kBM + quarter * 32 + lane;
      const bool row_ok = row < p.M;
      float xs = 0.0f;
      if (EPI == 0) {
        const int nb = n_blk * BN;
        __syncwarp();  // the previous tile's reads of the staging area are done
        for (int i = lane * 4; i < BN; i += 128) {
          float4 w4 = make_float4(0.f, 0.f, 0.f, 0.f);
          if (nb + i + 4 <= p.N && p.vec_ok) {
            w4 = __ldg(reinterpret_cast<const float4*>(p.w_scale + nb + i));
          } else {
            if (nb + i < p.N) w4.x = __ldg(p.w_scale + nb + i);
            if (nb + i + 1 < p.N) w4.y = __ldg(p.w_scale + nb + i + 1);
            if (nb + i + 2 < p.N) w4.z = __ldg(p.w_scale + nb + i + 2);
            if (nb + i + 3 < p.N) w4.w = __ldg(p.w_scale + nb + i + 3);
          }
          *reinterpret_cast<float4*>(ep_ws + i) = w4;
        }
        for (int i = lane; i < BN; i += 32)
          ep_b[i] = (p.bias != nullptr && nb + i < p.N)
                        ? __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + nb + i)) << 16)
                        : 0.0f;
        xs = row_ok ? __ldg(p.x_scale + row) : 0.0f;
        __syncwarp();
      }
      // every lane observes the phase itself; the vote keeps the warp uniform
      // for the warp-collective tcgen05.ld even if lanes disagree on a timeout
      const bool mine = !*abort_flag && mbar_wait_bounded(&tfull[acc], acc_phase, p.timeout_ns);
      if (!__all_sync(0xFFFFFFFFu, mine)) {
        if (lane == 0 && !*abort_flag) flag_timeout(abort_flag);
        break;
      }
      tc_fence_after();
      const uint32_t t_base =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * CHAINS * BN);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld_32cols(t_base + static_cast<uint32_t>(c0), r);
        tmem_ld_wait();
#pragma unroll
        for (int ch = 1; ch < CHAINS; ++ch) {
          uint32_t r2[32];
          tmem_ld_32cols(t_base + static_cast<uint32_t>(ch * BN + c0), r2);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] += r2[j];
        }
        const int n0 = n_blk * BN + c0;
        if (n0 >= p.N) continue;  // tile overhang past N (warp-uniform)
        const bool full_chunk = (n0 + 32 <= p.N);
        const bool vec = full_chunk && p.vec_ok;
        if (EPI == 0) {
          uint32_t packed[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float y0 =
                __fmaf_rn(__int2float_rn(static_cast<int>(r[j])), __fmul_rn(xs, ep_ws[c0 + j]), ep_b[c0 + j]);
            const float y1 = __fmaf_rn(__int2float_rn(static_cast<int>(r[j + 1])), __fmul_rn(xs, ep_ws[c0 + j + 1]),
                                       ep_b[c0 + j + 1]);
            packed[j / 2] = pack_bf16x2(y0, y1);
          }
          if (row_ok) {
            uint16_t* yrow = static_cast<uint16_t*>(p.out) + static_cast<int64_t>(row) * p.N + n0;
            if (vec) {
              uint4* dst = reinterpret_cast<uint4*>(yrow);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                dst[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (n0 + j < p.N) yrow[j] = static_cast<uint16_t>(packed[j / 2] >> ((j & 1) * 16));
            }
          }
        } else {
          if (row_ok) {
            int32_t* arow = static_cast<int32_t*>(p.out) + static_cast<int64_t>(row) * p.N + n0;
            if (vec) {
              uint4* dst = reinterpret_cast<uint4*>(arow);
#pragma unroll
              for (int j = 0; j < 8; ++j) dst[j] = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (n0 + j < p.N) arow[j] = static_cast<int32_t>(r[j]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (warp == 2 && lane == 0) SQ_BIG_MARK(3);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace
}  // namespace sq

#include "sq_gemm_small.cuh"
#include "sq_gemm_splitk.cuh"

namespace sq {
namespace {
#include "sq_gemm_pair.cuh"
#include "sq_gemm_prologue.cuh"
}  // namespace
}  // namespace sq

namespace sq {
namespace {

// ----------------------------------------------------------- host helpers
// test hook state (sq_debug_pipeline_stall)
std::atomic<int> g_debug_stall{0};
std::atomic<unsigned long long> g_debug_timeout_ns{kWaitTimeoutNs};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2-D int8 tensor map over a row-major [rows][K] matrix, box = box_rows x 128 bytes,
// 128-byte swizzle, zero fill outside the matrix.
bool make_tmap_i8(CUtensorMap* map, const int8_t* base, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// m-blocks per tile group: the group's Xq rows (group_m * bm * K bytes) are
// kept near SQ_GEMM_GROUP_BYTES so that they stay in L2 while the group sweeps
// every Wq slice.
#ifndef SQ_GEMM_GROUP_BYTES  // build-time knob
#define SQ_GEMM_GROUP_BYTES (32ll << 20)
#endif
int tile_group_m(int bm, int64_t K, int num_m_blocks) {
  const int64_t per_block = static_cast<int64_t>(bm) * K;
  const int64_t g = std::max<int64_t>(1, SQ_GEMM_GROUP_BYTES / per_block);
  return static_cast<int>(std::min<int64_t>(g, num_m_blocks));
}

template <int BN, int STAGES, int EPI, int CHAINS>
cudaError_t run_gemm(const GemmArgs& a, cudaStream_t st, const DeviceInfo& dev, const char** why) {
  using L = SmemLayout<BN, STAGES>;
  CUtensorMap tmA, tmB;
  if (!make_tmap_i8(&tmA, a.A, a.M, a.K, kBM) || !make_tmap_i8(&tmB, a.B, a.N, a.K, BN)) {
    *why = "cuTensorMapEncodeTiled failed or unavailable";
    return cudaErrorInvalidValue;
  }
  KParams p;
  p.timeout_ns = g_debug_stall.load() ? g_debug_timeout_ns.load() : kWaitTimeoutNs;
  p.skip_first_load = g_debug_stall.load() ? 1 : 0;
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.num_m_blocks = static_cast<int>((a.M + kBM - 1) / kBM);
  p.num_n_blocks = static_cast<int>((a.N + BN - 1) / BN);
  p.num_k_blocks = static_cast<int>((a.K + kBK - 1) / kBK);
  p.group_m = tile_group_m(kBM, a.K, p.num_m_blocks);
  p.x_scale = a.x_scale;
  p.w_scale = a.w_scale;
  p.bias = a.bias;
  p.out = a.out;
  const int elem = (EPI == 0) ? 2 : 4;
  p.vec_ok = ((a.N * elem) % 16 == 0) && (reinterpret_cast<uintptr_t>(a.out) % 16 == 0) &&
             (reinterpret_cast<uintptr_t>(a.w_scale) % 16 == 0 || EPI != 0) &&
             (a.bias == nullptr || reinterpret_cast<uintptr_t>(a.bias) % 16 == 0);
  auto kern = gemm_i8_kernel<BN, STAGES, EPI, CHAINS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, kCarveoutMaxShared);
  if (e != cudaSuccess) {
    *why = "cudaFuncSetAttribute failed";
    return e;
  }
  const int tiles = p.num_m_blocks * p.num_n_blocks;
  const int grid = std::min(tiles, dev.sm_count);
  return launch_pdl(kern, dim3(grid), dim3(kThreads), L::kAlloc, st, tmA, tmB, p);
}

template <int NT, bool kFused>
cudaError_t run_small(const SmallArgs& a, cudaStream_t st, const DeviceInfo& dev, const char** why) {
  const int nrb = static_cast<int>((a.N + kSmallRows - 1) / kSmallRows);
  const int nk = static_cast<int>((a.K + kBK - 1) / kBK);
  const int smem_cap = static_cast<int>(dev.max_smem_optin) - 1024;
  const int part_bytes = kSmallRows * NT * 4;
  const int stage_bytes = kSmallABytes + (kFused ? 0 : NT * kBK);
  const int fixed = part_bytes + 128 + 18 * NT * 4 + 2 * kSmallRows * 4 + 256 + 16;
  // split K over a cluster of S CTAs: as many splits as keep one wave of CTAs
  // (S <= 8, at least two k-blocks each), more if the fused codes would not fit
  int S = 1;
  while (S < 8 && static_cast<int64_t>(nrb) * S * 2 <= dev.sm_count && (nk + 2 * S - 1) / (2 * S) >= 2) S *= 2;
  auto b_bytes_for = [&](int splits) { return kFused ? ((nk + splits - 1) / splits) * NT * kBK : 0; };
  while (S < 8 && b_bytes_for(S) + fixed + 2 * stage_bytes > smem_cap) S *= 2;
  const int kps = (nk + S - 1) / S;
  const int b_bytes = b_bytes_for(S);
  const int stages = std::min(kSmallMaxStages, (smem_cap - b_bytes - fixed) / stage_bytes);
  if (stages < 2) {
    *why = "small-M kernel: K too large for shared memory";
    return cudaErrorNotSupported;
  }
  SmallParams p{};
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.nk = nk;
  p.kb_per_split = kps;
  p.stages = stages;
  p.stage_bytes = stage_bytes;
  p.X = a.X;
  p.s = a.s;
  p.x_scale = a.x_scale;
  p.w_scale = a.w_scale;
  p.bias = a.bias;
  p.timeout_ns = g_debug_stall.load() ? g_debug_timeout_ns.load() : kWaitTimeoutNs;
  p.skip_first_load = g_debug_stall.load() ? 1 : 0;
  p.Y = a.Y;
  p.b_off = stages * stage_bytes;
  p.part_off = p.b_off + b_bytes;
  p.xs_off = p.part_off + part_bytes;
  p.red_off = p.xs_off + 128;
  p.wsb_off = p.red_off + 18 * NT * 4;
  p.bar_off = p.wsb_off + 2 * kSmallRows * 4;
  p.misc_off = p.bar_off + 256;
  const int alloc = p.misc_off + 16 + 1024;
  CUtensorMap tmW, tmX;
  if (!make_tmap_i8(&tmW, a.Wq, a.N, a.K, kSmallRows) ||
      (!kFused && !make_tmap_i8(&tmX, a.Xq, a.M, a.K, NT))) {
    *why = "cuTensorMapEncodeTiled failed or unavailable";
    return cudaErrorInvalidValue;
  }
  if (kFused) tmX = tmW;  // unused
  auto kern = gemm_small_m_kernel<NT, kFused>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, alloc);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, kCarveoutMaxShared);
  if (e != cudaSuccess) {
    *why = "cudaFuncSetAttribute failed";
    return e;
  }
  e = launch_pdl_cluster(kern, dim3(static_cast<unsigned>(S), static_cast<unsigned>(nrb), 1), dim3(kSmallThreads),
                         static_cast<size_t>(alloc), st, static_cast<unsigned>(S), tmW, tmX, p);
  if (e != cudaSuccess) *why = "cluster launch of the small-M kernel failed";
  return e;
}

// Clusters of two CTAs of `kern` (threads, smem bytes) that can run at once:
// the persistent grid of a CTA-pair kernel.  Cached per device in `cache`.
template <typename Kern>
int max_pair_clusters(Kern kern, int threads, int smem, const DeviceInfo& dev, int (&cache)[64]) {
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  if (dev.device < 0 || dev.device >= 64) return 0;
  if (cache[dev.device] != 0) return cache[dev.device];
  int n = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * static_cast<unsigned>(dev.sm_count / 2));
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess)
    n = 0;
  cache[dev.device] = n > 0 ? n : -1;
  return cache[dev.device];
}

int pair_clusters(const DeviceInfo& dev) {
  static int cache[64] = {};
  return max_pair_clusters(gemm_i8_pair_kernel<0>, kPairThreads, kPairAlloc, dev, cache);
}

int prologue_clusters(const DeviceInfo& dev) {
  static int cache[64] = {};
  return max_pair_clusters(gemm_i8_prologue_kernel, kFThreads, kFAlloc, dev, cache);
}

template <int EPI>
cudaError_t run_pair(const GemmArgs& a, cudaStream_t st, const DeviceInfo& dev, int clusters, const char** why) {
  CUtensorMap tmA, tmB;
  if (!make_tmap_i8(&tmA, a.A, a.M, a.K, kPairHalf) || !make_tmap_i8(&tmB, a.B, a.N, a.K, kPairHalf)) {
    *why = "cuTensorMapEncodeTiled failed or unavailable";
    return cudaErrorInvalidValue;
  }
  PairParams p;
  p.timeout_ns = g_debug_stall.load() ? g_debug_timeout_ns.load() : kWaitTimeoutNs;
  p.skip_first_load = g_debug_stall.load() ? 1 : 0;
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.num_m_blocks = static_cast<int>((a.M + kPairBM - 1) / kPairBM);
  p.num_n_blocks = static_cast<int>((a.N + kPairBN - 1) / kPairBN);
  p.num_k_blocks = static_cast<int>((a.K + kBK - 1) / kBK);
  p.group_m = tile_group_m(kPairBM, a.K, p.num_m_blocks);
  p.x_scale = a.x_scale;
  p.w_scale = a.w_scale;
  p.bias = a.bias;
  p.out = a.out;
  const int elem = (EPI == 0) ? 2 : 4;
  p.vec_ok = ((a.N * elem) % 16 == 0) && (reinterpret_cast<uintptr_t>(a.out) % 16 == 0) &&
             (reinterpret_cast<uintptr_t>(a.w_scale) % 16 == 0 || EPI != 0) &&
             (a.bias == nullptr || reinterpret_cast<uintptr_t>(a.bias) % 16 == 0);
  auto kern = gemm_i8_pair_kernel<EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kPairAlloc);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, kCarveoutMaxShared);
  if (e != cudaSuccess) {
    *why = "cudaFuncSetAttribute failed";
    return e;
  }
  const int tiles = p.num_m_blocks * p.num_n_blocks;
  const int pairs = std::min(tiles, clusters);
  e = launch_pdl_cluster(kern, dim3(2u * static_cast<unsigned>(pairs)), dim3(kPairThreads),
                         static_cast<size_t>(kPairAlloc), st, 2u, tmA, tmB, p);
  if (e != cudaSuccess) *why = "cluster launch of the CTA-pair GEMM failed";
  return e;
}

// K split over a CTA pair (cluster of 2); the pair exchanges partial sums
// through `a.ws` (at least splitk_workspace_bytes).
cudaError_t run_splitk(const GemmArgs& a, cudaStream_t st, const char** why) {
  CUtensorMap tmA, tmB;
  if (!make_tmap_i8(&tmA, a.A, a.M, a.K, kBM) || !make_tmap_i8(&tmB, a.B, a.N, a.K, kSkBN)) {
    *why = "cuTensorMapEncodeTiled failed or unavailable";
    return cudaErrorInvalidValue;
  }
  SkParams p{};
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.num_m_blocks = static_cast<int>((a.M + kBM - 1) / kBM);
  p.nk = static_cast<int>((a.K + kBK - 1) / kBK);
  p.kb_per_split = (p.nk + 1) / 2;
  p.x_scale = a.x_scale;
  p.w_scale = a.w_scale;
  p.bias = a.bias;
  p.out = static_cast<uint16_t*>(a.out);
  p.part = static_cast<uint4*>(a.ws);
  p.vec_ok = ((a.N * 2) % 16 == 0) && (reinterpret_cast<uintptr_t>(a.out) % 16 == 0);
  // Y by TMA stores of 32 x 32 boxes (64-byte rows, 64-byte swizzle) when its
  // row pitch allows a tensor map; otherwise per-thread stores
  CUtensorMap tmY = tmA;  // unused unless tma_store
  p.tma_store = p.vec_ok && make_tmap_2d(&tmY, a.out, a.M, a.N, 2, kSkChunkCols, 32, 64) ? 1 : 0;
  p.skip_first_load = g_debug_stall.load() ? 1 : 0;
  p.timeout_ns = g_debug_stall.load() ? g_debug_timeout_ns.load() : kWaitTimeoutNs;
  const int tiles = p.num_m_blocks * static_cast<int>((a.N + kSkBN - 1) / kSkBN);
  auto kern = gemm_i8_splitk_kernel;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSkAlloc);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, kCarveoutMaxShared);
  if (e != cudaSuccess) {
    *why = "cudaFuncSetAttribute failed";
    return e;
  }
  e = launch_pdl_cluster(kern, dim3(2u, static_cast<unsigned>(tiles), 1), dim3(kSkThreads),
                         static_cast<size_t>(kSkAlloc), st, 2u, tmA, tmB, tmY, p);
  if (e != cudaSuccess) *why = "cluster launch of the split-K GEMM failed";
  return e;
}

}  // namespace

cudaError_t launch_small_m(const SmallArgs& a, cudaStream_t st, const DeviceInfo& dev, const char** why) {
  if (a.M < 1 || a.M > kSmallMaxM) return cudaErrorNotSupported;
  const bool fused = a.X != nullptr;
  if (a.M <= 16) return fused ? run_small<16, true>(a, st, dev, why) : run_small<16, false>(a, st, dev, why);
  return fused ? run_small<32, true>(a, st, dev, why) : run_small<32, false>(a, st, dev, why);
}

// Split K over a CTA pair when 128 x 256 tiles fill at most half the SMs and
// K has at least four 128-byte k-blocks (bf16 epilogue only).
static bool use_splitk(int64_t M, int64_t N, int64_t K, int sm_count) {
  const int64_t tiles256 = ((M + kBM - 1) / kBM) * ((N + 255) / 256);
  const int64_t nk = (K + kBK - 1) / kBK;
  return SQ_GEMM_SPLITK && SQ_GEMM_BN == 0 && 2 * tiles256 <= sm_count && nk >= 4;
}

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int sm_count) {
  if (!use_splitk(M, N, K, sm_count)) return 0;
  const int64_t tiles256 = ((M + kBM - 1) / kBM) * ((N + 255) / 256);
  return static_cast<size_t>(tiles256) * 2 * kSkSlotBytes;
}

cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t st, const DeviceInfo& dev, const char** why) {
  // An M=128 int8 MMA costs about the same for N=128 as for N=256, so the main
  // loop of an SM takes as long for a 128 x 128 tile as for a 128 x 256 one.
  // With t tiles of 128 x 256:
  //   2t <= SMs: split each tile's K over a CTA pair (twice the SMs, half the
  //              main loop each, plus one exchange of partial sums), given a
  //              workspace for that exchange; without one, 128 x 128 tiles;
  //   else:      128 x 256 tiles, persistent (128-wide tiles would give an SM
  //              two tiles' worth of MMAs where a 256-wide one gives it one).
  const int64_t tiles256 = ((a.M + kBM - 1) / kBM) * ((a.N + 255) / 256);
  if (a.epi == Epilogue::kBf16Dequant && a.ws != nullptr) {
    const size_t need = gemm_workspace_bytes(a.M, a.N, a.K, dev.sm_count);
    if (need > 0 && a.ws_bytes >= need) return run_splitk(a, st, why);
  }
  // Output tiles of 256 x 256 on CTA pairs whenever they fill every pair at
  // least once: each CTA then reads a third less operand data per MMA than
  // with 128 x 256 tiles of its own.
  if (SQ_GEMM_PAIR && SQ_GEMM_BN == 0) {
    const int64_t pair_tiles = ((a.M + kPairBM - 1) / kPairBM) * ((a.N + kPairBN - 1) / kPairBN);
    const int clusters = pair_clusters(dev);
    if (clusters > 0 && pair_tiles >= clusters)
      return a.epi == Epilogue::kBf16Dequant ? run_pair<0>(a, st, dev, clusters, why)
                                             : run_pair<1>(a, st, dev, clusters, why);
  }
  const bool wide = SQ_GEMM_BN == 256 || (SQ_GEMM_BN == 0 && 2 * tiles256 > dev.sm_count);
  if (a.epi == Epilogue::kBf16Dequant) {
    return wide ? run_gemm<256, 4, 0, 1>(a, st, dev, why) : run_gemm<128, 6, 0, SQ_GEMM_CHAINS128>(a, st, dev, why);
  }
  return wide ? run_gemm<256, 4, 1, 1>(a, st, dev, why) : run_gemm<128, 6, 1, SQ_GEMM_CHAINS128>(a, st, dev, why);
}

cudaError_t launch_forward_prologue(const PrologueArgs& a, cudaStream_t st, const DeviceInfo& dev, const char** why) {
  // pre-pass: x_scale[M] and RN(1/s)[K]
  cudaError_t e = launch_act_scales(a.X, a.M, a.K, a.s, a.x_scale, a.rs, st, dev);
  if (e != cudaSuccess) {
    *why = "scale pre-pass launch";
    return e;
  }
  const int clusters = prologue_clusters(dev);
  if (clusters <= 0) {
    *why = "the fused-prologue GEMM cannot be resident on this device";
    return cudaErrorNotSupported;
  }
  CUtensorMap tmX, tmB;
  if (!make_tmap_2d(&tmX, a.X, a.M, a.K, 2, kFXCols, kFHalf) || !make_tmap_i8(&tmB, a.Wq, a.N, a.K, kFHalf)) {
    *why = "cuTensorMapEncodeTiled failed or unavailable";
    return cudaErrorInvalidValue;
  }
  PrologueParams p;
  p.timeout_ns = g_debug_stall.load() ? g_debug_timeout_ns.load() : kWaitTimeoutNs;
  p.skip_first_load = g_debug_stall.load() ? 1 : 0;
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.num_m_blocks = static_cast<int>((a.M + kFBM - 1) / kFBM);
  p.num_n_blocks = static_cast<int>((a.N + kFBN - 1) / kFBN);
  p.num_k_blocks = static_cast<int>((a.K + kBK - 1) / kBK);
  p.group_m = tile_group_m(kFBM, 2 * a.K, p.num_m_blocks);  // groups of bf16 X rows
  p.s = a.s;
  p.rs = a.rs;
  p.x_scale = a.x_scale;
  p.w_scale = a.w_scale;
  p.bias = a.bias;
  p.out = a.Y;
  p.vec_ok = (a.N % 8 == 0) && (reinterpret_cast<uintptr_t>(a.Y) % 16 == 0) &&
             (reinterpret_cast<uintptr_t>(a.w_scale) % 16 == 0) &&
             (a.bias == nullptr || reinterpret_cast<uintptr_t>(a.bias) % 16 == 0);
  auto kern = gemm_i8_prologue_kernel;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kFAlloc);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, kCarveoutMaxShared);
  if (e != cudaSuccess) {
    *why = "cudaFuncSetAttribute failed";
    return e;
  }
  const int tiles = p.num_m_blocks * p.num_n_blocks;
  const int pairs = std::min(tiles, clusters);
  e = launch_pdl_cluster(kern, dim3(2u * static_cast<unsigned>(pairs)), dim3(kFThreads), static_cast<size_t>(kFAlloc),
                         st, 2u, tmX, tmB, p);
  if (e != cudaSuccess) *why = "cluster launch of the fused-prologue GEMM failed";
  return e;
}

#ifdef SQ_TRACE
extern "C" __attribute__((visibility("default"))) int sq_trace_read_sk(unsigned long long* host, int n) {
  return cudaMemcpyFromSymbol(host, g_sk_trace, sizeof(unsigned long long) * 8 * static_cast<size_t>(n)) ==
                 cudaSuccess
             ? 0
             : 1;
}
extern "C" __attribute__((visibility("default"))) int sq_trace_read_big(unsigned long long* host, int n) {
  return cudaMemcpyFromSymbol(host, g_big_trace, sizeof(unsigned long long) * 5 * static_cast<size_t>(n)) ==
                 cudaSuccess
             ? 0
             : 1;
}
extern "C" __attribute__((visibility("default"))) int sq_trace_read_prologue(unsigned long long* conv,
                                                                             unsigned long long* x) {
  return cudaMemcpyFromSymbol(conv, sq::g_pro_trace, sizeof(sq::g_pro_trace)) == cudaSuccess &&
                 cudaMemcpyFromSymbol(x, sq::g_pro_xtrace, sizeof(sq::g_pro_xtrace)) == cudaSuccess
             ? 0
             : 1;
}
extern "C" __attribute__((visibility("default"))) int sq_trace_read(unsigned long long* host, int n) {
  return cudaMemcpyFromSymbol(host, g_small_trace, sizeof(unsigned long long) * 12 * static_cast<size_t>(n)) ==
                 cudaSuccess
             ? 0
             : 1;
}
#endif

void debug_pipeline_stall(bool enable, unsigned long long timeout_ns) {
  g_debug_timeout_ns.store(timeout_ns > 0 ? timeout_ns : kWaitTimeoutNs);
  g_debug_stall.store(enable ? 1 : 0);
}

bool debug_stall_state(unsigned long long* timeout_ns) {
  const bool on = g_debug_stall.load() != 0;
  *timeout_ns = on ? g_debug_timeout_ns.load() : kWaitTimeoutNs;
  return on;
}

cudaError_t read_device_status(uint32_t* flags, bool clear) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return e;
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_sq_device_status, sizeof(v));
  if (e != cudaSuccess) return e;
  if (clear) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_sq_device_status, &z, sizeof(z));
    if (e != cudaSuccess) return e;
  }
  uint32_t q = 0, w = 0, b = 0;
  e = read_quant_status(&q, clear);
  if (e == cudaSuccess) e = read_weight_only_status(&w, clear);
  if (e == cudaSuccess) e = read_ste_status(&b, clear);
  if (e != cudaSuccess) return e;
  *flags = v | q | w | b;
  return cudaSuccess;
}

bool make_tmap_2d(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int elem_bytes, int box_cols,
                  int box_rows, int swizzle_bytes, int64_t pitch_bytes) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  CUtensorMapDataType dt;
  switch (elem_bytes) {
    case 1: dt = CU_TENSOR_MAP_DATA_TYPE_UINT8; break;
    case 2: dt = CU_TENSOR_MAP_DATA_TYPE_UINT16; break;
    case 4: dt = CU_TENSOR_MAP_DATA_TYPE_UINT32; break;
    default: return false;
  }
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {pitch_bytes > 0 ? static_cast<cuuint64_t>(pitch_bytes)
                                           : static_cast<cuuint64_t>(cols) * static_cast<cuuint64_t>(elem_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUtensorMapSwizzle sw;
  switch (swizzle_bytes) {
    case 0: sw = CU_TENSOR_MAP_SWIZZLE_NONE; break;
    case 32: sw = CU_TENSOR_MAP_SWIZZLE_32B; break;
    case 64: sw = CU_TENSOR_MAP_SWIZZLE_64B; break;
    case 128: sw = CU_TENSOR_MAP_SWIZZLE_128B; break;
    default: return false;
  }
  CUresult r = enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace sq
