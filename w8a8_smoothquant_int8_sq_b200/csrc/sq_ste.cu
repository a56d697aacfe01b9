// sq_ste.cu -- backward pass of the learnable-alpha SmoothQuant layer under
// the straight-through estimator.
//
// Page: "w8a8_smoothquant.py -- W8A8 com SmoothQuant e alpha APRENDIVEL (V5)":
// SmoothQuantW8A8.forward in quantised mode recomputes
//     s = clamp(mx^alpha / mw^(1-alpha), 1e-8),  alpha = sigmoid(eta_alpha),
// smooths X / s and weight_fp * s, fake-quantises both with STEQuantize
// (per token and per output channel; round and clamp pass the gradient
// through, the scales get none) and returns X_q_deq @ W_q_deq^T + bias.
// With G = dL/dY, Wdq = Wq * w_scale and Xdq = Xq * x_scale the chain rule
// gives
//     dXs = G Wdq,  dX = dXs / s          dWs = G^T Xdq,  dW = dWs * s
//     db  = sum over tokens of G
//     ds_k s_k = sum_n dWs[n][k] (W[n][k] s_k - Wdq[n][k])
//              - sum_m dXs[m][k] (X[m][k] / s_k - Xdq[m][k])
//     d eta = alpha (1 - alpha) sum_k ds_k raw_k (ln mx_k + ln mw_k) [raw_k >= 1e-8]
// The ds form above equals the page's sum_n dWs W - sum_m dXs X / s^2 (the
// two differ by sum_n dWs Wdq - sum_m dXs Xdq, which is zero), written with
// the quantisation errors so that no two large sums cancel.
//
// Precision.  Both products take the int8 codes as exact bf16 operands and
// move the scale onto the gradient side, where it is split in two bf16 halves:
//     dXs^T[k][m] = sum_n q_w[n][k] (Ghi + Glo)[m][n],  G' = G[m][n] w_scale[n]
//     dWs^T[k][n] = sum_m q_x[m][k] (Gthi + Gtlo)[n][m], G'' = G[m][n] x_scale[m]
// with hi = bf16(v), lo = bf16(v - hi), so the operands carry 2^-16 relative
// error instead of bf16's 2^-8 (two MMAs per step instead of one).  That
// keeps each channel's ds accurate enough for d eta, a sum over channels
// that cancels heavily.
//
// Kernels (all chained with programmatic dependent launch):
//   transpose_codes_kernel  Wt[k][n] = Wq[n][k], Xt[k][m] = Xq[m][k] as bf16;
//                           the first launch also zeroes the per-channel sums,
//                           db and the finish counter
//   split_g_kernel          Ghi/Glo[m][n] from G w_scale, Gthi/Gtlo[n][m] from
//                           G x_scale (transposed), db[n] += sum_m G[m][n]
//   ste_gemm_kernel<DX>     dXs^T on the tensor cores (bf16 in, fp32 in TMEM);
//                           epilogue writes dX and adds lane k's
//                           sum_m dXs (X/s - Xdq)
//   ste_gemm_kernel<DW>     dWs^T; epilogue writes dW, adds
//                           sum_n dWs (W s - Wdq) and max |W| per k
//   ste_finish_kernel       d eta from the per-channel sums
// The GEMMs put the channel k on the MMA's M side (TMEM lanes), so the sums
// over tokens or output rows that ds needs run inside one thread.
#include <algorithm>
#include <cstdint>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {
namespace {

__device__ unsigned int g_sq_ste_status = 0u;

constexpr int kTT = 64;            // transpose tile (64 x 64 elements)
constexpr int kTThreads = 256;
constexpr int kSBM = 128;          // GEMM tile rows (channels k) = MMA M
constexpr int kSBN = 128;          // GEMM tile columns (tokens or output rows) = MMA N
constexpr int kSBK = 64;           // contraction elements per stage (128 bytes of bf16)
constexpr int kSUmmaK = 16;        // contraction per tcgen05.mma kind::f16
constexpr int kSStages = 4;
constexpr int kSEpiWarps = 8;     // two per TMEM lane quarter, each taking half of the tile's columns
constexpr int kSThreads = 64 + 32 * kSEpiWarps;
constexpr int kSABytes = kSBM * kSBK * 2;
constexpr int kSBBytes = kSBN * kSBK * 2;  // one half (hi or lo)
constexpr int kSStageBytes = kSABytes + 2 * kSBBytes;
constexpr int kSBarOffset = kSStages * kSStageBytes;
constexpr int kSNumBars = 2 * kSStages + 4 + 1;
// per epilogue warp: a 32 x 32 block of src (bf16, 80-byte rows) and of q
// (int8, 48-byte rows) staged for the transposed read, and the block's 32
// column scales; the row pitches keep the 16-byte stores of 8 consecutive
// lanes on distinct bank groups
constexpr int kStgSrcPitch = 80;
constexpr int kStgQPitch = 48;
constexpr int kStgBytes = 32 * kStgSrcPitch + 32 * kStgQPitch + 32 * 4;
constexpr int kSStgOffset = (kSBarOffset + kSNumBars * 8 + 15) / 16 * 16;
constexpr int kSMiscOffset = kSStgOffset + kSEpiWarps * kStgBytes;
constexpr int kSAlloc = kSMiscOffset + 16 + 1024;
constexpr int kSAccCols = 2 * kSBN;         // one accumulator: A Bh^T in columns [0, 128), A Bl^T in [128, 256)
constexpr uint32_t kSTmemCols = 2 * kSAccCols;
constexpr int kEpiDX = 0;
constexpr int kEpiDW = 1;

// Warp-wide load of 8 consecutive 32-bit TMEM columns; lane i of the warp gets
// TMEM lane (warp quarter * 32 + i).
__device__ __forceinline__ void tmem_ld_8cols(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}

__device__ __forceinline__ uint16_t bf16_bits_rn(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }

// store the first min(4, n) of v0..v3 at dst (8-byte aligned when n >= 4)
__device__ __forceinline__ void store4(uint16_t* dst, int n, uint16_t v0, uint16_t v1, uint16_t v2, uint16_t v3) {
  if (n >= 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(static_cast<uint32_t>(v0) | (static_cast<uint32_t>(v1) << 16),
                                                static_cast<uint32_t>(v2) | (static_cast<uint32_t>(v3) << 16));
  } else {
    dst[0] = v0;
    if (n > 1) dst[1] = v1;
    if (n > 2) dst[2] = v2;
  }
}

// Per-call sums that the later kernels accumulate into, zeroed by the first
// transpose (before the split of G adds to db and the GEMMs to tx, tw, mw).
struct SteZero {
  float* tx;
  float* tw;
  unsigned int* mwbits;
  int K;
  float* db;  // may be null
  int N;
  unsigned int* counter;
};

// out[c][r] = in[r][c] as bf16 (exact for int8 codes) for r < R, c < C.  in:
// int8, row pitch C (C % 4 == 0); out: row pitch ldo elements (ldo % 8 == 0).
// Thread (ty, tx) of a 16 x 16 block loads 4 codes of rows ty + 16i and
// stores 4 outputs of rows ty + 16i of the transposed tile.  With zero.tx not
// null the grid also zeroes the words of `zero`.
__global__ void __launch_bounds__(kTThreads) transpose_codes_kernel(const int8_t* in, int R, int C, uint16_t* out,
                                                                     int ldo, SteZero zero) {
  __shared__ uint16_t tile[kTT][kTT + 2];
  const int c0 = blockIdx.x * kTT, r0 = blockIdx.y * kTT;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  griddep_wait();
  griddep_launch_dependents();
  if (zero.tx != nullptr) {
    const int nb = gridDim.x * gridDim.y;
    const int b = blockIdx.y * gridDim.x + blockIdx.x;
    const int stride = nb * kTThreads;
    for (int i = b * kTThreads + threadIdx.x; i < zero.K; i += stride) {
      zero.tx[i] = 0.0f;
      zero.tw[i] = 0.0f;
      zero.mwbits[i] = 0u;
    }
    if (zero.db != nullptr)
      for (int i = b * kTThreads + threadIdx.x; i < zero.N; i += stride) zero.db[i] = 0.0f;
    if (b == 0 && threadIdx.x == 0) *zero.counter = 0u;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rl = ty + 16 * i, r = r0 + rl, c = c0 + 4 * tx;
    uint32_t w = 0u;
    if (r < R && c < C) w = *reinterpret_cast<const uint32_t*>(in + static_cast<int64_t>(r) * C + c);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int q = static_cast<int>(static_cast<int8_t>(w >> (8 * j)));
      tile[4 * tx + j][rl] = bf16_bits_rn(static_cast<float>(q));
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int cl = ty + 16 * i, c = c0 + cl, r = r0 + 4 * tx;
    if (c >= C || r >= R) continue;
    store4(out + static_cast<int64_t>(c) * ldo + r, R - r, tile[cl][4 * tx], tile[cl][4 * tx + 1],
           tile[cl][4 * tx + 2], tile[cl][4 * tx + 3]);
  }
}

// From G[R = M][C = N] (bf16, row pitch C, C % 4 == 0):
//   gh/gl[r][c]   = hi/lo of G[r][c] * cscale[c]      (row pitch C)
//   gth/gtl[c][r] = hi/lo of G[r][c] * rscale[r]      (row pitch ldt, ldt % 8 == 0)
//   colsum[c]    += sum_r G[r][c]                     (when not null)
// hi = bf16(v), lo = bf16(v - hi); v - hi is exact in fp32.
__global__ void __launch_bounds__(kTThreads) split_g_kernel(const uint16_t* G, int R, int C, const float* cscale,
                                                             const float* rscale, uint16_t* gh, uint16_t* gl,
                                                             uint16_t* gth, uint16_t* gtl, int ldt, float* colsum) {
  __shared__ float tile[kTT][kTT + 1];  // [c][r], G * rscale[r]
  __shared__ float gcol[kTT][kTT + 1];  // [c][r], G
  const int c0 = blockIdx.x * kTT, r0 = blockIdx.y * kTT;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  griddep_wait();
  griddep_launch_dependents();
  float cs[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) cs[j] = (c0 + 4 * tx + j < C) ? cscale[c0 + 4 * tx + j] : 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rl = ty + 16 * i, r = r0 + rl, c = c0 + 4 * tx;
    uint2 w = make_uint2(0u, 0u);
    float rs = 0.0f;
    const bool ok = r < R && c < C;
    if (ok) {
      w = *reinterpret_cast<const uint2*>(G + static_cast<int64_t>(r) * C + c);
      rs = rscale[r];
    }
    const float g[4] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y)};
    uint16_t h[4], l[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float v = __fmul_rn(g[j], cs[j]);
      h[j] = bf16_bits_rn(v);
      l[j] = bf16_bits_rn(__fsub_rn(v, __uint_as_float(static_cast<uint32_t>(h[j]) << 16)));
      tile[4 * tx + j][rl] = __fmul_rn(g[j], rs);
      gcol[4 * tx + j][rl] = g[j];
    }
    if (ok) {
      const int64_t e = static_cast<int64_t>(r) * C + c;
      *reinterpret_cast<uint2*>(gh + e) = make_uint2(static_cast<uint32_t>(h[0]) | (static_cast<uint32_t>(h[1]) << 16),
                                                     static_cast<uint32_t>(h[2]) | (static_cast<uint32_t>(h[3]) << 16));
      *reinterpret_cast<uint2*>(gl + e) = make_uint2(static_cast<uint32_t>(l[0]) | (static_cast<uint32_t>(l[1]) << 16),
                                                     static_cast<uint32_t>(l[2]) | (static_cast<uint32_t>(l[3]) << 16));
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int cl = ty + 16 * i, c = c0 + cl, r = r0 + 4 * tx;
    float sum = 0.0f;
    if (c < C && r < R) {
      uint16_t h[4], l[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float v = tile[cl][4 * tx + j];
        h[j] = bf16_bits_rn(v);
        l[j] = bf16_bits_rn(__fsub_rn(v, __uint_as_float(static_cast<uint32_t>(h[j]) << 16)));
        sum += gcol[cl][4 * tx + j];  // entries past R are zeros
      }
      const int64_t e = static_cast<int64_t>(c) * ldt + r;
      store4(gth + e, R - r, h[0], h[1], h[2], h[3]);
      store4(gtl + e, R - r, l[0], l[1], l[2], l[3]);
    }
    // the 16 threads of a half warp hold the same output row c
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    if (colsum != nullptr && tx == 0 && c < C) atomicAdd(colsum + c, sum);
  }
}

struct SteGemmParams {
  int I, J, C;  // output rows (channels k), output columns, contraction length
  int num_i_blocks, num_j_blocks, num_c_blocks;
  const float* s;          // [I]
  const uint16_t* src;     // X or W: element (j, i) at src[j * I + i]
  const int8_t* q;         // Xq or Wq: element (j, i) at q[j * I + i]
  const float* qscale;     // x_scale or w_scale, per column j
  float* out;              // dX or dW: element (j, i) at out[j * I + i]
  float* tsum;             // [I] sum over j of dXs * dX_q (or dWs * dW_q)
  unsigned int* mwbits;    // DW: [I] max |W| as fp32 bits
  unsigned long long timeout_ns;  // limit of every mbarrier wait
  int skip_first_load;            // test hook: the producer never loads its first stage
};

#ifdef SQ_TRACE
// Optional per-tile timestamps (build with -DSQ_TRACE), CTAs 0..3, first 16
// tiles of each: MMA thread at 0 accumulator free, 1 last MMA issued;
// epilogue warp 0 (lane 0) at 2 block loads issued, 3 accumulator ready,
// 4 first 32 columns done, 5 tile done.  [EPI][cta][tile][mark]
__device__ unsigned long long g_ste_trace[2][4][16][6];
#define SQ_STE_MARK(t, i)                                                                              \
  do {                                                                                                 \
    if (blockIdx.x < 4 && (t) < 16) g_ste_trace[EPI][blockIdx.x][(t)][(i)] = globaltimer_ns();         \
  } while (0)
extern "C" __attribute__((visibility("default"))) int sq_trace_read_ste(unsigned long long* host) {
  return cudaMemcpyFromSymbol(host, g_ste_trace, sizeof(g_ste_trace)) == cudaSuccess ? 0 : 1;
}
#else
#define SQ_STE_MARK(t, i) \
  do {                    \
  } while (0)
#endif

__device__ __forceinline__ void ste_flag_timeout(volatile int* abort_flag) {
  *abort_flag = 1;
  atomicOr(&g_sq_ste_status, 1u);
}

// D[i][j] = sum_c A[i][c] (Bh[j][c] + Bl[j][c]) with A [I][C], Bh and Bl
// [J][C] bf16 (row-major, loaded by TMA in 128 x 64-element boxes with the
// 128-byte swizzle), one CTA per SM persistent over 128 x 128 tiles: warp 0
// loads (and prefetches the tile's src and q blocks into L2 for the
// epilogue), warp 1 issues tcgen05.mma kind::f16 with N = 256 -- the Bh and
// Bl boxes sit back to back in shared memory and form one 256-row operand, so
// one MMA yields A Bh^T and A Bl^T side by side -- into one of two TMEM
// accumulators, warps 2..5 run the epilogue of EPI on TMEM lanes (rows i)
// 32 (warp % 4) .. + 31, adding the two halves.
template <int EPI>
__global__ void __launch_bounds__(kSThreads, 1)
    ste_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmBh,
                    const __grid_constant__ CUtensorMap tmBl, const __grid_constant__ CUtensorMap tmSrc,
                    const __grid_constant__ CUtensorMap tmQ, const SteGemmParams p) {
  extern __shared__ uint8_t ste_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ste_smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSBarOffset);
  uint64_t* full = bars;
  uint64_t* empty = bars + kSStages;
  uint64_t* tfull = bars + 2 * kSStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSMiscOffset);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSMiscOffset + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kSEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmBh);
    tma_prefetch_desc(&tmBl);
    tma_prefetch_desc(&tmSrc);
    tma_prefetch_desc(&tmQ);
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(tmem_slot, kSTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();
  griddep_launch_dependents();

  const int num_tiles = p.num_i_blocks * p.num_j_blocks;
  const int nk = p.num_c_blocks;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued[kSStages];
      uint32_t issued_phase[kSStages];
#pragma unroll
      for (int i = 0; i < kSStages; ++i) issued[i] = 0, issued_phase[i] = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const int i_blk = tile % p.num_i_blocks;
        const int j_blk = tile / p.num_i_blocks;
        // the epilogue's src and q blocks of this tile, into L2
        tma_prefetch_l2_2d(&tmSrc, i_blk * kSBM, j_blk * kSBN);
        tma_prefetch_l2_2d(&tmQ, i_blk * kSBM, j_blk * kSBN);
        for (int kb = 0; kb < nk; ++kb) {
          if (*abort_flag || !mbar_wait_bounded(&empty[stage], phase ^ 1u, p.timeout_ns)) {
            if (!*abort_flag) ste_flag_timeout(abort_flag);
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * kSStageBytes;
          uint8_t* sb = sa + kSABytes;
          if (!(p.skip_first_load && tile == static_cast<int>(blockIdx.x) && kb == 0)) {
            mbar_arrive_expect_tx(&full[stage], kSStageBytes);
            tma_load_2d(sa, &tmA, kb * kSBK, i_blk * kSBM, &full[stage]);
            tma_load_2d(sb, &tmBh, kb * kSBK, j_blk * kSBN, &full[stage]);
            tma_load_2d(sb + kSBBytes, &tmBl, kb * kSBK, j_blk * kSBN, &full[stage]);
            issued[stage] = 1;  // (test hook: a skipped stage is not waited for)
            issued_phase[stage] = phase;
          }
          if (++stage == kSStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
#pragma unroll
        for (int i = 0; i < kSStages; ++i)
          if (issued[i]) (void)mbar_wait_bounded(&full[i], issued_phase[i], p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kSBM, 2 * kSBN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (*abort_flag || !mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, p.timeout_ns)) {
          if (!*abort_flag) ste_flag_timeout(abort_flag);
          break;
        }
        SQ_STE_MARK(it, 0);
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kSAccCols);
        for (int kb = 0; kb < nk; ++kb) {
          if (*abort_flag || !mbar_wait_bounded(&full[stage], phase, p.timeout_ns)) {
            if (!*abort_flag) ste_flag_timeout(abort_flag);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kSStageBytes);
          const uint32_t sb = sa + kSABytes;
          const uint64_t adesc = smem_desc_k_sw128(sa);
          const uint64_t bdesc = smem_desc_k_sw128(sb);  // Bh rows 0..127, Bl rows 128..255
#pragma unroll
          for (int kk = 0; kk < kSBK / kSUmmaK; ++kk)  // 32 bytes per step inside the swizzle atom
            mma_bf16(d_tmem, adesc + static_cast<uint64_t>(kk * 2), bdesc + static_cast<uint64_t>(kk * 2), idesc,
                     (kb != 0 || kk != 0) ? 1u : 0u);
          mma_commit(&empty[stage]);
          if (++stage == kSStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        SQ_STE_MARK(it, 1);
        mma_commit(&tfull[acc]);
      }
      mma_commit(drain);
      (void)mbar_wait_bounded(drain, 0, p.timeout_ns);
    }
  } else {
    const int quarter = warp & 3;          // TMEM lanes 32 quarter .. + 31
    const int ew = warp - 2;               // epilogue warp 0 .. kSEpiWarps - 1
    const int half = ew / 4;               // columns [64 half, 64 half + 64) of each tile
    uint8_t* stg = smem + kSStgOffset + ew * kStgBytes;
    uint16_t* stg_src = reinterpret_cast<uint16_t*>(stg);                 // [32 j][kStgSrcPitch bytes]
    int8_t* stg_q = reinterpret_cast<int8_t*>(stg + 32 * kStgSrcPitch);  // [32 j][kStgQPitch bytes]
    float* stg_qs = reinterpret_cast<float*>(stg + 32 * (kStgSrcPitch + kStgQPitch));  // [32 j]
    constexpr int kChunks = kSBN / 32 / 2;  // 32-column chunks per warp and tile
    // this warp's 32 x 64 block of src and q of a tile and its column scales:
    // lane l holds row j_blk * 128 + 64 half + 32 cc + l, the warp's 32
    // columns from i0 (those that exist; the rest stay zero).  A tile's blocks
    // are fetched while the previous tile's last chunk is processed (the
    // first tile's before its accumulator is ready), so the loads overlap the
    // epilogue and the MMAs.
    uint4 ra[kChunks][4], rb[kChunks][2];
    float rq[kChunks];
    auto load_blocks = [&](int t) {
      const int ib = t % p.num_i_blocks;
      const int jb = t / p.num_i_blocks;
      const int r0 = ib * kSBM + quarter * 32;
      // rows of this warp that exist: 0, 16 or 32 (I % 16 == 0, r0 % 32 == 0)
      const int nr = max(0, min(32, p.I - r0));
#pragma unroll
      for (int cc = 0; cc < kChunks; ++cc) {
        const int j = jb * kSBN + half * 64 + cc * 32 + lane;
#pragma unroll
        for (int u = 0; u < 4; ++u) ra[cc][u] = make_uint4(0u, 0u, 0u, 0u);
        rb[cc][0] = rb[cc][1] = make_uint4(0u, 0u, 0u, 0u);
        rq[cc] = 0.0f;
        if (j < p.J) {
          rq[cc] = __ldg(p.qscale + j);
          if (nr > 0) {
            const int64_t e = static_cast<int64_t>(j) * p.I + r0;
            const uint4* sv = reinterpret_cast<const uint4*>(p.src + e);
            const uint4* qv = reinterpret_cast<const uint4*>(p.q + e);
            ra[cc][0] = sv[0];
            ra[cc][1] = sv[1];
            rb[cc][0] = qv[0];
            if (nr > 16) {
              ra[cc][2] = sv[2];
              ra[cc][3] = sv[3];
              rb[cc][1] = qv[1];
            }
          }
        }
      }
    };
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      const int i_blk = tile % p.num_i_blocks;
      const int j_blk = tile / p.num_i_blocks;
      const int i0 = i_blk * kSBM + quarter * 32;  // this warp's first row
      const int i = i0 + lane;
      const bool row_ok = i < p.I;
      const float s_i = row_ok ? __ldg(p.s + i) : 1.0f;
      const float rs_i = __frcp_rn(s_i);
      if (it == 0) load_blocks(tile);
      if (ew == 0 && lane == 0) SQ_STE_MARK(it, 2);
      const bool mine = !*abort_flag && mbar_wait_bounded(&tfull[acc], acc_phase, p.timeout_ns);
      if (!__all_sync(0xFFFFFFFFu, mine)) {
        if (lane == 0 && !*abort_flag) ste_flag_timeout(abort_flag);
        break;
      }
      tc_fence_after();
      if (ew == 0 && lane == 0) SQ_STE_MARK(it, 3);
      const uint32_t t_base =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * kSAccCols);
      float tsum = 0.0f;
      uint32_t mbits = 0u;
#pragma unroll
      for (int cc = 0; cc < kChunks; ++cc) {
        const int c0 = half * 64 + cc * 32;
        const int j0 = j_blk * kSBN + c0;
        const int jn = min(32, p.J - j0);
        __syncwarp();  // the previous chunk's reads of the staging area are done
        {
          uint4* ds = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(stg_src) + lane * kStgSrcPitch);
#pragma unroll
          for (int u = 0; u < 4; ++u) ds[u] = ra[cc][u];
          uint4* dq = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(stg_q) + lane * kStgQPitch);
          dq[0] = rb[cc][0];
          dq[1] = rb[cc][1];
          stg_qs[lane] = rq[cc];
        }
        // the blocks of this warp's next tile, in flight while this chunk and
        // the tile hand-over run
        if (cc == kChunks - 1 && tile + static_cast<int>(gridDim.x) < num_tiles)
          load_blocks(tile + static_cast<int>(gridDim.x));
        __syncwarp();
        // Columns past J and rows past I hold zeros in every operand (TMA
        // fills the boxes past the matrix with zeros, and the staged blocks
        // start from zero), so they add nothing to the sums; only the stores
        // are predicated, and the loop has no early exit.  Eight columns at a
        // time: each group's TMEM loads end in a wait, which also bounds how
        // far the compiler hoists the staging reads (register pressure).
        const bool st_ok = row_ok && j0 < p.J;
        float* op = p.out + (static_cast<int64_t>(j0) * p.I + i);  // advanced by a row per column
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t r[8], rl[8];
          tmem_ld_8cols(t_base + static_cast<uint32_t>(c0 + 8 * g), r);          // A Bh^T
          tmem_ld_8cols(t_base + static_cast<uint32_t>(kSBN + c0 + 8 * g), rl);  // A Bl^T
          tmem_ld_wait();
          // an opaque copy of the staging pointer: the group's staging reads
          // cannot be hoisted above this point
          const uint8_t* sg = stg;
          asm volatile("" : "+l"(sg));
          const float* sqs = reinterpret_cast<const float*>(sg + 32 * (kStgSrcPitch + kStgQPitch));
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int jj = 8 * g + u;
            const float v = __fadd_rn(__uint_as_float(r[u]), __uint_as_float(rl[u]));
            const uint16_t xb = *reinterpret_cast<const uint16_t*>(sg + jj * kStgSrcPitch + lane * 2);
            const float x = __uint_as_float(static_cast<uint32_t>(xb) << 16);
            const float dq = static_cast<float>(*reinterpret_cast<const int8_t*>(sg + 32 * kStgSrcPitch +
                                                                                 jj * kStgQPitch + lane));
            float o;
            if (EPI == kEpiDX) {
              o = __fmul_rn(v, rs_i);                                           // dXs / s
              const float err = __fmaf_rn(-dq, sqs[jj], __fmul_rn(x, rs_i));  // X/s - Xdq
              tsum = __fmaf_rn(v, err, tsum);
            } else {
              o = __fmul_rn(v, s_i);                                            // dWs * s
              const float err = __fmaf_rn(-dq, sqs[jj], __fmul_rn(x, s_i));   // W*s - Wdq
              tsum = __fmaf_rn(v, err, tsum);
              mbits = max(mbits, static_cast<uint32_t>(xb & 0x7FFFu) << 16);
            }
            if (st_ok && jj < jn) *op = o;
            op += p.I;
          }
        }
        if (cc == 0 && ew == 0 && lane == 0) SQ_STE_MARK(it, 4);
      }
      tc_fence_before();
      __syncwarp();
      if (ew == 0 && lane == 0) SQ_STE_MARK(it, 5);
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (row_ok) {
        atomicAdd(p.tsum + i, tsum);
        if (EPI == kEpiDW) atomicMax(p.mwbits + i, mbits);
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kSTmemCols);
  }
}

// ds_k = T_k / s_k with T_k = tw_k - tx_k, and d eta = alpha (1 - alpha)
// sum_k ds_k raw_k (ln mx_k + ln mw_k) over the channels whose raw_k =
// mx_k^alpha / mw_k^(1-alpha) (both clamped at 1e-8) is not below 1e-8.
// float64; one channel per thread, block sums in `partial`, and the last
// block to finish (arrival counter, zeroed by the first transpose) adds the block
// sums in block order and writes d eta.
constexpr int kFinishThreads = 256;
__global__ void __launch_bounds__(kFinishThreads) ste_finish_kernel(const float* tx, const float* tw,
                                                                     const unsigned int* mwbits, const float* mx,
                                                                     const float* s, float alpha, int K,
                                                                     float* ds_out, double* partial,
                                                                     unsigned int* counter, float* d_eta) {
  __shared__ double part[kFinishThreads / 32];
  __shared__ bool last;
  griddep_wait();
  griddep_launch_dependents();
  const double a = static_cast<double>(alpha);
  const double floor_v = static_cast<double>(kClampFloor);
  double acc = 0.0;
  const int k = blockIdx.x * kFinishThreads + threadIdx.x;
  if (k < K) {
    const double mxc = fmax(static_cast<double>(mx[k]), floor_v);
    const double mwc = fmax(static_cast<double>(__uint_as_float(mwbits[k])), floor_v);
    const double raw = pow(mxc, a) / pow(mwc, 1.0 - a);
    const double ds = (static_cast<double>(tw[k]) - static_cast<double>(tx[k])) / static_cast<double>(s[k]);
    if (ds_out != nullptr) ds_out[k] = static_cast<float>(ds);
    if (raw >= floor_v) acc = ds * raw * (log(mxc) + log(mwc));
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double v = 0.0;
    for (int w = 0; w < kFinishThreads / 32; ++w) v += part[w];
    partial[blockIdx.x] = v;
    __threadfence();
    last = atomicAdd(counter, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (last && threadIdx.x == 0) {
    __threadfence();
    double v = 0.0;
    for (unsigned b = 0; b < gridDim.x; ++b) v += *(volatile double*)(partial + b);
    d_eta[0] = static_cast<float>(a * (1.0 - a) * v);
  }
}

int64_t round_up64(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

struct SteLayout {
  int64_t Mp;
  size_t wt, xt, gh, gl, gth, gtl, tx, tw, mw, fin, total;
};

SteLayout ste_layout(int64_t M, int64_t N, int64_t K) {
  SteLayout L;
  L.Mp = round_up64(M, 8);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = static_cast<size_t>(round_up64(static_cast<int64_t>(off + bytes), 1024));
    return at;
  };
  L.wt = take(static_cast<size_t>(K) * N * 2);
  L.xt = take(static_cast<size_t>(K) * L.Mp * 2);
  L.gh = take(static_cast<size_t>(M) * N * 2);
  L.gl = take(static_cast<size_t>(M) * N * 2);
  L.gth = take(static_cast<size_t>(N) * L.Mp * 2);
  L.gtl = take(static_cast<size_t>(N) * L.Mp * 2);
  L.tx = take(static_cast<size_t>(K) * 4);
  L.tw = take(static_cast<size_t>(K) * 4);
  L.mw = take(static_cast<size_t>(K) * 4);
  L.fin = take(static_cast<size_t>((K + kFinishThreads - 1) / kFinishThreads) * 8 + 16);  // block sums, counter
  L.total = off;
  return L;
}

template <int EPI>
cudaError_t run_ste_gemm(const void* A, const void* Bh, const void* Bl, int64_t I, int64_t J, int64_t C,
                         int64_t pitch_elems, const SteGemmParams& base, cudaStream_t st, const DeviceInfo& dev,
                         const char** why) {
  CUtensorMap tmA, tmBh, tmBl, tmSrc, tmQ;
  if (!make_tmap_2d(&tmA, A, I, C, 2, kSBK, kSBM, 128, pitch_elems * 2) ||
      !make_tmap_2d(&tmBh, Bh, J, C, 2, kSBK, kSBN, 128, pitch_elems * 2) ||
      !make_tmap_2d(&tmBl, Bl, J, C, 2, kSBK, kSBN, 128, pitch_elems * 2) ||
      !make_tmap_2d(&tmSrc, base.src, J, I, 2, kSBM, kSBN, 0) ||
      !make_tmap_2d(&tmQ, base.q, J, I, 1, kSBM, kSBN, 0)) {
    *why = "cuTensorMapEncodeTiled failed or unavailable";
    return cudaErrorInvalidValue;
  }
  SteGemmParams p = base;
  p.skip_first_load = debug_stall_state(&p.timeout_ns) ? 1 : 0;
  p.I = static_cast<int>(I);
  p.J = static_cast<int>(J);
  p.C = static_cast<int>(C);
  p.num_i_blocks = static_cast<int>((I + kSBM - 1) / kSBM);
  p.num_j_blocks = static_cast<int>((J + kSBN - 1) / kSBN);
  p.num_c_blocks = static_cast<int>((C + kSBK - 1) / kSBK);
  auto kern = ste_gemm_kernel<EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSAlloc);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, kCarveoutMaxShared);
  if (e != cudaSuccess) {
    *why = "cudaFuncSetAttribute failed";
    return e;
  }
  const int tiles = p.num_i_blocks * p.num_j_blocks;
  const int grid = std::min(tiles, dev.sm_count);
  return launch_pdl(kern, dim3(grid), dim3(kSThreads), kSAlloc, st, tmA, tmBh, tmBl, tmSrc, tmQ, p);
}

}  // namespace

size_t ste_workspace_bytes(int64_t M, int64_t N, int64_t K) { return ste_layout(M, N, K).total; }

cudaError_t read_ste_status(uint32_t* flags, bool clear) {
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_sq_ste_status, sizeof(v));
  if (e != cudaSuccess) return e;
  if (clear && v != 0u) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_sq_ste_status, &z, sizeof(z));
    if (e != cudaSuccess) return e;
  }
  *flags = v;
  return cudaSuccess;
}

cudaError_t launch_ste_backward(const SteArgs& a, cudaStream_t st, const DeviceInfo& dev, const char** why) {
  const SteLayout L = ste_layout(a.M, a.N, a.K);
  if (a.ws == nullptr || a.ws_bytes < L.total) {
    *why = "workspace too small";
    return cudaErrorInvalidValue;
  }
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  uint16_t* Wt = reinterpret_cast<uint16_t*>(ws + L.wt);
  uint16_t* Xt = reinterpret_cast<uint16_t*>(ws + L.xt);
  uint16_t* Gh = reinterpret_cast<uint16_t*>(ws + L.gh);
  uint16_t* Gl = reinterpret_cast<uint16_t*>(ws + L.gl);
  uint16_t* Gth = reinterpret_cast<uint16_t*>(ws + L.gth);
  uint16_t* Gtl = reinterpret_cast<uint16_t*>(ws + L.gtl);
  float* tx = reinterpret_cast<float*>(ws + L.tx);
  float* tw = reinterpret_cast<float*>(ws + L.tw);
  unsigned int* mw = reinterpret_cast<unsigned int*>(ws + L.mw);
  const int fin_blocks = (static_cast<int>(a.K) + kFinishThreads - 1) / kFinishThreads;
  double* fin_partial = reinterpret_cast<double*>(ws + L.fin);
  unsigned int* fin_counter = reinterpret_cast<unsigned int*>(ws + L.fin + static_cast<size_t>(fin_blocks) * 8);
  const int M = static_cast<int>(a.M), N = static_cast<int>(a.N), K = static_cast<int>(a.K);
  const int Mp = static_cast<int>(L.Mp);

  // the codes transposed first: the first transpose also zeroes the sums that
  // the split of G (db) and the GEMMs (tx, tw, mw) accumulate into
  const SteZero zero{tx, tw, mw, K, a.db, N, fin_counter};
  const SteZero no_zero{nullptr, nullptr, nullptr, 0, nullptr, 0, nullptr};
  cudaError_t e = launch_pdl(transpose_codes_kernel, dim3((K + kTT - 1) / kTT, (N + kTT - 1) / kTT), dim3(kTThreads),
                             0, st, a.Wq, N, K, Wt, N, zero);
  if (e != cudaSuccess) return *why = "transpose of Wq", e;
  e = launch_pdl(transpose_codes_kernel, dim3((K + kTT - 1) / kTT, (M + kTT - 1) / kTT), dim3(kTThreads), 0, st, a.Xq,
                 M, K, Xt, Mp, no_zero);
  if (e != cudaSuccess) return *why = "transpose of Xq", e;
  e = launch_pdl(split_g_kernel, dim3((N + kTT - 1) / kTT, (M + kTT - 1) / kTT), dim3(kTThreads), 0, st, a.G, M, N,
                 a.w_scale, a.x_scale, Gh, Gl, Gth, Gtl, Mp, a.db);
  if (e != cudaSuccess) return *why = "split of G", e;

  SteGemmParams p{};
  p.s = a.s;
  p.src = a.X;
  p.q = a.Xq;
  p.qscale = a.x_scale;
  p.out = a.dX;
  p.tsum = tx;
  p.mwbits = nullptr;
  // dXs^T[k][m] = sum_n Wt[k][n] (Gh + Gl)[m][n]
  e = run_ste_gemm<kEpiDX>(Wt, Gh, Gl, a.K, a.M, a.N, a.N, p, st, dev, why);
  if (e != cudaSuccess) return e;
  p.src = a.W;
  p.q = a.Wq;
  p.qscale = a.w_scale;
  p.out = a.dW;
  p.tsum = tw;
  p.mwbits = mw;
  // dWs^T[k][n] = sum_m Xt[k][m] (Gth + Gtl)[n][m]
  e = run_ste_gemm<kEpiDW>(Xt, Gth, Gtl, a.K, a.N, a.M, L.Mp, p, st, dev, why);
  if (e != cudaSuccess) return e;
  e = launch_pdl(ste_finish_kernel, dim3(fin_blocks), dim3(kFinishThreads), 0, st, static_cast<const float*>(tx),
                 static_cast<const float*>(tw), static_cast<const unsigned int*>(mw), a.mx, a.s, a.alpha, K, a.ds,
                 fin_partial, fin_counter, a.d_eta);
  if (e != cudaSuccess) return *why = "finish launch", e;
  return cudaSuccess;
}

}  // namespace sq
