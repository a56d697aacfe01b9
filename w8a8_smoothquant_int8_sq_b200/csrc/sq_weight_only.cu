// sq_weight_only.cu -- the int8 weight-only linear, the decode comparison
// point beside the W8A8 path.
//
// Page: torchao, Int8WeightOnlyQuantizedLinearWeight._quantized_op: the
// activations stay in floating point and
//     y[m][n] = (sum_k x[m][k] * Wq[n][k]) * w_scale[n] + bias[n].
// There is no int8 x bf16 tensor-core product, so the multiply-adds run on the
// CUDA cores in fp32 (packed f32x2 FMAs), reading Wq from HBM once.
//
// Grid: (K splits) x (128-row blocks of Wq) x (groups of 8 tokens); the K
// splits of a row block form one thread-block cluster.
//   * The CTA's slice of X (8 tokens x its K range) is converted once to fp32
//     in shared memory, laid out per column as four (token 2p, token 2p+1)
//     pairs, so one 16-byte broadcast load gives two pairs to every lane.
//   * Wq streams through a ring of shared-memory stages, each a TMA box of 128
//     rows x 128 bytes of K (128-byte swizzle); one thread issues the boxes,
//     completion is counted on mbarriers (bounded waits), and the block
//     synchronises once per stage before its buffer is refilled.
//   * Lane l of every warp owns rows l, l+32, l+64, l+96 of the block; warp w
//     takes columns 16w..16w+15 of every stage.  Per stage a lane reads the 16
//     codes of each of its rows (conflict-free thanks to the swizzle), turns
//     them into fp32 four at a time (byte permute into the mantissa of
//     2^23 + 128 + q, then one packed subtract), and accumulates 4 rows x 8
//     tokens with packed FMAs: acc(t, t+1) += (x_t, x_t+1) * (w, w).
//   * The eight warps' sums are added in shared memory; the K splits push
//     theirs into rank 0's shared memory (distributed shared memory, 4 KB per
//     rank), and after one cluster barrier rank 0 adds them, applies
//     fma(sum, w_scale, bias) and stores bf16.
// Every mbarrier wait is bounded; a timeout latches bit 0 of the status word
// and the block stops loading (its output is then undefined).  Every thread
// reaches every __syncthreads and the cluster barrier.
#include <algorithm>
#include <cstdint>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {
namespace {

constexpr int kWoThreads = 256;                  // 8 warps
constexpr int kWoWarps = kWoThreads / 32;
constexpr int kWoTok = 8;                        // tokens per CTA
constexpr int kWoRowsPerLane = 4;
constexpr int kWoRows = 32 * kWoRowsPerLane;     // rows of Wq per CTA
constexpr int kWoStep = 16;                      // columns per step (one 16-byte vector of codes)
constexpr int kWoMaxCols = 4096;                 // columns of X per CTA (fp32 pairs: 32 B per column)
constexpr int kWoMaxSplit = 4;
constexpr int kWoXBytes = kWoMaxCols * 32;                      // 128 KB
constexpr int kWoRedBytes = kWoWarps * kWoTok * kWoRows * 4;    // 32 KB (reuses the X area)
constexpr int kWoStageCols = 128;                               // columns of Wq per stage (one TMA box)
constexpr int kWoStageBytes = kWoRows * kWoStageCols;           // 16 KB
#ifndef SQ_WO_STAGES
#define SQ_WO_STAGES 4
#endif
constexpr int kWoStages = SQ_WO_STAGES;
constexpr int kWoRingOffset = kWoXBytes;
constexpr int kWoRecvOffset = kWoRingOffset + kWoStages * kWoStageBytes;
constexpr int kWoMaxRecvSplit = 4;                              // K splits whose partials fit below
constexpr int kWoRecvBytes = kWoMaxRecvSplit * kWoTok * kWoRows * 4;  // 16 KB
constexpr int kWoBarOffset = kWoRecvOffset + kWoRecvBytes;
constexpr int kWoSmemBytes = kWoBarOffset + kWoStages * 8 + 16 + 1024;
static_assert(kWoStageCols == kWoWarps * kWoStep, "one 16-column step per warp per stage");
static_assert(kWoRedBytes <= kWoXBytes, "the warp sums reuse the X area");
static_assert(kWoMaxSplit <= kWoMaxRecvSplit, "every split's partial has a slot");
static_assert(kWoSmemBytes <= 232448, "shared memory per block");

struct WoParams {
  const uint16_t* X;  // [M][K] bf16
  const int8_t* Wq;   // [N][K]
  const float* w_scale;
  const uint16_t* bias;  // [N] or null
  uint16_t* Y;           // [M][N] bf16
  int M, N, K;
  int kc;  // columns per K split (a multiple of kWoStageCols)
  unsigned long long timeout_ns;  // limit of every mbarrier wait
  int skip_first_load;            // test hook: the first stage is never loaded
};

__device__ unsigned int g_sq_wo_status = 0u;

__device__ __forceinline__ void st_cluster_f4(uint32_t addr, float4 v) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w)
               : "memory");
}
__device__ __forceinline__ uint32_t wo_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t wo_map_rank(uint32_t smem_addr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(smem_addr), "r"(rank));
  return d;
}

// four signed int8 codes of w -> four floats, as two pairs (codes 0,1 and 2,3)
__device__ __forceinline__ void codes4_to_f2(uint32_t w, f2x& lo, f2x& hi) {
  const uint32_t u = w ^ 0x80808080u;  // q + 128 in [0, 255]
  const float b = 8388736.0f;          // 2^23 + 128
  // 0x4B0000bb: byte k of u as the low mantissa byte of 2^23 (selector
  // nibbles, low to high: byte k of u, two zero bytes and 0x4B of the constant)
  const uint32_t e0 = __byte_perm(u, 0x4B000000u, 0x7550);
  const uint32_t e1 = __byte_perm(u, 0x4B000000u, 0x7551);
  const uint32_t e2 = __byte_perm(u, 0x4B000000u, 0x7552);
  const uint32_t e3 = __byte_perm(u, 0x4B000000u, 0x7553);
  const f2x nb = f2_pack(-b, -b);
  lo = f2_add(f2_pack(__uint_as_float(e0), __uint_as_float(e1)), nb);
  hi = f2_add(f2_pack(__uint_as_float(e2), __uint_as_float(e3)), nb);
}

__global__ void __launch_bounds__(kWoThreads, 1) weight_only_kernel(const __grid_constant__ CUtensorMap tmW,
                                                                    const WoParams p) {
  extern __shared__ uint8_t wo_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(wo_smem_raw) + 1023) & ~uintptr_t(1023));
  float4* x2 = reinterpret_cast<float4*>(smem);  // [col][2]: (x0,x1,x2,x3), (x4,x5,x6,x7)
  const ulonglong2* xq = reinterpret_cast<const ulonglong2*>(smem);  // the same, as fp32 pairs (x0,x1), (x2,x3)...
  float* red = reinterpret_cast<float*>(smem);   // after the main loop: [warp][token][row]
  uint8_t* ring = smem + kWoRingOffset;          // [stage][128 rows][128 bytes], 128-byte swizzle
  float* recv = reinterpret_cast<float*>(smem + kWoRecvOffset);  // rank 0: [rank][token][row]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kWoBarOffset);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + kWoStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = wo_cluster_rank();
  const int nsplit = static_cast<int>(cluster_nctarank());
  const int row0 = blockIdx.y * kWoRows;
  const int tok0 = blockIdx.z * kWoTok;
  const int k_lo = static_cast<int>(rank) * p.kc;
  const int k_hi = min(p.K, k_lo + p.kc);
  const int ncols = max(0, k_hi - k_lo);

  const int nstages = (ncols + kWoStageCols - 1) / kWoStageCols;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kWoStages; ++i) mbar_init(&full[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
  }
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();
  int issued = 0;  // thread 0: stages issued so far (0 .. issued - 1)
  auto issue_stage = [&](int j) {  // thread 0 only
    if (!(p.skip_first_load && j == 0)) {  // test hook: the first stage never fills
      mbar_arrive_expect_tx(&full[j % kWoStages], kWoStageBytes);
      tma_load_2d(ring + (j % kWoStages) * kWoStageBytes, &tmW, k_lo + j * kWoStageCols, row0, &full[j % kWoStages]);
    }
    issued = j + 1;
  };
  if (threadIdx.x == 0)
    for (int j = 0; j < min(kWoStages, nstages); ++j) issue_stage(j);

  // ---- X slice -> fp32 pairs in shared memory (tokens past M are zeros).
  // Thread i takes token i % 8 of vector i / 8 (8 columns); a warp's lanes
  // cover 8 tokens x 4 vectors, and at step j lane (t, v) writes column
  // (j + v) % 8 of its vector, so the 32 stores of a step land in 32 banks.
  // The global loads are issued kWoXBatch at a time before any is used, so
  // their latencies overlap.
  {
    constexpr int kWoXBatch = 8;
    const int nvec = (ncols + 7) / 8;  // 16-byte vectors of bf16 per token row
    const int total = kWoTok * nvec;
    for (int base = threadIdx.x; base < total; base += kWoXBatch * kWoThreads) {
      uint4 wv[kWoXBatch];
#pragma unroll
      for (int u = 0; u < kWoXBatch; ++u) {
        const int i = base + u * kWoThreads;
        const int t = i % kWoTok, v = i / kWoTok;
        wv[u] = make_uint4(0u, 0u, 0u, 0u);
        if (i < total && tok0 + t < p.M)
          wv[u] = *reinterpret_cast<const uint4*>(p.X + static_cast<int64_t>(tok0 + t) * p.K + k_lo + v * 8);
      }
#pragma unroll
      for (int u = 0; u < kWoXBatch; ++u) {
        const int i = base + u * kWoThreads;
        if (i >= total) break;
        const int t = i % kWoTok, v = i / kWoTok;
        float* dst = reinterpret_cast<float*>(x2) + (v * 8) * 8 + t;  // column-major: [col][token]
        const uint32_t ws[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
        float f[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) f[2 * j] = bf16_lo(ws[j]), f[2 * j + 1] = bf16_hi(ws[j]);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int col = (j + v) & 7;
          float val = f[0];
#pragma unroll
          for (int q = 1; q < 8; ++q) val = col == q ? f[q] : val;
          dst[col * 8] = val;
        }
      }
    }
  }
  __syncthreads();

  // ---- main loop: stage j holds columns 128j..128j+127 of this split; warp w
  // takes the 16 columns 16w..16w+15 of every stage
  f2x acc[kWoRowsPerLane][kWoTok / 2];
#pragma unroll
  for (int r = 0; r < kWoRowsPerLane; ++r)
#pragma unroll
    for (int q = 0; q < kWoTok / 2; ++q) acc[r][q] = 0ull;
  for (int j = 0; j < nstages; ++j) {
    const int st = j % kWoStages;
    const bool ok = !*abort_flag && mbar_wait_bounded(&full[st], static_cast<uint32_t>((j / kWoStages) & 1), p.timeout_ns);
    if (!__all_sync(0xFFFFFFFFu, ok)) {
      if (lane == 0) {
        *abort_flag = 1;
        atomicOr(&g_sq_wo_status, 1u);
      }
    } else {
      const int c = j * kWoStageCols + warp * kWoStep;  // first column of this warp's step
      if (c < ncols) {
        const uint8_t* stage = ring + st * kWoStageBytes;
        uint4 w[kWoRowsPerLane];
#pragma unroll
        for (int r = 0; r < kWoRowsPerLane; ++r) {
          const int row = r * 32 + lane;  // row within the box; 16-byte unit `warp` of it, swizzled
          w[r] = *reinterpret_cast<const uint4*>(stage + row * 128 + ((warp ^ (row & 7)) << 4));
        }
        // X pairs of four columns at a time, the next four loaded while the
        // current four are used (two named buffers, no copies)
        f2x xA[4][4], xB[4][4];
        auto load_x = [&](int col0, f2x (&xs)[4][4]) {
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const ulonglong2 a = xq[(col0 + jj) * 2], b = xq[(col0 + jj) * 2 + 1];  // tokens (0,1)(2,3), (4,5)(6,7)
            xs[jj][0] = a.x, xs[jj][1] = a.y, xs[jj][2] = b.x, xs[jj][3] = b.y;
          }
        };
        auto compute4 = [&](int g, const f2x (&xs)[4][4]) {  // columns 4g..4g+3 of the step
          f2x wlo[kWoRowsPerLane], whi[kWoRowsPerLane];
#pragma unroll
          for (int r = 0; r < kWoRowsPerLane; ++r) {
            const uint32_t word = g == 0 ? w[r].x : g == 1 ? w[r].y : g == 2 ? w[r].z : w[r].w;
            codes4_to_f2(word, wlo[r], whi[r]);
          }
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
            for (int r = 0; r < kWoRowsPerLane; ++r) {
              const float wv = (jj & 1) ? f2_hi(jj < 2 ? wlo[r] : whi[r]) : f2_lo(jj < 2 ? wlo[r] : whi[r]);
              const f2x ww = f2_pack(wv, wv);
#pragma unroll
              for (int q = 0; q < kWoTok / 2; ++q) acc[r][q] = f2_fma(xs[jj][q], ww, acc[r][q]);
            }
          }
        };
        load_x(c, xA);
        load_x(c + 4, xB);
        compute4(0, xA);
        load_x(c + 8, xA);
        compute4(1, xB);
        load_x(c + 12, xB);
        compute4(2, xA);
        compute4(3, xB);
      }
    }
    __syncthreads();  // every warp is done with stage j: refill its buffer
    if (threadIdx.x == 0 && !*abort_flag && j + kWoStages < nstages) {
      fence_proxy_async_smem();
      issue_stage(j + kWoStages);
    }
  }
  if (*abort_flag && threadIdx.x == 0) {
    // let the copies issued and not yet consumed land before the block exits
    // (the last kWoStages issued; a skipped first stage never completes)
    for (int j = max(0, issued - kWoStages); j < issued; ++j)
      if (!(p.skip_first_load && j == 0))
        (void)mbar_wait_bounded(&full[j % kWoStages], static_cast<uint32_t>((j / kWoStages) & 1), p.timeout_ns);
  }

  // ---- the eight warps' sums -> one per (token, row)
  __syncthreads();  // every warp is done with the X area
#pragma unroll
  for (int r = 0; r < kWoRowsPerLane; ++r)
#pragma unroll
    for (int q = 0; q < kWoTok / 2; ++q) {
      red[(warp * kWoTok + 2 * q) * kWoRows + r * 32 + lane] = f2_lo(acc[r][q]);
      red[(warp * kWoTok + 2 * q + 1) * kWoRows + r * 32 + lane] = f2_hi(acc[r][q]);
    }
  __syncthreads();
  // thread i: token i / 32, rows 4 (i % 32) .. 4 (i % 32) + 3
  const int t = threadIdx.x / 32, rq = (threadIdx.x % 32) * 4;
  float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int w = 0; w < kWoWarps; ++w) {
    const float4 v = *reinterpret_cast<const float4*>(red + (w * kWoTok + t) * kWoRows + rq);
    sum.x += v.x, sum.y += v.y, sum.z += v.z, sum.w += v.w;
  }
  // ---- K splits: push to rank 0, one cluster barrier, rank 0 finishes
  if (nsplit > 1) {
    const uint32_t dst = wo_map_rank(smem_u32(recv + (static_cast<int>(rank) * kWoTok + t) * kWoRows + rq), 0u);
    st_cluster_f4(dst, sum);
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (rank != 0) return;
    sum = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < nsplit; ++q) {
      const float4 v = *reinterpret_cast<const float4*>(recv + (q * kWoTok + t) * kWoRows + rq);
      sum.x += v.x, sum.y += v.y, sum.z += v.z, sum.w += v.w;
    }
  }
  const int m = tok0 + t;
  if (m >= p.M) return;
  const float s4[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int n = row0 + rq + j;
    if (n < p.N) {
      const float b = p.bias != nullptr ? __uint_as_float(static_cast<uint32_t>(p.bias[n]) << 16) : 0.0f;
      p.Y[static_cast<int64_t>(m) * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmaf_rn(s4[j], p.w_scale[n], b)));
    }
  }
}

}  // namespace

cudaError_t read_weight_only_status(uint32_t* flags, bool clear) {
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_sq_wo_status, sizeof(v));
  if (e != cudaSuccess) return e;
  if (clear && v != 0u) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_sq_wo_status, &z, sizeof(z));
    if (e != cudaSuccess) return e;
  }
  *flags = v;
  return cudaSuccess;
}

cudaError_t launch_weight_only(const uint16_t* X, int64_t M, const int8_t* Wq, const float* w_scale,
                               const uint16_t* bias, int64_t N, int64_t K, uint16_t* Y, cudaStream_t st,
                               const DeviceInfo& dev) {
  const int rb = static_cast<int>((N + kWoRows - 1) / kWoRows);
  const int tg = static_cast<int>((M + kWoTok - 1) / kWoTok);
  // K splits (cluster size): enough CTAs to cover the SMs, and at most
  // kWoMaxCols columns of X per CTA
  int ks = 1;
  while (ks < kWoMaxSplit && static_cast<int64_t>(rb) * tg * ks * 2 <= dev.sm_count) ks *= 2;
  const int64_t unit = kWoStageCols;
  while (ks < kWoMaxSplit && (K + ks - 1) / ks > kWoMaxCols) ks *= 2;
  int64_t kc = ((K + ks - 1) / ks + unit - 1) / unit * unit;
  if (kc > kWoMaxCols) return cudaErrorNotSupported;  // K beyond kWoMaxSplit * kWoMaxCols
  WoParams p;
  p.X = X;
  p.Wq = Wq;
  p.w_scale = w_scale;
  p.bias = bias;
  p.Y = Y;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.kc = static_cast<int>(kc);
  p.skip_first_load = debug_stall_state(&p.timeout_ns) ? 1 : 0;
  CUtensorMap tmW;
  if (!make_tmap_2d(&tmW, Wq, N, K, 1, kWoStageCols, kWoRows, 128)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(weight_only_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kWoSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(weight_only_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, kCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  return launch_pdl_cluster(weight_only_kernel, dim3(static_cast<unsigned>(ks), static_cast<unsigned>(rb),
                                                     static_cast<unsigned>(tg)),
                            dim3(kWoThreads), static_cast<size_t>(kWoSmemBytes), st, static_cast<unsigned>(ks), tmW, p);
}

}  // namespace sq
