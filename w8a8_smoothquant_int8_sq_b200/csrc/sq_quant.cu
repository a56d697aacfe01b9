// sq_quant.cu -- the HBM-bound kernels of the SmoothQuant W8A8 path.
//
//   colmax_kernel        column max-abs of the calibration batch C[R][K] and of
//                        the weight W[N][K] (per input channel), then
//                        s_j = max(mx_j,1e-8)^a / max(mw_j,1e-8)^(1-a), >= 1e-8
//   row_quant_kernel     per-row symmetric int8 quantisation of W*s (weight
//                        prep, per output channel) or X/s (activations, per token)
//
// Page: "w8a8_smoothquant.py -- W8A8 com SmoothQuant e alpha APRENDIVEL (V5)",
// functions _per_channel_max_abs, calibrate_smoothquant,
// quantize_per_channel_symmetric, quantize_per_token_symmetric and the methods
// SmoothQuantW8A8.calibrate / freeze_quantization / forward.
#include <algorithm>
#include <cstdint>
#include <mutex>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {

// ====================================================== column max-abs (K1)
// Blocks are laid out as (256-column stripe) x (chunk of rows) x {C, W}; about
// two blocks per SM in total, each walking its chunk in batches of 8 rows per
// warp with the next batch's loads issued before the current one is reduced
// (16 loads of 16 bytes in flight per lane).  |x| is taken on the bf16 bit
// patterns with the sign bit cleared: for non-negative bf16 values the integer
// order of the patterns is the numeric order, so the max is exact and needs no
// conversion until the end.  Block results are merged with an unsigned
// atomicMax on the fp32 bit patterns (valid for values >= 0) into the
// workspace.  The last block of each stripe to finish (a per-stripe arrival
// counter) turns the stripe's maxima into s:
//     s_j = max( max(mx_j, 1e-8)^a / max(mw_j, 1e-8)^(1-a), 1e-8 )
// evaluated in double and rounded once to fp32 (calibrate_smoothquant), after
// merging the caller's running maximum (SmoothQuantW8A8.calibrate).
// Workspace layout (cleared by a memset before the launch): mx[K], mw[K]
// (fp32 bit patterns), count[stripes].
constexpr int kColThreads = 256;
constexpr int kColStripe = 256;
constexpr int kColBatch = 8;                              // rows per warp per batch
constexpr int kColBatchRows = kColBatch * (kColThreads / 32);  // rows per block per batch

__device__ __forceinline__ float smoothing_factor(float mx, float mw, double alpha) {
  const double floor = static_cast<double>(kClampFloor);
  const double x = fmax(static_cast<double>(mx), floor);
  const double w = fmax(static_cast<double>(mw), floor);
  const double v = fmax(pow(x, alpha) / pow(w, 1.0 - alpha), floor);
  return __double2float_rn(v);
}

__device__ __forceinline__ void colmax_load_batch(uint4 (&v)[kColBatch], const uint16_t* base, int64_t r, int64_t r1,
                                                  int K) {
#pragma unroll
  for (int i = 0; i < kColBatch; ++i)
    v[i] = (r + i < r1) ? __ldcg(reinterpret_cast<const uint4*>(base + (r + i) * K)) : make_uint4(0u, 0u, 0u, 0u);
}

__global__ void __launch_bounds__(kColThreads) colmax_kernel(const uint16_t* __restrict__ C, int64_t R,
                                                             const uint16_t* __restrict__ W, int64_t N, int K,
                                                             uint32_t* ws, int chunks_c, int chunks_w,
                                                             int64_t rows_c, int64_t rows_w, double alpha,
                                                             float* __restrict__ mx_inout, float* __restrict__ s) {
  griddep_wait();
  griddep_launch_dependents();
  const bool is_w = blockIdx.z == 1;
  const int chunks = is_w ? chunks_w : chunks_c;
  if (static_cast<int>(blockIdx.y) >= chunks) return;  // not counted: only chunks_c + chunks_w blocks arrive
  const uint16_t* A = is_w ? W : C;
  const int64_t rows = is_w ? N : R;
  const int64_t chunk_rows = is_w ? rows_w : rows_c;
  uint32_t* ws_mx = ws;
  uint32_t* ws_mw = ws + K;
  unsigned int* count = reinterpret_cast<unsigned int*>(ws + 2 * K);
  uint32_t* out = is_w ? ws_mw : ws_mx;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col = blockIdx.x * kColStripe + lane * 8;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * chunk_rows;
  const int64_t r1 = min(rows, r0 + chunk_rows);

  uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;  // packed pairs of |bf16| patterns
  if (col < K) {
    const uint16_t* base = A + col;
    uint4 cur[kColBatch], nxt[kColBatch];
    int64_t r = r0 + warp * kColBatch;
    colmax_load_batch(cur, base, r, r1, K);
    for (int64_t b0 = r0; b0 < r1; b0 += kColBatchRows, r += kColBatchRows) {
      const bool more = b0 + kColBatchRows < r1;
      if (more) colmax_load_batch(nxt, base, r + kColBatchRows, r1, K);
#pragma unroll
      for (int i = 0; i < kColBatch; ++i) {
        m0 = __vmaxu2(m0, cur[i].x & 0x7FFF7FFFu);
        m1 = __vmaxu2(m1, cur[i].y & 0x7FFF7FFFu);
        m2 = __vmaxu2(m2, cur[i].z & 0x7FFF7FFFu);
        m3 = __vmaxu2(m3, cur[i].w & 0x7FFF7FFFu);
      }
      if (!more) break;
#pragma unroll
      for (int i = 0; i < kColBatch; ++i) cur[i] = nxt[i];
    }
  }
  __shared__ uint32_t red[kColThreads / 32][kColStripe];
  __shared__ bool last;
  const uint32_t m[4] = {m0, m1, m2, m3};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    red[warp][lane * 8 + 2 * i] = (m[i] & 0xFFFFu) << 16;  // fp32 pattern of the bf16 value
    red[warp][lane * 8 + 2 * i + 1] = m[i] & 0xFFFF0000u;
  }
  __syncthreads();
  uint32_t vmax = 0;
#pragma unroll
  for (int w = 0; w < kColThreads / 32; ++w) vmax = max(vmax, red[w][threadIdx.x]);
  const int c = blockIdx.x * kColStripe + threadIdx.x;
  if (c < K && vmax != 0u) atomicMax(out + c, vmax);

  // arrival: the last block of this stripe computes s for the stripe
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned int total = static_cast<unsigned int>(chunks_c + chunks_w);
    last = (atomicAdd(count + blockIdx.x, 1u) == total - 1u);
  }
  __syncthreads();
  if (!last || c >= K) return;
  __threadfence();
  float mx = __uint_as_float(__ldcg(ws_mx + c));
  if (mx_inout != nullptr) {  // running max over calibration batches
    mx = fmaxf(mx, mx_inout[c]);
    mx_inout[c] = mx;
  }
  s[c] = smoothing_factor(mx, __uint_as_float(__ldcg(ws_mw + c)), alpha);
}

static int col_stripes(int64_t K) { return static_cast<int>((K + kColStripe - 1) / kColStripe); }

size_t calibrate_workspace_words(int64_t K) { return static_cast<size_t>(2 * K + col_stripes(K)); }

// rows per block for `rows` rows split into about `g` chunks (multiple of a batch)
static int64_t chunk_rows_for(int64_t rows, int64_t g) {
  const int64_t per = (rows + g - 1) / g;
  return std::max<int64_t>(kColBatchRows, (per + kColBatchRows - 1) / kColBatchRows * kColBatchRows);
}

cudaError_t launch_calibrate(const uint16_t* C, int64_t R, int64_t K, const uint16_t* W, int64_t N, float alpha,
                             float* s, float* mx_inout, void* ws, cudaStream_t st, const DeviceInfo& dev) {
  cudaError_t e = cudaMemsetAsync(ws, 0, calibrate_workspace_words(K) * sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  static bool attr_set = false;  // idempotent attribute; a race only repeats the call
  if (!attr_set) {
    e = cudaFuncSetAttribute(colmax_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, kCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  // about two blocks per SM over all stripes, split between C and W by rows
  const int stripes = col_stripes(K);
  const int64_t g_total = std::max<int64_t>(1, (2 * static_cast<int64_t>(dev.sm_count) + stripes - 1) / stripes);
  int64_t g_w = std::max<int64_t>(1, (g_total * N + (N + R) - 1) / (N + R));
  int64_t g_c = R > 0 ? std::max<int64_t>(1, g_total - g_w) : 0;
  const int64_t rows_w = chunk_rows_for(N, g_w);
  const int64_t rows_c = R > 0 ? chunk_rows_for(R, g_c) : kColBatchRows;
  const int chunks_w = static_cast<int>((N + rows_w - 1) / rows_w);
  const int chunks_c = R > 0 ? static_cast<int>((R + rows_c - 1) / rows_c) : 0;
  dim3 grid(static_cast<unsigned>(stripes), static_cast<unsigned>(std::max(chunks_c, chunks_w)), 2);
  return launch_pdl(colmax_kernel, grid, dim3(kColThreads), 0, st, C, R, W, N, static_cast<int>(K),
                    static_cast<uint32_t*>(ws), chunks_c, chunks_w, rows_c, rows_w, static_cast<double>(alpha),
                    mx_inout, s);
}

// ============================================ calibration without allocation
// Scratch for sq_calibrate_noalloc: the same words (2*K column maxima and a
// per-stripe counter) that
// sq_calibrate keeps in the caller's workspace, here in a fixed array that
// every device loading the library holds until the process exits (about
// 128 KiB).
// Host code must not pass the symbol itself to a kernel (on the host it only
// names a stand-in object); the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint32_t g_calib_noalloc_scratch[2 * kNoAllocMaxK + kNoAllocMaxK / 256];

cudaError_t launch_calibrate_noalloc(const uint16_t* C, int64_t R, int64_t K, const uint16_t* W, int64_t N,
                                     float alpha, float* s, float* mx_inout, cudaStream_t st, const DeviceInfo& dev) {
  // One-time set-up per device, done on that device's first call: look up the
  // device address of the scratch array while the device is current.
  static std::mutex mu;
  static void* addr[64] = {};
  void* ws = nullptr;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (dev.device < 0 || dev.device >= 64) return cudaErrorInvalidDevice;
    if (addr[dev.device] == nullptr) {
      void* p = nullptr;
      cudaError_t e = cudaGetSymbolAddress(&p, g_calib_noalloc_scratch);
      if (e != cudaSuccess) return e;
      addr[dev.device] = p;
    }
    ws = addr[dev.device];
  }
  // launch_calibrate clears the words it uses before the reduction, so the
  // previous call's contents never leak into this one.
  return launch_calibrate(C, R, K, W, N, alpha, s, mx_inout, ws, st, dev);
}

// ===================================================== row quantisers (K2/K3)
// A row is owned by a group of WPR warps; a 256-thread block holds 8/WPR rows
// at a time and walks the rows persistently.  Lane l of warp w (w-th of its
// group) owns the 16-byte vectors i*(32*WPR) + 32*w + l, i < VPL, so every warp
// load or store instruction touches one contiguous run of memory.  The next
// row's vectors are loaded into registers before the current row is reduced,
// so loads stay in flight while the block computes.  The smoothed values stay
// in registers between the row max and the codes: each element is read from
// HBM once and written once.
//   kMul == true  (weights):     t = fl(w * s_j)
//   kMul == false (activations): t = fl(x / s_j) = div_rn(x, s_j, RN(1/s_j))
// then scale = fl(max(max|t|, 1e-8) / 127) and q = rne(fl(t / scale)).  For
// finite inputs |t / scale| <= 127 * (1 + 2^-23) < 127.5, so the rounded code
// is already within +-127 and the clamp of the page is implied.
// s (and 1/s) sit in shared memory as four float4 arrays indexed by vector, so
// the table reads of a warp are contiguous and free of bank conflicts.
constexpr int kRowThreads = 256;

template <int VPL, int WPR>
__device__ __forceinline__ void load_row_vectors(uint4 (&xv)[VPL], const uint16_t* __restrict__ src, int64_t row,
                                                 int64_t rows, int K, int nvec, int wsub, int lane) {
  if (row < rows) {
    const uint4* xr = reinterpret_cast<const uint4*>(src + row * static_cast<int64_t>(K));
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int v = i * (32 * WPR) + wsub * 32 + lane;
      xv[i] = (v < nvec) ? __ldcs(xr + v) : make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

template <bool kMul, int WPR, int VPL>
__global__ void __launch_bounds__(kRowThreads) row_quant_kernel(const uint16_t* __restrict__ src, int64_t rows, int K,
                                                                const float* __restrict__ s, int8_t* __restrict__ q,
                                                                float* __restrict__ scale) {
  constexpr int RPC = 8 / WPR;  // rows per block in flight
  // Table, one float4 pair per 16-byte vector of 8 columns:
  //   weights:     sA = s[8v..8v+3], sB = s[8v+4..8v+7]
  //   activations: the same slots hold -s, and rA/rB hold RN(1/s)
  extern __shared__ float4 tab[];
  __shared__ float red[2][8];
  const int nvec = K >> 3;
  float4* sA = tab;
  float4* sB = tab + nvec;
  float4* rA = tab + 2 * nvec;
  float4* rB = tab + 3 * nvec;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slot = warp / WPR, wsub = warp % WPR;
  int64_t row = static_cast<int64_t>(blockIdx.x) * RPC + slot;
  const int64_t row_step = static_cast<int64_t>(gridDim.x) * RPC;

  griddep_wait();
  griddep_launch_dependents();
  uint4 xv[VPL];
  load_row_vectors<VPL, WPR>(xv, src, row, rows, K, nvec, wsub, lane);  // in flight during the table build

  const float4* s4 = reinterpret_cast<const float4*>(s);
  for (int v = tid; v < nvec; v += kRowThreads) {
    const float4 a = __ldg(s4 + 2 * v), b = __ldg(s4 + 2 * v + 1);
    if (kMul) {
      sA[v] = a;
      sB[v] = b;
    } else {
      sA[v] = make_float4(-a.x, -a.y, -a.z, -a.w);
      sB[v] = make_float4(-b.x, -b.y, -b.z, -b.w);
      rA[v] = make_float4(__frcp_rn(a.x), __frcp_rn(a.y), __frcp_rn(a.z), __frcp_rn(a.w));
      rB[v] = make_float4(__frcp_rn(b.x), __frcp_rn(b.y), __frcp_rn(b.z), __frcp_rn(b.w));
    }
  }
  __syncthreads();
  const f2x* sA2 = reinterpret_cast<const f2x*>(sA);
  const f2x* sB2 = reinterpret_cast<const f2x*>(sB);
  const f2x* rA2 = reinterpret_cast<const f2x*>(rA);
  const f2x* rB2 = reinterpret_cast<const f2x*>(rB);

  for (int it = 0; row < rows; ++it) {
    f2x t[VPL][4];  // smoothed values, pairs of columns
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int v = i * (32 * WPR) + wsub * 32 + lane;
      if (v < nvec) {
        const uint4 w = xv[i];
        const f2x x[4] = {f2_from_bf16x2(w.x), f2_from_bf16x2(w.y), f2_from_bf16x2(w.z), f2_from_bf16x2(w.w)};
        const f2x sv[4] = {sA2[2 * v], sA2[2 * v + 1], sB2[2 * v], sB2[2 * v + 1]};
        if (kMul) {
#pragma unroll
          for (int e = 0; e < 4; ++e) t[i][e] = f2_mul(x[e], sv[e]);
        } else {
          const f2x rv[4] = {rA2[2 * v], rA2[2 * v + 1], rB2[2 * v], rB2[2 * v + 1]};
#pragma unroll
          for (int e = 0; e < 4; ++e) t[i][e] = f2_div_rn(x[e], sv[e], rv[e]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) m = f2_absmax(m, t[i][e]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) t[i][e] = 0ull;
      }
    }
    const int64_t next = row + row_step;
    load_row_vectors<VPL, WPR>(xv, src, next, rows, K, nvec, wsub, lane);  // prefetch
    m = warp_max(m);
    if (WPR > 1) {
      if (lane == 0) red[it & 1][warp] = m;
      named_bar_sync(1 + slot, 32 * WPR);
#pragma unroll
      for (int w = 0; w < WPR; ++w) m = fmaxf(m, red[it & 1][slot * WPR + w]);
    }
    const float sc = __fdiv_rn(fmaxf(m, kClampFloor), kQmax);
    const float rsc = __frcp_rn(sc);
    const f2x nsc2 = f2_pack(-sc, -sc), rsc2 = f2_pack(rsc, rsc);
    int8_t* qr = q + row * static_cast<int64_t>(K);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int v = i * (32 * WPR) + wsub * 32 + lane;
      if (v < nvec) {
        f2x c[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) c[e] = f2_round_codes(f2_div_rn(t[i][e], nsc2, rsc2));
        *reinterpret_cast<uint2*>(qr + static_cast<int64_t>(v) * 8) = pack8_codes(c[0], c[1], c[2], c[3]);
      }
    }
    if (wsub == 0 && lane == 0) scale[row] = sc;
    row = next;
  }
}

template <bool kMul, int WPR, int VPL>
static cudaError_t launch_rq(const uint16_t* src, int64_t rows, int K, const float* s, int8_t* q, float* scale,
                             cudaStream_t st, const DeviceInfo& dev) {
  const size_t smem = static_cast<size_t>(K / 8) * sizeof(float4) * (kMul ? 2 : 4);
  auto kern = row_quant_kernel<kMul, WPR, VPL>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  cudaError_t ec = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, kCarveoutMaxShared);
  if (ec != cudaSuccess) return ec;
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kRowThreads, smem);
  if (e != cudaSuccess) return e;
  per_sm = std::max(per_sm, 1);
  constexpr int RPC = 8 / WPR;
  const int64_t groups = (rows + RPC - 1) / RPC;
  const int64_t grid = std::min<int64_t>(groups, static_cast<int64_t>(dev.sm_count) * per_sm);
  return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(kRowThreads), smem, st, src, rows, K, s, q, scale);
}

template <bool kMul>
static cudaError_t dispatch_rq(const uint16_t* src, int64_t rows, int K, const float* s, int8_t* q, float* scale,
                               cudaStream_t st, const DeviceInfo& dev) {
  // vectors per lane (up to 8), then warps per row (up to 8) to cover K
  const int nvec = K / 8;
  if (nvec <= 32) return launch_rq<kMul, 1, 1>(src, rows, K, s, q, scale, st, dev);
  if (nvec <= 64) return launch_rq<kMul, 1, 2>(src, rows, K, s, q, scale, st, dev);
  if (nvec <= 128) return launch_rq<kMul, 1, 4>(src, rows, K, s, q, scale, st, dev);
  if (nvec <= 256) return launch_rq<kMul, 1, 8>(src, rows, K, s, q, scale, st, dev);
  if (nvec <= 512) return launch_rq<kMul, 2, 8>(src, rows, K, s, q, scale, st, dev);
  if (nvec <= 1024) return launch_rq<kMul, 4, 8>(src, rows, K, s, q, scale, st, dev);
  return launch_rq<kMul, 8, 8>(src, rows, K, s, q, scale, st, dev);
}

cudaError_t launch_row_quant(bool multiply, const uint16_t* src, int64_t rows, int64_t K, const float* s, int8_t* q,
                             float* scale, cudaStream_t st, const DeviceInfo& dev) {
  const int Ki = static_cast<int>(K);
  return multiply ? dispatch_rq<true>(src, rows, Ki, s, q, scale, st, dev)
                  : dispatch_rq<false>(src, rows, Ki, s, q, scale, st, dev);
}

}  // namespace sq
