// sq_quant.cu -- the HBM-bound kernels of the SmoothQuant W8A8 path.
//
//   colmax_kernel        column max-abs of the calibration batch C[R][K] and of
//                        the weight W[N][K] (per input channel), then
//                        s_j = max(mx_j,1e-8)^a / max(mw_j,1e-8)^(1-a), >= 1e-8
//   row_quant_kernel     per-row symmetric int8 quantisation of W*s (weight
//                        prep, per output channel) or X/s (activations, per token)
//   pt_absmax_kernel,    one scale for a whole tensor (the per-tensor W8A8
//   pt_quant_kernel      baseline: page "quantized_linear.py -- QuantizedLinear
//                        + apply_w8a8", quantize_tensor)
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

// Latched by a wait in these kernels that ran out of time (bit 0), like the
// GEMM's status word; read and cleared through read_device_status.
__device__ unsigned int g_sq_quant_status = 0u;



#ifdef SQ_TRACE
// Optional block timestamps (build with -DSQ_TRACE): per kernel kind (0 colmax,
// 1 row quant of weights, 2 row quant of activations) and block, globaltimer at
// 0 block start, 1 past the wait for the previous kernel, 2 block end, 3 a
// kernel-specific point (colmax: the block's maxima merged, before arrival).
__device__ unsigned long long g_blk_trace[3][2048][4];
struct BlockTrace {
  int kind, id;
  __device__ BlockTrace(int k) : kind(k), id(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z)) {
    mark(0);
  }
  __device__ void mark(int i) const {
    if (threadIdx.x == 0 && id < 2048) g_blk_trace[kind][id][i] = globaltimer_ns();
  }
  __device__ ~BlockTrace() { mark(2); }
};
#define SQ_BLOCK_TRACE(kind) BlockTrace blk_trace_(kind)
#define SQ_BLOCK_MARK(i) blk_trace_.mark(i)
extern "C" __attribute__((visibility("default"))) int sq_trace_read_blocks(unsigned long long* host) {
  return cudaMemcpyFromSymbol(host, g_blk_trace, sizeof(g_blk_trace)) == cudaSuccess ? 0 : 1;
}
extern "C" __attribute__((visibility("default"))) int sq_trace_clear_blocks() {
  static unsigned long long zero[3][2048][4];
  return cudaMemcpyToSymbol(g_blk_trace, zero, sizeof(zero)) == cudaSuccess ? 0 : 1;
}
#else
#define SQ_BLOCK_TRACE(kind) \
  do {                       \
  } while (0)
#define SQ_BLOCK_MARK(i) \
  do {                   \
  } while (0)
#endif

// ====================================================== column max-abs (K1)
// Work unit: one 256-column stripe of a contiguous range of rows of C or of W;
// one thread block per unit.  A producer warp streams the unit as 32-row x
// 256-column boxes (16 KB of bf16) by TMA into a ring of shared-memory stages;
// eight consumer warps take four rows of every box each, lane l reading the
// 16 bytes of columns 8l..8l+7 of a row (one contiguous 512-byte row per warp
// instruction, free of bank conflicts).  Bytes in flight are set by the ring
// (six stages per block, two blocks per SM), not by registers.
// |x| is taken on the bf16 bit patterns with the sign bit cleared: for
// non-negative bf16 values the integer order of the patterns is the numeric
// order, so the max is exact and needs no conversion until the end.  Rows past
// the matrix end are zero-filled by TMA and rows past the unit's end belong to
// the same matrix, so neither changes a max.  Block results are merged with an
// unsigned atomicMax on the fp32 bit patterns (valid for values >= 0) into the
// workspace.  The last block of each stripe to finish (a per-stripe arrival
// counter) turns the stripe's maxima into s:
//     s_j = max( max(mx_j, 1e-8)^a / max(mw_j, 1e-8)^(1-a), 1e-8 )
// evaluated in double and rounded once to fp32 (calibrate_smoothquant), after
// merging the caller's running maximum (SmoothQuantW8A8.calibrate).
// Workspace layout: mx[K], mw[K] (fp32 bit patterns), count[stripes].  It must
// be zero when the kernel starts, and the last block of each stripe zeroes the
// stripe's words again once it has read them, so a call leaves the workspace
// zero (a caller workspace is cleared by a small kernel first, the library's own
// scratch is not).
constexpr int kColConsumers = 8;                                 // consumer warps
constexpr int kColThreads = 32 * (kColConsumers + 1);            // + one producer warp
constexpr int kColStripe = 256;                                  // columns per box (TMA box limit)
constexpr int kColBoxRows = 4 * kColConsumers;                   // rows per box
constexpr int kColStageBytes = kColStripe * kColBoxRows * 2;     // 16 KB
#ifndef SQ_COLMAX_STAGES  // build-time tuning knob: ring depth per block
#define SQ_COLMAX_STAGES 6
#endif
constexpr int kColStages = SQ_COLMAX_STAGES;
constexpr int kColRedOffset = kColStages * kColStageBytes;       // [8][256] u32 block reduction
constexpr int kColBarOffset = kColRedOffset + kColConsumers * kColStripe * 4;
constexpr int kColFlagOffset = kColBarOffset + 2 * kColStages * 8;
constexpr int kColSmemBytes = kColFlagOffset + 16 + 1024;        // + alignment slack

struct ColmaxParams {
  int K, box_cols, stripes;
  int chunks_c, chunks_w;  // row ranges per stripe of C and of W
  int rows_c, rows_w;      // rows per range (multiples of kColBoxRows)
  int R, N;
  uint32_t* ws;
  double alpha;
  float* mx_inout;
  float* s;
  unsigned long long timeout_ns;
  int skip_first_load;  // test hook: the first box of every block is never loaded
};

__device__ __forceinline__ float smoothing_factor(float mx, float mw, double alpha) {
  const double floor = static_cast<double>(kClampFloor);
  const double x = fmax(static_cast<double>(mx), floor);
  const double w = fmax(static_cast<double>(mw), floor);
  const double v = fmax(pow(x, alpha) / pow(w, 1.0 - alpha), floor);
  return __double2float_rn(v);
}

__global__ void __launch_bounds__(kColThreads) colmax_kernel(const __grid_constant__ CUtensorMap tmC,
                                                             const __grid_constant__ CUtensorMap tmW,
                                                             const ColmaxParams p) {
  SQ_BLOCK_TRACE(0);
  extern __shared__ uint8_t col_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(col_smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* red = reinterpret_cast<uint32_t*>(smem + kColRedOffset);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kColBarOffset);
  uint64_t* empty = full + kColStages;
  volatile int* flags = reinterpret_cast<volatile int*>(smem + kColFlagOffset);  // [0] abort, [1] last block

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int b = static_cast<int>(blockIdx.x);
  const bool is_w = b >= p.stripes * p.chunks_c;
  if (is_w) b -= p.stripes * p.chunks_c;
  const int stripe = b % p.stripes, chunk = b / p.stripes;
  const int rows = is_w ? p.N : p.R;
  const int chunk_rows = is_w ? p.rows_w : p.rows_c;
  const int r0 = chunk * chunk_rows;
  const int r1 = min(rows, r0 + chunk_rows);
  const int nbox = (r1 - r0 + kColBoxRows - 1) / kColBoxRows;
  const CUtensorMap* map = is_w ? &tmW : &tmC;
  const int row_bytes = p.box_cols * 2;  // a box row in shared memory

  if (threadIdx.x == 0) {
    for (int i = 0; i < kColStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kColConsumers);
    }
    flags[0] = 0;
    fence_mbar_init();
  }
  if (warp == kColConsumers && lane == 0) tma_prefetch_desc(map);
  __syncthreads();
  griddep_wait();
  SQ_BLOCK_MARK(1);
  griddep_launch_dependents();

  uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;  // packed pairs of |bf16| patterns
  if (warp == kColConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint32_t box_bytes = static_cast<uint32_t>(row_bytes * kColBoxRows);
      int j = 0;
      for (; j < nbox; ++j) {
        const int st = j % kColStages;
        if (j >= kColStages &&
            (flags[0] || !mbar_wait_bounded(&empty[st], static_cast<uint32_t>((j / kColStages - 1) & 1), p.timeout_ns))) {
          flags[0] = 1;
          atomicOr(&g_sq_quant_status, 1u);
          break;
        }
        if (p.skip_first_load && j == 0) continue;  // test hook: this box never fills
        mbar_arrive_expect_tx(&full[st], box_bytes);
        tma_load_2d(smem + st * kColStageBytes, map, stripe * p.box_cols, r0 + j * kColBoxRows, &full[st]);
      }
      if (j < nbox) {
        // gave up: let the copies already issued land before the block exits
        // (a skipped box never completes)
        for (int q = max(0, j - kColStages); q < j; ++q)
          if (!(p.skip_first_load && q == 0))
            (void)mbar_wait_bounded(&full[q % kColStages], static_cast<uint32_t>((q / kColStages) & 1), p.timeout_ns);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const bool active = lane * 8 < p.box_cols;
    const uint8_t* my_rows = smem + warp * 4 * row_bytes + lane * 16;
    for (int j = 0; j < nbox; ++j) {
      const int st = j % kColStages;
      if (flags[0] || !mbar_wait_bounded(&full[st], static_cast<uint32_t>((j / kColStages) & 1), p.timeout_ns)) {
        flags[0] = 1;
        atomicOr(&g_sq_quant_status, 1u);
        break;
      }
      if (active) {
        const uint8_t* src = my_rows + st * kColStageBytes;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v = *reinterpret_cast<const uint4*>(src + i * row_bytes);
          m0 = __vmaxu2(m0, v.x & 0x7FFF7FFFu);
          m1 = __vmaxu2(m1, v.y & 0x7FFF7FFFu);
          m2 = __vmaxu2(m2, v.z & 0x7FFF7FFFu);
          m3 = __vmaxu2(m3, v.w & 0x7FFF7FFFu);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    const uint32_t m[4] = {m0, m1, m2, m3};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      red[warp * kColStripe + lane * 8 + 2 * i] = (m[i] & 0xFFFFu) << 16;  // fp32 pattern of the bf16 value
      red[warp * kColStripe + lane * 8 + 2 * i + 1] = m[i] & 0xFFFF0000u;
    }
  }
  __syncthreads();
  uint32_t* ws_mx = p.ws;
  uint32_t* ws_mw = p.ws + p.K;
  unsigned int* count = reinterpret_cast<unsigned int*>(p.ws + 2 * p.K);
  const int c = stripe * kColStripe + static_cast<int>(threadIdx.x);
  if (threadIdx.x < kColStripe) {
    uint32_t vmax = 0;
#pragma unroll
    for (int w = 0; w < kColConsumers; ++w) vmax = max(vmax, red[w * kColStripe + threadIdx.x]);
    if (c < p.K && vmax != 0u) atomicMax((is_w ? ws_mw : ws_mx) + c, vmax);
  }

  // arrival: the last block of this stripe computes s for the stripe
  SQ_BLOCK_MARK(3);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned int total = static_cast<unsigned int>(p.chunks_c + p.chunks_w);
    flags[1] = (atomicAdd(count + stripe, 1u) == total - 1u) ? 1 : 0;
  }
  __syncthreads();
  if (!flags[1] || threadIdx.x >= kColStripe) return;
  __threadfence();
  if (threadIdx.x == 0) count[stripe] = 0u;  // every block of the stripe has arrived
  if (c >= p.K) return;
  float mx = __uint_as_float(__ldcg(ws_mx + c));
  const float mw = __uint_as_float(__ldcg(ws_mw + c));
  ws_mx[c] = 0u;  // leave the workspace as it was found: zero
  ws_mw[c] = 0u;
  if (p.mx_inout != nullptr) {  // running max over calibration batches
    mx = fmaxf(mx, p.mx_inout[c]);
    p.mx_inout[c] = mx;
  }
  p.s[c] = smoothing_factor(mx, mw, p.alpha);
}

#ifndef SQ_CALIB_MEMSET  // build-time knob: 1 clears the workspace with cudaMemsetAsync
#define SQ_CALIB_MEMSET 0
#endif

// Clears n words.  Nothing the previous kernel in the stream writes is touched
// before its results are visible (griddepcontrol.wait first).
__global__ void __launch_bounds__(256) zero_words_kernel(uint32_t* __restrict__ w, size_t n) {
  griddep_wait();
  griddep_launch_dependents();
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    w[i] = 0u;
}

static int col_stripes(int64_t K) { return static_cast<int>((K + kColStripe - 1) / kColStripe); }

size_t calibrate_workspace_words(int64_t K) { return static_cast<size_t>(2 * K + col_stripes(K)); }

// rows per range for `rows` rows split into about `g` ranges (multiple of a box)
static int64_t chunk_rows_for(int64_t rows, int64_t g) {
  const int64_t per = (rows + g - 1) / g;
  return std::max<int64_t>(kColBoxRows, (per + kColBoxRows - 1) / kColBoxRows * kColBoxRows);
}

cudaError_t launch_calibrate(const uint16_t* C, int64_t R, int64_t K, const uint16_t* W, int64_t N, float alpha,
                             float* s, float* mx_inout, void* ws, bool ws_is_zero, cudaStream_t st,
                             const DeviceInfo& dev) {
  cudaError_t e = cudaSuccess;
  if (!ws_is_zero) {
#if SQ_CALIB_MEMSET
    e = cudaMemsetAsync(ws, 0, calibrate_workspace_words(K) * sizeof(uint32_t), st);
#else
    // a small kernel rather than a memset node, so that it chains with its
    // neighbours through programmatic dependent launch
    const size_t words = calibrate_workspace_words(K);
    const unsigned blocks = static_cast<unsigned>(std::min<size_t>((words + 1023) / 1024, 4 * dev.sm_count));
    e = launch_pdl(zero_words_kernel, dim3(blocks), dim3(256), 0, st, static_cast<uint32_t*>(ws), words);
#endif
    if (e != cudaSuccess) return e;
  }
  static int per_sm = 0;  // idempotent set-up; a race only repeats it
  if (per_sm == 0) {
    e = cudaFuncSetAttribute(colmax_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kColSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(colmax_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, kCarveoutMaxShared);
    int n = 0;
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, colmax_kernel, kColThreads, kColSmemBytes);
    if (e != cudaSuccess) return e;
    per_sm = std::max(n, 1);
  }
  const int box_cols = static_cast<int>(std::min<int64_t>(K, kColStripe));
  CUtensorMap tmC, tmW;
  if (!make_tmap_2d(&tmW, W, N, K, 2, box_cols, kColBoxRows) ||
      !make_tmap_2d(&tmC, R > 0 ? C : W, R > 0 ? R : N, K, 2, box_cols, kColBoxRows))
    return cudaErrorInvalidValue;
  // about one wave of resident blocks over all stripes, split between C and W by rows
  const int stripes = col_stripes(K);
  const int64_t g_total = std::max<int64_t>(1, static_cast<int64_t>(per_sm) * dev.sm_count / stripes);
  const int64_t g_w = std::max<int64_t>(1, (g_total * N + (N + R) / 2) / (N + R));
  const int64_t g_c = R > 0 ? std::max<int64_t>(1, g_total - g_w) : 0;
  ColmaxParams p;
  p.K = static_cast<int>(K);
  p.box_cols = box_cols;
  p.stripes = stripes;
  p.rows_w = static_cast<int>(chunk_rows_for(N, g_w));
  p.rows_c = R > 0 ? static_cast<int>(chunk_rows_for(R, g_c)) : kColBoxRows;
  p.chunks_w = static_cast<int>((N + p.rows_w - 1) / p.rows_w);
  p.chunks_c = R > 0 ? static_cast<int>((R + p.rows_c - 1) / p.rows_c) : 0;
  p.R = static_cast<int>(R);
  p.N = static_cast<int>(N);
  p.ws = static_cast<uint32_t*>(ws);
  p.alpha = static_cast<double>(alpha);
  p.mx_inout = mx_inout;
  p.s = s;
  p.skip_first_load = debug_stall_state(&p.timeout_ns) ? 1 : 0;  // the normal limit: 2 s
  const int64_t grid = static_cast<int64_t>(stripes) * (p.chunks_c + p.chunks_w);
  return launch_pdl(colmax_kernel, dim3(static_cast<unsigned>(grid)), dim3(kColThreads),
                    static_cast<size_t>(kColSmemBytes), st, tmC, tmW, p);
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

// Reads the status word; clearing it also re-zeroes the no-allocation scratch,
// which a timed-out calibration may have left dirty.
cudaError_t read_quant_status(uint32_t* flags, bool clear) {
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_sq_quant_status, sizeof(v));
  if (e != cudaSuccess) return e;
  if (clear) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_sq_quant_status, &z, sizeof(z));
    if (e != cudaSuccess) return e;
    if (v != 0u) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_calib_noalloc_scratch);
      if (e == cudaSuccess) e = cudaMemset(p, 0, sizeof(g_calib_noalloc_scratch));
      if (e != cudaSuccess) return e;
    }
  }
  *flags = v;
  return cudaSuccess;
}

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
  // The array is zero at load time and every call leaves it zero, so no memset
  // is needed (read_quant_status(clear) re-zeroes it after a timed-out call).
  return launch_calibrate(C, R, K, W, N, alpha, s, mx_inout, ws, /*ws_is_zero=*/true, st, dev);
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
#ifndef SQ_RQ_L2_AHEAD  // build-time tuning knob: 1 prefetches the row after next into L2
#define SQ_RQ_L2_AHEAD 1
#endif
#ifndef SQ_RQ_EARLY_L2  // build-time tuning knob: rows per row group prefetched into L2 before the wait
#define SQ_RQ_EARLY_L2 2
#endif

// kExact: the row fills the WPR warps' VPL vectors exactly (K == 256 VPL WPR),
// so no vector index needs a bounds check.
template <int VPL, int WPR, bool kExact>
__device__ __forceinline__ void load_row_vectors(uint4 (&xv)[VPL], const uint16_t* __restrict__ src, int64_t row,
                                                 int64_t rows, int K, int nvec, int wsub, int lane) {
  if (row < rows) {
    const uint4* xr = reinterpret_cast<const uint4*>(src + row * static_cast<int64_t>(K));
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int v = i * (32 * WPR) + wsub * 32 + lane;
      xv[i] = (kExact || v < nvec) ? __ldcs(xr + v) : make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

// kExact: K == 256 * VPL * WPR (every vector index in range; no bounds checks).
// kCodes == false (activations only): the scales alone, no codes (q unused);
// block 0 also writes RN(1/s_j) to recip[K] when recip is not null.  This is
// the pre-pass of the GEMM that quantises its A operand itself.
template <bool kMul, int WPR, int VPL, bool kCodes, bool kExact>
__global__ void __launch_bounds__(kRowThreads) row_quant_kernel(const uint16_t* __restrict__ src, int64_t rows, int K,
                                                                const float* __restrict__ s, int8_t* __restrict__ q,
                                                                float* __restrict__ scale,
                                                                float* __restrict__ recip) {
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

  SQ_BLOCK_TRACE(kMul ? 1 : 2);
#if SQ_RQ_EARLY_L2
  // While the previous kernel is still running, pull this block's first rows
  // into L2.  A prefetch is only a hint and L2 is where every SM's writes
  // land, so even rows the previous kernel is still writing are read
  // correctly after the wait below.
  if (wsub == 0 && lane == 0) {
    for (int i = 0; i < SQ_RQ_EARLY_L2; ++i) {
      const int64_t r = row + i * row_step;
      if (r < rows) bulk_prefetch_l2(src + r * static_cast<int64_t>(K), static_cast<uint32_t>(K) * 2u);
    }
  }
#endif
  griddep_wait();
  SQ_BLOCK_MARK(1);
  griddep_launch_dependents();
  // The table, kTabChunk vectors per thread at a time: all of a chunk's loads
  // of s are issued before any of them is used (one memory round trip per
  // chunk instead of one per vector), and the first chunk's before the loads
  // of the first row, so that s does not queue behind a row per block (and
  // the rows prefetched above) in the memory system.
  uint4 xv[VPL];
  bool row_issued = false;
  const float4* s4 = reinterpret_cast<const float4*>(s);
  constexpr int kTabChunk = 4;
  for (int v0 = tid; v0 < nvec; v0 += kTabChunk * kRowThreads) {
    float4 a[kTabChunk], b[kTabChunk];
#pragma unroll
    for (int j = 0; j < kTabChunk; ++j) {
      const int v = v0 + j * kRowThreads;
      if (v < nvec) {
        a[j] = __ldg(s4 + 2 * v);
        b[j] = __ldg(s4 + 2 * v + 1);
      }
    }
    if (!row_issued) {  // the first row, in flight during the table build
      load_row_vectors<VPL, WPR, kExact>(xv, src, row, rows, K, nvec, wsub, lane);
      row_issued = true;
    }
#pragma unroll
    for (int j = 0; j < kTabChunk; ++j) {
      const int v = v0 + j * kRowThreads;
      if (v >= nvec) break;
      if (kMul) {
        sA[v] = a[j];
        sB[v] = b[j];
      } else {
        sA[v] = make_float4(-a[j].x, -a[j].y, -a[j].z, -a[j].w);
        sB[v] = make_float4(-b[j].x, -b[j].y, -b[j].z, -b[j].w);
        const float4 ra = make_float4(__frcp_rn(a[j].x), __frcp_rn(a[j].y), __frcp_rn(a[j].z), __frcp_rn(a[j].w));
        const float4 rb = make_float4(__frcp_rn(b[j].x), __frcp_rn(b[j].y), __frcp_rn(b[j].z), __frcp_rn(b[j].w));
        rA[v] = ra;
        rB[v] = rb;
        if (!kCodes && recip != nullptr && blockIdx.x == 0) {
          reinterpret_cast<float4*>(recip)[2 * v] = ra;
          reinterpret_cast<float4*>(recip)[2 * v + 1] = rb;
        }
      }
    }
  }
  if (!row_issued) load_row_vectors<VPL, WPR, kExact>(xv, src, row, rows, K, nvec, wsub, lane);
  __syncthreads();
  SQ_BLOCK_MARK(3);
  const float r127 = __frcp_rn(kQmax);  // RN(1/127), for the correctly rounded max / 127

  for (int it = 0; row < rows; ++it) {
    f2x t[VPL][4];  // smoothed values, pairs of columns
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int v = i * (32 * WPR) + wsub * 32 + lane;
      if (kExact || v < nvec) {
        const uint4 w = xv[i];
        const f2x x[4] = {f2_from_bf16x2(w.x), f2_from_bf16x2(w.y), f2_from_bf16x2(w.z), f2_from_bf16x2(w.w)};
        // one 16-byte table read per float4: consecutive lanes, consecutive
        // 16 bytes (no bank conflicts)
        const float4 sa = sA[v], sb = sB[v];
        const f2x sv[4] = {f2_pack(sa.x, sa.y), f2_pack(sa.z, sa.w), f2_pack(sb.x, sb.y), f2_pack(sb.z, sb.w)};
        if (kMul) {
#pragma unroll
          for (int e = 0; e < 4; ++e) t[i][e] = f2_mul(x[e], sv[e]);
        } else {
          const float4 ra = rA[v], rb = rB[v];
          const f2x rv[4] = {f2_pack(ra.x, ra.y), f2_pack(ra.z, ra.w), f2_pack(rb.x, rb.y), f2_pack(rb.z, rb.w)};
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
    load_row_vectors<VPL, WPR, kExact>(xv, src, next, rows, K, nvec, wsub, lane);  // prefetch
#if SQ_RQ_L2_AHEAD
    {
      // and the row after that into L2, so the register prefetch above finds
      // its row in L2 instead of paying a DRAM latency per row
      const int64_t ahead = next + row_step;
      if (wsub == 0 && lane == 0 && ahead < rows)
        bulk_prefetch_l2(src + ahead * static_cast<int64_t>(K), static_cast<uint32_t>(K) * 2u);
    }
#endif
    m = warp_max(m);
    if (WPR > 1) {
      if (lane == 0) red[it & 1][warp] = m;
      named_bar_sync(1 + slot, 32 * WPR);
#pragma unroll
      for (int w = 0; w < WPR; ++w) m = fmaxf(m, red[it & 1][slot * WPR + w]);
    }
    // fl(max / 127): Markstein's correction of the product with RN(1/127),
    // equal to the IEEE quotient for every fp32 from 1e-8 up (checked
    // exhaustively on the CPU)
    const float sc = div_rn(fmaxf(m, kClampFloor), kQmax, r127);
    if (kCodes) {
      const float rsc = __frcp_rn(sc);
      const f2x nsc2 = f2_pack(-sc, -sc), rsc2 = f2_pack(rsc, rsc);
      int8_t* qr = q + row * static_cast<int64_t>(K);
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int v = i * (32 * WPR) + wsub * 32 + lane;
        if (kExact || v < nvec) {
          f2x c[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) c[e] = f2_round_codes(f2_div_rn(t[i][e], nsc2, rsc2));
          *reinterpret_cast<uint2*>(qr + static_cast<int64_t>(v) * 8) = pack8_codes(c[0], c[1], c[2], c[3]);
        }
      }
    }
    if (wsub == 0 && lane == 0) scale[row] = sc;
    row = next;
  }
}

template <bool kMul, int WPR, int VPL, bool kCodes>
static cudaError_t launch_rq(const uint16_t* src, int64_t rows, int K, const float* s, int8_t* q, float* scale,
                             float* recip, cudaStream_t st, const DeviceInfo& dev) {
  const size_t smem = static_cast<size_t>(K / 8) * sizeof(float4) * (kMul ? 2 : 4);
  // rows that fill the warps' vectors exactly take the kernel without bounds checks
  auto kern = (K == 256 * VPL * WPR) ? row_quant_kernel<kMul, WPR, VPL, kCodes, true>
                                     : row_quant_kernel<kMul, WPR, VPL, kCodes, false>;
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
  return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(kRowThreads), smem, st, src, rows, K, s, q, scale,
                    recip);
}

#ifndef SQ_RQ_VPL  // build-time tuning knob: most 16-byte vectors a lane holds (4 or 8)
#define SQ_RQ_VPL 4
#endif

template <bool kMul, bool kCodes = true>
static cudaError_t dispatch_rq(const uint16_t* src, int64_t rows, int K, const float* s, int8_t* q, float* scale,
                               cudaStream_t st, const DeviceInfo& dev, float* recip = nullptr) {
  // vectors per lane (up to SQ_RQ_VPL), then warps per row (up to 8) to cover K
  constexpr int V = SQ_RQ_VPL;
  static_assert(V == 4 || V == 8, "SQ_RQ_VPL must be 4 or 8");
  const int nvec = K / 8;
  if (nvec <= 32) return launch_rq<kMul, 1, 1, kCodes>(src, rows, K, s, q, scale, recip, st, dev);
  if (nvec <= 64) return launch_rq<kMul, 1, 2, kCodes>(src, rows, K, s, q, scale, recip, st, dev);
  if (nvec <= 128) return launch_rq<kMul, 1, 4, kCodes>(src, rows, K, s, q, scale, recip, st, dev);
  if (nvec <= 32 * V) return launch_rq<kMul, 1, V, kCodes>(src, rows, K, s, q, scale, recip, st, dev);
  if (nvec <= 64 * V) return launch_rq<kMul, 2, V, kCodes>(src, rows, K, s, q, scale, recip, st, dev);
  if (nvec <= 128 * V) return launch_rq<kMul, 4, V, kCodes>(src, rows, K, s, q, scale, recip, st, dev);
  if (nvec <= 256 * V) return launch_rq<kMul, 8, V, kCodes>(src, rows, K, s, q, scale, recip, st, dev);
  return launch_rq<kMul, 8, 8, kCodes>(src, rows, K, s, q, scale, recip, st, dev);  // K up to 16384
}

// ============================================ per-tensor quantisation (baseline)
// quantize_tensor of the QuantizedLinear page: scale = max|x| / 127 in fp32
// (1.0 when below 1e-8), codes rne(fl(x / scale)) clamped to [-128, 127].
// Since scale = fl(max|x| / 127), |x / scale| exceeds 127 by at most one ulp
// and every code already lies in [-127, 127]: the clamp is implied.
// Pass 1 writes one partial maximum per block (plain stores, no atomics and so
// nothing to clear); pass 2 reduces them in every block and quantises.  The
// tensor is read as a flat array of 16-byte vectors (rows * K is a multiple
// of 8), four vectors in flight per thread.
constexpr int kPtThreads = 256;
constexpr int kPtVecs = 4;  // vectors per thread per iteration
constexpr int kPtMaxBlocks = 1024;

__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < static_cast<int>(blockDim.x >> 5) ? red[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  return red[0];
}

__global__ void __launch_bounds__(kPtThreads) pt_absmax_kernel(const uint4* __restrict__ x, int64_t nvec,
                                                               uint32_t* __restrict__ part) {
  __shared__ uint32_t red[kPtThreads / 32];
  griddep_wait();
  griddep_launch_dependents();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kPtThreads;
  uint32_t m = 0;  // packed pair of |bf16| patterns
  for (int64_t v0 = static_cast<int64_t>(blockIdx.x) * kPtThreads + threadIdx.x; v0 < nvec; v0 += kPtVecs * stride) {
    uint4 a[kPtVecs];
#pragma unroll
    for (int i = 0; i < kPtVecs; ++i) {
      const int64_t v = v0 + i * stride;
      a[i] = v < nvec ? __ldcs(x + v) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < kPtVecs; ++i) {
      m = __vmaxu2(m, a[i].x & 0x7FFF7FFFu);
      m = __vmaxu2(m, a[i].y & 0x7FFF7FFFu);
      m = __vmaxu2(m, a[i].z & 0x7FFF7FFFu);
      m = __vmaxu2(m, a[i].w & 0x7FFF7FFFu);
    }
  }
  const uint32_t h = block_max_u32(max(m & 0xFFFFu, m >> 16), red);
  if (threadIdx.x == 0) part[blockIdx.x] = h << 16;  // fp32 pattern of the bf16 maximum
}

__global__ void __launch_bounds__(kPtThreads) pt_quant_kernel(const uint4* __restrict__ x, int64_t nvec,
                                                              const uint32_t* __restrict__ part, int nparts,
                                                              int64_t rows, uint2* __restrict__ q,
                                                              float* __restrict__ scale_rows) {
  __shared__ uint32_t red[kPtThreads / 32];
  griddep_wait();
  griddep_launch_dependents();
  uint32_t m = 0;
  for (int i = threadIdx.x; i < nparts; i += kPtThreads) m = max(m, __ldcg(part + i));
  const float mx = __uint_as_float(block_max_u32(m, red));
  float sc = __fdiv_rn(mx, kQmax);
  if (sc < kClampFloor) sc = 1.0f;
  const float rsc = __frcp_rn(sc);
  const f2x nsc2 = f2_pack(-sc, -sc), rsc2 = f2_pack(rsc, rsc);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kPtThreads;
  for (int64_t v0 = static_cast<int64_t>(blockIdx.x) * kPtThreads + threadIdx.x; v0 < nvec; v0 += kPtVecs * stride) {
    uint4 a[kPtVecs];
#pragma unroll
    for (int i = 0; i < kPtVecs; ++i) {
      const int64_t v = v0 + i * stride;
      a[i] = v < nvec ? __ldcs(x + v) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < kPtVecs; ++i) {
      const int64_t v = v0 + i * stride;
      if (v < nvec) {
        f2x c[4];
        c[0] = f2_round_codes(f2_div_rn(f2_from_bf16x2(a[i].x), nsc2, rsc2));
        c[1] = f2_round_codes(f2_div_rn(f2_from_bf16x2(a[i].y), nsc2, rsc2));
        c[2] = f2_round_codes(f2_div_rn(f2_from_bf16x2(a[i].z), nsc2, rsc2));
        c[3] = f2_round_codes(f2_div_rn(f2_from_bf16x2(a[i].w), nsc2, rsc2));
        q[v] = pack8_codes(c[0], c[1], c[2], c[3]);
      }
    }
  }
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * kPtThreads + threadIdx.x; r < rows; r += stride)
    scale_rows[r] = sc;
}

size_t per_tensor_workspace_bytes() { return kPtMaxBlocks * sizeof(uint32_t); }

cudaError_t launch_quantize_per_tensor(const uint16_t* src, int64_t rows, int64_t K, int8_t* q, float* scale_rows,
                                       void* ws, cudaStream_t st, const DeviceInfo& dev) {
  const int64_t nvec = rows * K / 8;
  const int64_t want = (nvec + kPtVecs * kPtThreads - 1) / (kPtVecs * kPtThreads);
  const int blocks = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>({want, static_cast<int64_t>(4) * dev.sm_count, static_cast<int64_t>(kPtMaxBlocks)})));
  uint32_t* part = static_cast<uint32_t*>(ws);
  const uint4* x = reinterpret_cast<const uint4*>(src);
  cudaError_t e = launch_pdl(pt_absmax_kernel, dim3(blocks), dim3(kPtThreads), 0, st, x, nvec, part);
  if (e != cudaSuccess) return e;
  return launch_pdl(pt_quant_kernel, dim3(blocks), dim3(kPtThreads), 0, st, x, nvec,
                    static_cast<const uint32_t*>(part), blocks, rows, reinterpret_cast<uint2*>(q), scale_rows);
}

cudaError_t launch_row_quant(bool multiply, const uint16_t* src, int64_t rows, int64_t K, const float* s, int8_t* q,
                             float* scale, cudaStream_t st, const DeviceInfo& dev) {
  const int Ki = static_cast<int>(K);
  return multiply ? dispatch_rq<true>(src, rows, Ki, s, q, scale, st, dev)
                  : dispatch_rq<false>(src, rows, Ki, s, q, scale, st, dev);
}

cudaError_t launch_act_scales(const uint16_t* X, int64_t rows, int64_t K, const float* s, float* scale, float* recip,
                              cudaStream_t st, const DeviceInfo& dev) {
  return dispatch_rq<false, false>(X, rows, static_cast<int>(K), s, nullptr, scale, st, dev, recip);
}

}  // namespace sq
