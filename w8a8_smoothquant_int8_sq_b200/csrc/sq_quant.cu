// sq_quant.cu -- the HBM-bound kernels of the SmoothQuant W8A8 path.
//
//   colmax_kernel        column max-abs of the calibration batch C[R][K] and of
//                        the weight W[N][K] (per input channel)
//   calib_finalize_kernel s_j = max(mx_j,1e-8)^a / max(mw_j,1e-8)^(1-a), >= 1e-8
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
// A block covers a stripe of 256 columns (one 16-byte vector of 8 bf16 per
// lane) and a chunk of kColRows rows; its 8 warps walk the chunk's rows.  |x|
// is taken on the bf16 bit patterns (sign bit cleared): for non-negative bf16
// values the integer order of the patterns is the numeric order, so the max is
// exact and needs no conversion until the end.  Block results are merged with
// an unsigned atomicMax on the fp32 bit patterns (valid for values >= 0).
constexpr int kColThreads = 256;
constexpr int kColStripe = 256;
constexpr int kColRows = 128;

__global__ void __launch_bounds__(kColThreads) colmax_kernel(const uint16_t* __restrict__ C, int64_t R,
                                                             const uint16_t* __restrict__ W, int64_t N, int K,
                                                             uint32_t* __restrict__ ws_mx,
                                                             uint32_t* __restrict__ ws_mw, int chunks_c,
                                                             int chunks_w) {
  const bool is_w = blockIdx.z == 1;
  const int chunks = is_w ? chunks_w : chunks_c;
  if (static_cast<int>(blockIdx.y) >= chunks) return;
  const uint16_t* A = is_w ? W : C;
  const int64_t rows = is_w ? N : R;
  uint32_t* out = is_w ? ws_mw : ws_mx;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col = blockIdx.x * kColStripe + lane * 8;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kColRows;
  const int64_t r1 = min(rows, r0 + kColRows);

  uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;  // packed pairs of |bf16| patterns
  if (col < K) {
    const uint16_t* base = A + col;
    int64_t r = r0 + warp;
    for (; r + 24 < r1; r += 32) {  // four independent 16-byte loads in flight
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(base + r * K));
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(base + (r + 8) * K));
      const uint4 c = __ldg(reinterpret_cast<const uint4*>(base + (r + 16) * K));
      const uint4 d = __ldg(reinterpret_cast<const uint4*>(base + (r + 24) * K));
      m0 = __vmaxu2(__vmaxu2(m0, a.x & 0x7FFF7FFFu), __vmaxu2(b.x & 0x7FFF7FFFu, __vmaxu2(c.x & 0x7FFF7FFFu, d.x & 0x7FFF7FFFu)));
      m1 = __vmaxu2(__vmaxu2(m1, a.y & 0x7FFF7FFFu), __vmaxu2(b.y & 0x7FFF7FFFu, __vmaxu2(c.y & 0x7FFF7FFFu, d.y & 0x7FFF7FFFu)));
      m2 = __vmaxu2(__vmaxu2(m2, a.z & 0x7FFF7FFFu), __vmaxu2(b.z & 0x7FFF7FFFu, __vmaxu2(c.z & 0x7FFF7FFFu, d.z & 0x7FFF7FFFu)));
      m3 = __vmaxu2(__vmaxu2(m3, a.w & 0x7FFF7FFFu), __vmaxu2(b.w & 0x7FFF7FFFu, __vmaxu2(c.w & 0x7FFF7FFFu, d.w & 0x7FFF7FFFu)));
    }
    for (; r < r1; r += 8) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(base + r * K));
      m0 = __vmaxu2(m0, a.x & 0x7FFF7FFFu);
      m1 = __vmaxu2(m1, a.y & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, a.z & 0x7FFF7FFFu);
      m3 = __vmaxu2(m3, a.w & 0x7FFF7FFFu);
    }
  }
  __shared__ uint32_t red[kColThreads / 32][kColStripe];
  const uint32_t m[4] = {m0, m1, m2, m3};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    red[warp][lane * 8 + 2 * i] = (m[i] & 0xFFFFu) << 16;  // fp32 pattern of the bf16 value
    red[warp][lane * 8 + 2 * i + 1] = m[i] & 0xFFFF0000u;
  }
  __syncthreads();
  uint32_t v = 0;
#pragma unroll
  for (int w = 0; w < kColThreads / 32; ++w) v = max(v, red[w][threadIdx.x]);
  const int c = blockIdx.x * kColStripe + threadIdx.x;
  if (c < K && v != 0u) atomicMax(out + c, v);
}

// ============================================================ finalise s (K1)
__global__ void calib_finalize_kernel(const uint32_t* __restrict__ ws_mx, const uint32_t* __restrict__ ws_mw, int K,
                                      double alpha, float* __restrict__ mx_inout, float* __restrict__ s) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  float mx = __uint_as_float(ws_mx[j]);
  if (mx_inout != nullptr) {  // running max over calibration batches
    mx = fmaxf(mx, mx_inout[j]);
    mx_inout[j] = mx;
  }
  const float mw = __uint_as_float(ws_mw[j]);
  const double floor = static_cast<double>(kClampFloor);
  const double x = fmax(static_cast<double>(mx), floor);
  const double w = fmax(static_cast<double>(mw), floor);
  double v = pow(x, alpha) / pow(w, 1.0 - alpha);
  v = fmax(v, floor);
  s[j] = __double2float_rn(v);
}

cudaError_t launch_calibrate(const uint16_t* C, int64_t R, int64_t K, const uint16_t* W, int64_t N, float alpha,
                             float* s, float* mx_inout, void* ws, cudaStream_t st, const DeviceInfo& dev) {
  (void)dev;
  uint32_t* ws_mx = static_cast<uint32_t*>(ws);
  uint32_t* ws_mw = ws_mx + K;
  cudaError_t e = cudaMemsetAsync(ws, 0, static_cast<size_t>(2 * K) * sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  const int chunks_c = static_cast<int>((R + kColRows - 1) / kColRows);
  const int chunks_w = static_cast<int>((N + kColRows - 1) / kColRows);
  dim3 grid(static_cast<unsigned>((K + kColStripe - 1) / kColStripe), static_cast<unsigned>(std::max(chunks_c, chunks_w)),
            2);
  colmax_kernel<<<grid, kColThreads, 0, st>>>(C, R, W, N, static_cast<int>(K), ws_mx, ws_mw, chunks_c, chunks_w);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  calib_finalize_kernel<<<static_cast<unsigned>((K + 255) / 256), 256, 0, st>>>(ws_mx, ws_mw, static_cast<int>(K),
                                                                                static_cast<double>(alpha),
                                                                                mx_inout, s);
  return cudaGetLastError();
}

// ============================================ calibration without allocation
// Scratch for sq_calibrate_noalloc: the same 2*K words of column maxima that
// sq_calibrate keeps in the caller's workspace, here in a fixed array that
// every device loading the library holds until the process exits (128 KiB).
// Host code must not pass the symbol itself to a kernel (on the host it only
// names a stand-in object); the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint32_t g_calib_noalloc_scratch[2 * kNoAllocMaxK];

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
  // launch_calibrate clears the 2*K words it uses before the reduction, so the
  // previous call's contents never leak into this one.
  return launch_calibrate(C, R, K, W, N, alpha, s, mx_inout, ws, st, dev);
}

// ===================================================== row quantisers (K2/K3)
// One thread block quantises one row at a time (persistent over rows).  Each
// thread owns VPT 16-byte vectors (8 bf16 each) of the row, strided by the
// block size so that every load and store instruction of a warp is contiguous.
// The smoothed values stay in registers between the max-abs reduction and the
// code computation, so the row is read from HBM exactly once.
//   kMul == true  (weights):     t = fl(w * s_j)              s_j from shared memory
//   kMul == false (activations): t = fl(x / s_j) = div_rn(x, s_j, RN(1/s_j))
// then scale = fl(max(max|t|, 1e-8) / 127), q = clamp(rne(fl(t / scale))).
constexpr int kRowThreads = 256;

template <bool kMul, int VPT>
__global__ void __launch_bounds__(kRowThreads) row_quant_kernel(const uint16_t* __restrict__ src, int64_t rows, int K,
                                                                const float* __restrict__ s, int8_t* __restrict__ q,
                                                                float* __restrict__ scale) {
  extern __shared__ __align__(16) float smem_sr[];  // kMul: s[K]; else (s_j, 1/s_j) pairs [K]
  __shared__ float red[kRowThreads / 32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (kMul) {
    for (int j = tid; j < K; j += kRowThreads) smem_sr[j] = s[j];
  } else {
    for (int j = tid; j < K; j += kRowThreads) {
      const float sj = s[j];
      smem_sr[2 * j] = sj;
      smem_sr[2 * j + 1] = __frcp_rn(sj);
    }
  }
  __syncthreads();
  const int nvec = K >> 3;

  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const uint4* xr = reinterpret_cast<const uint4*>(src + row * static_cast<int64_t>(K));
    float t[VPT][8];
    float m = 0.0f;
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int idx = tid + v * kRowThreads;
      if (idx < nvec) {
        const uint4 w = __ldg(xr + idx);
        const float x[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                            bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
        const int c = idx * 8;
        if (kMul) {
          const float4 s0 = *reinterpret_cast<const float4*>(smem_sr + c);
          const float4 s1 = *reinterpret_cast<const float4*>(smem_sr + c + 4);
          const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) t[v][e] = __fmul_rn(x[e], sv[e]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const float4 p = *reinterpret_cast<const float4*>(smem_sr + 2 * (c + e));
            t[v][e] = div_rn(x[e], p.x, p.y);
            t[v][e + 1] = div_rn(x[e + 1], p.z, p.w);
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(t[v][e]));
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) t[v][e] = 0.0f;
      }
    }
    m = warp_max(m);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    float mm = red[0];
#pragma unroll
    for (int w = 1; w < kRowThreads / 32; ++w) mm = fmaxf(mm, red[w]);
    const float sc = __fdiv_rn(fmaxf(mm, kClampFloor), kQmax);
    const float rsc = __frcp_rn(sc);
    int8_t* qr = q + row * static_cast<int64_t>(K);
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int idx = tid + v * kRowThreads;
      if (idx < nvec) {
        int c[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) c[e] = rne_clamp_q(div_rn(t[v][e], sc, rsc));
        uint2 packed;
        packed.x = pack4_i8(c[0], c[1], c[2], c[3]);
        packed.y = pack4_i8(c[4], c[5], c[6], c[7]);
        *reinterpret_cast<uint2*>(qr + idx * 8) = packed;
      }
    }
    if (tid == 0) scale[row] = sc;
    __syncthreads();  // `red` is reused by the next row
  }
}

template <bool kMul, int VPT>
static cudaError_t launch_rq(const uint16_t* src, int64_t rows, int K, const float* s, int8_t* q, float* scale,
                             cudaStream_t st, const DeviceInfo& dev) {
  const size_t smem = static_cast<size_t>(K) * (kMul ? 4 : 8);
  auto kern = row_quant_kernel<kMul, VPT>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kRowThreads, smem);
  if (e != cudaSuccess) return e;
  per_sm = std::max(per_sm, 1);
  const int64_t grid = std::min<int64_t>(rows, static_cast<int64_t>(dev.sm_count) * per_sm);
  kern<<<static_cast<unsigned>(grid), kRowThreads, smem, st>>>(src, rows, K, s, q, scale);
  return cudaGetLastError();
}

cudaError_t launch_row_quant(bool multiply, const uint16_t* src, int64_t rows, int64_t K, const float* s, int8_t* q,
                             float* scale, cudaStream_t st, const DeviceInfo& dev) {
  const int Ki = static_cast<int>(K);
  const int64_t nvec = K / 8;
  const int vpt = static_cast<int>((nvec + kRowThreads - 1) / kRowThreads);
  if (multiply) {
    if (vpt <= 1) return launch_rq<true, 1>(src, rows, Ki, s, q, scale, st, dev);
    if (vpt <= 2) return launch_rq<true, 2>(src, rows, Ki, s, q, scale, st, dev);
    if (vpt <= 4) return launch_rq<true, 4>(src, rows, Ki, s, q, scale, st, dev);
    return launch_rq<true, 8>(src, rows, Ki, s, q, scale, st, dev);
  }
  if (vpt <= 1) return launch_rq<false, 1>(src, rows, Ki, s, q, scale, st, dev);
  if (vpt <= 2) return launch_rq<false, 2>(src, rows, Ki, s, q, scale, st, dev);
  if (vpt <= 4) return launch_rq<false, 4>(src, rows, Ki, s, q, scale, st, dev);
  return launch_rq<false, 8>(src, rows, Ki, s, q, scale, st, dev);
}

}  // namespace sq
