// sq_aux.cu -- the relative-MSE auxiliary loss of the learnable-alpha layer
// and its gradient with respect to the quantised output.
//
// Page: "w8a8_smoothquant.py -- W8A8 com SmoothQuant e alpha APRENDIVEL (V5)",
// module docstring: aux = ||Y_fp - Y_q||_F^2 / ||Y_fp||_F^2 (relative MSE),
// added to the total loss so that its gradient reaches eta_alpha.  Y_fp (the
// unquantised layer) does not depend on alpha, so the gradient that matters
// is d aux / d Y_q = 2 (Y_q - Y_fp) / den, den = max(||Y_fp||^2, 1e-24) (the
// square of the 1e-12 floor that quantization_error puts on the norm).
//
// Two passes over the n = M N bf16 elements of Y_fp and Y_q, 16-byte vectors
// (8 elements) per thread and four vectors in flight, sums in float64 (the
// square of the difference of two bf16 values is exact in float64; only the
// additions round):
//   aux_reduce_kernel  per-block partial sums of (Y_fp - Y_q)^2 and Y_fp^2
//                      into the workspace (plain stores: nothing to clear);
//   aux_update_kernel  every block adds all partials in one fixed order, so
//                      every block holds the same den; block 0 writes the
//                      loss; with a gradient it writes
//                      G_out = bf16(G_in + lambda * 2 (Y_q - Y_fp) / den),
//                      evaluated in float64 and rounded once.
#include <algorithm>
#include <cstdint>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {
namespace {

constexpr int kAuxThreads = 256;
constexpr int kAuxVecs = 4;          // 16-byte vectors in flight per thread and array
constexpr int kAuxMaxBlocks = 1184;  // partial sums the workspace holds
constexpr double kAuxDenFloor = 1e-24;

__device__ __forceinline__ double bf16_f64(uint32_t bits16) {
  return static_cast<double>(__uint_as_float(bits16 << 16));
}

// adds (a - b)^2 and a^2 over the 8 bf16 pairs of two vectors
__device__ __forceinline__ void acc8(const uint4 a, const uint4 b, double& num, double& den) {
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const double a0 = bf16_f64(wa[e] & 0xFFFFu), a1 = bf16_f64(wa[e] >> 16);
    const double d0 = a0 - bf16_f64(wb[e] & 0xFFFFu), d1 = a1 - bf16_f64(wb[e] >> 16);
    num = fma(d0, d0, num);
    num = fma(d1, d1, num);
    den = fma(a0, a0, den);
    den = fma(a1, a1, den);
  }
}

// sum over the block in a fixed order (shuffle tree, then warps in order)
__device__ __forceinline__ void block_sum2(double& x, double& y, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
    y += __shfl_xor_sync(0xFFFFFFFFu, y, o);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // earlier readers of red are done
  if (lane == 0) {
    red[2 * warp] = x;
    red[2 * warp + 1] = y;
  }
  __syncthreads();
  x = 0.0;
  y = 0.0;
  for (int w = 0; w < kAuxThreads / 32; ++w) {
    x += red[2 * w];
    y += red[2 * w + 1];
  }
}

__global__ void __launch_bounds__(kAuxThreads) aux_reduce_kernel(const uint16_t* __restrict__ yfp,
                                                                 const uint16_t* __restrict__ yq, int64_t n,
                                                                 double* __restrict__ part) {
  __shared__ double red[2 * kAuxThreads / 32];
  griddep_wait();
  griddep_launch_dependents();
  const int64_t nvec = n >> 3;
  const uint4* a4 = reinterpret_cast<const uint4*>(yfp);
  const uint4* b4 = reinterpret_cast<const uint4*>(yq);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kAuxThreads;
  double num = 0.0, den = 0.0;
  for (int64_t v0 = static_cast<int64_t>(blockIdx.x) * kAuxThreads + threadIdx.x; v0 < nvec;
       v0 += kAuxVecs * stride) {
    uint4 a[kAuxVecs], b[kAuxVecs];
#pragma unroll
    for (int i = 0; i < kAuxVecs; ++i) {
      const int64_t v = v0 + i * stride;
      a[i] = v < nvec ? __ldcs(a4 + v) : make_uint4(0u, 0u, 0u, 0u);
      b[i] = v < nvec ? __ldcs(b4 + v) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < kAuxVecs; ++i) acc8(a[i], b[i], num, den);
  }
  if (blockIdx.x == 0) {  // the elements past the last whole vector
    const int64_t e = (nvec << 3) + threadIdx.x;
    if (e < n) {
      const double a0 = bf16_f64(yfp[e]), d0 = a0 - bf16_f64(yq[e]);
      num = fma(d0, d0, num);
      den = fma(a0, a0, den);
    }
  }
  block_sum2(num, den, red);
  if (threadIdx.x == 0) {
    part[2 * blockIdx.x] = num;
    part[2 * blockIdx.x + 1] = den;
  }
}

__global__ void __launch_bounds__(kAuxThreads) aux_update_kernel(
    const uint16_t* __restrict__ yfp, const uint16_t* __restrict__ yq, int64_t n, const double* __restrict__ part,
    int nparts, double lambda, const uint16_t* g_in, uint16_t* g_out, double* __restrict__ loss) {
  __shared__ double red[2 * kAuxThreads / 32];
  griddep_wait();
  griddep_launch_dependents();
  double num = 0.0, den = 0.0;
  for (int i = threadIdx.x; i < nparts; i += kAuxThreads) {
    num += part[2 * i];
    den += part[2 * i + 1];
  }
  block_sum2(num, den, red);
  const double den_eff = fmax(den, kAuxDenFloor);
  if (blockIdx.x == 0 && threadIdx.x == 0) *loss = num / den_eff;
  if (g_out == nullptr) return;
  const double coef = lambda * 2.0 / den_eff;
  const int64_t nvec = n >> 3;
  const uint4* a4 = reinterpret_cast<const uint4*>(yfp);
  const uint4* b4 = reinterpret_cast<const uint4*>(yq);
  const uint4* g4 = reinterpret_cast<const uint4*>(g_in);
  uint4* o4 = reinterpret_cast<uint4*>(g_out);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kAuxThreads;
  for (int64_t v0 = static_cast<int64_t>(blockIdx.x) * kAuxThreads + threadIdx.x; v0 < nvec;
       v0 += kAuxVecs * stride) {
    uint4 a[kAuxVecs], b[kAuxVecs], g[kAuxVecs];
#pragma unroll
    for (int i = 0; i < kAuxVecs; ++i) {
      const int64_t v = v0 + i * stride;
      const bool ok = v < nvec;
      a[i] = ok ? __ldcs(a4 + v) : make_uint4(0u, 0u, 0u, 0u);
      b[i] = ok ? __ldcs(b4 + v) : make_uint4(0u, 0u, 0u, 0u);
      g[i] = ok ? __ldcs(g4 + v) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < kAuxVecs; ++i) {
      const int64_t v = v0 + i * stride;
      if (v >= nvec) break;
      const uint32_t wa[4] = {a[i].x, a[i].y, a[i].z, a[i].w}, wb[4] = {b[i].x, b[i].y, b[i].z, b[i].w};
      const uint32_t wg[4] = {g[i].x, g[i].y, g[i].z, g[i].w};
      uint32_t out[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const double lo = fma(coef, bf16_f64(wb[e] & 0xFFFFu) - bf16_f64(wa[e] & 0xFFFFu), bf16_f64(wg[e] & 0xFFFFu));
        const double hi = fma(coef, bf16_f64(wb[e] >> 16) - bf16_f64(wa[e] >> 16), bf16_f64(wg[e] >> 16));
        out[e] = static_cast<uint32_t>(__bfloat16_as_ushort(__double2bfloat16(lo))) |
                 (static_cast<uint32_t>(__bfloat16_as_ushort(__double2bfloat16(hi))) << 16);
      }
      __stcs(o4 + v, make_uint4(out[0], out[1], out[2], out[3]));
    }
  }
  if (blockIdx.x == 0) {
    const int64_t e = (nvec << 3) + threadIdx.x;
    if (e < n) {
      const double val = fma(coef, bf16_f64(yq[e]) - bf16_f64(yfp[e]), bf16_f64(g_in[e]));
      g_out[e] = __bfloat16_as_ushort(__double2bfloat16(val));
    }
  }
}

int aux_blocks(int64_t n, const DeviceInfo& dev) {
  const int64_t per_block = static_cast<int64_t>(kAuxThreads) * kAuxVecs * 8;
  const int64_t want = (n + per_block - 1) / per_block;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>({want, kAuxMaxBlocks, 8ll * dev.sm_count})));
}

}  // namespace

size_t rel_mse_workspace_bytes() { return static_cast<size_t>(2 * kAuxMaxBlocks) * sizeof(double); }

cudaError_t launch_rel_mse(const uint16_t* yfp, const uint16_t* yq, int64_t n, double lambda, const uint16_t* g_in,
                           uint16_t* g_out, double* loss, void* ws, cudaStream_t st, const DeviceInfo& dev) {
  double* part = static_cast<double*>(ws);
  const int nb = aux_blocks(n, dev);
  cudaError_t e = launch_pdl(aux_reduce_kernel, dim3(static_cast<unsigned>(nb)), dim3(kAuxThreads), 0, st, yfp, yq,
                             n, part);
  if (e != cudaSuccess) return e;
  const int nu = g_out != nullptr ? nb : 1;
  return launch_pdl(aux_update_kernel, dim3(static_cast<unsigned>(nu)), dim3(kAuxThreads), 0, st, yfp, yq, n,
                    static_cast<const double*>(part), nb, lambda, g_in, g_out, loss);
}

}  // namespace sq
