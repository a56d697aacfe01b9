// sq_internal.h -- launchers shared between the libsq translation units.
// Arguments are validated by the C ABI layer (sq_api.cu) before these run.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <utility>

namespace sq {

// Largest K the row quantisers handle: a row is held in registers by at most
// eight warps of eight 16-byte vectors per lane.
constexpr int64_t kMaxQuantK = 16384;

// cudaSharedmemCarveoutMaxShared: every libsq kernel asks for the same L1 /
// shared-memory split, so back-to-back kernels need no reconfiguration.
constexpr int kCarveoutMaxShared = 100;

// Launch a kernel with programmatic stream serialization (it may begin while
// the previous kernel in the stream drains; the kernel itself waits for that
// kernel's results before touching global memory) and, when cluster_x >= 1,
// as clusters of cluster_x CTAs along x (cluster_x == 0: no cluster launch).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                               unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  unsigned n = 1;
  if (cluster_x >= 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  return launch_pdl_cluster(kern, grid, block, smem, st, 0u, std::forward<Args>(args)...);
}

struct DeviceInfo {
  int device = -1;
  int sm_count = 0;
  int major = 0, minor = 0;
  size_t max_smem_optin = 0;
};

// Cached properties of the current device.
cudaError_t current_device_info(DeviceInfo* out);

// 2-D tensor map over a row-major [rows][cols] matrix of elem_bytes-wide
// elements (row pitch pitch_bytes, or cols * elem_bytes when 0), box
// box_cols x box_rows, zero fill outside the matrix; swizzle_bytes 0 (none),
// 32, 64 or 128 (the shared-memory box's 16-byte units permuted as the
// hardware swizzle mode of that span).  False when the driver's encoder is
// unavailable or rejects the arguments.
bool make_tmap_2d(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int elem_bytes, int box_cols,
                  int box_rows, int swizzle_bytes = 0, int64_t pitch_bytes = 0);

// Status word of the HBM-bound kernels (bit 0: a wait timed out).  Clearing a
// set word also re-zeroes the no-allocation calibration scratch.
cudaError_t read_quant_status(uint32_t* flags, bool clear);

// ---- calibration (sq_quant.cu)
// 32-bit words of calibration scratch: mx[K], mw[K], one counter per 256 columns.
size_t calibrate_workspace_words(int64_t K);
// ws_is_zero: the caller guarantees the workspace words are zero (no memset).
// Every call leaves them zero.
cudaError_t launch_calibrate(const uint16_t* C, int64_t R, int64_t K, const uint16_t* W, int64_t N, float alpha,
                             float* s, float* mx_inout, void* ws, bool ws_is_zero, cudaStream_t st,
                             const DeviceInfo& dev);

// Largest K accepted by sq_calibrate_noalloc (its fixed scratch holds 2*K words).
constexpr int64_t kNoAllocMaxK = 16384;

// Same as launch_calibrate, with the scratch in a fixed device array instead
// of a caller workspace; looks up that array's address on a device's first call.
cudaError_t launch_calibrate_noalloc(const uint16_t* C, int64_t R, int64_t K, const uint16_t* W, int64_t N,
                                     float alpha, float* s, float* mx_inout, cudaStream_t st, const DeviceInfo& dev);

// ---- row quantisers (sq_quant.cu)
// multiply == true : weight path,   t = fl(w * s_j)
// multiply == false: activation path, t = fl(x / s_j)
cudaError_t launch_row_quant(bool multiply, const uint16_t* src, int64_t rows, int64_t K, const float* s,
                             int8_t* q, float* scale, cudaStream_t st, const DeviceInfo& dev);

// Activation scales only (the pre-pass of launch_forward_prologue):
// scale[m] exactly as launch_row_quant(false, ...) computes it, no codes, and
// RN(1/s_j) into recip[K] (16-byte aligned).
cudaError_t launch_act_scales(const uint16_t* X, int64_t rows, int64_t K, const float* s, float* scale, float* recip,
                              cudaStream_t st, const DeviceInfo& dev);

// ---- per-tensor quantisation, the baseline beside SmoothQuant (sq_quant.cu)
// Workspace: one partial maximum per pass-1 block.
size_t per_tensor_workspace_bytes();
// Aq = clamp(rne(fl(A / scale)), -128, 127) with scale = fl(max|A| / 127)
// (1.0 below 1e-8); every entry of scale_rows[rows] receives the scale.
cudaError_t launch_quantize_per_tensor(const uint16_t* src, int64_t rows, int64_t K, int8_t* q, float* scale_rows,
                                       void* ws, cudaStream_t st, const DeviceInfo& dev);

// ---- int8 weight-only linear, the decode comparison point (sq_weight_only.cu)
// Y = bf16((X Wq^T) * w_scale + bias) with X in bf16; cudaErrorNotSupported
// when K exceeds the kernel's 4 x 4096 columns.
cudaError_t launch_weight_only(const uint16_t* X, int64_t M, const int8_t* Wq, const float* w_scale,
                               const uint16_t* bias, int64_t N, int64_t K, uint16_t* Y, cudaStream_t st,
                               const DeviceInfo& dev);

// Status word of the weight-only kernel (bit 0: a wait timed out).
cudaError_t read_weight_only_status(uint32_t* flags, bool clear);

// ---- GEMM (sq_gemm.cu)
enum class Epilogue { kBf16Dequant = 0, kS32 = 1 };

struct GemmArgs {
  const int8_t* A;          // Xq [M][K]
  const int8_t* B;          // Wq [N][K]
  int64_t M, N, K;
  const float* x_scale;     // [M]   (bf16 epilogue)
  const float* w_scale;     // [N]   (bf16 epilogue)
  const uint16_t* bias;     // [N] or null
  void* out;                // Y bf16 [M][N] or acc int32 [M][N]
  Epilogue epi;
  void* ws = nullptr;       // optional scratch (16-byte aligned) for the split-K exchange
  size_t ws_bytes = 0;
};
cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t st, const DeviceInfo& dev, const char** why);

// Scratch the GEMM can use for an M x N x K problem on a device with sm_count
// SMs (0: none; the split-K path is taken only when at least this much is given).
size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int sm_count);

// Few tokens (M <= kSmallMaxM): weight-streaming kernel, split-K over a thread
// block cluster.  With X != null the per-token quantisation of X / s is fused
// (codes and scales identical to launch_row_quant); otherwise Xq and x_scale
// come from the caller.  Returns cudaErrorNotSupported when the shape does not
// fit the kernel (the caller then uses the general path).
constexpr int64_t kSmallMaxM = 32;
// sq_forward fuses the activation quantisation into that kernel up to this
// many tokens; above it (to kSmallMaxM) the row quantiser runs first.
#ifndef SQ_SMALL_FUSED_MAX  // build-time knob
#define SQ_SMALL_FUSED_MAX 8
#endif
constexpr int64_t kSmallFusedMaxM = SQ_SMALL_FUSED_MAX;
struct SmallArgs {
  const uint16_t* X;      // fused: bf16 [M][K]
  const float* s;         // fused: [K]
  const int8_t* Xq;       // prequantised: [M][K]
  const float* x_scale;   // prequantised: [M]
  const int8_t* Wq;       // [N][K]
  const float* w_scale;   // [N]
  const uint16_t* bias;   // [N] or null
  int64_t M, N, K;
  uint16_t* Y;            // [M][N]
};
cudaError_t launch_small_m(const SmallArgs& a, cudaStream_t st, const DeviceInfo& dev, const char** why);

// Many tokens, activation quantisation fused into the GEMM: a pre-pass writes
// x_scale[M] and RN(1/s)[K] (caller scratch, 16-byte aligned), then a CTA-pair
// GEMM converts bf16 X to codes in shared memory as it goes (codes, scales and
// Y identical to launch_row_quant followed by launch_gemm).  Needs K % 16 == 0.
struct PrologueArgs {
  const uint16_t* X;      // [M][K] bf16
  const float* s;         // [K]
  const int8_t* Wq;       // [N][K]
  const float* w_scale;   // [N]
  const uint16_t* bias;   // [N] or null
  int64_t M, N, K;
  uint16_t* Y;            // [M][N]
  float* x_scale;         // scratch [M]
  float* rs;              // scratch [K]
};
cudaError_t launch_forward_prologue(const PrologueArgs& a, cudaStream_t st, const DeviceInfo& dev, const char** why);

// Test hook: while enabled, the GEMMs' producers skip their first stage and
// every wait gives up after timeout_ns (the kernel then reports bit 0).
void debug_pipeline_stall(bool enable, unsigned long long timeout_ns);
// Whether that hook is on; *timeout_ns receives the wait limit to use (the
// hook's while it is on, the normal one otherwise).
bool debug_stall_state(unsigned long long* timeout_ns);

// Device status word (bit 0: pipeline wait timeout).
cudaError_t read_device_status(uint32_t* flags, bool clear);

// ---- relative-MSE auxiliary loss (sq_aux.cu)
// loss = sum (Y_fp - Y_q)^2 / max(sum Y_fp^2, 1e-24) over n elements (float64);
// with g_out != null also g_out = bf16(g_in + lambda * 2 (Y_q - Y_fp) / den)
// (g_in and g_out may be the same array).  ws: rel_mse_workspace_bytes(),
// 16-byte aligned.
size_t rel_mse_workspace_bytes();
cudaError_t launch_rel_mse(const uint16_t* yfp, const uint16_t* yq, int64_t n, double lambda, const uint16_t* g_in,
                           uint16_t* g_out, double* loss, void* ws, cudaStream_t st, const DeviceInfo& dev);

// ---- straight-through backward of the learnable-alpha layer (sq_ste.cu)
struct SteArgs {
  const uint16_t* G;      // [M][N] bf16, dL/dY
  const uint16_t* X;      // [M][K] bf16
  const uint16_t* W;      // [N][K] bf16
  const float* s;         // [K]
  const float* mx;        // [K] running activation max
  float alpha;
  const int8_t* Xq;       // [M][K]
  const float* x_scale;   // [M]
  const int8_t* Wq;       // [N][K]
  const float* w_scale;   // [N]
  int64_t M, N, K;
  float* dX;              // [M][K]
  float* dW;              // [N][K]
  float* db;              // [N] or null
  float* ds;              // [K] or null
  float* d_eta;           // [1]
  void* ws;
  size_t ws_bytes;
};
size_t ste_workspace_bytes(int64_t M, int64_t N, int64_t K);
cudaError_t launch_ste_backward(const SteArgs& a, cudaStream_t st, const DeviceInfo& dev, const char** why);
cudaError_t read_ste_status(uint32_t* flags, bool clear);

}  // namespace sq
