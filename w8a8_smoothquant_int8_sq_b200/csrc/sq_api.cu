// sq_api.cu -- the C ABI of libsq: argument validation, workspace carving,
// launch, status codes.  Declarations and contracts: include/sq.h.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/sq.h"
#include "sq_internal.h"

namespace sq {

// ------------------------------------------------------------ device info
cudaError_t current_device_info(DeviceInfo* out) {
  static std::mutex mu;
  static std::vector<DeviceInfo> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  if (dev < static_cast<int>(cache.size()) && cache[dev].device == dev) {
    *out = cache[dev];
    return cudaSuccess;
  }
  DeviceInfo d;
  d.device = dev;
  if ((e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) return e;
  int smem = 0;
  if ((e = cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  d.max_smem_optin = static_cast<size_t>(smem);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1);
  cache[dev] = d;
  *out = d;
  return cudaSuccess;
}

}  // namespace sq

namespace {

thread_local std::string g_last_error;
std::atomic<int> g_fail_after{-1};

constexpr int64_t kMaxGemmK = 133143;  // 127^2 * K must stay below 2^31

sq_status fail(sq_status st, const std::string& msg) {
  g_last_error = std::string(sq_status_string(st)) + ": " + msg;
  return st;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Host-side fault injection: consume one "launch credit".
bool injected_failure() {
  int cur = g_fail_after.load();
  while (cur >= 0) {
    if (cur == 0) return true;
    if (g_fail_after.compare_exchange_weak(cur, cur - 1)) return false;
  }
  return false;
}

sq_status prologue(sq::DeviceInfo* dev) {
  cudaError_t e = sq::current_device_info(dev);
  if (e != cudaSuccess) return fail(SQ_ERR_CUDA, std::string("device query: ") + cudaGetErrorString(e));
  if (dev->major != 10)
    return fail(SQ_ERR_UNSUPPORTED, "libsq needs an sm_100 device (compute capability 10.x); found " +
                                        std::to_string(dev->major) + "." + std::to_string(dev->minor));
  if (injected_failure()) return fail(SQ_ERR_CUDA, "injected failure (sq_debug_fail_after)");
  return SQ_OK;
}

sq_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return SQ_OK;
  return fail(SQ_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

sq_status check_k(int64_t K, int64_t kmax) {
  if (K < 16 || K > kmax) return fail(SQ_ERR_SHAPE, "K=" + std::to_string(K) + " outside [16, " + std::to_string(kmax) + "]");
  if (K % 16 != 0) return fail(SQ_ERR_ALIGN, "K=" + std::to_string(K) + " is not a multiple of 16");
  return SQ_OK;
}

sq_status check_rows(int64_t v, const char* name, int64_t lo = 1) {
  if (v < lo || v > INT32_MAX) return fail(SQ_ERR_SHAPE, std::string(name) + "=" + std::to_string(v) + " out of range");
  return SQ_OK;
}

#define SQ_TRY(x)                 \
  do {                            \
    sq_status _st = (x);          \
    if (_st != SQ_OK) return _st; \
  } while (0)

#define SQ_NONNULL(p)                                                       \
  do {                                                                      \
    if ((p) == nullptr) return fail(SQ_ERR_NULL, #p " is NULL");            \
    if (!aligned16(p)) return fail(SQ_ERR_ALIGN, #p " is not 16-byte aligned"); \
  } while (0)

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

extern "C" {

int sq_version(void) { return 100; }

const char* sq_last_error(void) { return g_last_error.c_str(); }

const char* sq_status_string(sq_status st) {
  switch (st) {
    case SQ_OK: return "SQ_OK";
    case SQ_ERR_NULL: return "SQ_ERR_NULL";
    case SQ_ERR_SHAPE: return "SQ_ERR_SHAPE";
    case SQ_ERR_ALIGN: return "SQ_ERR_ALIGN";
    case SQ_ERR_ARG: return "SQ_ERR_ARG";
    case SQ_ERR_UNSUPPORTED: return "SQ_ERR_UNSUPPORTED";
    case SQ_ERR_CUDA: return "SQ_ERR_CUDA";
    case SQ_ERR_TIMEOUT: return "SQ_ERR_TIMEOUT";
    case SQ_ERR_WORKSPACE: return "SQ_ERR_WORKSPACE";
  }
  return "SQ_ERR_UNKNOWN";
}

void sq_debug_fail_after(int n) { g_fail_after.store(n < 0 ? -1 : n); }

void sq_debug_pipeline_stall(int enable, int64_t timeout_ns) {
  sq::debug_pipeline_stall(enable != 0, timeout_ns > 0 ? static_cast<unsigned long long>(timeout_ns) : 0ull);
}

// ------------------------------------------------------------ calibration
size_t sq_calibrate_workspace_bytes(int64_t K) {
  if (K <= 0) return 0;
  return round_up(sq::calibrate_workspace_words(K) * sizeof(uint32_t), 256);
}

sq_status sq_calibrate(const sq_bf16* C, int64_t R, int64_t K, const sq_bf16* W, int64_t N, float alpha, float* s,
                       float* mx_inout, void* workspace, size_t workspace_bytes, void* stream) {
  SQ_TRY(check_k(K, INT32_MAX - 15));
  SQ_TRY(check_rows(N, "N"));
  SQ_TRY(check_rows(R, "R", 0));
  if (!(alpha >= 0.0f && alpha <= 1.0f)) return fail(SQ_ERR_ARG, "alpha must lie in [0, 1]");
  if (R > 0) SQ_NONNULL(C);
  if (R == 0 && mx_inout == nullptr) return fail(SQ_ERR_NULL, "R == 0 needs the running max mx_inout");
  SQ_NONNULL(W);
  SQ_NONNULL(s);
  if (mx_inout != nullptr && !aligned16(mx_inout)) return fail(SQ_ERR_ALIGN, "mx_inout is not 16-byte aligned");
  if (workspace == nullptr || workspace_bytes < sq_calibrate_workspace_bytes(K))
    return fail(SQ_ERR_WORKSPACE, "workspace must hold sq_calibrate_workspace_bytes(K) = " +
                                      std::to_string(sq_calibrate_workspace_bytes(K)) + " bytes");
  if (!aligned16(workspace)) return fail(SQ_ERR_ALIGN, "workspace is not 16-byte aligned");
  sq::DeviceInfo dev;
  SQ_TRY(prologue(&dev));
  return cuda_status(sq::launch_calibrate(C, R, K, W, N, alpha, s, mx_inout, workspace, /*ws_is_zero=*/false,
                                          static_cast<cudaStream_t>(stream), dev),
                     "calibrate launch");
}

// For callers that cannot pass scratch memory: the column maxima live in a
// fixed array inside the library (see include/sq.h for the limits and the
// sharing rule); nothing is allocated.
sq_status sq_calibrate_noalloc(const sq_bf16* C, int64_t R, int64_t K, const sq_bf16* W, int64_t N, float alpha,
                               float* s, float* mx_inout, void* stream) {
  SQ_TRY(check_k(K, INT32_MAX - 15));
  if (K > sq::kNoAllocMaxK)
    return fail(SQ_ERR_SHAPE, "sq_calibrate_noalloc supports K <= " + std::to_string(sq::kNoAllocMaxK) + " (got " +
                                  std::to_string(K) + "); use sq_calibrate with a workspace");
  SQ_TRY(check_rows(N, "N"));
  SQ_TRY(check_rows(R, "R", 0));
  if (!(alpha >= 0.0f && alpha <= 1.0f)) return fail(SQ_ERR_ARG, "alpha must lie in [0, 1]");
  if (R > 0) SQ_NONNULL(C);
  if (R == 0 && mx_inout == nullptr) return fail(SQ_ERR_NULL, "R == 0 needs the running max mx_inout");
  SQ_NONNULL(W);
  SQ_NONNULL(s);
  if (mx_inout != nullptr && !aligned16(mx_inout)) return fail(SQ_ERR_ALIGN, "mx_inout is not 16-byte aligned");
  sq::DeviceInfo dev;
  SQ_TRY(prologue(&dev));
  return cuda_status(sq::launch_calibrate_noalloc(C, R, K, W, N, alpha, s, mx_inout,
                                                  static_cast<cudaStream_t>(stream), dev),
                     "calibrate (no-alloc) launch");
}

// ---------------------------------------------------------- weight prepare
sq_status sq_prepare_weight(const sq_bf16* W, int64_t N, int64_t K, const float* s, int8_t* Wq, float* w_scale,
                            void* stream) {
  SQ_TRY(check_k(K, sq::kMaxQuantK));
  SQ_TRY(check_rows(N, "N"));
  SQ_NONNULL(W);
  SQ_NONNULL(s);
  SQ_NONNULL(Wq);
  SQ_NONNULL(w_scale);
  sq::DeviceInfo dev;
  SQ_TRY(prologue(&dev));
  return cuda_status(sq::launch_row_quant(true, W, N, K, s, Wq, w_scale, static_cast<cudaStream_t>(stream), dev),
                     "prepare_weight launch");
}

// -------------------------------------------------------- activation quant
sq_status sq_quantize_act(const sq_bf16* X, int64_t M, int64_t K, const float* s, int8_t* Xq, float* x_scale,
                          void* stream) {
  SQ_TRY(check_k(K, sq::kMaxQuantK));
  SQ_TRY(check_rows(M, "M"));
  SQ_NONNULL(X);
  SQ_NONNULL(s);
  SQ_NONNULL(Xq);
  SQ_NONNULL(x_scale);
  sq::DeviceInfo dev;
  SQ_TRY(prologue(&dev));
  return cuda_status(sq::launch_row_quant(false, X, M, K, s, Xq, x_scale, static_cast<cudaStream_t>(stream), dev),
                     "quantize_act launch");
}

// --------------------------------------------- per-tensor baseline quantiser
size_t sq_quantize_per_tensor_workspace_bytes(void) { return sq::per_tensor_workspace_bytes(); }

sq_status sq_quantize_per_tensor(const sq_bf16* A, int64_t rows, int64_t K, int8_t* Aq, float* scale_rows,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  SQ_TRY(check_k(K, INT32_MAX - 15));
  SQ_TRY(check_rows(rows, "rows"));
  SQ_NONNULL(A);
  SQ_NONNULL(Aq);
  SQ_NONNULL(scale_rows);
  if (workspace == nullptr || workspace_bytes < sq::per_tensor_workspace_bytes())
    return fail(SQ_ERR_WORKSPACE, "workspace must hold sq_quantize_per_tensor_workspace_bytes() = " +
                                      std::to_string(sq::per_tensor_workspace_bytes()) + " bytes");
  if (!aligned16(workspace)) return fail(SQ_ERR_ALIGN, "workspace is not 16-byte aligned");
  sq::DeviceInfo dev;
  SQ_TRY(prologue(&dev));
  return cuda_status(sq::launch_quantize_per_tensor(A, rows, K, Aq, scale_rows, workspace,
                                                    static_cast<cudaStream_t>(stream), dev),
                     "quantize_per_tensor launch");
}

// ------------------------------------------------- int8 weight-only linear
sq_status sq_linear_weight_only(const sq_bf16* X, int64_t M, const int8_t* Wq, const float* w_scale,
                                const sq_bf16* bias, int64_t N, int64_t K, sq_bf16* Y, void* stream) {
  SQ_TRY(check_k(K, sq::kMaxQuantK));
  SQ_TRY(check_rows(M, "M"));
  SQ_TRY(check_rows(N, "N"));
  SQ_NONNULL(X);
  SQ_NONNULL(Wq);
  SQ_NONNULL(w_scale);
  SQ_NONNULL(Y);
  if (bias != nullptr && !aligned16(bias)) return fail(SQ_ERR_ALIGN, "bias is not 16-byte aligned");
  sq::DeviceInfo dev;
  SQ_TRY(prologue(&dev));
  return cuda_status(sq::launch_weight_only(X, M, Wq, w_scale, bias, N, K, Y, static_cast<cudaStream_t>(stream), dev),
                     "weight-only linear launch");
}

// ------------------------------------- learnable-alpha straight-through backward
size_t sq_ste_backward_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return sq::ste_workspace_bytes(M, N, K);
}

sq_status sq_ste_backward(const sq_bf16* G, const sq_bf16* X, const sq_bf16* W, const float* s, const float* mx,
                          float alpha, const int8_t* Xq, const float* x_scale, const int8_t* Wq,
                          const float* w_scale, int64_t M, int64_t N, int64_t K, float* dX, float* dW, float* db,
                          float* ds, float* d_eta, void* workspace, size_t workspace_bytes, void* stream) {
  SQ_TRY(check_k(K, sq::kMaxQuantK));
  SQ_TRY(check_rows(M, "M"));
  SQ_TRY(check_rows(N, "N"));
  if (N % 8 != 0) return fail(SQ_ERR_ALIGN, "N=" + std::to_string(N) + " is not a multiple of 8");
  if (!(alpha >= 0.0f && alpha <= 1.0f)) return fail(SQ_ERR_ARG, "alpha outside [0, 1]");
  SQ_NONNULL(G);
  SQ_NONNULL(X);
  SQ_NONNULL(W);
  SQ_NONNULL(s);
  SQ_NONNULL(mx);
  SQ_NONNULL(Xq);
  SQ_NONNULL(x_scale);
  SQ_NONNULL(Wq);
  SQ_NONNULL(w_scale);
  SQ_NONNULL(dX);
  SQ_NONNULL(dW);
  SQ_NONNULL(d_eta);
  SQ_NONNULL(workspace);
  if (db != nullptr && !aligned16(db)) return fail(SQ_ERR_ALIGN, "db is not 16-byte aligned");
  if (ds != nullptr && !aligned16(ds)) return fail(SQ_ERR_ALIGN, "ds is not 16-byte aligned");
  const size_t need = sq::ste_workspace_bytes(M, N, K);
  if (workspace_bytes < need)
    return fail(SQ_ERR_WORKSPACE, "workspace of " + std::to_string(workspace_bytes) + " bytes; " +
                                      std::to_string(need) + " needed");
  sq::DeviceInfo dev;
  SQ_TRY(prologue(&dev));
  sq::SteArgs a;
  a.G = G;
  a.X = X;
  a.W = W;
  a.s = s;
  a.mx = mx;
  a.alpha = alpha;
  a.Xq = Xq;
  a.x_scale = x_scale;
  a.Wq = Wq;
  a.w_scale = w_scale;
  a.M = M;
  a.N = N;
  a.K = K;
  a.dX = dX;
  a.dW = dW;
  a.db = db;
  a.ds = ds;
  a.d_eta = d_eta;
  a.ws = workspace;
  a.ws_bytes = workspace_bytes;
  const char* why = "launch";
  cudaError_t e = sq::launch_ste_backward(a, static_cast<cudaStream_t>(stream), dev, &why);
  if (e != cudaSuccess) return fail(SQ_ERR_CUDA, std::string("straight-through backward: ") + why + ": " +
                                                     cudaGetErrorString(e));
  return SQ_OK;
}

// ------------------------------------------------------------- int8 linear
// SMs assumed when no device can be queried (a B200), so that sizes asked
// before a device is current are the ones a B200 will want.
constexpr int kDefaultSmCount = 148;

size_t sq_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= sq::kSmallMaxM || M <= 0 || N <= 0 || K <= 0) return 0;  // the few-token kernel needs none
  sq::DeviceInfo dev;
  const int sms = sq::current_device_info(&dev) == cudaSuccess ? dev.sm_count : kDefaultSmCount;
  return sq::gemm_workspace_bytes(M, N, K, sms);
}

static sq_status gemm_common(const int8_t* Xq, const float* x_scale, const int8_t* Wq, const float* w_scale,
                             const sq_bf16* bias, int64_t M, int64_t N, int64_t K, void* out, sq::Epilogue epi,
                             void* stream, const sq::DeviceInfo& dev, void* ws = nullptr, size_t ws_bytes = 0) {
  sq::GemmArgs a;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  a.A = Xq;
  a.B = Wq;
  a.M = M;
  a.N = N;
  a.K = K;
  a.x_scale = x_scale;
  a.w_scale = w_scale;
  a.bias = bias;
  a.out = out;
  a.epi = epi;
  const char* why = "kernel launch";
  cudaError_t e = sq::launch_gemm(a, static_cast<cudaStream_t>(stream), dev, &why);
  return cuda_status(e, why);
}

sq_status sq_linear(const int8_t* Xq, const float* x_scale, const int8_t* Wq, const float* w_scale,
                    const sq_bf16* bias, int64_t M, int64_t N, int64_t K, sq_bf16* Y, void* workspace,
                    size_t workspace_bytes, void* stream) {
  SQ_TRY(check_k(K, kMaxGemmK));
  SQ_TRY(check_rows(M, "M"));
  SQ_TRY(check_rows(N, "N"));
  SQ_NONNULL(Xq);
  SQ_NONNULL(x_scale);
  SQ_NONNULL(Wq);
  SQ_NONNULL(w_scale);
  SQ_NONNULL(Y);
  if (bias != nullptr && !aligned16(bias)) return fail(SQ_ERR_ALIGN, "bias is not 16-byte aligned");
  if (workspace != nullptr && !aligned16(workspace)) return fail(SQ_ERR_ALIGN, "workspace is not 16-byte aligned");
  sq::DeviceInfo dev;
  SQ_TRY(prologue(&dev));
  if (M <= sq::kSmallMaxM) {  // few tokens: weight-streaming split-K kernel
    sq::SmallArgs a{nullptr, nullptr, Xq, x_scale, Wq, w_scale, bias, M, N, K, Y};
    const char* why = "small-M kernel";
    cudaError_t e = sq::launch_small_m(a, static_cast<cudaStream_t>(stream), dev, &why);
    if (e != cudaErrorNotSupported) return cuda_status(e, why);
  }
  return gemm_common(Xq, x_scale, Wq, w_scale, bias, M, N, K, Y, sq::Epilogue::kBf16Dequant, stream, dev,
                     workspace, workspace == nullptr ? 0 : workspace_bytes);
}

// ------------------------------------------------ auxiliary loss (learnable alpha)
size_t sq_rel_mse_workspace_bytes(void) { return round_up(sq::rel_mse_workspace_bytes(), 256); }

sq_status sq_rel_mse(const sq_bf16* Y_fp, const sq_bf16* Y_q, int64_t M, int64_t N, double lambda,
                     const sq_bf16* G_in, sq_bf16* G_out, double* loss_out, void* workspace, size_t workspace_bytes,
                     void* stream) {
  SQ_TRY(check_rows(M, "M"));
  SQ_TRY(check_rows(N, "N"));
  SQ_NONNULL(Y_fp);
  SQ_NONNULL(Y_q);
  if (loss_out == nullptr) return fail(SQ_ERR_NULL, "loss_out is NULL");
  if ((reinterpret_cast<uintptr_t>(loss_out) & 7u) != 0) return fail(SQ_ERR_ALIGN, "loss_out is not 8-byte aligned");
  if ((G_in == nullptr) != (G_out == nullptr)) return fail(SQ_ERR_ARG, "G_in and G_out must both be given or both be NULL");
  if (G_in != nullptr && (!aligned16(G_in) || !aligned16(G_out)))
    return fail(SQ_ERR_ALIGN, "G_in / G_out are not 16-byte aligned");
  if (!std::isfinite(lambda)) return fail(SQ_ERR_ARG, "lambda is not finite");
  if (workspace == nullptr || workspace_bytes < sq_rel_mse_workspace_bytes())
    return fail(SQ_ERR_WORKSPACE, "workspace must hold sq_rel_mse_workspace_bytes() = " +
                                      std::to_string(sq_rel_mse_workspace_bytes()) + " bytes");
  if (!aligned16(workspace)) return fail(SQ_ERR_ALIGN, "workspace is not 16-byte aligned");
  sq::DeviceInfo dev;
  SQ_TRY(prologue(&dev));
  return cuda_status(sq::launch_rel_mse(Y_fp, Y_q, M * N, lambda, G_in, G_out, loss_out, workspace,
                                        static_cast<cudaStream_t>(stream), dev),
                     "relative-MSE loss launch");
}

// ----------------------------------------------------------- fused forward
static size_t forward_xq_bytes(int64_t M, int64_t K) { return round_up(static_cast<size_t>(M * K), 256); }

size_t sq_forward_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || K <= 0) return 0;
  return forward_xq_bytes(M, K) + round_up(static_cast<size_t>(M) * sizeof(float), 256) + sq_workspace_bytes(M, N, K);
}

sq_status sq_forward(const sq_bf16* X, const float* s, const int8_t* Wq, const float* w_scale, const sq_bf16* bias,
                     int64_t M, int64_t N, int64_t K, sq_bf16* Y, void* workspace, size_t workspace_bytes,
                     void* stream) {
  SQ_TRY(check_k(K, sq::kMaxQuantK));
  SQ_TRY(check_rows(M, "M"));
  SQ_TRY(check_rows(N, "N"));
  SQ_NONNULL(X);
  SQ_NONNULL(s);
  SQ_NONNULL(Wq);
  SQ_NONNULL(w_scale);
  SQ_NONNULL(Y);
  if (bias != nullptr && !aligned16(bias)) return fail(SQ_ERR_ALIGN, "bias is not 16-byte aligned");
  if (workspace == nullptr || workspace_bytes < sq_forward_workspace_bytes(M, N, K))
    return fail(SQ_ERR_WORKSPACE, "workspace must hold sq_forward_workspace_bytes(M, N, K) = " +
                                      std::to_string(sq_forward_workspace_bytes(M, N, K)) + " bytes");
  if (!aligned16(workspace)) return fail(SQ_ERR_ALIGN, "workspace is not 16-byte aligned");
  sq::DeviceInfo dev;
  SQ_TRY(prologue(&dev));
  if (M <= sq::kSmallFusedMaxM) {  // few tokens: quantisation fused into the weight-streaming kernel
    sq::SmallArgs a{X, s, nullptr, nullptr, Wq, w_scale, bias, M, N, K, Y};
    const char* why = "fused small-M kernel";
    cudaError_t e = sq::launch_small_m(a, static_cast<cudaStream_t>(stream), dev, &why);
    if (e != cudaErrorNotSupported) return cuda_status(e, why);
  }
  int8_t* Xq = static_cast<int8_t*>(workspace);
  const size_t xs_off = forward_xq_bytes(M, K);
  float* xs = reinterpret_cast<float*>(static_cast<char*>(workspace) + xs_off);
  const size_t gemm_off = xs_off + round_up(static_cast<size_t>(M) * sizeof(float), 256);
  sq_status st = cuda_status(
      sq::launch_row_quant(false, X, M, K, s, Xq, xs, static_cast<cudaStream_t>(stream), dev), "quantize_act launch");
  if (st != SQ_OK) return st;
  if (M <= sq::kSmallMaxM) {  // few tokens, quantised first: the weight-streaming kernel on the codes
    sq::SmallArgs a{nullptr, nullptr, Xq, xs, Wq, w_scale, bias, M, N, K, Y};
    const char* why = "small-M kernel";
    cudaError_t e = sq::launch_small_m(a, static_cast<cudaStream_t>(stream), dev, &why);
    if (e != cudaErrorNotSupported) return cuda_status(e, why);
  }
  return gemm_common(Xq, xs, Wq, w_scale, bias, M, N, K, Y, sq::Epilogue::kBf16Dequant, stream, dev,
                     static_cast<char*>(workspace) + gemm_off, workspace_bytes - gemm_off);
}

// ------------------------------------- forward, quantisation in the GEMM
size_t sq_forward_prologue_workspace_bytes(int64_t M, int64_t K) {
  if (M <= 0 || K <= 0) return 0;
  return round_up(static_cast<size_t>(M) * sizeof(float), 256) + round_up(static_cast<size_t>(K) * sizeof(float), 256);
}

sq_status sq_forward_prologue(const sq_bf16* X, const float* s, const int8_t* Wq, const float* w_scale,
                              const sq_bf16* bias, int64_t M, int64_t N, int64_t K, sq_bf16* Y, void* workspace,
                              size_t workspace_bytes, void* stream) {
  SQ_TRY(check_k(K, sq::kMaxQuantK));
  SQ_TRY(check_rows(M, "M"));
  SQ_TRY(check_rows(N, "N"));
  SQ_NONNULL(X);
  SQ_NONNULL(s);
  SQ_NONNULL(Wq);
  SQ_NONNULL(w_scale);
  SQ_NONNULL(Y);
  if (bias != nullptr && !aligned16(bias)) return fail(SQ_ERR_ALIGN, "bias is not 16-byte aligned");
  if (workspace == nullptr || workspace_bytes < sq_forward_prologue_workspace_bytes(M, K))
    return fail(SQ_ERR_WORKSPACE, "workspace must hold sq_forward_prologue_workspace_bytes(M, K) = " +
                                      std::to_string(sq_forward_prologue_workspace_bytes(M, K)) + " bytes");
  if (!aligned16(workspace)) return fail(SQ_ERR_ALIGN, "workspace is not 16-byte aligned");
  sq::DeviceInfo dev;
  SQ_TRY(prologue(&dev));
  float* xs = static_cast<float*>(workspace);
  float* rs = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                       round_up(static_cast<size_t>(M) * sizeof(float), 256));
  sq::PrologueArgs a{X, s, Wq, w_scale, bias, M, N, K, Y, xs, rs};
  const char* why = "fused-prologue forward";
  return cuda_status(sq::launch_forward_prologue(a, static_cast<cudaStream_t>(stream), dev, &why), why);
}

// ---------------------------------------------------------------- test hook
sq_status sq_gemm_s32(const int8_t* Xq, const int8_t* Wq, int64_t M, int64_t N, int64_t K, int32_t* acc,
                      void* stream) {
  SQ_TRY(check_k(K, kMaxGemmK));
  SQ_TRY(check_rows(M, "M"));
  SQ_TRY(check_rows(N, "N"));
  SQ_NONNULL(Xq);
  SQ_NONNULL(Wq);
  SQ_NONNULL(acc);
  sq::DeviceInfo dev;
  SQ_TRY(prologue(&dev));
  return gemm_common(Xq, nullptr, Wq, nullptr, nullptr, M, N, K, acc, sq::Epilogue::kS32, stream, dev);
}

// ------------------------------------------------------------ device status
sq_status sq_device_status(uint32_t* flags, int clear) {
  if (flags == nullptr) return fail(SQ_ERR_NULL, "flags is NULL");
  cudaError_t e = sq::read_device_status(flags, clear != 0);
  if (e != cudaSuccess) return cuda_status(e, "device status read");
  if (*flags != 0u) return fail(SQ_ERR_TIMEOUT, "a device-side pipeline wait timed out");
  return SQ_OK;
}

}  // extern "C"
