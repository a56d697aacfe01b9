// sq_gemm_small.cuh -- the int8 linear for few tokens (M <= 32), optionally with
// the per-token activation quantisation fused in.  Included by sq_gemm.cu (one
// translation unit: it shares the device status word and the host helpers).
//
// Page: "w8a8_smoothquant.py -- W8A8 com SmoothQuant e alpha APRENDIVEL (V5)",
// SmoothQuantW8A8.forward (X / s, per-token quantisation, int8 product,
// dequantisation and bias).  With few tokens the layer is a stream of the int8
// weight: the kernel is built to read Wq from HBM once, at full bandwidth.
//
//   * swap-AB: the MMA's M = 128 rows of Wq, its N = the tokens padded to
//     NT = 16 or 32 (tcgen05.mma kind::i8, M=128, N=NT, K=32).  A CTA owns
//     256 rows of Wq, fetched as one 256-row x 128-byte TMA box per stage
//     (large boxes stream HBM markedly faster than 128-row ones) and fed to the
//     tensor core as two 128-row halves with their own accumulators.  An M=128
//     int8 MMA costs about the same whatever its N, so the tensor core takes
//     about 4 KB of Wq per MMA; spreading the rows over ~128 CTAs keeps that
//     above the HBM rate.
//   * split-K over a thread-block cluster of S CTAs: each CTA streams its
//     share of the row block's K; at the end every CTA pushes its partial
//     int32 sums of each row (real tokens only) into the shared memory of the
//     rank that reduces that row with st.async, whose bytes count on that
//     rank's mbarrier, and once its phase completes each rank adds the S
//     partials of its rows from its own shared memory (exact, no global
//     scratch, no remote load and no cluster barrier at the end).
//   * prequantised codes (sq_linear): the codes travel by TMA in the same
//     stage as the weight box (NT-row box, rows past M zero-filled), so the
//     first MMA waits only for the first stage.
//   * fused quantisation (sq_forward, up to 8 tokens): eight warps quantise
//     this CTA's K-slice of X / s (correctly rounded fp32 division, as
//     sq_quantize_act), holding their X vectors in registers between the two
//     passes.  The per-token maxima over the whole row are assembled from the
//     S ranks' slice maxima: every rank stores its maxima into every rank's
//     shared memory with st.async, which counts the bytes on the receiver's
//     own mbarrier (no cluster barrier, no cluster-scope release: under the
//     weight stream a cluster barrier here took ~5 us, the asynchronous
//     stores ~0.4 us); the codes then go straight into the shared-memory B
//     operand in the 128-byte-swizzled K-major layout the tensor core reads.
//     The MMAs cannot start before the codes exist, and past that point the
//     kernel runs at the weight-stream rate, so the fused path is only about
//     as fast as quantising first; beyond 8 tokens sq_forward quantises first.
//
// Warps: 0 TMA producer, 1 TMEM owner + MMA issuer, 2..9 quantisation and
// reduction (2..5 also drain TMEM: lane quarters 2, 3, 0, 1).  Every mbarrier
// wait is bounded; every thread takes part in the one cluster phase (arrived
// after the barrier set-up, waited for before its first remote store or at
// the end).

namespace sq {
namespace {

// Build-time knob: when the fused kernel's producer starts streaming the
// weight (0 at once, 1 once the activation loads have returned, 2 once the row
// scales are known, 3 once the codes are written).
// Build-time knob: weight boxes (k-blocks) per CTA prefetched into L2 before
// the wait for the previous kernel (in a stream of calls, the CTAs that start
// while the previous call's last CTAs finish get their first stages early).
#ifndef SQ_SMALL_EARLY_L2
#define SQ_SMALL_EARLY_L2 2
#endif
#ifndef SQ_SMALL_GATE
#define SQ_SMALL_GATE 0
#endif
// Build-time knob: 1 = the fused kernel's ranks exchange their slice maxima by
// asynchronous remote stores that complete bytes on the receiver's own
// mbarrier (st.async), 0 = plain remote loads after a cluster barrier.
#ifndef SQ_SMALL_XCHG_ASYNC
#define SQ_SMALL_XCHG_ASYNC 1
#endif

constexpr int kSmallThreads = 320;
constexpr int kSmallQuantThreads = 256;  // warps 2..9
constexpr int kSmallMaxStages = 8;
constexpr int kSmallRows = 2 * kBM;             // Wq rows per CTA (two MMA halves)
constexpr int kSmallABytes = kSmallRows * kBK;  // 256 rows of Wq x 128 bytes of K

struct SmallParams {
  int M, N, K;
  int nk;            // k-blocks of 128 bytes over K
  int kb_per_split;  // k-blocks per cluster rank
  int stages;
  int stage_bytes;   // Wq box (+ codes box when prequantised)
  const uint16_t* X;     // fused: bf16 activations [M][K]
  const float* s;        // fused: smoothing factor [K]
  const float* x_scale;  // prequantised scales [M]
  const float* w_scale;  // [N]
  const uint16_t* bias;  // [N] or null
  uint16_t* Y;           // [M][N]
  // shared-memory layout (bytes from the 1024-aligned base)
  int b_off, part_off, xs_off, red_off, wsb_off, bar_off, misc_off;
  unsigned long long timeout_ns;  // limit of every mbarrier wait
  int skip_first_load;            // test hook: the producer never loads its first stage
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }
// 4-byte store into a cluster peer's shared memory whose completion is
// counted (in bytes) on the peer's mbarrier at remote_bar; no fence, no
// release: the receiver sees the value once that barrier's phase completes.
__device__ __forceinline__ void st_async_f32(uint32_t remote_addr, float v, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(remote_addr),
               "r"(__float_as_uint(v)), "r"(remote_bar)
               : "memory");
}
// The same for 16 bytes (16-byte aligned destination).
__device__ __forceinline__ void st_async_v4(uint32_t remote_addr, uint4 v, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   remote_addr),
               "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(remote_bar)
               : "memory");
}
__device__ __forceinline__ uint32_t map_cluster_rank(uint32_t smem_addr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(smem_addr), "r"(rank));
  return d;
}
__device__ __forceinline__ uint4 ld_cluster_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// Byte offset of code (token m, local column c) in the B operand: k-block
// c/128 holds NT rows of 128 bytes in 8-row atoms of 1024 bytes, each row's
// 16-byte chunks permuted by XOR with (row % 8) -- the layout a TMA load with
// 128-byte swizzle produces and the descriptor's 128-byte swizzle mode reads.
template <int NT>
__device__ __forceinline__ uint32_t b_code_offset(int m, int c) {
  const int j = c >> 7, b = c & 127;
  return static_cast<uint32_t>(j * (NT * 128) + (m >> 3) * 1024 + (m & 7) * 128 + (((b >> 4) ^ (m & 7)) << 4) +
                               (b & 15));
}

#ifdef SQ_TRACE
// Optional phase timestamps (build with -DSQ_TRACE): per CTA, globaltimer at
// 0 start, 1 codes ready, 2 first stage consumed, 3 last MMA issued,
// 4 accumulators read, 5 after the reduction barrier, 6 end; fused: 7 pass-1
// loads returned, 8 slice maxima reduced, 9 after the exchange barrier,
// 10 scales formed, 11 codes written (warp 2, lane 0).
__device__ unsigned long long g_small_trace[1024][12];
#define SQ_TRACE_MARK(i)                                        \
  do {                                                          \
    const int cta_ = blockIdx.y * gridDim.x + blockIdx.x;       \
    if (cta_ < 1024) g_small_trace[cta_][i] = globaltimer_ns(); \
  } while (0)
#else
#define SQ_TRACE_MARK(i) \
  do {                   \
  } while (0)
#endif

// fl(x / s) for the 8 columns of one 16-byte bf16 vector, as four fp32 pairs
__device__ __forceinline__ void smooth8(const uint4 w, const f2x (&ns)[4], const f2x (&rs)[4], f2x (&t)[4]) {
  t[0] = f2_div_rn(f2_from_bf16x2(w.x), ns[0], rs[0]);
  t[1] = f2_div_rn(f2_from_bf16x2(w.y), ns[1], rs[1]);
  t[2] = f2_div_rn(f2_from_bf16x2(w.z), ns[2], rs[2]);
  t[3] = f2_div_rn(f2_from_bf16x2(w.w), ns[3], rs[3]);
}
// -s and RN(1/s) for the 8 columns of vector v, as fp32 pairs
__device__ __forceinline__ void load_s8(const float4* s4, int v, f2x (&ns)[4], f2x (&rs)[4]) {
  const float4 a = __ldg(s4 + 2 * v), b = __ldg(s4 + 2 * v + 1);
  ns[0] = f2_pack(-a.x, -a.y), ns[1] = f2_pack(-a.z, -a.w), ns[2] = f2_pack(-b.x, -b.y), ns[3] = f2_pack(-b.z, -b.w);
  rs[0] = f2_pack(__frcp_rn(a.x), __frcp_rn(a.y)), rs[1] = f2_pack(__frcp_rn(a.z), __frcp_rn(a.w));
  rs[2] = f2_pack(__frcp_rn(b.x), __frcp_rn(b.y)), rs[3] = f2_pack(__frcp_rn(b.z), __frcp_rn(b.w));
}

// Warp max of 16 per-lane values rm[0..15] by reduce-scatter: 16 shuffles
// instead of 16 x 5.  Afterwards lane l holds the max of value l >> 1.
__device__ __forceinline__ float warp_max16_scatter(const float (&rm)[16], int lane) {
  float a[8];
  const bool hi4 = lane & 16;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float give = hi4 ? rm[j] : rm[8 + j];
    const float keep = hi4 ? rm[8 + j] : rm[j];
    a[j] = fmaxf(keep, __shfl_xor_sync(0xFFFFFFFFu, give, 16));
  }
  float b[4];
  const bool hi3 = lane & 8;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float give = hi3 ? a[j] : a[4 + j];
    const float keep = hi3 ? a[4 + j] : a[j];
    b[j] = fmaxf(keep, __shfl_xor_sync(0xFFFFFFFFu, give, 8));
  }
  float c[2];
  const bool hi2 = lane & 4;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float give = hi2 ? b[j] : b[2 + j];
    const float keep = hi2 ? b[2 + j] : b[j];
    c[j] = fmaxf(keep, __shfl_xor_sync(0xFFFFFFFFu, give, 4));
  }
  const bool hi1 = lane & 2;
  float d = fmaxf(hi1 ? c[1] : c[0], __shfl_xor_sync(0xFFFFFFFFu, hi1 ? c[0] : c[1], 2));
  return fmaxf(d, __shfl_xor_sync(0xFFFFFFFFu, d, 1));
}

// Fused quantisation, pass 1, for one 16-byte vector v of the K-slice and the
// first R token rows held in registers: loads (s, then the R rows of X, all
// issued before any arithmetic), -s and RN(1/s), and the rows' max |fl(x/s)|.
template <int R>
__device__ __forceinline__ void fused_pass1(const uint4* X4, const float4* s4, int nvec, int v, bool has, int M,
                                            uint4 (&xr)[16], f2x (&ns)[4], f2x (&rs)[4], float (&rmax)[16]) {
  float4 sa = make_float4(1.f, 1.f, 1.f, 1.f), sb = sa;
  if (has) {
    sa = __ldg(s4 + 2 * v);
    sb = __ldg(s4 + 2 * v + 1);
  }
#pragma unroll
  for (int r = 0; r < R; ++r)
    xr[r] = (has && r < M) ? __ldg(X4 + static_cast<int64_t>(r) * nvec + v) : make_uint4(0u, 0u, 0u, 0u);
  ns[0] = f2_pack(-sa.x, -sa.y), ns[1] = f2_pack(-sa.z, -sa.w), ns[2] = f2_pack(-sb.x, -sb.y), ns[3] = f2_pack(-sb.z, -sb.w);
  rs[0] = f2_pack(__frcp_rn(sa.x), __frcp_rn(sa.y)), rs[1] = f2_pack(__frcp_rn(sa.z), __frcp_rn(sa.w));
  rs[2] = f2_pack(__frcp_rn(sb.x), __frcp_rn(sb.y)), rs[3] = f2_pack(__frcp_rn(sb.z), __frcp_rn(sb.w));
  // every one of the R rows, real or padding (zeros), with no branch, so the
  // rows' dependency chains interleave
#pragma unroll
  for (int r = 0; r < R; ++r) {
    f2x t[4];
    smooth8(xr[r], ns, rs, t);
#pragma unroll
    for (int e = 0; e < 4; ++e) rmax[r] = f2_absmax(rmax[r], t[e]);
  }
}

// Fused quantisation, pass 2: the codes of the first R rows of vector v into
// the swizzled B operand (padding rows get code 0; their accumulator columns
// are never read).
template <int NT, int R>
__device__ __forceinline__ void fused_pass2(const uint4 (&xr)[16], const f2x (&ns)[4], const f2x (&rs)[4],
                                            const float* xs_s, const float* rxs_s, uint8_t* bsm, int c) {
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const float sc = xs_s[r], rsc = rxs_s[r];
    const f2x nsc2 = f2_pack(-sc, -sc), rsc2 = f2_pack(rsc, rsc);
    f2x t[4];
    smooth8(xr[r], ns, rs, t);
#pragma unroll
    for (int e = 0; e < 4; ++e) t[e] = f2_round_codes(f2_div_rn(t[e], nsc2, rsc2));
    *reinterpret_cast<uint2*>(bsm + b_code_offset<NT>(r, c)) = pack8_codes(t[0], t[1], t[2], t[3]);
  }
}

template <int NT, bool kFused>
__global__ void __launch_bounds__(kSmallThreads, 1)
    gemm_small_m_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                        const SmallParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* bsm = smem + p.b_off;  // fused: the codes of this CTA's K-slice
  int32_t* part = reinterpret_cast<int32_t*>(smem + p.part_off);
  float* xs_s = reinterpret_cast<float*>(smem + p.xs_off);
  float* red = reinterpret_cast<float*>(smem + p.red_off);  // [8 warps][NT], then the slice maxima [NT]
  float* cmax = red + 8 * NT;
  float* rxs_s = red + 9 * NT;  // fused: RN(1 / x_scale) per token
  float* recv = red + 10 * NT;  // fused: [rank][NT] slice maxima received from every rank
  float* wsb = reinterpret_cast<float*>(smem + p.wsb_off);  // w_scale[256], bias[256] of this row block
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.bar_off);
  uint64_t* full = bars;
  uint64_t* empty = bars + kSmallMaxStages;
  uint64_t* b_ready = bars + 2 * kSmallMaxStages;
  uint64_t* acc_full = b_ready + 1;
  uint64_t* drain = b_ready + 2;
  uint64_t* x_in = b_ready + 3;  // fused: every quantisation warp holds its slice of X
  uint64_t* xchg = b_ready + 4;  // fused: the slice maxima of every rank have landed in recv
  uint64_t* red_bar = b_ready + 5;  // every rank's partial sums of the rows this rank reduces have landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + p.misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + p.misc_off + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int S = static_cast<int>(cluster_nctarank());
  const int rb = blockIdx.y;  // 256-row block of Wq (= 256 outputs)
  const int kb0 = static_cast<int>(rank) * p.kb_per_split;
  const int kb1 = min(p.nk, kb0 + p.kb_per_split);
  const int my_nkb = max(0, kb1 - kb0);
  const int stages = p.stages;
  // The four K=32 steps of a k-block write four separate TMEM accumulators
  // (NT columns each) per 128-row half; the epilogue adds them (exact int32).
  constexpr int kChains = 4;
  constexpr int kHalfCols = kChains * NT;
  constexpr uint32_t kTmemCols = 2 * kHalfCols;

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(b_ready, 1);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    mbar_init(x_in, kSmallQuantThreads / 32);
    if (kFused && SQ_SMALL_XCHG_ASYNC) {
      mbar_init(xchg, 1);
      mbar_arrive_expect_tx(xchg, static_cast<uint32_t>(S * NT * 4));
    }
    // the partial sums arrive by st.async: S senders x (256 / S) rows x the
    // token quads that hold real tokens x 16 bytes
    mbar_init(red_bar, 1);
    mbar_arrive_expect_tx(red_bar, static_cast<uint32_t>(kSmallRows * ((p.M + 3) / 4) * 16));
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  // A cluster phase that says every rank's barriers are initialised: arrived
  // now, waited for just before a thread's first remote store (the fused
  // kernel's exchange, or the partial sums), or at the end by the warps that
  // store nothing remotely.  (The fused kernel with the exchange by cluster
  // barrier has its quantisation warps take that barrier instead.)
  if (!kFused || SQ_SMALL_XCHG_ASYNC) cluster_arrive_relaxed();
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    if (!kFused) tma_prefetch_desc(&tmX);
    // the first weight boxes of this CTA into L2 while the previous kernel may
    // still run (a hint only: writes land in L2, so the loads after the wait
    // read current data)
    for (int kb = kb0; kb < min(kb1, kb0 + SQ_SMALL_EARLY_L2); ++kb)
      tma_prefetch_l2_2d(&tmW, kb * kBK, rb * kSmallRows);
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
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x == 0) SQ_TRACE_MARK(0);
  // fused: warps 0 and 1 take no part in the mid-kernel exchange of row maxima;
  // they arrive now and complete that phase at the end
  if (kFused && !SQ_SMALL_XCHG_ASYNC && warp < 2) cluster_arrive_relaxed();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && my_nkb > 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      // fused: start the weight stream only once the activation loads have
      // returned; issued behind a full ring of weight boxes they would wait for
      // the whole ring to drain from HBM, and the MMAs wait for their codes
      if (kFused && SQ_SMALL_GATE > 0 &&
          (*abort_flag || !mbar_wait_bounded(SQ_SMALL_GATE == 3 ? b_ready : x_in, 0, p.timeout_ns))) {
        if (!*abort_flag) flag_timeout(abort_flag);
        ok = false;
      }
      for (int kb = kb0; ok && kb < kb1; ++kb) {
        if (*abort_flag || !mbar_wait_bounded(&empty[stage], phase ^ 1u, p.timeout_ns)) {
          if (!*abort_flag) flag_timeout(abort_flag);
          ok = false;
          break;
        }
        uint8_t* dst = smem + stage * p.stage_bytes;
        if (!(p.skip_first_load && kb == kb0)) {  // test hook: the first stage never fills
          mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(p.stage_bytes));
          tma_load_2d(dst, &tmW, kb * kBK, rb * kSmallRows, &full[stage]);
          if (!kFused) tma_load_2d(dst + kSmallABytes, &tmX, kb * kBK, 0, &full[stage]);
        }
        ++issued;
        if (++stage == stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {  // drain the copies in flight (the last min(issued, stages) loads; a skipped one never completes)
        for (int i = 0; i < min(issued, stages); ++i) {
          const int q = issued - 1 - i;
          if (p.skip_first_load && q == 0) continue;
          (void)mbar_wait_bounded(&full[q % stages], static_cast<uint32_t>((q / stages) & 1), p.timeout_ns);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kBM, NT);
      bool ok = true;
      if (kFused) {
        ok = !*abort_flag && mbar_wait_bounded(b_ready, 0, p.timeout_ns);
        if (!ok && !*abort_flag) flag_timeout(abort_flag);
      }
      SQ_TRACE_MARK(1);
      int stage = 0;
      uint32_t phase = 0;
      for (int j = 0; ok && j < my_nkb; ++j) {
        if (*abort_flag || !mbar_wait_bounded(&full[stage], phase, p.timeout_ns)) {
          if (!*abort_flag) flag_timeout(abort_flag);
          ok = false;
          break;
        }
        tc_fence_after();
        if (j == 0) SQ_TRACE_MARK(2);
        const uint32_t st = smem_u32(smem + stage * p.stage_bytes);
        const uint64_t bdesc = kFused ? smem_desc_k_sw128(smem_u32(bsm + j * (NT * kBK)))
                                      : smem_desc_k_sw128(st + kSmallABytes);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint64_t adesc = smem_desc_k_sw128(st + h * (kBM * kBK));
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk)
            mma_i8(tmem_base + static_cast<uint32_t>(h * kHalfCols + kk * NT), adesc + static_cast<uint64_t>(kk * 2),
                   bdesc + static_cast<uint64_t>(kk * 2), idesc, j != 0 ? 1u : 0u);
        }
        mma_commit(&empty[stage]);
        if (++stage == stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      SQ_TRACE_MARK(3);
      if (ok) mma_commit(acc_full);
      mma_commit(drain);
      (void)mbar_wait_bounded(drain, 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------- quantisation (warps 2..9)
    const int qt = threadIdx.x - 64;
    const int qw = qt >> 5;
    const int M = p.M;
    if (kFused) {
      const int K = p.K;
      const int nvec = K >> 3;
      const int v_lo = kb0 * (kBK / 8);
      const int v_hi = min(nvec, kb1 * (kBK / 8));
      const uint4* X4 = reinterpret_cast<const uint4*>(p.X);
      const float4* s4 = reinterpret_cast<const float4*>(p.s);
      // With at most one 16-byte vector of the K-slice per thread and at most
      // 16 tokens, each thread keeps its X vectors in registers from pass 1 to
      // pass 2: all of its global loads are issued at once, before any
      // arithmetic, and nothing is read twice.
      constexpr int kRegRows = 16;
      const bool in_regs = NT == kRegRows && v_hi - v_lo <= kSmallQuantThreads;
      uint4 xr[kRegRows];
      f2x rns[4], rrs[4];
      float rmax[NT];
#pragma unroll
      for (int m = 0; m < NT; ++m) rmax[m] = 0.0f;
      if (in_regs) {
        float rm16[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) rm16[m] = 0.0f;
        const int v = v_lo + qt;
        const bool has = v < v_hi;
        if (M <= 8)
          fused_pass1<8>(X4, s4, nvec, v, has, M, xr, rns, rrs, rm16);
        else
          fused_pass1<16>(X4, s4, nvec, v, has, M, xr, rns, rrs, rm16);
        __syncwarp();
        if (SQ_SMALL_GATE == 1 && lane == 0) mbar_arrive(x_in);  // this warp's pass-1 loads have all returned
        if (warp == 2 && lane == 0) SQ_TRACE_MARK(7);
        const float wm = warp_max16_scatter(rm16, lane);
        if ((lane & 1) == 0) red[qw * NT + (lane >> 1)] = wm;
      }
      // pass 1: max of |fl(X / s)| over this CTA's K-slice, eight rows at a time
      // with all of a group's loads issued before any arithmetic
      for (int v = v_lo + qt; !in_regs && v < v_hi; v += kSmallQuantThreads) {
        f2x ns[4], rs[4];
        load_s8(s4, v, ns, rs);
#pragma unroll
        for (int g = 0; g < NT; g += 8) {
          if (g < M) {
            uint4 w[8];
#pragma unroll
            for (int r = 0; r < 8; ++r)
              w[r] = (g + r < M) ? __ldg(X4 + static_cast<int64_t>(g + r) * nvec + v) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int r = 0; r < 8; ++r) {
              f2x t[4];
              smooth8(w[r], ns, rs, t);
#pragma unroll
              for (int e = 0; e < 4; ++e) rmax[g + r] = f2_absmax(rmax[g + r], t[e]);
            }
          }
        }
      }
      if (!in_regs) {
        __syncwarp();
        if (SQ_SMALL_GATE == 1 && lane == 0) mbar_arrive(x_in);  // this warp's pass-1 loads have all returned
#pragma unroll
        for (int m = 0; m < NT; ++m) {
          const float r = warp_max(rmax[m]);
          if (lane == 0) red[qw * NT + m] = r;
        }
      }
      named_bar_sync(1, kSmallQuantThreads);
      if (qt < NT) {
        float mx = 0.0f;
#pragma unroll
        for (int w = 0; w < kSmallQuantThreads / 32; ++w) mx = fmaxf(mx, red[w * NT + qt]);
        cmax[qt] = mx;
      }
      if (warp == 2 && lane == 0) SQ_TRACE_MARK(8);
      // exchange of the slice maxima across the cluster
      if (SQ_SMALL_XCHG_ASYNC) {
        cluster_wait();  // every rank's exchange barrier is initialised
        if (qt < NT) {
          const uint32_t slot = smem_u32(recv + static_cast<int>(rank) * NT + qt);
          const uint32_t bar = smem_u32(xchg);
          for (int r = 0; r < S; ++r)
            st_async_f32(map_cluster_rank(slot, static_cast<uint32_t>(r)), cmax[qt],
                         map_cluster_rank(bar, static_cast<uint32_t>(r)));
        }
        if (!mbar_wait_bounded(xchg, 0, p.timeout_ns) && lane == 0) flag_timeout(abort_flag);
      } else {  // warps 0, 1 arrived early
        asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
      }
      if (warp == 2 && lane == 0) SQ_TRACE_MARK(9);
      if (SQ_SMALL_XCHG_ASYNC && qt < NT) {
        float mx = 0.0f;
        for (int r = 0; r < S; ++r) mx = fmaxf(mx, recv[r * NT + qt]);
        const float sc = __fdiv_rn(fmaxf(mx, kClampFloor), kQmax);
        xs_s[qt] = sc;
        rxs_s[qt] = __frcp_rn(sc);
      }
      if (!SQ_SMALL_XCHG_ASYNC && qt < NT) {
        // all S remote loads are issued before the first use of any of them
        const uint32_t a = smem_u32(cmax + qt);
        float part_max[8];
#pragma unroll
        for (int r = 0; r < 8; ++r)
          if (r < S) part_max[r] = ld_cluster_f32(map_cluster_rank(a, static_cast<uint32_t>(r)));
        float mx = 0.0f;
#pragma unroll
        for (int r = 0; r < 8; ++r)
          if (r < S) mx = fmaxf(mx, part_max[r]);
        const float sc = __fdiv_rn(fmaxf(mx, kClampFloor), kQmax);
        xs_s[qt] = sc;
        rxs_s[qt] = __frcp_rn(sc);
      }
      named_bar_sync(1, kSmallQuantThreads);
      if (SQ_SMALL_GATE == 2 && lane == 0) mbar_arrive(x_in);  // the row scales are known
      if (warp == 2 && lane == 0) SQ_TRACE_MARK(10);
      // pass 2: the codes of this CTA's K-slice, into the swizzled B operand
      if (in_regs && v_lo + qt < v_hi) {
        const int c = (v_lo + qt) * 8 - kb0 * kBK;
        if (M <= 8)
          fused_pass2<NT, 8>(xr, rns, rrs, xs_s, rxs_s, bsm, c);
        else
          fused_pass2<NT, 16>(xr, rns, rrs, xs_s, rxs_s, bsm, c);
      }
      for (int v = v_lo + qt; !in_regs && v < v_hi; v += kSmallQuantThreads) {
        f2x ns[4], rs[4];
        load_s8(s4, v, ns, rs);
        const int c = v * 8 - kb0 * kBK;
#pragma unroll
        for (int g = 0; g < NT; g += 8) {
          if (g < M) {
            uint4 w[8];
#pragma unroll
            for (int r = 0; r < 8; ++r)
              w[r] = (g + r < M) ? __ldg(X4 + static_cast<int64_t>(g + r) * nvec + v) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int r = 0; r < 8; ++r) {
              if (g + r < M) {
                const float sc = xs_s[g + r];
                const float rsc = rxs_s[g + r];
                const f2x nsc2 = f2_pack(-sc, -sc), rsc2 = f2_pack(rsc, rsc);
                f2x t[4];
                smooth8(w[r], ns, rs, t);
#pragma unroll
                for (int e = 0; e < 4; ++e) t[e] = f2_round_codes(f2_div_rn(t[e], nsc2, rsc2));
                *reinterpret_cast<uint2*>(bsm + b_code_offset<NT>(g + r, c)) = pack8_codes(t[0], t[1], t[2], t[3]);
              }
            }
          }
        }
      }
      if (warp == 2 && lane == 0) SQ_TRACE_MARK(11);
      // make the generic-proxy smem writes visible to the tensor core, then release the MMA warp
      fence_proxy_async_smem();
      named_bar_sync(1, kSmallQuantThreads);
      if (qt == 0) mbar_arrive(b_ready);
    } else {
      if (qt < NT) xs_s[qt] = (qt < M) ? __ldg(p.x_scale + qt) : 0.0f;
    }
    // stage this row block's w_scale and bias for the reduction (off the critical path)
    {
      const int n = rb * kSmallRows + qt;  // one row per quantisation thread
      wsb[qt] = (n < p.N) ? __ldg(p.w_scale + n) : 0.0f;
      wsb[kSmallRows + qt] =
          (p.bias != nullptr && n < p.N) ? __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + n)) << 16) : 0.0f;
    }

    // ------------------------------------------------- accumulators to shared memory (warps 2..5)
    if (warp < 6) {
      const int quarter = warp & 3;
      if (!kFused) cluster_wait();  // every rank's red_bar is initialised
      bool have = my_nkb > 0;
      if (have) {
        const bool mine = !*abort_flag && mbar_wait_bounded(acc_full, 0, p.timeout_ns);
        have = __all_sync(0xFFFFFFFFu, mine);
        if (!have && lane == 0 && !*abort_flag) flag_timeout(abort_flag);
      }
      if (have) tc_fence_after();
      if (warp == 2 && lane == 0) SQ_TRACE_MARK(4);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int n_local = h * kBM + quarter * 32 + lane;
        uint32_t acc[NT];
#pragma unroll
        for (int i = 0; i < NT; ++i) acc[i] = 0u;
        if (have) {
          const uint32_t taddr =
              tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(h * kHalfCols);
#pragma unroll
          for (int c = 0; c < kHalfCols; c += 32) {
            uint32_t r32[32];
            tmem_ld_32cols(taddr + static_cast<uint32_t>(c), r32);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[(c + i) % NT] += r32[i];
          }
        }
        // push the row's partial sums to the rank that reduces this row, into
        // that rank's slot for this sender, by st.async: the bytes count on
        // the owner's red_bar, which the owner waits for (no cluster barrier)
        const int rpr = kSmallRows / S;
        const int owner = n_local / rpr;
        const uint32_t dst = map_cluster_rank(
            smem_u32(part + (static_cast<int>(rank) * rpr + (n_local - owner * rpr)) * NT), static_cast<uint32_t>(owner));
        const uint32_t dst_bar = map_cluster_rank(smem_u32(red_bar), static_cast<uint32_t>(owner));
        const int nq = (p.M + 3) / 4;  // token quads that hold real tokens
#pragma unroll
        for (int i = 0; i < NT / 4; ++i)
          if (i < nq)
            st_async_v4(dst + 16u * i, make_uint4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]), dst_bar);
      }
    }
  }

  // ------------------------------------------- split-K reduction over the cluster
  // Rank q reduces rows [q*256/S, (q+1)*256/S): every rank pushes its partial
  // sums of those rows into rank q's shared memory (one slot per sender) with
  // st.async, counted on rank q's red_bar; once its phase completes the S
  // partials of a row are local loads; the sum is dequantised and stored.
  // Token quads past M are skipped.  A rank leaves only after every byte
  // addressed to it has landed, and no rank reads another's shared memory,
  // so no cluster barrier is needed at the end.
  tc_fence_before();
  __syncthreads();  // w_scale, bias and the token scales staged above
  // completes the start phase for the warps that stored nothing remotely
  if (kFused ? warp < 2 : (warp < 2 || warp >= 6)) cluster_wait();
  if (warp >= 2) {
    if (!mbar_wait_bounded(red_bar, 0, p.timeout_ns) && lane == 0) flag_timeout(abort_flag);
  }
  if (threadIdx.x == 64) SQ_TRACE_MARK(5);
  if (warp >= 2) {
    const int rpr = kSmallRows / S;
    const int r_lo = static_cast<int>(rank) * rpr;
    const int items = rpr * ((p.M + 3) / 4);
    for (int it = threadIdx.x - 64; it < items; it += kSmallQuantThreads) {
      // consecutive threads take consecutive rows (outputs n) of one token
      // quad, so a warp's Y stores for a token cover one contiguous run
      const int lr = it % rpr;
      const int q4 = it / rpr;
      uint4 v[8];
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < S) v[r] = *reinterpret_cast<const uint4*>(part + (r * rpr + lr) * NT + q4 * 4);
      int32_t acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < S) {
          acc[0] += static_cast<int32_t>(v[r].x), acc[1] += static_cast<int32_t>(v[r].y);
          acc[2] += static_cast<int32_t>(v[r].z), acc[3] += static_cast<int32_t>(v[r].w);
        }
      const int n_local = r_lo + lr;
      const int n = rb * kSmallRows + n_local;
      if (n < p.N) {
        const float ws = wsb[n_local];
        const float b = wsb[kSmallRows + n_local];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int m = q4 * 4 + j;
          if (m < p.M) {
            const float y = __fmaf_rn(__int2float_rn(acc[j]), __fmul_rn(xs_s[m], ws), b);
            p.Y[static_cast<int64_t>(m) * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) SQ_TRACE_MARK(6);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace
}  // namespace sq
