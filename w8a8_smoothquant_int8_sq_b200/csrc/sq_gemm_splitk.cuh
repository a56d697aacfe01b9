// sq_gemm_splitk.cuh -- the int8 GEMM for problems with fewer 128 x 256 output
// tiles than SMs: each tile's K is split over a thread-block cluster of S CTAs
// and the partial accumulators are summed through distributed shared memory.
// Included by sq_gemm.cu (one translation unit with the persistent kernel).
//
// Page: "w8a8_smoothquant.py -- W8A8 com SmoothQuant e alpha APRENDIVEL (V5)",
// SmoothQuantW8A8.forward: acc = Xq Wq^T (INT8 x INT8 -> INT32), then
// Y = bf16(acc * x_scale[m] * w_scale[n] + bias[n]).
//
// A tcgen05.mma kind::i8 with M = 128 takes about the same time for N = 128 as
// for N = 256, so output tiles are always 128 x 256; when there are fewer such
// tiles than SMs the K dimension is split instead of the tile shrunk.
//   warp 0      TMA producer: 128 x 128-byte Xq and 256 x 128-byte Wq slices of
//               this rank's K range into a 4-stage ring.
//   warp 1      TMEM owner (256 columns) and MMA issuer.
//   warps 2..5  stage the tile's scales and bias, then push the int32
//               accumulator rows from TMEM to the rank that owns them (rank q
//               owns rows [q*128/S, (q+1)*128/S)): remote rows with
//               distributed-shared-memory stores into the owner's (now idle)
//               ring memory, own rows with local stores.
//   all warps   after one cluster barrier, each rank sums the S copies of its
//               rows from its own shared memory, dequantises and stores.
// Every mbarrier wait is bounded; every thread reaches the cluster barrier.

namespace sq {
namespace {

constexpr int kSkBN = 256;
constexpr int kSkStages = 4;
constexpr int kSkThreads = 192;
constexpr int kSkStageBytes = kBM * kBK + kSkBN * kBK;  // 48 KB
constexpr int kSkRingBytes = kSkStages * kSkStageBytes;
// shared memory after the ring: w_scale[256], bias[256], x_scale[128], barriers, misc
constexpr int kSkWsOffset = kSkRingBytes;
constexpr int kSkBiasOffset = kSkWsOffset + kSkBN * 4;
constexpr int kSkXsOffset = kSkBiasOffset + kSkBN * 4;
constexpr int kSkBarOffset = kSkXsOffset + kBM * 4;
constexpr int kSkMiscOffset = kSkBarOffset + (2 * kSkStages + 2) * 8;
constexpr int kSkAlloc = kSkMiscOffset + 16 + 1024;
static_assert(kBM * kSkBN * 4 <= kSkRingBytes, "the partial tile reuses the ring");

struct SkParams {
  int M, N, K;
  int num_m_blocks;
  int nk, kb_per_split;
  const float* x_scale;
  const float* w_scale;
  const uint16_t* bias;
  void* out;  // bf16 Y or int32 acc, [M][N]
  int vec_ok;
};

// Byte offset of the 16-byte unit u (4 int32 columns) of row slot r in a
// receive buffer: rows of 1 KB, units permuted by XOR with (r % 8) so that
// eight lanes writing the same unit of eight rows hit eight bank groups.
__device__ __forceinline__ uint32_t sk_part_offset(int r, int u) {
  return static_cast<uint32_t>(r * (kSkBN * 4) + ((u ^ (r & 7)) << 4));
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

#ifdef SQ_TRACE
// Optional phase timestamps (build with -DSQ_TRACE): per CTA, globaltimer at
// 0 start, 1 first stage consumed, 2 last MMA issued, 3 accumulator ready,
// 4 after the first cluster barrier, 5 after the pushes' barrier, 6 end.
__device__ unsigned long long g_sk_trace[1024][8];
#define SQ_SK_MARK(i)                                             \
  do {                                                            \
    const int cta_ = blockIdx.y * gridDim.x + blockIdx.x;         \
    if (cta_ < 1024) g_sk_trace[cta_][i] = globaltimer_ns();      \
  } while (0)
#else
#define SQ_SK_MARK(i) \
  do {                \
  } while (0)
#endif

template <int EPI>
__global__ void __launch_bounds__(kSkThreads, 1)
    gemm_i8_splitk_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const SkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* ws_s = reinterpret_cast<float*>(smem + kSkWsOffset);
  float* b_s = reinterpret_cast<float*>(smem + kSkBiasOffset);
  float* xs_s = reinterpret_cast<float*>(smem + kSkXsOffset);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kSkBarOffset);
  uint64_t* empty = full + kSkStages;
  uint64_t* acc_full = empty + kSkStages;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSkMiscOffset);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSkMiscOffset + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int S = static_cast<int>(cluster_nctarank());
  const int tile = blockIdx.y;
  const int m_blk = tile % p.num_m_blocks;
  const int n_blk = tile / p.num_m_blocks;
  const int kb0 = static_cast<int>(rank) * p.kb_per_split;
  const int kb1 = min(p.nk, kb0 + p.kb_per_split);
  const int my_nkb = max(0, kb1 - kb0);
  constexpr uint32_t kTmemCols = kSkBN;
  bool have_acc = false;  // epilogue warps: the accumulator is complete and valid

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSkStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
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
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x == 0) SQ_SK_MARK(0);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && my_nkb > 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (*abort_flag || !mbar_wait_bounded(&empty[stage], phase ^ 1u, kWaitTimeoutNs)) {
          if (!*abort_flag) flag_timeout(abort_flag);
          ok = false;
          break;
        }
        uint8_t* sa = smem + stage * kSkStageBytes;
        mbar_arrive_expect_tx(&full[stage], kSkStageBytes);
        tma_load_2d(sa, &tmA, kb * kBK, m_blk * kBM, &full[stage]);
        tma_load_2d(sa + kBM * kBK, &tmB, kb * kBK, n_blk * kSkBN, &full[stage]);
        ++issued;
        if (++stage == kSkStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {  // drain the copies in flight
        for (int i = 0; i < min(issued, kSkStages); ++i) {
          const int q = issued - 1 - i;
          (void)mbar_wait_bounded(&full[q % kSkStages], static_cast<uint32_t>((q / kSkStages) & 1), kWaitTimeoutNs);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kBM, kSkBN);
      bool ok = true;
      int stage = 0;
      uint32_t phase = 0;
      for (int j = 0; j < my_nkb; ++j) {
        if (*abort_flag || !mbar_wait_bounded(&full[stage], phase, kWaitTimeoutNs)) {
          if (!*abort_flag) flag_timeout(abort_flag);
          ok = false;
          break;
        }
        tc_fence_after();
        if (j == 0) SQ_SK_MARK(1);
        const uint32_t sa = smem_u32(smem + stage * kSkStageBytes);
        const uint64_t adesc = smem_desc_k_sw128(sa);
        const uint64_t bdesc = smem_desc_k_sw128(sa + kBM * kBK);
#pragma unroll
        for (int kk = 0; kk < kBK / kUmmaK; ++kk)
          mma_i8(tmem_base, adesc + static_cast<uint64_t>(kk * 2), bdesc + static_cast<uint64_t>(kk * 2), idesc,
                 (j | kk) != 0 ? 1u : 0u);
        mma_commit(&empty[stage]);
        if (++stage == kSkStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      SQ_SK_MARK(2);
      if (ok) mma_commit(acc_full);
      mma_commit(drain);
      (void)mbar_wait_bounded(drain, 0, kWaitTimeoutNs);
    }
  } else {
    // ------------------------------------------- stage scales, wait for the accumulator
    const int et = threadIdx.x - 64;  // 0..127
    if (EPI == 0) {
      const int nb = n_blk * kSkBN;
      for (int i = et; i < kSkBN; i += 128) {
        const int n = nb + i;
        ws_s[i] = n < p.N ? __ldg(p.w_scale + n) : 0.0f;
        b_s[i] = (p.bias != nullptr && n < p.N) ? __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + n)) << 16)
                                                : 0.0f;
      }
      const int m = m_blk * kBM + et;
      xs_s[et] = m < p.M ? __ldg(p.x_scale + m) : 0.0f;
    }
    bool have = my_nkb > 0;
    if (have) {
      const bool mine = !*abort_flag && mbar_wait_bounded(acc_full, 0, kWaitTimeoutNs);
      have = __all_sync(0xFFFFFFFFu, mine);
      if (!have && lane == 0 && !*abort_flag) flag_timeout(abort_flag);
    }
    have_acc = have;
    if (warp == 2 && lane == 0) SQ_SK_MARK(3);
  }

  // ------------------------------------------- push the partial rows to their owners
  // After the first cluster barrier every CTA's MMAs are complete (its epilogue
  // warps saw acc_full and its MMA thread drained), so every ring is idle and
  // can receive rows.  Rank q owns rows [q*128/S, (q+1)*128/S); its ring holds
  // slot (sender, local row) = sender * 128/S + local row for every sender.
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (threadIdx.x == 0) SQ_SK_MARK(4);
  if (warp >= 2) {
    tc_fence_after();
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // tile row = TMEM lane
    const int rows_per_rank = kBM / S;
    const int owner = r / rows_per_rank;
    const int slot = static_cast<int>(rank) * rows_per_rank + (r - owner * rows_per_rank);
    const uint32_t dst_base = map_cluster_rank(smem_u32(smem), static_cast<uint32_t>(owner));
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
    for (int c0 = 0; c0 < kSkBN; c0 += 32) {
      uint32_t v[32];
      if (have_acc) {
        tmem_ld_32cols(taddr + static_cast<uint32_t>(c0), v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0u;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        st_cluster_v4(dst_base + sk_part_offset(slot, c0 / 4 + u),
                      make_uint4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]));
    }
  }

  // ------------------------------------------- split-K reduction over the cluster
  cluster_sync_all();  // all pushes have landed
  if (threadIdx.x == 0) SQ_SK_MARK(5);
  {
    const int rows_per_rank = kBM / S;
    const int r_lo = static_cast<int>(rank) * rows_per_rank;
    const int items = rows_per_rank * (kSkBN / 4);  // 16-byte units of 4 columns
    for (int it = threadIdx.x; it < items; it += kSkThreads) {
      const int rr = it / (kSkBN / 4);
      const int u = it % (kSkBN / 4);
      int32_t acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (q < S) {
          const uint4 v = *reinterpret_cast<const uint4*>(smem + sk_part_offset(q * rows_per_rank + rr, u));
          acc[0] += static_cast<int32_t>(v.x), acc[1] += static_cast<int32_t>(v.y);
          acc[2] += static_cast<int32_t>(v.z), acc[3] += static_cast<int32_t>(v.w);
        }
      const int r = r_lo + rr;
      const int m = m_blk * kBM + r;
      const int n0 = n_blk * kSkBN + 4 * u;
      if (m < p.M && n0 < p.N) {
        if (EPI == 0) {
          const float xs = xs_s[r];
          float y[4];
#pragma unroll
          for (int j = 0; j < 4; ++j)
            y[j] = __fmaf_rn(__int2float_rn(acc[j]), __fmul_rn(xs, ws_s[4 * u + j]), b_s[4 * u + j]);
          uint16_t* yrow = static_cast<uint16_t*>(p.out) + static_cast<int64_t>(m) * p.N + n0;
          if (n0 + 4 <= p.N && p.vec_ok) {
            *reinterpret_cast<uint2*>(yrow) = make_uint2(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]));
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              if (n0 + j < p.N) yrow[j] = __bfloat16_as_ushort(__float2bfloat16_rn(y[j]));
          }
        } else {
          int32_t* arow = static_cast<int32_t*>(p.out) + static_cast<int64_t>(m) * p.N + n0;
          if (n0 + 4 <= p.N && p.vec_ok) {
            *reinterpret_cast<int4*>(arow) = make_int4(acc[0], acc[1], acc[2], acc[3]);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              if (n0 + j < p.N) arow[j] = acc[j];
          }
        }
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) SQ_SK_MARK(6);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace
}  // namespace sq
