// sq_gemm_splitk.cuh -- the int8 GEMM for problems with fewer 128 x 256 output
// tiles than SMs: each tile's K is split between the two CTAs of a cluster and
// the partial accumulators are exchanged through the caller's workspace (L2).
// Included by sq_gemm.cu (one translation unit with the persistent kernel).
//
// Page: "w8a8_smoothquant.py -- W8A8 com SmoothQuant e alpha APRENDIVEL (V5)",
// SmoothQuantW8A8.forward: acc = Xq Wq^T (INT8 x INT8 -> INT32), then
// Y = bf16(acc * x_scale[m] * w_scale[n] + bias[n]).
//
// A tcgen05.mma kind::i8 with M = 128 takes about the same time for N = 128 as
// for N = 256, so output tiles are always 128 x 256; when there are fewer such
// tiles than SMs the K dimension is split in two instead of the tile shrunk.
//   warp 0      TMA producer: 128 x 128-byte Xq and 256 x 128-byte Wq slices of
//               this CTA's half of K into a 4-stage ring.
//   warp 1      TMEM owner (256 columns) and MMA issuer.
//   warps 2..5  epilogue.  Rank q of the pair owns output columns
//               [128q, 128q + 128) of the tile.  Each CTA stores the partial
//               sums of the columns the other rank owns (128 x 128 int32,
//               64 KB) into its slot of the workspace; after one cluster
//               barrier (release / acquire at cluster scope) one thread brings
//               the peer's partial of its own columns into the idle ring with a
//               single 64 KB bulk copy (L2 hits), and the warps add their own
//               sums from TMEM, dequantise and store.  Distributed shared
//               memory was measured slower for this exchange on B200, and
//               per-thread loads of the partial paid one L2 latency per chunk.
// Workspace slot layout: [tile][sender rank][32-column chunk c][16-byte unit
// u][row r], so the 32 lanes of a warp (32 consecutive rows) store or load one
// contiguous 512-byte run per instruction.
// Every mbarrier wait is bounded; every thread reaches the cluster barrier.

namespace sq {
namespace {

constexpr int kSkBN = 256;
constexpr int kSkHalf = kSkBN / 2;      // output columns owned by each rank
constexpr int kSkStages = 4;
constexpr int kSkThreads = 192;
constexpr int kSkStageBytes = kBM * kBK + kSkBN * kBK;  // 48 KB
constexpr int kSkRingBytes = kSkStages * kSkStageBytes;
constexpr int kSkChunkCols = 32;                          // columns per tcgen05.ld
constexpr int kSkChunks = kSkHalf / kSkChunkCols;         // 4
constexpr size_t kSkSlotBytes = static_cast<size_t>(kBM) * kSkHalf * 4;  // 64 KB per (tile, sender)
// ring reuse after the main loop: [0, 64 KB) the peer's partial, then the
// output boxes (4 warps x 4 chunks x 32 rows x 64 bytes = 32 KB)
constexpr int kSkYOffset = static_cast<int>(kSkSlotBytes);
static_assert(kSkYOffset + 4 * 4 * 32 * 64 <= kSkRingBytes, "the output boxes reuse the ring");
// shared memory after the ring: w_scale[128], bias[128], x_scale[128] of the owned half, barriers, misc
constexpr int kSkWsOffset = kSkRingBytes;
constexpr int kSkBiasOffset = kSkWsOffset + kSkHalf * 4;
constexpr int kSkXsOffset = kSkBiasOffset + kSkHalf * 4;
constexpr int kSkBarOffset = kSkXsOffset + kBM * 4;
constexpr int kSkNumBars = 2 * kSkStages + 3;  // full, empty, acc_full, drain, peer partial
constexpr int kSkMiscOffset = kSkBarOffset + kSkNumBars * 8;
constexpr int kSkAlloc = kSkMiscOffset + 16 + 1024;

struct SkParams {
  int M, N, K;
  int num_m_blocks;
  int nk, kb_per_split;
  const float* x_scale;
  const float* w_scale;
  const uint16_t* bias;
  uint16_t* out;  // bf16 Y [M][N]
  uint4* part;    // workspace: 2 slots of kSkSlotBytes per tile
  int vec_ok;
  int tma_store;        // Y written by TMA stores (tmY valid)
  int skip_first_load;  // test hook: never load the first stage
  unsigned long long timeout_ns;
};

// 16-byte unit index of (chunk c, unit u, row r) within a slot
__device__ __forceinline__ int sk_unit(int c, int u, int r) { return (c * 8 + u) * kBM + r; }

#ifdef SQ_TRACE
// Optional phase timestamps (build with -DSQ_TRACE): per CTA, globaltimer at
// 0 past the wait for the previous kernel, 1 first stage consumed, 2 last MMA
// issued, 3 accumulator ready, 4 partial stored, 5 after the cluster barrier,
// 6 stores done, 7 end.
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

__global__ void __launch_bounds__(kSkThreads, 1)
    gemm_i8_splitk_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmY, const SkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* ws_s = reinterpret_cast<float*>(smem + kSkWsOffset);
  float* b_s = reinterpret_cast<float*>(smem + kSkBiasOffset);
  float* xs_s = reinterpret_cast<float*>(smem + kSkXsOffset);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kSkBarOffset);
  uint64_t* empty = full + kSkStages;
  uint64_t* acc_full = empty + kSkStages;
  uint64_t* drain = acc_full + 1;
  uint64_t* part_full = drain + 1;  // the peer's partial has landed in the ring
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSkMiscOffset);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSkMiscOffset + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
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
    mbar_init(part_full, 1);
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
        if (*abort_flag || !mbar_wait_bounded(&empty[stage], phase ^ 1u, p.timeout_ns)) {
          if (!*abort_flag) flag_timeout(abort_flag);
          ok = false;
          break;
        }
        uint8_t* sa = smem + stage * kSkStageBytes;
        if (!(p.skip_first_load && kb == kb0)) {
          mbar_arrive_expect_tx(&full[stage], kSkStageBytes);
          tma_load_2d(sa, &tmA, kb * kBK, m_blk * kBM, &full[stage]);
          tma_load_2d(sa + kBM * kBK, &tmB, kb * kBK, n_blk * kSkBN, &full[stage]);
        }
        ++issued;
        if (++stage == kSkStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {  // drain the copies in flight (a skipped first load never completes: no wait for it)
        for (int i = 0; i < min(issued, kSkStages); ++i) {
          const int q = issued - 1 - i;
          if (p.skip_first_load && q == 0) continue;
          (void)mbar_wait_bounded(&full[q % kSkStages], static_cast<uint32_t>((q / kSkStages) & 1), p.timeout_ns);
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
        if (*abort_flag || !mbar_wait_bounded(&full[stage], phase, p.timeout_ns)) {
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
      (void)mbar_wait_bounded(drain, 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------- stage scales, wait for the accumulator
    const int et = threadIdx.x - 64;  // 0..127
    const int n = n_blk * kSkBN + static_cast<int>(rank) * kSkHalf + et;
    ws_s[et] = n < p.N ? __ldg(p.w_scale + n) : 0.0f;
    b_s[et] = (p.bias != nullptr && n < p.N) ? __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + n)) << 16)
                                             : 0.0f;
    const int m = m_blk * kBM + et;
    xs_s[et] = m < p.M ? __ldg(p.x_scale + m) : 0.0f;
    bool have = my_nkb > 0;
    if (have) {
      const bool mine = !*abort_flag && mbar_wait_bounded(acc_full, 0, p.timeout_ns);
      have = __all_sync(0xFFFFFFFFu, mine);
      if (!have && lane == 0 && !*abort_flag) flag_timeout(abort_flag);
    }
    have_acc = have;
    if (warp == 2 && lane == 0) SQ_SK_MARK(3);
    // ------------------------------------------- store the partial sums of the peer's columns
    tc_fence_after();
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // tile row = TMEM lane
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    uint4* mine_slot = p.part + (static_cast<size_t>(tile) * 2 + rank) * (kSkSlotBytes / 16);
#pragma unroll 1
    for (int c = 0; c < kSkChunks; ++c) {
      uint32_t v[32];
      if (have_acc) {
        tmem_ld_32cols(taddr + static_cast<uint32_t>(static_cast<int>(peer) * kSkHalf + c * kSkChunkCols), v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0u;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        __stcg(mine_slot + sk_unit(c, u, r), make_uint4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]));
    }
    if (warp == 2 && lane == 0) SQ_SK_MARK(4);
  }

  // Release / acquire at cluster scope: the peer's partial stores are visible
  // to this CTA's loads after the barrier.
  cluster_sync_all();
  if (threadIdx.x == 0) SQ_SK_MARK(5);
  if (warp >= 2) {
    // ------------------------------------------- own columns: add the peer's partial, dequantise, store
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint4* peer_slot = p.part + (static_cast<size_t>(tile) * 2 + peer) * (kSkSlotBytes / 16);
    const uint4* staged = reinterpret_cast<const uint4*>(smem);  // the ring is idle: every MMA has completed
    if (warp == 2 && lane == 0) {
      fence_proxy_async_global();  // the acquired partial stores, then the bulk read
      mbar_arrive_expect_tx(part_full, static_cast<uint32_t>(kSkSlotBytes));
      bulk_load(smem, peer_slot, static_cast<uint32_t>(kSkSlotBytes), part_full);
    }
    const int m = m_blk * kBM + r;
    const bool row_ok = m < p.M;
    const float xs = xs_s[r];
    const bool got = mbar_wait_bounded(part_full, 0, p.timeout_ns);
    if (!__all_sync(0xFFFFFFFFu, got) && lane == 0 && !*abort_flag) flag_timeout(abort_flag);
#pragma unroll 1
    for (int c = 0; c < kSkChunks; ++c) {
      uint4 q[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) q[u] = staged[sk_unit(c, u, r)];
      uint32_t v[32];
      if (have_acc) {
        tmem_ld_32cols(taddr + static_cast<uint32_t>(static_cast<int>(rank) * kSkHalf + c * kSkChunkCols), v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0u;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) v[4 * u] += q[u].x, v[4 * u + 1] += q[u].y, v[4 * u + 2] += q[u].z, v[4 * u + 3] += q[u].w;
      const int cc = c * kSkChunkCols;  // column within the owned half
      const int n0 = n_blk * kSkBN + static_cast<int>(rank) * kSkHalf + cc;
      if (n0 >= p.N) continue;  // warp-uniform
      uint32_t packed[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float y0 = __fmaf_rn(__int2float_rn(static_cast<int>(v[j])), __fmul_rn(xs, ws_s[cc + j]), b_s[cc + j]);
        const float y1 = __fmaf_rn(__int2float_rn(static_cast<int>(v[j + 1])), __fmul_rn(xs, ws_s[cc + j + 1]),
                                   b_s[cc + j + 1]);
        packed[j / 2] = pack_bf16x2(y0, y1);
      }
      if (p.tma_store) {
        // this warp's 32 rows x 32 columns into its own 2 KB box (row = lane,
        // 64 bytes; 16-byte unit u of row r at u ^ ((r >> 1) & 3), the 64-byte
        // swizzle, so the 32 lanes' writes spread over all banks), then one
        // TMA store; rows past M and columns past N are not written
        uint8_t* box = smem + kSkYOffset + ((quarter * kSkChunks + c) * 32) * (kSkChunkCols * 2);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          *reinterpret_cast<uint4*>(box + lane * 64 + ((u ^ ((lane >> 1) & 3)) << 4)) =
              make_uint4(packed[4 * u], packed[4 * u + 1], packed[4 * u + 2], packed[4 * u + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmY, n0, m_blk * kBM + quarter * 32, box);
          bulk_commit_group();
        }
        continue;
      }
      if (!row_ok) continue;
      uint16_t* yrow = p.out + static_cast<int64_t>(m) * p.N + n0;
      if (n0 + kSkChunkCols <= p.N && p.vec_ok) {
        uint4* dst = reinterpret_cast<uint4*>(yrow);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          dst[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (n0 + j < p.N) yrow[j] = static_cast<uint16_t>(packed[j / 2] >> ((j & 1) * 16));
      }
    }
    if (p.tma_store && lane == 0) bulk_wait_group_read0();  // the boxes are read before the block exits
    if (warp == 2 && lane == 0) SQ_SK_MARK(6);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) SQ_SK_MARK(7);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace
}  // namespace sq
