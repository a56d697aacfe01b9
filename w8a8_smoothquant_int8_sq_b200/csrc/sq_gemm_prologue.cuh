// sq_gemm_prologue.cuh -- the int8 GEMM that quantises its own A operand
// (activation quantisation fused into the GEMM prologue, for many tokens).
// Included by sq_gemm.cu (inside namespace sq, anonymous namespace).
//
// SmoothQuantW8A8.forward on the SmoothQuant page, once frozen: X~ = X / s,
// Xq = quantize_per_token_symmetric(X~) (per token: scale = max|row| / 127,
// codes round-half-even clamped to +-127), then acc = Xq Wq^T in int32 and
// Y = bf16(acc * x_scale[m] * w_scale[n] + bias[n]).  A pre-pass (the row
// quantiser without codes) has written x_scale[M] and RN(1/s_j)[K]; this
// kernel reads X in bf16 and writes the codes straight into the tensor core's
// shared-memory A operand, so Xq never exists in global memory.  The codes are
// those of the row quantiser bit for bit: t = fl(x / s_j) and fl(t / scale)
// are both correctly rounded divisions (Markstein's correction of the product
// with the correctly rounded reciprocal), rounded half-to-even by the fp32
// adder.
//
// Tiles are 256 x 512 outputs on a CTA pair (tcgen05 cta_group::2):
//   * CTA r of the pair owns rows [128 r, 128 r + 128) of the tile's 256 rows;
//     per k-block (128 columns of K) it holds its 128 rows of A codes and, for
//     each of the two 256-column halves of the tile, its 128 rows of that
//     half's Wq slice (TMA, 128-byte swizzle).  One thread of the even CTA
//     issues two M = 256, N = 256 MMAs per 32 columns of K, one per half, into
//     the two 256-column accumulators that fill tensor memory.  A code is
//     computed once per 512 output columns, not once per 256: the conversion is
//     the costly part of this kernel, the tensor pipe the cheap one.
//   * an X-producer warp streams the CTA's bf16 rows by TMA in slots of
//     128 rows x 64 columns (16 KB, no swizzle), each with the 64 matching
//     values of s and RN(1/s) (bulk copies), through a ring of four slots;
//   * sixteen converter warps turn two slots into one k-block of codes: lane l
//     of a warp takes 8 columns (8 (l % 8) .. + 7) of two rows, dividing by
//     s_j and by the row's scale and packing the codes into the swizzled
//     layout the MMA descriptors read; the writes are made visible to the
//     tensor core (fence.proxy.async) and each warp arrives on a barrier of
//     its own CTA (release at CTA scope).  The even CTA's full barrier counts
//     its producer's Wq bytes (both CTAs' loads), its own converter warps, and
//     one arrival from a relay thread of the odd CTA, which waits for the odd
//     CTA's converter warps and then releases their codes at cluster scope:
//     one cluster-scope release per stage instead of one per warp (each cost
//     a converter warp about 0.7 us, measured);
//   * four epilogue warps, one per TMEM lane quarter, read both accumulators
//     and write Y after the last k-block.  Both accumulators are in use for a
//     whole tile, so the next tile's MMAs wait for the epilogue; the
//     converters and the Wq producer run ahead into the ring meanwhile, and
//     the epilogue sleeps between polls of its barrier so that its warps leave
//     the issue slots to the converters during the main loop.
// Pair p takes tiles p, p + pairs, ... in the grouped order of tile_coords.
// Every wait is bounded; a timeout latches bit 0 of the device status word,
// the CTA leaves its loops, and both CTAs meet at a cluster barrier before
// freeing tensor memory.
//
// Measured against the row quantiser followed by the CTA-pair GEMM, this
// kernel is slower wherever a code feeds many output columns: each element of
// X is converted N / 512 times (56 times for N = 28672), two correctly
// rounded divisions and the packing each time, and the converter warps supply
// about 9 codes per cycle per SM where the tensor pipe consumes 16.

#ifndef SQ_PRO_EPI_SLEEP  // build-time knob: ns the epilogue sleeps between polls of its accumulator barrier
#define SQ_PRO_EPI_SLEEP 256
#endif

constexpr int kFHalf = 128;                  // rows of A, and rows of each Wq half, per CTA
constexpr int kFBM = 256;                    // tile rows
constexpr int kFSub = 256;                   // columns per MMA (one accumulator)
constexpr int kFBN = 2 * kFSub;              // tile columns
#ifndef SQ_PRO_CONV_WARPS  // build-time knob: converter warps (8 or 16)
#define SQ_PRO_CONV_WARPS 16
#endif
#ifndef SQ_PRO_EPI_WARPS  // build-time knob: epilogue warps (4: each takes both halves, or 8)
#define SQ_PRO_EPI_WARPS 4
#endif
constexpr int kFConvWarps = SQ_PRO_CONV_WARPS;
constexpr int kFEpiWarps = SQ_PRO_EPI_WARPS;
constexpr int kFRowsPerThread = 32 / kFConvWarps;  // rows of a slot per converter lane
static_assert(kFConvWarps == 8 || kFConvWarps == 16, "converter warps");
static_assert(kFEpiWarps == 4 || kFEpiWarps == 8, "epilogue warps");
constexpr int kFEpiWarp0 = 3;                // warps: 0 Wq producer, 1 MMA, 2 X producer
constexpr int kFConvWarp0 = kFEpiWarp0 + kFEpiWarps;
constexpr int kFThreads = 32 * (kFConvWarp0 + kFConvWarps);
#ifndef SQ_PRO_STAGES  // build-time knob: ring depth of A codes + both Wq halves
#define SQ_PRO_STAGES 3
#endif
#ifndef SQ_PRO_XSLOTS  // build-time knob: ring depth of bf16 X slots
#define SQ_PRO_XSLOTS 4
#endif
constexpr int kFStages = SQ_PRO_STAGES;
constexpr int kFABytes = kFHalf * kBK;       // 16 KB
constexpr int kFBHalfBytes = kFHalf * kBK;   // 16 KB per 256-column half
constexpr int kFStageBytes = kFABytes + 2 * kFBHalfBytes;  // 48 KB
constexpr int kFXCols = 64;                  // columns of X per slot
constexpr int kFXSlots = SQ_PRO_XSLOTS;
constexpr int kFXBytes = kFHalf * kFXCols * 2;             // 16 KB of bf16
constexpr int kFXSlotBytes = kFXBytes + 2 * kFXCols * 4;   // + s and RN(1/s) of its columns
constexpr int kFXOffset = kFStages * kFStageBytes;
constexpr int kFBarOffset = kFXOffset + kFXSlots * kFXSlotBytes;
constexpr int kFNumBars = 3 * kFStages + 2 * kFXSlots + 3;  // full, empty, cfull, xfull, xempty, tfull, tempty, drain
constexpr int kFMiscOffset = (kFBarOffset + kFNumBars * 8 + 15) / 16 * 16;
constexpr int kFBytes = kFMiscOffset + 16;
constexpr int kFAlloc = kFBytes + 1024;      // manual 1024-byte alignment
constexpr uint32_t kFTmemCols = kFBN;        // both accumulators: all 512 columns
static_assert(kFStageBytes % 1024 == 0 && kFXSlotBytes % 16 == 0, "stage alignment");
static_assert(kFAlloc <= 227 * 1024, "shared memory");

struct PrologueParams {
  unsigned long long timeout_ns;
  int skip_first_load;  // test hook: the Wq producers never load the first stage
  int M, N, K;
  int num_m_blocks, num_n_blocks, num_k_blocks;
  int group_m;
  const float* s;        // [K]
  const float* rs;       // [K] RN(1/s_j)
  const float* x_scale;  // [M]
  const float* w_scale;  // [N]
  const uint16_t* bias;  // [N] or null
  uint16_t* out;         // Y [M][N]
  int vec_ok;            // 16-byte loads of w_scale / bias and stores of Y allowed
};

#ifdef SQ_TRACE
// Optional stage timestamps (build with -DSQ_TRACE), pair 0, first 64 stages,
// per CTA rank: converter warp 0 lane 0 at 0 stage free, 1 first slot landed,
// 2 first slot converted, 3 second slot landed, 4 second slot converted,
// 5 codes published; 6 the MMA's full wait done (even CTA); 7 the Wq producer's
// empty wait done; 8 past the proxy fence; 9 the last converter warp at 5.  X producer issue times
// per slot in g_pro_xtrace.
__device__ unsigned long long g_pro_trace[2][64][10];
__device__ unsigned long long g_pro_xtrace[2][128];
#define SQ_PRO_MARK(seq, i)                                                                             \
  do {                                                                                                  \
    if (blockIdx.x < 2 && (seq) < 64) g_pro_trace[blockIdx.x][(seq)][(i)] = globaltimer_ns();           \
  } while (0)
#define SQ_PRO_XMARK(seq)                                                                               \
  do {                                                                                                  \
    if (blockIdx.x < 2 && (seq) < 128) g_pro_xtrace[blockIdx.x][(seq)] = globaltimer_ns();              \
  } while (0)
#else
#define SQ_PRO_MARK(seq, i) \
  do {                      \
  } while (0)
#define SQ_PRO_XMARK(seq) \
  do {                    \
  } while (0)
#endif

// Row (within the CTA's 128) of converter warp cw's instruction i
// (0 <= i < kFRowsPerThread), lane group
// rq = lane / 8: a warp instruction covers rows {b, b+4, b+1, b+5} or
// {b+2, b+6, b+3, b+7} of an 8-row swizzle atom b, so its four 64-byte code
// writes fall into distinct bank halves (two wavefronts for 256 bytes) and its
// four 128-byte X reads into four (the minimum for 512 bytes).
__device__ __forceinline__ int prologue_row(int cw, int i, int rq) {
  const int q = cw * kFRowsPerThread + i;
  return 8 * (q >> 1) + 2 * (q & 1) + ((rq & 1) << 2) + (rq >> 1);
}

__global__ void __launch_bounds__(kFThreads, 1)
    gemm_i8_prologue_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                            const PrologueParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kFBarOffset);
  uint64_t* full = bars;                      // even CTA: Wq bytes of both CTAs + 16 converter warps
  uint64_t* empty = bars + kFStages;          // each CTA: the stage may be refilled
  uint64_t* cfull = empty + kFStages;         // odd CTA: its converter warps published a stage
  uint64_t* xfull = cfull + kFStages;         // each CTA: an X slot landed
  uint64_t* xempty = xfull + kFXSlots;        // each CTA: an X slot was converted
  uint64_t* tfull = xempty + kFXSlots;        // each CTA: the accumulators are final
  uint64_t* tempty = tfull + 1;               // even CTA: both CTAs' epilogues are done with them
  uint64_t* drain = tempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kFMiscOffset);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kFMiscOffset + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_cta_rank();
  const int pair = static_cast<int>(blockIdx.x) >> 1;
  const int num_pairs = static_cast<int>(gridDim.x) >> 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kFStages; ++i) {
      // even CTA: its producer's expect_tx, its converter warps, and the odd
      // CTA's converter warps (or their relay)
      mbar_init(&full[i], 1 + kFConvWarps + 1);
      mbar_init(&empty[i], 1);
      mbar_init(&cfull[i], kFConvWarps);
    }
    for (int i = 0; i < kFXSlots; ++i) {
      mbar_init(&xfull[i], 1);
      mbar_init(&xempty[i], kFConvWarps);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 2 * kFEpiWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc_pair(tmem_slot, kFTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_barrier_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();
  griddep_launch_dependents();

  const int num_tiles = p.num_m_blocks * p.num_n_blocks;
  const int nk = p.num_k_blocks;

  if (warp == 0) {
    // ---------------------------------------------- Wq producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int64_t seq = 0;
      for (int tile = pair; ok && tile < num_tiles; tile += num_pairs) {
        int m_blk, n_blk;
        tile_coords(tile, p.num_m_blocks, p.num_n_blocks, p.group_m, m_blk, n_blk);
        const int b_row = n_blk * kFBN + static_cast<int>(rank) * kFHalf;
        for (int kb = 0; kb < nk; ++kb, ++seq) {
          if (*abort_flag || !mbar_wait_bounded(&empty[stage], phase ^ 1u, p.timeout_ns)) {
            if (!*abort_flag) flag_timeout(abort_flag);
            ok = false;
            break;
          }
          SQ_PRO_MARK(seq, 7);
          if (!(p.skip_first_load && seq == 0)) {  // test hook: this stage never gets its Wq bytes
            uint8_t* sb = smem + stage * kFStageBytes + kFABytes;
            const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * 2 * kFBHalfBytes);
            tma_load_2d_pair(sb, &tmB, kb * kBK, b_row, bar);
            tma_load_2d_pair(sb + kFBHalfBytes, &tmB, kb * kBK, b_row + kFSub, bar);
          } else if (rank == 0) {
            mbar_arrive_expect_tx(&full[stage], 2 * 2 * kFBHalfBytes);
          }
          if (++stage == kFStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 2) {
    // ----------------------------------------------- X producer (both CTAs)
    if (lane == 0) {
      int slot = 0;
      uint32_t phase = 0;
      bool ok = true;
      int xseq = 0;
      for (int tile = pair; ok && tile < num_tiles; tile += num_pairs) {
        int m_blk, n_blk;
        tile_coords(tile, p.num_m_blocks, p.num_n_blocks, p.group_m, m_blk, n_blk);
        const int a_row = m_blk * kFBM + static_cast<int>(rank) * kFHalf;
        for (int h = 0; h < 2 * nk; ++h, ++xseq) {
          if (*abort_flag || !mbar_wait_bounded(&xempty[slot], phase ^ 1u, p.timeout_ns)) {
            if (!*abort_flag) flag_timeout(abort_flag);
            ok = false;
            break;
          }
          SQ_PRO_XMARK(xseq);
          (void)xseq;
          const int c0 = h * kFXCols;
          const int cols = min(kFXCols, p.K - c0);  // a multiple of 16; <= 0 past K
          uint8_t* xs = smem + kFXOffset + slot * kFXSlotBytes;
          if (cols > 0) {
            const uint32_t tab = static_cast<uint32_t>(cols) * 4u;
            mbar_arrive_expect_tx(&xfull[slot], kFXBytes + 2 * tab);
            tma_load_2d(xs, &tmX, c0, a_row, &xfull[slot]);
            bulk_load(xs + kFXBytes, p.s + c0, tab, &xfull[slot]);
            bulk_load(xs + kFXBytes + kFXCols * 4, p.rs + c0, tab, &xfull[slot]);
          } else {
            mbar_arrive(&xfull[slot]);  // columns past K: the converters write zero codes
          }
          if (++slot == kFXSlots) {
            slot = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (even CTA)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kFBM, kFSub);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < num_tiles; tile += num_pairs, ++it) {
        if (*abort_flag || !mbar_wait_cluster_bounded(tempty, (it & 1) ^ 1u, p.timeout_ns)) {
          if (!*abort_flag) flag_timeout(abort_flag);
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb) {
          // converter arrivals come from both CTAs: acquire at cluster scope
          if (*abort_flag || !mbar_wait_cluster_bounded(&full[stage], phase, p.timeout_ns)) {
            if (!*abort_flag) flag_timeout(abort_flag);
            ok = false;
            break;
          }
          SQ_PRO_MARK(it * nk + kb, 6);
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kFStageBytes);
          const uint64_t adesc = smem_desc_k_sw128(sa);
          const uint64_t b0desc = smem_desc_k_sw128(sa + kFABytes);
          const uint64_t b1desc = smem_desc_k_sw128(sa + kFABytes + kFBHalfBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            const uint32_t acc = (kb != 0 || kk != 0) ? 1u : 0u;
            const uint64_t adv = static_cast<uint64_t>(kk * 2);  // +32 bytes inside the swizzle atom
            mma_i8_pair(tmem_base, adesc + adv, b0desc + adv, idesc, acc);
            mma_i8_pair(tmem_base + kFSub, adesc + adv, b1desc + adv, idesc, acc);
          }
          mma_commit_pair(&empty[stage], 0x3);
          if (++stage == kFStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair(tfull, 0x3);
      }
      mma_commit_pair(drain, 0x1);
      (void)mbar_wait_bounded(drain, 0, p.timeout_ns);
    } else if (rank == 1 && lane == 0) {
      // relay (odd CTA): once all of this CTA's converter warps have published
      // a stage (release / acquire at CTA scope, cheap for them), one arrive
      // on the even CTA's full barrier releases their codes at cluster scope
      const uint32_t full_even = mapa_shared(smem_u32(&full[0]), 0);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < num_tiles; tile += num_pairs) {
        for (int kb = 0; kb < nk; ++kb) {
          if (*abort_flag || !mbar_wait_bounded(&cfull[stage], phase, p.timeout_ns)) {
            if (!*abort_flag) flag_timeout(abort_flag);
            ok = false;
            break;
          }
          mbar_arrive_cluster(full_even + static_cast<uint32_t>(stage * 8));
          if (++stage == kFStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp < kFConvWarp0) {
    // --------------------------------------------- epilogue (both CTAs)
    const int quarter = warp & 3;                  // TMEM lanes [32 quarter, 32 quarter + 32)
    // with eight warps, warp w takes half (w - 3) / 4; with four, both halves
    const int half0 = kFEpiWarps == 8 ? (warp - kFEpiWarp0) >> 2 : 0;
    constexpr int kHalves = kFEpiWarps == 8 ? 1 : 2;
    const uint32_t tempty_even = mapa_shared(smem_u32(tempty), 0);
    int it = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs, ++it) {
      int m_blk, n_blk;
      tile_coords(tile, p.num_m_blocks, p.num_n_blocks, p.group_m, m_blk, n_blk);
      const int row = m_blk * kFBM + static_cast<int>(rank) * kFHalf + quarter * 32 + lane;
      const bool row_ok = row < p.M;
      const float xs = row_ok ? __ldg(p.x_scale + row) : 0.0f;
      const bool mine = !*abort_flag && (SQ_PRO_EPI_SLEEP > 0
                                             ? mbar_wait_bounded_sleep(tfull, it & 1, p.timeout_ns, SQ_PRO_EPI_SLEEP)
                                             : mbar_wait_bounded(tfull, it & 1, p.timeout_ns));
      if (!__all_sync(0xFFFFFFFFu, mine)) {
        if (lane == 0 && !*abort_flag) flag_timeout(abort_flag);
        break;
      }
      tc_fence_after();
      const uint32_t t_base =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(half0 * kFSub);
#pragma unroll 1
      for (int c0 = 0; c0 < kHalves * kFSub; c0 += 32) {
        uint32_t r[32];
        tmem_ld_32cols(t_base + static_cast<uint32_t>(c0), r);
        tmem_ld_wait();
        const int n0 = n_blk * kFBN + half0 * kFSub + c0;
        if (n0 >= p.N) continue;  // tile overhang past N (warp-uniform)
        const bool vec = (n0 + 32 <= p.N) && p.vec_ok;
        uint16_t* yrow = p.out + static_cast<int64_t>(row) * p.N + n0;
        if (vec) {
          // 8 columns at a time: two float4 of w_scale, 8 bf16 of bias, one 16-byte store
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            const float4 wa = __ldg(reinterpret_cast<const float4*>(p.w_scale + n0 + j));
            const float4 wb = __ldg(reinterpret_cast<const float4*>(p.w_scale + n0 + j + 4));
            const float ws[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
            uint4 b8 = make_uint4(0u, 0u, 0u, 0u);
            if (p.bias != nullptr) b8 = __ldg(reinterpret_cast<const uint4*>(p.bias + n0 + j));
            const uint32_t bw[4] = {b8.x, b8.y, b8.z, b8.w};
            uint32_t packed[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float y0 =
                  __fmaf_rn(__int2float_rn(static_cast<int>(r[j + 2 * u])), __fmul_rn(xs, ws[2 * u]), bf16_lo(bw[u]));
              const float y1 = __fmaf_rn(__int2float_rn(static_cast<int>(r[j + 2 * u + 1])),
                                         __fmul_rn(xs, ws[2 * u + 1]), bf16_hi(bw[u]));
              packed[u] = pack_bf16x2(y0, y1);
            }
            if (row_ok)
              *reinterpret_cast<uint4*>(yrow + j) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (n0 + j < p.N) {
              const float ws = __ldg(p.w_scale + n0 + j);
              const float b =
                  p.bias != nullptr ? __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + n0 + j)) << 16) : 0.0f;
              const float y = __fmaf_rn(__int2float_rn(static_cast<int>(r[j])), __fmul_rn(xs, ws), b);
              if (row_ok) yrow[j] = static_cast<uint16_t>(pack_bf16x2(y, 0.0f));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_even);
    }
  } else {
    // -------------------------------------------- converters (both CTAs)
    const int cw = warp - kFConvWarp0;
    const int v = lane & 7;    // 8-column vector of the slot
    const int rq = lane >> 3;  // row within the warp instruction
    int rl[kFRowsPerThread];
#pragma unroll
    for (int i = 0; i < kFRowsPerThread; ++i) rl[i] = prologue_row(cw, i, rq);
    int stage = 0, slot = 0;
    uint32_t phase = 0, xphase = 0;
    bool ok = true;
    int cseq = 0;  // stages converted (trace index)
    const bool tr0 = cw == 0 && lane == 0, trl = cw == kFConvWarps - 1 && lane == 0;
    (void)tr0;
    (void)trl;
    for (int tile = pair; ok && tile < num_tiles; tile += num_pairs) {
      int m_blk, n_blk;
      tile_coords(tile, p.num_m_blocks, p.num_n_blocks, p.group_m, m_blk, n_blk);
      const int row0 = m_blk * kFBM + static_cast<int>(rank) * kFHalf;
      // the row scales of this tile: -scale and RN(1/scale), as lane pairs
      f2x nsc[kFRowsPerThread], rsc[kFRowsPerThread];
#pragma unroll
      for (int i = 0; i < kFRowsPerThread; ++i) {
        const int row = row0 + rl[i];
        const float sc = row < p.M ? __ldg(p.x_scale + row) : 1.0f;
        const float r = __frcp_rn(sc);
        nsc[i] = f2_pack(-sc, -sc);
        rsc[i] = f2_pack(r, r);
      }
      for (int kb = 0; kb < nk; ++kb) {
        bool got = !*abort_flag && mbar_wait_bounded(&empty[stage], phase ^ 1u, p.timeout_ns);
        if (!__all_sync(0xFFFFFFFFu, got)) {
          if (lane == 0 && !*abort_flag) flag_timeout(abort_flag);
          ok = false;
          break;
        }
        if (tr0) SQ_PRO_MARK(cseq, 0);
        uint8_t* a = smem + stage * kFStageBytes;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          got = !*abort_flag && mbar_wait_bounded(&xfull[slot], xphase, p.timeout_ns);
          if (!__all_sync(0xFFFFFFFFu, got)) {
            if (lane == 0 && !*abort_flag) flag_timeout(abort_flag);
            ok = false;
            break;
          }
          if (tr0) SQ_PRO_MARK(cseq, 1 + 2 * h);
          const uint8_t* xs = smem + kFXOffset + slot * kFXSlotBytes;
          const bool col_ok = (kb * kBK + h * kFXCols + 8 * v) < p.K;  // K % 16 == 0: whole vectors
          f2x ns[4], rs[4];
          {
            const float4* st = reinterpret_cast<const float4*>(xs + kFXBytes) + 2 * v;
            const float4* rt = reinterpret_cast<const float4*>(xs + kFXBytes + kFXCols * 4) + 2 * v;
            const float4 s0 = st[0], s1 = st[1], r0 = rt[0], r1 = rt[1];
            ns[0] = f2_pack(-s0.x, -s0.y), ns[1] = f2_pack(-s0.z, -s0.w);
            ns[2] = f2_pack(-s1.x, -s1.y), ns[3] = f2_pack(-s1.z, -s1.w);
            rs[0] = f2_pack(r0.x, r0.y), rs[1] = f2_pack(r0.z, r0.w);
            rs[2] = f2_pack(r1.x, r1.y), rs[3] = f2_pack(r1.z, r1.w);
          }
          const int c16 = h * 4 + (v >> 1);  // 16-byte chunk of the 128-byte code row
#pragma unroll
          for (int i = 0; i < kFRowsPerThread; ++i) {
            const int r = rl[i];
            uint2 codes = make_uint2(0u, 0u);
            if (col_ok) {
              const uint4 w = *reinterpret_cast<const uint4*>(xs + r * (kFXCols * 2) + v * 16);
              const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
              f2x c[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const f2x t = f2_div_rn(f2_from_bf16x2(wv[e]), ns[e], rs[e]);
                c[e] = f2_round_codes(f2_div_rn(t, nsc[i], rsc[i]));
              }
              codes = pack8_codes(c[0], c[1], c[2], c[3]);
            }
            const int off = (r >> 3) * 1024 + (r & 7) * 128 + ((c16 ^ (r & 7)) << 4) + ((v & 1) << 3);
            *reinterpret_cast<uint2*>(a + off) = codes;
          }
          __syncwarp();
          if (tr0) SQ_PRO_MARK(cseq, 2 + 2 * h);
          if (lane == 0) mbar_arrive(&xempty[slot]);
          if (++slot == kFXSlots) {
            slot = 0;
            xphase ^= 1u;
          }
        }
        if (!ok) break;
        // the codes, to the tensor core: async-proxy visibility, then the even
        // CTA's full barrier (the odd CTA's warps through the relay)
        fence_proxy_async_smem();
        if (tr0) SQ_PRO_MARK(cseq, 8);
        __syncwarp();
        if (lane == 0) mbar_arrive(rank == 0 ? &full[stage] : &cfull[stage]);
        if (tr0) SQ_PRO_MARK(cseq, 5);
        if (trl) SQ_PRO_MARK(cseq, 9);
        ++cseq;
        if (++stage == kFStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_barrier_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kFTmemCols);
  }
}
