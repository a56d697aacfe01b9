// sq_gemm_pair.cuh -- the int8 GEMM for many output tiles, on CTA pairs.
// Included by sq_gemm.cu (inside namespace sq, anonymous namespace).
//
// Same product and epilogue as gemm_i8_kernel (SmoothQuantW8A8.forward on the
// SmoothQuant page: acc = Xq Wq^T exact in int32, Y = bf16(acc * x_scale[m] *
// w_scale[n] + bias[n])), with output tiles of 256 x 256 shared by the two
// CTAs of a cluster (tcgen05 cta_group::2):
//   * CTA r of the pair loads rows [128 r, 128 r + 128) of the tile's Xq slice
//     and rows [128 r, 128 r + 128) of its Wq slice (128-byte K slices,
//     128-byte swizzle) into its own shared memory, at the same offsets in
//     both CTAs.  Each CTA reads half of the B operand it would read for a
//     128 x 256 tile on its own: 32 KB per k-block instead of 48 KB.
//   * Both CTAs' loads count their bytes on the even CTA's full barrier; one
//     thread of the even CTA issues tcgen05.mma.cta_group::2 (M = 256, N = 256,
//     K = 32), which reads A and B from both CTAs' shared memory and writes
//     accumulator rows 0-127 into the even CTA's tensor memory and rows
//     128-255 into the odd CTA's, at the same columns.
//   * tcgen05.commit with a two-CTA mask frees the ring stage in both CTAs and
//     announces a finished accumulator to both CTAs' epilogues; the epilogue
//     warps of both CTAs release an accumulator on the even CTA's barrier.
//   * Two accumulators of 256 columns (all 512 columns of tensor memory) let
//     the epilogue of one tile overlap the main loop of the next.
// Tiles go round the pairs persistently (pair p takes tiles p, p + pairs, ...)
// in the grouped order of tile_coords.  Every wait is bounded; a timeout latches bit 0 of the
// device status word and the CTA leaves its loop; both CTAs meet at a cluster
// barrier before freeing tensor memory and exiting.

constexpr int kPairBM = 256;                 // tile rows (128 per CTA)
constexpr int kPairBN = 256;                 // tile columns (128 rows of Wq per CTA)
constexpr int kPairHalf = 128;               // rows of A and of B per CTA
constexpr int kPairThreads = 192;            // producer, MMA, 4 epilogue warps
#ifndef SQ_PAIR_STAGES  // build-time knob: ring depth
#define SQ_PAIR_STAGES 6
#endif
constexpr int kPairStages = SQ_PAIR_STAGES;
constexpr int kPairABytes = kPairHalf * kBK;             // 16 KB
constexpr int kPairStageBytes = 2 * kPairABytes;         // A half + B half: 32 KB
constexpr int kPairRingBytes = kPairStages * kPairStageBytes;
constexpr int kPairBarOffset = kPairRingBytes;
constexpr int kPairNumBars = 2 * kPairStages + 4 + 1;    // full, empty, tfull[2], tempty[2], drain
constexpr int kPairEpiOffset = (kPairBarOffset + kPairNumBars * 8 + 15) / 16 * 16;
constexpr int kPairEpiBytes = 4 * 2 * kPairBN * 4;       // per epilogue warp: w_scale[256], bias[256]
constexpr int kPairMiscOffset = kPairEpiOffset + kPairEpiBytes;
constexpr int kPairBytes = kPairMiscOffset + 16;
constexpr int kPairAlloc = kPairBytes + 1024;            // manual 1024-byte alignment
constexpr uint32_t kPairTmemCols = 2 * kPairBN;          // two accumulators

struct PairParams {
  unsigned long long timeout_ns;
  int skip_first_load;  // test hook: the producers never load the first stage
  int M, N, K;
  int num_m_blocks, num_n_blocks, num_k_blocks;
  int group_m;  // m-blocks per tile group (tile_coords)
  const float* x_scale;
  const float* w_scale;
  const uint16_t* bias;
  void* out;
  int vec_ok;
};

template <int EPI>
__global__ void __launch_bounds__(kPairThreads, 1)
    gemm_i8_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const PairParams p) {
  extern __shared__ uint8_t smem_raw[];
  // the same alignment in both CTAs: the MMA reads both at the same offsets
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPairBarOffset);
  uint64_t* full = bars;                   // even CTA: both CTAs' loads of a stage
  uint64_t* empty = bars + kPairStages;    // each CTA: its stage may be refilled
  uint64_t* tfull = bars + 2 * kPairStages;  // each CTA: accumulator ready
  uint64_t* tempty = tfull + 2;            // even CTA: both CTAs' epilogues done with it
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kPairMiscOffset);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kPairMiscOffset + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_cta_rank();  // 0: issues the MMAs
  const int pair = static_cast<int>(blockIdx.x) >> 1;
  const int num_pairs = static_cast<int>(gridDim.x) >> 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kPairStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 8);  // one arrive per epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc_pair(tmem_slot, kPairTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // barriers of both CTAs initialised (the peer's loads count on ours) and
  // tensor memory allocated in both before anything crosses the pair
  cluster_barrier_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();
  griddep_launch_dependents();

  const int num_tiles = p.num_m_blocks * p.num_n_blocks;
  const int nk = p.num_k_blocks;

  if (warp == 0) {
    // ------------------------------------------------- producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int64_t seq = 0;
      for (int tile = pair; ok && tile < num_tiles; tile += num_pairs) {
        int m_blk, n_blk;
        tile_coords(tile, p.num_m_blocks, p.num_n_blocks, p.group_m, m_blk, n_blk);
        const int a_row = m_blk * kPairBM + static_cast<int>(rank) * kPairHalf;
        const int b_row = n_blk * kPairBN + static_cast<int>(rank) * kPairHalf;
        for (int kb = 0; kb < nk; ++kb, ++seq) {
          if (p.skip_first_load && seq == 0) {  // test hook: this stage never fills
            if (++stage == kPairStages) {
              stage = 0;
              phase ^= 1u;
            }
            continue;
          }
          if (*abort_flag || !mbar_wait_bounded(&empty[stage], phase ^ 1u, p.timeout_ns)) {
            if (!*abort_flag) flag_timeout(abort_flag);
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * kPairStageBytes;
          uint8_t* sb = sa + kPairABytes;
          const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
          // the even CTA's barrier expects both CTAs' bytes of this stage
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * kPairStageBytes);
          tma_load_2d_pair(sa, &tmA, kb * kBK, a_row, bar);
          tma_load_2d_pair(sb, &tmB, kb * kBK, b_row, bar);
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (even CTA)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kPairBM, kPairBN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < num_tiles; tile += num_pairs, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (*abort_flag || !mbar_wait_cluster_bounded(&tempty[acc], acc_phase ^ 1u, p.timeout_ns)) {
          if (!*abort_flag) flag_timeout(abort_flag);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kPairBN);
        for (int kb = 0; kb < nk; ++kb) {
          if (*abort_flag || !mbar_wait_bounded(&full[stage], phase, p.timeout_ns)) {
            if (!*abort_flag) flag_timeout(abort_flag);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kPairStageBytes);
          const uint32_t sb = sa + kPairABytes;
          const uint64_t adesc = smem_desc_k_sw128(sa);
          const uint64_t bdesc = smem_desc_k_sw128(sb);
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            // K advance inside the 128-byte swizzle atom: +32 bytes (encoded >> 4)
            mma_i8_pair(d_tmem, adesc + static_cast<uint64_t>(kk * 2), bdesc + static_cast<uint64_t>(kk * 2), idesc,
                        (kb != 0 || kk != 0) ? 1u : 0u);
          }
          mma_commit_pair(&empty[stage], 0x3);  // frees the stage in both CTAs
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair(&tfull[acc], 0x3);  // the accumulator, to both CTAs' epilogues
      }
      // drain: every MMA this thread issued has completed (a pair commit
      // tracks the pair MMAs; only this CTA's drain barrier is signalled)
      mma_commit_pair(drain, 0x1);
      (void)mbar_wait_bounded(drain, 0, p.timeout_ns);
    }
  } else {
    // --------------------------------------------- epilogue (both CTAs)
    const int quarter = warp & 3;  // TMEM lanes [32 quarter, 32 quarter + 32)
    float* ep_ws = reinterpret_cast<float*>(smem + kPairEpiOffset) + (warp - 2) * (2 * kPairBN);
    float* ep_b = ep_ws + kPairBN;
    const uint32_t tempty_even = mapa_shared(smem_u32(&tempty[0]), 0);
    int it = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      int m_blk, n_blk;
      tile_coords(tile, p.num_m_blocks, p.num_n_blocks, p.group_m, m_blk, n_blk);
      const int row = m_blk * kPairBM + static_cast<int>(rank) * kPairHalf + quarter * 32 + lane;
      const bool row_ok = row < p.M;
      float xs = 0.0f;
      if (EPI == 0) {
        const int nb = n_blk * kPairBN;
        __syncwarp();  // the previous tile's reads of the staging area are done
        for (int i = lane * 4; i < kPairBN; i += 128) {
          float4 w4 = make_float4(0.f, 0.f, 0.f, 0.f);
          if (nb + i + 4 <= p.N && p.vec_ok) {
            w4 = __ldg(reinterpret_cast<const float4*>(p.w_scale + nb + i));
          } else {
            if (nb + i < p.N) w4.x = __ldg(p.w_scale + nb + i);
            if (nb + i + 1 < p.N) w4.y = __ldg(p.w_scale + nb + i + 1);
            if (nb + i + 2 < p.N) w4.z = __ldg(p.w_scale + nb + i + 2);
            if (nb + i + 3 < p.N) w4.w = __ldg(p.w_scale + nb + i + 3);
          }
          *reinterpret_cast<float4*>(ep_ws + i) = w4;
        }
        for (int i = lane; i < kPairBN; i += 32)
          ep_b[i] = (p.bias != nullptr && nb + i < p.N)
                        ? __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + nb + i)) << 16)
                        : 0.0f;
        xs = row_ok ? __ldg(p.x_scale + row) : 0.0f;
        __syncwarp();
      }
      const bool mine = !*abort_flag && mbar_wait_bounded(&tfull[acc], acc_phase, p.timeout_ns);
      if (!__all_sync(0xFFFFFFFFu, mine)) {
        if (lane == 0 && !*abort_flag) flag_timeout(abort_flag);
        break;
      }
      tc_fence_after();
      const uint32_t t_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                              static_cast<uint32_t>(acc * kPairBN);
#pragma unroll 1
      for (int c0 = 0; c0 < kPairBN; c0 += 32) {
        uint32_t r[32];
        tmem_ld_32cols(t_base + static_cast<uint32_t>(c0), r);
        tmem_ld_wait();
        const int n0 = n_blk * kPairBN + c0;
        if (n0 >= p.N) continue;  // tile overhang past N (warp-uniform)
        const bool vec = (n0 + 32 <= p.N) && p.vec_ok;
        if (EPI == 0) {
          uint32_t packed[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float y0 =
                __fmaf_rn(__int2float_rn(static_cast<int>(r[j])), __fmul_rn(xs, ep_ws[c0 + j]), ep_b[c0 + j]);
            const float y1 = __fmaf_rn(__int2float_rn(static_cast<int>(r[j + 1])), __fmul_rn(xs, ep_ws[c0 + j + 1]),
                                       ep_b[c0 + j + 1]);
            packed[j / 2] = pack_bf16x2(y0, y1);
          }
          if (row_ok) {
            uint16_t* yrow = static_cast<uint16_t*>(p.out) + static_cast<int64_t>(row) * p.N + n0;
            if (vec) {
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
        } else {
          if (row_ok) {
            int32_t* arow = static_cast<int32_t*>(p.out) + static_cast<int64_t>(row) * p.N + n0;
            if (vec) {
              uint4* dst = reinterpret_cast<uint4*>(arow);
#pragma unroll
              for (int j = 0; j < 8; ++j) dst[j] = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (n0 + j < p.N) arow[j] = static_cast<int32_t>(r[j]);
            }
          }
        }
      }
      // this warp's rows of the accumulator are read: release it on the even CTA
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_even + static_cast<uint32_t>(acc * 8));
    }
  }

  // both CTAs done with each other's shared memory and tensor memory
  __syncwarp();
  tc_fence_before();
  cluster_barrier_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kPairTmemCols);
  }
}
