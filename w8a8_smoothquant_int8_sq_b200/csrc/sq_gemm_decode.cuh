// sq_gemm_decode.cuh -- the int8 linear for few tokens (M <= 32): a stream of
// the int8 weight through the tensor cores.  Included by sq_gemm.cu (inside
// namespace sq, anonymous namespace).
//
// Page: "w8a8_smoothquant.py -- W8A8 com SmoothQuant e alpha APRENDIVEL (V5)",
// SmoothQuantW8A8.forward: X / s, per-token quantisation, the int8 product,
// dequantisation and bias.  With few tokens the layer reads each byte of Wq
// once and does M multiply-adds with it: the time is the weight stream.
//
// Operands.  The MMA's M side holds the tokens and its N side 256 rows of Wq
// (tcgen05.mma kind::i8, M = 128, N = 256, K = 32): one MMA consumes 8 KB of
// the weight, twice what an MMA with the weight on the M side (128 rows x 32
// bytes) takes in about the same time, so the tensor core keeps ahead of HBM.
// The token rows of the A operand are the first ceil(M/8) 8-row atoms of
// each k-block; the A tiles of consecutive k-blocks sit one after another, so
// the MMA's other rows read the next k-blocks' atoms (and, for the last ones,
// the start of the weight ring that follows the A region).  Those rows of the
// product land in tensor-memory lanes the kernel never reads: only lanes
// 0..M-1 are used, and every row the MMA reads lies inside this CTA's shared
// memory.
//
//   * a CTA owns 256 rows of Wq and a K-slice; a cluster of S CTAs splits K.
//     The producer streams 256-row x 128-byte Wq boxes (128-byte swizzle)
//     through a ring; one thread issues the MMAs into one 256-column int32
//     accumulator.
//   * the codes: prequantised (sq_linear), the producer loads this CTA's
//     slice of Xq up front (rows past M zero-filled); fused (sq_forward, up to
//     8 tokens), eight warps divide their slice of X by s (correctly rounded,
//     as sq_quantize_act) and write the codes into the swizzled A atoms.  The
//     per-token scales come from row_scale_kernel, launched just before; X,
//     s and Wq are not written by that kernel, so they are read before the
//     wait for it: the weight stream starts at once.
//   * split-K: each rank copies its accumulator rows 0..M-1 to shared memory
//     and pushes the columns that rank q reduces into rank q's shared memory
//     (one slot per sender); after one cluster barrier each rank adds the S
//     partials of its 256/S columns, dequantises and stores Y.
// Warps: 0 producer, 1 tensor-memory owner + MMA issuer, 2..9 codes (fused),
// reduction and output.  Every mbarrier wait is bounded.

#ifdef SQ_TRACE
// Optional phase timestamps (build with -DSQ_TRACE): per CTA, globaltimer at
// 0 start, 1 codes ready (MMA warp), 2 first stage consumed, 3 last MMA
// issued, 4 accumulator read, 5 after the reduction barrier, 6 end,
// 7 past the wait for the previous kernel (code warps); per token of the
// scale pre-pass: [1023 - m][0] start, [1023 - m][1] end.
__device__ unsigned long long g_dec_trace[1024][8];
#define SQ_DEC_MARK(i)                                                  \
  do {                                                                  \
    const int cta_ = blockIdx.y * gridDim.x + blockIdx.x;               \
    if (cta_ < 1000) g_dec_trace[cta_][i] = globaltimer_ns();           \
  } while (0)
#else
#define SQ_DEC_MARK(i) \
  do {                 \
  } while (0)
#endif

constexpr int kDecThreads = 320;
constexpr int kDecRows = 256;                // Wq rows per CTA = MMA N
constexpr int kDecStageBytes = kDecRows * kBK;  // 32 KB
constexpr int kDecMaxStages = 8;
constexpr uint32_t kDecTmemCols = kDecRows;  // one int32 accumulator, 256 columns

struct DecParams {
  int M, N, K;
  int nk;            // k-blocks of 128 bytes over K
  int kb_per_split;  // k-blocks per cluster rank
  int stages;
  int a_atoms;       // 8-row atoms of tokens per k-block (ceil(M / 8))
  int mp;            // tokens padded to a multiple of 4 (partial-sum rows)
  const uint16_t* X;     // fused: [M][K] bf16
  const float* s;        // fused: [K]
  const float* x_scale;  // [M] (fused: written by row_scale_kernel)
  const float* w_scale;  // [N]
  const uint16_t* bias;  // [N] or null
  uint16_t* Y;           // [M][N]
  int ring_off, part_off, bar_off, misc_off;  // shared-memory layout (atoms at 0)
  unsigned long long timeout_ns;
};

// Byte offset of the code of token m, column c (0..127) of k-block j in the
// A region: atom (m / 8) of k-block j, row m % 8, 16-byte chunk c / 16
// permuted by XOR with the row (the 128-byte swizzle the descriptor reads).
__device__ __forceinline__ uint32_t dec_a_offset(int a_atoms, int j, int m, int c) {
  return static_cast<uint32_t>((j * a_atoms + (m >> 3)) * 1024 + (m & 7) * 128 + ((((c >> 4) ^ (m & 7)) & 7) << 4) +
                               (c & 15));
}

template <bool kFused>
__global__ void __launch_bounds__(kDecThreads, 2)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const DecParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* asm_ = smem;                                             // token atoms of every k-block
  uint8_t* ring = smem + p.ring_off;                                // weight boxes, right after the atoms
  int32_t* part = reinterpret_cast<int32_t*>(smem + p.part_off);    // [S senders][256/S cols][mp]
  // [256 cols][mp] this rank's sums, in the ring once every MMA has completed
  int32_t* mine = reinterpret_cast<int32_t*>(ring);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.bar_off);
  uint64_t* full = bars;
  uint64_t* empty = bars + kDecMaxStages;
  uint64_t* a_ready = bars + 2 * kDecMaxStages;
  uint64_t* acc_full = a_ready + 1;
  uint64_t* drain = a_ready + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + p.misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + p.misc_off + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_cta_rank();
  const int S = static_cast<int>(cluster_nctarank());
  const int rb = blockIdx.y;  // 256-row block of Wq
  const int kb0 = static_cast<int>(rank) * p.kb_per_split;
  const int kb1 = min(p.nk, kb0 + p.kb_per_split);
  const int my_nkb = max(0, kb1 - kb0);
  const int stages = p.stages;

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(a_ready, 1);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    if (!kFused) tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(tmem_slot, kDecTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (threadIdx.x == 0) SQ_DEC_MARK(0);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && my_nkb > 0) {
      // fused: Wq is not written by the previous kernel (the row scales are),
      // so the stream starts before the wait; prequantised: the codes may be
      // the previous kernel's output, so everything waits
      if (!kFused) griddep_wait();
      bool ok = true;
      if (!kFused) {
        // this CTA's codes, all k-blocks up front (rows past M read as zero)
        mbar_arrive_expect_tx(a_ready, static_cast<uint32_t>(my_nkb * p.a_atoms * 1024));
        for (int j = 0; j < my_nkb; ++j)
          tma_load_2d(asm_ + j * p.a_atoms * 1024, &tmX, (kb0 + j) * kBK, 0, a_ready);
      }
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int kb = kb0; ok && kb < kb1; ++kb) {
        if (*abort_flag || !mbar_wait_bounded(&empty[stage], phase ^ 1u, p.timeout_ns)) {
          if (!*abort_flag) flag_timeout(abort_flag);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(kDecStageBytes));
        tma_load_2d(ring + stage * kDecStageBytes, &tmW, kb * kBK, rb * kDecRows, &full[stage]);
        ++issued;
        if (++stage == stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {  // the copies in flight land before the CTA leaves
        for (int i = 0; i < min(issued, stages); ++i) {
          const int q = issued - 1 - i;
          (void)mbar_wait_bounded(&full[q % stages], static_cast<uint32_t>((q / stages) & 1), p.timeout_ns);
        }
        if (!kFused) (void)mbar_wait_bounded(a_ready, 0, p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && my_nkb > 0) {
      constexpr uint32_t idesc = idesc_i8(128, kDecRows);
      bool ok = !*abort_flag && mbar_wait_bounded(a_ready, 0, p.timeout_ns);
      if (!ok && !*abort_flag) flag_timeout(abort_flag);
      SQ_DEC_MARK(1);
      int stage = 0;
      uint32_t phase = 0;
      for (int j = 0; ok && j < my_nkb; ++j) {
        if (*abort_flag || !mbar_wait_bounded(&full[stage], phase, p.timeout_ns)) {
          if (!*abort_flag) flag_timeout(abort_flag);
          ok = false;
          break;
        }
        tc_fence_after();
        if (j == 0) SQ_DEC_MARK(2);
        const uint64_t adesc = smem_desc_k_sw128(smem_u32(asm_ + j * p.a_atoms * 1024));
        const uint64_t bdesc = smem_desc_k_sw128(smem_u32(ring + stage * kDecStageBytes));
#pragma unroll
        for (int kk = 0; kk < kBK / kUmmaK; ++kk)
          mma_i8(tmem_base, adesc + static_cast<uint64_t>(kk * 2), bdesc + static_cast<uint64_t>(kk * 2), idesc,
                 (j != 0 || kk != 0) ? 1u : 0u);
        mma_commit(&empty[stage]);
        if (++stage == stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      SQ_DEC_MARK(3);
      if (ok) mma_commit(acc_full);
      mma_commit(drain);
      (void)mbar_wait_bounded(drain, 0, p.timeout_ns);
    }
  } else {
    // --------------------------------------------- codes (fused, warps 2..9)
    const int qt = threadIdx.x - 64;  // 0..255
    if (kFused) {
      // thread qt: the 16-byte vector qt of this CTA's K-slice (8 columns)
      // for every token; X / s before the wait, the codes after it
      const int nvec = p.K >> 3;
      const int v = kb0 * (kBK / 8) + qt;
      const bool has = my_nkb > 0 && qt < my_nkb * (kBK / 8) && v < nvec;
      uint4 xw[8];
      f2x ns[4], rs[4];
      if (has) {
        const uint4* X4 = reinterpret_cast<const uint4*>(p.X);
        const float4* s4 = reinterpret_cast<const float4*>(p.s);
#pragma unroll
        for (int m = 0; m < 8; ++m)
          xw[m] = m < p.M ? __ldg(X4 + static_cast<int64_t>(m) * nvec + v) : make_uint4(0u, 0u, 0u, 0u);
        const float4 sa = __ldg(s4 + 2 * v), sb = __ldg(s4 + 2 * v + 1);
        ns[0] = f2_pack(-sa.x, -sa.y);
        ns[1] = f2_pack(-sa.z, -sa.w);
        ns[2] = f2_pack(-sb.x, -sb.y);
        ns[3] = f2_pack(-sb.z, -sb.w);
        rs[0] = f2_pack(__frcp_rn(sa.x), __frcp_rn(sa.y));
        rs[1] = f2_pack(__frcp_rn(sa.z), __frcp_rn(sa.w));
        rs[2] = f2_pack(__frcp_rn(sb.x), __frcp_rn(sb.y));
        rs[3] = f2_pack(__frcp_rn(sb.z), __frcp_rn(sb.w));
      }
      griddep_wait();  // the row scales of the previous kernel are visible
      griddep_launch_dependents();
      if (qt == 0) SQ_DEC_MARK(7);
      if (has) {
        const int j = qt >> 4;            // k-block of this vector within the slice
        const int c = (qt & 15) * 8;      // its first column within the k-block
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          if (m < p.M) {
            const float sc = __ldg(p.x_scale + m);
            const float rsc = __frcp_rn(sc);
            const f2x nsc2 = f2_pack(-sc, -sc), rsc2 = f2_pack(rsc, rsc);
            const f2x x[4] = {f2_from_bf16x2(xw[m].x), f2_from_bf16x2(xw[m].y), f2_from_bf16x2(xw[m].z),
                              f2_from_bf16x2(xw[m].w)};
            f2x cd[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) cd[e] = f2_round_codes(f2_div_rn(f2_div_rn(x[e], ns[e], rs[e]), nsc2, rsc2));
            *reinterpret_cast<uint2*>(asm_ + dec_a_offset(p.a_atoms, j, m, c)) = pack8_codes(cd[0], cd[1], cd[2], cd[3]);
          }
        }
      }
      // the generic-proxy shared-memory writes, visible to the tensor core
      fence_proxy_async_smem();
      named_bar_sync(1, 256);
      if (qt == 0) mbar_arrive(a_ready);
    } else {
      griddep_wait();
      griddep_launch_dependents();
    }

    // ----------------------- accumulator rows 0..M-1 to shared memory (warp 4)
    // warp 4 reads tensor-memory lanes 0..31: lane m holds token m's sums
    if (warp == 4) {
      bool have = my_nkb > 0;
      if (have) {
        const bool got = !*abort_flag && mbar_wait_bounded(acc_full, 0, p.timeout_ns);
        have = __all_sync(0xFFFFFFFFu, got);
        if (!have && lane == 0 && !*abort_flag) flag_timeout(abort_flag);
      }
      if (have) tc_fence_after();
      if (lane == 0) SQ_DEC_MARK(4);
#pragma unroll 1
      for (int c0 = 0; c0 < kDecRows; c0 += 32) {
        uint32_t r[32];
        if (have) {
          tmem_ld_32cols(tmem_base + static_cast<uint32_t>(c0), r);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = 0u;
        }
        if (lane < p.mp) {
#pragma unroll
          for (int i = 0; i < 32; ++i) mine[(c0 + i) * p.mp + lane] = lane < p.M ? static_cast<int32_t>(r[i]) : 0;
        }
      }
    }
    named_bar_sync(2, 256);
    // push the columns rank q reduces into rank q's slot for this sender
    {
      const int cpr = kDecRows / S;  // columns per rank
      const int col = qt;            // one column per thread
      const int owner = col / cpr;
      const uint32_t dst = mapa_shared(
          smem_u32(part + (static_cast<int>(rank) * cpr + (col - owner * cpr)) * p.mp), static_cast<uint32_t>(owner));
      const int4* src = reinterpret_cast<const int4*>(mine + col * p.mp);
      for (int i = 0; i < p.mp / 4; ++i) {
        const int4 v4 = src[i];
        asm volatile("st.shared::cluster.v4.s32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 16u * i), "r"(v4.x), "r"(v4.y),
                     "r"(v4.z), "r"(v4.w)
                     : "memory");
      }
    }
  }

  // ------------------------------------------- split-K reduction over the cluster
  tc_fence_before();
  __syncthreads();
  cluster_barrier_sync();  // every rank's pushes have landed
  if (threadIdx.x == 0) SQ_DEC_MARK(5);
  if (warp >= 2) {
    const int cpr = kDecRows / S;
    const int items = cpr * p.M;
    for (int it = threadIdx.x - 64; it < items; it += 256) {
      // consecutive threads: consecutive columns (outputs n) of one token
      const int lc = it % cpr;
      const int m = it / cpr;
      int32_t acc = 0;
      for (int r = 0; r < S; ++r) acc += part[(r * cpr + lc) * p.mp + m];
      const int n = rb * kDecRows + static_cast<int>(rank) * cpr + lc;
      if (n < p.N) {
        const float ws = __ldg(p.w_scale + n);
        const float b = p.bias != nullptr ? __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + n)) << 16) : 0.0f;
        const float y = __fmaf_rn(__int2float_rn(acc), __fmul_rn(__ldg(p.x_scale + m), ws), b);
        p.Y[static_cast<int64_t>(m) * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) SQ_DEC_MARK(6);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kDecTmemCols);
  }
}

// Per-token scale of X / s for few tokens, the pre-pass of the fused decode
// path: x_scale[m] = fl(max(max_j |fl(X[m][j] / s_j)|, 1e-8) / 127), the same
// correctly rounded fp32 operations as sq_quantize_act.  One block per token.
__global__ void __launch_bounds__(256) row_scale_kernel(const uint16_t* __restrict__ X, int K,
                                                        const float* __restrict__ s, float* __restrict__ x_scale) {
  __shared__ float red[8];
#ifdef SQ_TRACE
  if (threadIdx.x == 0) g_dec_trace[1023 - blockIdx.x][0] = globaltimer_ns();
#endif
  griddep_wait();
  // the decode GEMM may start streaming its weight now
  griddep_launch_dependents();
  const int nvec = K >> 3;
  const uint4* xr = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(blockIdx.x) * K);
  const float4* s4 = reinterpret_cast<const float4*>(s);
  float m = 0.0f;
  for (int v = threadIdx.x; v < nvec; v += 256) {
    const uint4 w = __ldg(xr + v);
    const float4 sa = __ldg(s4 + 2 * v), sb = __ldg(s4 + 2 * v + 1);
    const f2x ns[4] = {f2_pack(-sa.x, -sa.y), f2_pack(-sa.z, -sa.w), f2_pack(-sb.x, -sb.y), f2_pack(-sb.z, -sb.w)};
    const f2x rs[4] = {f2_pack(__frcp_rn(sa.x), __frcp_rn(sa.y)), f2_pack(__frcp_rn(sa.z), __frcp_rn(sa.w)),
                       f2_pack(__frcp_rn(sb.x), __frcp_rn(sb.y)), f2_pack(__frcp_rn(sb.z), __frcp_rn(sb.w))};
    const f2x x[4] = {f2_from_bf16x2(w.x), f2_from_bf16x2(w.y), f2_from_bf16x2(w.z), f2_from_bf16x2(w.w)};
#pragma unroll
    for (int e = 0; e < 4; ++e) m = f2_absmax(m, f2_div_rn(x[e], ns[e], rs[e]));
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
    m = fmaxf(m, red[0]);
    x_scale[blockIdx.x] = __fdiv_rn(fmaxf(m, kClampFloor), kQmax);
#ifdef SQ_TRACE
    g_dec_trace[1023 - blockIdx.x][1] = globaltimer_ns();
#endif
  }
}
