// Q-ARVD dual-scale W4A8 integer GEMM ("Q-ARVD: Autoregressive Video
// Diffusion Models의 양자화", Methodology and Technical details: Q_dual(W) =
// [Q_outlier(W_outliers) | Q_normal(W_normal)] with per-channel weight and
// per-tensor activation quantization).
//
// The activations arrive in the weights' channel order (normal channels,
// zero padding to 32, outlier channels, zero padding to 32), so each class
// is a contiguous, MMA-aligned K range and gets its own int32 accumulator:
//   Y[m, n] = bf16(s_x * (s_norm[n] * acc_normal[m, n] + s_out[n] * acc_outlier[m, n])).
// The MMA is tcgen05 kind::i8 (int32 accumulation, exact).  Two kernels:
//   k_gemm_qarvd_pre  weights kept as int8 (expand_i8): CTA pairs, both
//                     operands by TMA (described further down);
//   k_gemm_qarvd      INT4 weights widened on chip, below.
// Activations may carry INT8 or INT6 codes (W4A6); the product is the same.
//
// k_gemm_qarvd: persistent, warp-specialized, one CTA (512 threads) per SM:
//   warps 0-7   transform: INT4 nibbles -> sign-extended int8 in the
//               128-byte-swizzled K-major layout;
//   warp 8      TMA producer: int8 activations straight into the MMA layout
//               (128-byte swizzle), raw INT4 weight tiles;
//   warp 9      MMA issuer (each 32-wide K step goes to its class's accumulator);
//   warp 10     TMEM allocator (2 tiles x 2 classes x 128 columns = 512);
//   warps 12-15 epilogue (column scales staged in shared memory per tile).
#include "ql_common.cuh"
#include "gemm_common.cuh"
#include "launchers.h"

namespace ql {

template <int S>
struct QarvdCfg {
  static constexpr int BM = 128, BN = 128;
  static constexpr int BK = 128;                 // K bytes (= int8 elements) per stage
  static constexpr int CONV_A = BM * BK;         // int8, swizzled, written by TMA
  static constexpr int CONV_B = BN * BK;         // int8, swizzled, written by the transform
  static constexpr int RAW_B = BN * BK / 2;      // INT4
  static constexpr int OFF_CA = 0;
  static constexpr int OFF_CB = OFF_CA + S * CONV_A;
  static constexpr int OFF_C = OFF_CB + S * CONV_B;
  static constexpr int OFF_RB = OFF_C + 2 * kEpiChunkBytes;
  static constexpr int OFF_CS = OFF_RB + S * RAW_B;          // column scales: 2 x BN floats
  static constexpr int OFF_BAR = OFF_CS + 2 * BN * 4;
  static constexpr int NBAR = 4 * S + 2 * 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr int XFORM_THREADS = 256;
  static_assert(SMEM <= 232448, "shared memory budget");
  // kind::i8 descriptor: D = S32 (2 at bit 4), A = B = signed int8 (1),
  // K-major, N >> 3 at bit 17, M >> 4 at bit 24.
  static constexpr uint32_t IDESC =
      (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
};

// Eight two's-complement nibbles (byte j: elements 2j low, 2j+1 high) ->
// eight int8 in element order.
__device__ __forceinline__ uint2 int4x8_to_int8(uint32_t w) {
  uint32_t lo = w & 0x0F0F0F0Fu;             // elements 0, 2, 4, 6
  uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;      // elements 1, 3, 5, 7
  lo |= (lo & 0x08080808u) * 0x1Eu;          // sign-extend: bit 3 -> bits 4..7
  hi |= (hi & 0x08080808u) * 0x1Eu;
  return make_uint2(__byte_perm(lo, hi, 0x5140u), __byte_perm(lo, hi, 0x7362u));
}

__device__ __forceinline__ uint32_t sw128q(uint32_t r, uint32_t c) {
  return r * 128u + ((c ^ (r & 7u)) << 4);
}

__device__ __forceinline__ bool warp_wait2q(uint64_t* a, uint32_t pa, uint64_t* b, uint32_t pb,
                                            long long limit, volatile int* abort_flag) {
  int ok = 0;
  if (lane_id() == 0)
    ok = (*abort_flag == 0) && mbar_wait(a, pa, limit) && mbar_wait(b, pb, limit);
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

template <int S>
__global__ void __launch_bounds__(512, 1)
    k_gemm_qarvd(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const __grid_constant__ CUtensorMap tm_y, const GemmArgs p) {
  using C = QarvdCfg<S>;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);     // A (TMA) + raw B (TMA)
  uint64_t* raw_empty = full + S;                                     // transform done with raw B
  uint64_t* conv_full = raw_empty + S;                                // transform wrote B
  uint64_t* empty = conv_full + S;                                    // MMA done with the stage
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  pdl_wait();   // before the first global access
  // Class sizes (device-resident, written by the weight preparation).
  const int k_norm_pad = p.kinfo[1];
  const int k_out_pad = p.kinfo[3];
  const int k_used = k_norm_pad + k_out_pad;
  const int num_kst = (k_used + C::BK - 1) / C::BK;

  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_y);
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&raw_empty[i], C::XFORM_THREADS / 32);
      mbar_init(&conv_full[i], C::XFORM_THREADS / 32);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 10) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 8) {
    // ------------------------------------------------------------ transform
    const uint32_t tid = threadIdx.x;
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
      for (int ks = 0; ks < num_kst; ++ks, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        // raw B landed (full) and the MMA is done with this stage's B (empty)
        if (!warp_wait2q(&full[s], ph, &empty[s], ph ^ 1, p.wait_limit, abort_flag)) {
          ok = false;
          break;
        }
        const uint8_t* rb = smem + C::OFF_RB + s * C::RAW_B;
        uint8_t* cb = smem + C::OFF_CB + s * C::CONV_B;
#pragma unroll
        for (int i = 0; i < 4; ++i) {   // BN rows x 8 chunks of 16 int8 (8 raw bytes)
          const uint32_t idx = tid + C::XFORM_THREADS * i;
          const uint32_t r = idx >> 3, c = idx & 7u;
          const uint2 q = *reinterpret_cast<const uint2*>(rb + idx * 8);
          const uint2 a = int4x8_to_int8(q.x);
          const uint2 b = int4x8_to_int8(q.y);
          *reinterpret_cast<uint4*>(cb + sw128q(r, c)) = make_uint4(a.x, a.y, b.x, b.y);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane_id() == 0) {
          mbar_arrive(&raw_empty[s]);
          mbar_arrive(&conv_full[s]);
        }
      }
    }
    if (!ok && lane_id() == 0) fail_timeout(p.status, abort_flag);
  } else if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        for (int ks = 0; ks < num_kst; ++ks, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          // the MMA is done with A (empty) and the transform with raw B (raw_empty)
          if (*abort_flag || !mbar_wait(&empty[s], ph ^ 1, p.wait_limit) ||
              !mbar_wait(&raw_empty[s], ph ^ 1, p.wait_limit)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], C::CONV_A + C::RAW_B);
          tma_load_2d(smem + C::OFF_CA + s * C::CONV_A, &tm_a, &full[s], ks * C::BK, mb * C::BM);
          tma_load_2d(smem + C::OFF_RB + s * C::RAW_B, &tm_b, &full[s], ks * (C::BK / 2), nb * BN);
        }
      }
      if (!ok) fail_timeout(p.status, abort_flag);
      drain_loads(full, it, S, p.status);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      int it = 0, local = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t aph = (local >> 1) & 1;
        if (*abort_flag || !mbar_wait(&tempty[acc], aph ^ 1, p.wait_limit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_norm = tmem + acc * 2 * BN;
        const uint32_t d_out = d_norm + BN;
        bool started_norm = false, started_out = false;
        for (int ks = 0; ks < num_kst; ++ks, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (*abort_flag || !mbar_wait(&conv_full[s], ph, p.wait_limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + C::OFF_CA + s * C::CONV_A);
          const uint32_t b_base = smem_u32(smem + C::OFF_CB + s * C::CONV_B);
#pragma unroll
          for (int i = 0; i < C::BK / 32; ++i) {
            const int kk = ks * C::BK + 32 * i;
            if (kk >= k_used) break;
            const bool normal = kk < k_norm_pad;
            const uint64_t adesc = smem_desc(a_base + 32 * i, 0, 1024, kSwizzle128B);
            const uint64_t bdesc = smem_desc(b_base + 32 * i, 0, 1024, kSwizzle128B);
            tc_mma_i8(normal ? d_norm : d_out, adesc, bdesc, C::IDESC,
                      (normal ? started_norm : started_out) ? 1u : 0u);
            if (normal) started_norm = true; else started_out = true;
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
      }
      if (!ok) fail_timeout(p.status, abort_flag);
      drain_mma(drain, p.status);
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ epilogue
    const float sx = ld_dep(p.g_a);
    const int ew = warp & 3;
    const int lane = lane_id();
    const int row = threadIdx.x & 127;
    float* cs = reinterpret_cast<float*>(smem + C::OFF_CS);
    EpilogueState es{};
    int local = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++local) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int acc = local & 1;
      const uint32_t aph = (local >> 1) & 1;
      // column scales of this tile (columns past N read as 0)
      const int n = nb * BN + row;
      const float sn = (n < p.N) ? __ldg(p.col_scale0 + n) : 0.f;
      const float so = (n < p.N) ? __ldg(p.col_scale1 + n) : 0.f;
      if (!epilogue_wait_uniform(&tfull[acc], aph, p.wait_limit, abort_flag, p.status)) break;
      cs[row] = sn;           // safe: the previous tile's readers passed the barrier above
      cs[BN + row] = so;
      named_bar_sync(1, 128);
      tc_fence_after();
      const uint32_t base = tmem + acc * 2 * BN + (static_cast<uint32_t>(ew * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < BN / kEpiChunkCols; ++c) {
        uint32_t packed[32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t an[32], ao[32];
          const uint32_t col = c * kEpiChunkCols + h * 32;
          tmem_ld32(base + col, an);
          tmem_ld32(base + BN + col, ao);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float y[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int jj = 2 * j + e;
              const float fn = k_norm_pad ? static_cast<float>(static_cast<int32_t>(an[jj])) : 0.f;
              const float fo = k_out_pad ? static_cast<float>(static_cast<int32_t>(ao[jj])) : 0.f;
              const float v = __fadd_rn(__fmul_rn(cs[col + jj], fn), __fmul_rn(cs[BN + col + jj], fo));
              y[e] = __fmul_rn(sx, v);
            }
            packed[16 * h + j] = pack_bf16x2(y[0], y[1]);
          }
        }
        if (c == BN / kEpiChunkCols - 1) {
          tc_fence_before();
          if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        if (nb * BN + c * kEpiChunkCols < p.N)
          epilogue_store_chunk(packed, smem + C::OFF_C, &tm_y, nb * BN + c * kEpiChunkCols, mb * C::BM, es);
      }
    }
    epilogue_finish(es);
  }

  pdl_release();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 10) tmem_dealloc(tmem, 512);
}

// --------------------------------------------------------------------------
// Weights kept as int8 (prepared with expand_i8): both operands come by TMA
// in the 128-byte-swizzled K-major layout and no warp touches them.
//
// 384 threads per CTA, one CTA per SM, the W4A4 kernel's roles:
//   warp 0      TMA producer;
//   warp 1      MMA issuer (kind::i8, each 32-wide K step to its class's
//               accumulator);
//   warp 2      tensor-memory allocation;
//   warps 4-11  epilogue, two warps per TMEM lane quarter, each with about
//               half of the tile's 32-column boxes, stored by TMA.
//   PAIR = true   two SMs of a cluster share each 256 x BN tile through
//                 tcgen05 cta_group::2 (each CTA holds its 128 activation
//                 rows and BN/2 of the weight rows); the leader issues.
//   PAIR = false  one SM per 128 x BN tile (M <= 128).
// Tensor memory (512 columns): two tiles x two class accumulators of BN
// columns.  A stage holds BK bytes of K as BK/128 chunks of one 128-byte
// swizzle span each; with BK = 256 a stage feeds eight MMAs, which halves
// the barrier round trips per MMA against BK = 128 (measured 15-18% faster
// on the CogVideoX-5B linears with the same shared-memory depth).
// --------------------------------------------------------------------------
template <bool PAIR, int STAGES, int BN_, int BK_>
struct QarvdPreCfg {
  static constexpr int CTAS = PAIR ? 2 : 1;
  static constexpr int BM = 128;              // activation rows per CTA
  static constexpr int BN = BN_;              // tile columns (MMA N)
  static constexpr int BNL = BN / CTAS;       // weight rows held by each CTA
  static constexpr int BK = BK_;              // K bytes (= int8 elements) per stage
  static constexpr int KC = BK / 128;         // 128-byte K chunks (one swizzle span) per stage
  static constexpr int A_CHUNK = BM * 128;    // one chunk: rows x 128 bytes, 128-byte swizzle
  static constexpr int B_CHUNK = BNL * 128;
  static constexpr int A_BYTES = KC * A_CHUNK;
  static constexpr int B_BYTES = KC * B_CHUNK;
  static constexpr int EPI_WARPS = 8;
  static constexpr int EPI_BUF = 2;
  static constexpr int NBOX = BN / kWarpBoxCols;     // 32-column boxes per tile row
  static constexpr int BOX0 = (NBOX + 1) / 2;        // boxes of the first column half
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_C = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_BAR = OFF_C + EPI_WARPS * EPI_BUF * kWarpBoxBytes;
  static constexpr int NBAR = 2 * STAGES + 2 * 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(B_CHUNK % 1024 == 0 && BK % 128 == 0, "1024-byte aligned chunks");
  static_assert(BN % kWarpBoxCols == 0 && BN % 16 == 0 && 4 * BN <= 512, "tile width");
  static constexpr uint32_t IDESC = (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) |
                                    (uint32_t((BM * CTAS) >> 4) << 24);
};

template <bool PAIR, int STAGES, int BN_, int BK_>
__global__ void __launch_bounds__(384, 1)
    k_gemm_qarvd_pre(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_y, const GemmArgs p) {
  using C = QarvdPreCfg<PAIR, STAGES, BN_, BK_>;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);   // pair: the leader's is used
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;                                     // pair: the leader's is used
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  pdl_wait();   // before the first global access
  const int k_norm_pad = p.kinfo[1];
  const int k_out_pad = p.kinfo[3];
  const int k_used = k_norm_pad + k_out_pad;
  const int num_kst = (k_used + C::BK - 1) / C::BK;

  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5;
  const int unit = PAIR ? (blockIdx.x >> 1) : blockIdx.x;
  const int nunits = PAIR ? (gridDim.x >> 1) : gridDim.x;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_y);
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], C::EPI_WARPS * C::CTAS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if constexpr (PAIR) cluster_sync();   // both CTAs' barriers exist before any remote use
  if (warp == 2) {
    if constexpr (PAIR)
      tmem_alloc_pair(tmem_slot, 512);
    else
      tmem_alloc(tmem_slot, 512);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      int it = 0;
      bool ok = true;
      constexpr uint32_t tx = C::A_BYTES + C::B_BYTES;
      for (int t = unit; t < p.num_tiles && ok; t += nunits) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        const int a_row = mb * C::BM * C::CTAS + static_cast<int>(rank) * C::BM;
        const int b_row = nb * BN + static_cast<int>(rank) * C::BNL;
        for (int ks = 0; ks < num_kst; ++ks, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (*abort_flag || !mbar_wait(&empty[s], ph ^ 1, p.wait_limit)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + C::OFF_A + s * C::A_BYTES;
          uint8_t* sb = smem + C::OFF_B + s * C::B_BYTES;
          if constexpr (PAIR) {
            // Both CTAs' bytes complete on the leader's barrier.
            if (leader) mbar_arrive_expect_tx(&full[s], 2 * tx);
            const uint32_t bar = map_to_rank(smem_u32(&full[s]), 0);
#pragma unroll
            for (int c = 0; c < C::KC; ++c) {
              tma_load_2d_pair(sa + c * C::A_CHUNK, &tm_a, bar, ks * C::BK + 128 * c, a_row);
              tma_load_2d_pair(sb + c * C::B_CHUNK, &tm_b, bar, ks * C::BK + 128 * c, b_row);
            }
          } else {
            mbar_arrive_expect_tx(&full[s], tx);
#pragma unroll
            for (int c = 0; c < C::KC; ++c) {
              tma_load_2d(sa + c * C::A_CHUNK, &tm_a, &full[s], ks * C::BK + 128 * c, a_row);
              tma_load_2d(sb + c * C::B_CHUNK, &tm_b, &full[s], ks * C::BK + 128 * c, b_row);
            }
          }
        }
      }
      if (!ok) fail_timeout(p.status, abort_flag);
      if (leader) {
        drain_loads(full, it, STAGES, p.status);   // pair: covers both CTAs' bytes
      } else {
        // The peer's loads complete on the leader's barriers; the leader frees
        // each stage (empty) only after the MMAs consumed both halves.
        for (int j = max(0, it - STAGES); j < it; ++j)
          if (!mbar_wait(&empty[j % STAGES], (j / STAGES) & 1, kDrainLimit)) record_error(p.status, QL_ERR_TIMEOUT);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (leader && elect_one()) {
      int it = 0, local = 0;
      bool ok = true;
      auto commit_to = [&](uint64_t* bar) {
        if constexpr (PAIR) {
          tc_commit_pair(map_to_rank(smem_u32(bar), 0));
          tc_commit_pair(map_to_rank(smem_u32(bar), 1));
        } else {
          tc_commit(bar);
        }
      };
      for (int t = unit; t < p.num_tiles && ok; t += nunits, ++local) {
        const int acc = local & 1;
        if (*abort_flag || !mbar_wait(&tempty[acc], ((local >> 1) & 1) ^ 1, p.wait_limit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_norm = tmem + acc * 2 * BN;
        const uint32_t d_out = d_norm + BN;
        bool started_norm = false, started_out = false;
        for (int ks = 0; ks < num_kst; ++ks, ++it) {
          const int s = it % STAGES;
          if (*abort_flag || !mbar_wait(&full[s], (it / STAGES) & 1, p.wait_limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + C::OFF_A + s * C::A_BYTES);
          const uint32_t b_base = smem_u32(smem + C::OFF_B + s * C::B_BYTES);
#pragma unroll
          for (int i = 0; i < C::BK / 32; ++i) {
            const int kk = ks * C::BK + 32 * i;
            if (kk >= k_used) break;
            const bool normal = kk < k_norm_pad;
            const uint32_t koff = 32 * (i & 3);
            const uint64_t adesc = smem_desc(a_base + (i >> 2) * C::A_CHUNK + koff, 0, 1024, kSwizzle128B);
            const uint64_t bdesc = smem_desc(b_base + (i >> 2) * C::B_CHUNK + koff, 0, 1024, kSwizzle128B);
            const uint32_t accum = (normal ? started_norm : started_out) ? 1u : 0u;
            if constexpr (PAIR)
              tc_mma_i8_pair(normal ? d_norm : d_out, adesc, bdesc, C::IDESC, accum);
            else
              tc_mma_i8(normal ? d_norm : d_out, adesc, bdesc, C::IDESC, accum);
            if (normal) started_norm = true; else started_out = true;
          }
          commit_to(&empty[s]);
        }
        if (!ok) break;
        commit_to(&tfull[acc]);
      }
      if (!ok) fail_timeout(p.status, abort_flag);
      if constexpr (PAIR) {
        tc_commit_pair(map_to_rank(smem_u32(drain), 0));
        if (!mbar_wait(drain, 0, kDrainLimit)) record_error(p.status, QL_ERR_TIMEOUT);
      } else {
        drain_mma(drain, p.status);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    // y = bf16(s_x * (s_norm[n] * acc_normal + s_out[n] * acc_outlier)); a
    // class without channels contributes 0 (its accumulator is never written).
    const float sx = ld_dep(p.g_a);
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    const int lane = lane_id();
    const bool has_norm = k_norm_pad != 0, has_out = k_out_pad != 0;
    const int box0 = half ? C::BOX0 : 0;                      // first box of this warp
    const int nbox = half ? C::NBOX - C::BOX0 : C::BOX0;      // boxes of this warp
    uint8_t* stage = smem + C::OFF_C + (warp - 4) * C::EPI_BUF * kWarpBoxBytes;
    const uint32_t swz = (lane >> 1) & 3;
    int next_buf = 0;
    int local = 0;
    for (int t = unit; t < p.num_tiles; t += nunits, ++local) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int acc = local & 1;
      const int row0 = mb * C::BM * C::CTAS + static_cast<int>(rank) * C::BM + 32 * quarter;
      const int c0 = nb * BN + box0 * kWarpBoxCols;
      // lane i holds the scales of column c0 + 32 c + i (0 past N)
      float sn[C::BOX0], so[C::BOX0];
#pragma unroll
      for (int c = 0; c < C::BOX0; ++c) {
        const int n = c0 + kWarpBoxCols * c + lane;
        const bool in = c < nbox && n < p.N;
        sn[c] = in ? __ldg(p.col_scale0 + n) : 0.f;
        so[c] = in ? __ldg(p.col_scale1 + n) : 0.f;
      }
      if (!warp_wait_uniform(&tfull[acc], (local >> 1) & 1, p.wait_limit, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t release = PAIR ? map_to_rank(smem_u32(&tempty[acc]), 0) : smem_u32(&tempty[acc]);
      const uint32_t lanes = static_cast<uint32_t>(32 * quarter) << 16;
      const uint32_t t_norm = tmem + acc * 2 * BN + box0 * kWarpBoxCols + lanes;
      const uint32_t t_out = t_norm + BN;
      uint32_t packed[C::BOX0][16];
#pragma unroll
      for (int c = 0; c < C::BOX0; ++c) {
        if (c < nbox) {   // warp-uniform
          uint32_t an[32], ao[32];
          tmem_ld32(t_norm + kWarpBoxCols * c, an);
          tmem_ld32(t_out + kWarpBoxCols * c, ao);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float y[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int jj = 2 * j + e;
              const float fn = has_norm ? static_cast<float>(static_cast<int32_t>(an[jj])) : 0.f;
              const float fo = has_out ? static_cast<float>(static_cast<int32_t>(ao[jj])) : 0.f;
              const float cn = __shfl_sync(0xffffffffu, sn[c], jj);
              const float co = __shfl_sync(0xffffffffu, so[c], jj);
              y[e] = __fmul_rn(sx, __fadd_rn(__fmul_rn(cn, fn), __fmul_rn(co, fo)));
            }
            packed[c][j] = pack_bf16x2(y[0], y[1]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(release);
      if (row0 >= p.M) continue;   // warp-uniform
#pragma unroll
      for (int c = 0; c < C::BOX0; ++c) {
        const int col = c0 + kWarpBoxCols * c;
        if (c >= nbox || col >= p.N) break;   // warp-uniform; TMA clips partial boxes
        uint8_t* buf = stage + next_buf * kWarpBoxBytes;
        if (lane == 0) bulk_wait_read<C::EPI_BUF - 1>();
        __syncwarp();
        uint8_t* dst = buf + lane * 64;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(dst + ((q ^ swz) << 4)) =
              make_uint4(packed[c][4 * q], packed[c][4 * q + 1], packed[c][4 * q + 2], packed[c][4 * q + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_y, buf, col, row0);
          bulk_commit();
        }
        next_buf = (next_buf + 1 == C::EPI_BUF) ? 0 : next_buf + 1;
      }
    }
    epilogue_warp_finish();
  }

  pdl_release();
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();   // no CTA leaves while its peer may still signal it
  tc_fence_after();
  if (warp == 2) {
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem, 512);
    else
      tmem_dealloc(tmem, 512);
  }
}

template <bool PAIR, int STAGES, int BN_, int BK_>
static ql_status launch_qarvd_pre(const void* a_codes, const float* s_x, int64_t M, const ql_weights* w, void* Y,
                                  cudaStream_t st, int* status) {
  using C = QarvdPreCfg<PAIR, STAGES, BN_, BK_>;
  const int N = w->N, Kp = w->Kp;
  CUtensorMap ta, tb, ty;
  if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, Kp, M, Kp, 128, C::BM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->w8, Kp, N, Kp, 128, C::BNL,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, N, M, static_cast<int64_t>(N) * 2,
                    kWarpBoxCols, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return QL_ERR_CUDA;
  GemmArgs p{};
  fill_gemm_args(p, M, N, Kp, C::BN, status);
  p.tiles_m = static_cast<int32_t>((M + C::BM * C::CTAS - 1) / (C::BM * C::CTAS));
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.g_a = s_x;
  p.col_scale0 = w->s_norm;
  p.col_scale1 = w->s_out;
  p.kinfo = w->kinfo;
  auto kern = k_gemm_qarvd_pre<PAIR, STAGES, BN_, BK_>;
  if (!set_smem_attr(reinterpret_cast<const void*>(kern), C::SMEM)) return QL_ERR_CUDA;
  const int units = std::min(p.num_tiles, num_sms() / C::CTAS);
  if (launch_pdl(kern, dim3(static_cast<unsigned>(units * C::CTAS)), dim3(384), C::SMEM, st, C::CTAS, ta, tb, ty,
                 p) != cudaSuccess) {
    (void)cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

// Sign-extend the packed INT4 weight codes to int8 ([N, Kp/2] bytes ->
// [N, Kp] int8), 8 bytes per thread.
__global__ void k_expand_int4_i8(const uint2* __restrict__ in, uint4* __restrict__ out, int64_t n8) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint2 q = in[i];
    const uint2 a = int4x8_to_int8(q.x);
    const uint2 b = int4x8_to_int8(q.y);
    out[i] = make_uint4(a.x, a.y, b.x, b.y);
  }
}

ql_status launch_expand_int4_i8(const void* codes, int32_t N, int32_t Kp, void* out, cudaStream_t st) {
  const int64_t n8 = static_cast<int64_t>(N) * Kp / 16;   // 8-byte groups (Kp % 32 == 0)
  const int grid = hbm_grid(n8, 256 * 4);
  k_expand_int4_i8<<<grid, 256, 0, st>>>(static_cast<const uint2*>(codes), static_cast<uint4*>(out), n8);
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

ql_status launch_gemm_qarvd(const void* a_codes, const float* s_x, int64_t M, const ql_weights* w, void* Y,
                            cudaStream_t st, int* status) {
  if (M == 0) return QL_OK;
  if (w->w8 != nullptr) {
    if (M > 128) return launch_qarvd_pre<true, 4, 128, 256>(a_codes, s_x, M, w, Y, st, status);
    return launch_qarvd_pre<false, 5, 128, 128>(a_codes, s_x, M, w, Y, st, status);
  }
  constexpr int S = 4;
  using C = QarvdCfg<S>;
  const int N = w->N, Kp = w->Kp;
  CUtensorMap ta, tb, ty;
  if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, Kp, M, Kp, C::BK, C::BM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, Kp / 2, N, Kp / 2, C::BK / 2, C::BN,
                    CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, N, M, static_cast<int64_t>(N) * 2, 64, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return QL_ERR_CUDA;
  GemmArgs p{};
  fill_gemm_args(p, M, N, Kp, C::BN, status);
  p.g_a = s_x;
  p.col_scale0 = w->s_norm;
  p.col_scale1 = w->s_out;
  p.kinfo = w->kinfo;
  auto kern = k_gemm_qarvd<S>;
  if (!set_smem_attr(reinterpret_cast<const void*>(kern), C::SMEM)) return QL_ERR_CUDA;
  const int grid = std::min(p.num_tiles, num_sms());
  if (launch_pdl(kern, dim3(grid), dim3(512), C::SMEM, st, 1, ta, tb, ty, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

}  // namespace ql
