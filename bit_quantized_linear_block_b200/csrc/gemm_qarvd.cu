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
//   k_gemm_qarvd_ts   INT4 weights widened on chip into tensor memory as the
//                     MMA's A operand (described further down);
//   k_gemm_qarvd_pre  weights kept as int8 (expand_i8): CTA pairs, both
//                     operands by TMA (described further down).
// Activations may carry INT8 or INT6 codes (W4A6); the product is the same.
#include "ql_common.cuh"
#include "gemm_common.cuh"
#include "launchers.h"

namespace ql {

// Eight two's-complement nibbles (byte j: elements 2j low, 2j+1 high) ->
// eight int8 in element order (the int8 weight copy).
__device__ __forceinline__ uint2 int4x8_to_int8(uint32_t w) {
  uint32_t lo = w & 0x0F0F0F0Fu;             // elements 0, 2, 4, 6
  uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;      // elements 1, 3, 5, 7
  lo |= (lo & 0x08080808u) * 0x1Eu;          // sign-extend: bit 3 -> bits 4..7
  hi |= (hi & 0x08080808u) * 0x1Eu;
  return make_uint2(__byte_perm(lo, hi, 0x5140u), __byte_perm(lo, hi, 0x7362u));
}

__device__ __forceinline__ bool warp_wait2q(uint64_t* a, uint32_t pa, uint64_t* b, uint32_t pb,
                                            long long limit, volatile int* abort_flag) {
  int ok = 0;
  if (lane_id() == 0)
    ok = (*abort_flag == 0) && mbar_wait(a, pa, limit) && mbar_wait(b, pb, limit);
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
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

// ---------------------------------------------------------------------------
// INT4 weights without the int8 copy, as the MMA's A operand in tensor
// memory: the widened weights never pass through shared memory.  The tile is
// transposed, D_c[n, m] = sum_{k in class c} 16 W[n, k] q[m, k]: 128 weight
// rows on the TMEM lanes (the MMA's M), 128 tokens as the MMA's N.
//
// Widening: a nibble moved to the high half of its byte is the int8 value
// 16 w (the nibble's sign bit lands on the byte's), so one mask, one shift
// and two byte permutes widen eight codes; the accumulators hold 16 x the
// integer sums (|16 acc| < 2^31 for K <= 16384), and the epilogue shifts the
// factor out exactly before the oracle's rounding order
// s_x (s_norm[n] acc_n + s_out[n] acc_o).
//
// Persistent, one CTA (512 to 768 threads) per SM, weight tiles fastest:
//   warp 0      TMA producer: int8 activation tile (128 tokens x 128 K bytes,
//               128-byte swizzle) and INT4 weight tile (128 rows x 64 bytes);
//   warp 1      TMEM allocator and MMA issuer (kind::i8, 128 x 128 x 32, A
//               from tensor memory; each 32-deep K step goes to its class);
//   4 XG transform warps (from warp 4), XG groups of four: group g widens
//               the stages it with it % XG == g; lane l of warp w owns weight
//               row 32 (w % 4) + l and writes its 128 widened K bytes of a
//               stage into one of four 32-column A slots with tcgen05.st;
//   8 epilogue warps: a TMEM lane quarter and half of the 128 token columns
//               each; y stored in 32 x 32 boxes (tokens x weight rows) by TMA.
// Tensor memory: normal-class accumulators for two tiles (0-255), ONE
// outlier-class accumulator (256-383) and the A slots (384-511).  The
// outlier K steps come last in a tile, so the MMA waits for the previous
// tile's epilogue to release the outlier accumulator only when it reaches
// them, while that epilogue has had the whole normal class to run.
// ---------------------------------------------------------------------------
template <int RS, int XG>
struct QarvdTsCfg {
  static constexpr int BMT = 128;                  // tokens per tile (MMA N)
  static constexpr int BK = 128;                   // K bytes (int8 elements) per stage
  static constexpr int AS = 4;                     // A slots of 32 columns
  static constexpr int ACC_OUT = 2 * BMT;          // outlier accumulator column
  static constexpr int A_COL = 3 * BMT;            // first A slot column
  static constexpr int B_BYTES = BMT * BK;         // int8 activations, 128-byte rows
  static constexpr int W_BYTES = 128 * BK / 2;     // INT4 codes, 64 bytes per weight row
  static constexpr int OFF_B = 0;
  static constexpr int OFF_W = OFF_B + RS * B_BYTES;
  static constexpr int OFF_C = OFF_W + RS * W_BYTES;       // 8 epilogue warps x 2 staging boxes
  static constexpr int OFF_BAR = OFF_C + 8 * 2 * kWarpBoxBytes;
  static constexpr int NBAR = 2 * RS + 2 * AS + 2 * 2 + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr int EPI0 = 4 + 4 * XG;
  static constexpr int THREADS = (EPI0 + 8) * 32;
  static constexpr int EPI_CH = BMT / 2 / 32;
  static_assert(XG >= 1 && XG <= 3, "transform warp groups");
  static_assert(A_COL + 32 * AS <= 512, "tensor memory budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  // kind::i8: D = S32 (2 at bit 4), A = B = signed int8, K-major, N = BMT, M = 128
  static constexpr uint32_t IDESC =
      (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(BMT >> 3) << 17) | (uint32_t(128 >> 4) << 24);
};

// Eight two's-complement nibbles (byte j: elements 2j low, 2j+1 high) ->
// eight int8 = 16 x the codes, in element order.
__device__ __forceinline__ uint2 int4x8_to_int8_x16(uint32_t w) {
  const uint32_t hi = w & 0xF0F0F0F0u;           // 16 e1, 16 e3, 16 e5, 16 e7
  const uint32_t lo = (w << 4) & 0xF0F0F0F0u;    // 16 e0, 16 e2, 16 e4, 16 e6
  return make_uint2(__byte_perm(lo, hi, 0x5140u), __byte_perm(lo, hi, 0x7362u));
}

template <int RS, int XG>
__global__ void __launch_bounds__(QarvdTsCfg<RS, XG>::THREADS, 1)
    k_gemm_qarvd_ts(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                    const __grid_constant__ CUtensorMap tm_y, const GemmArgs p) {
  using C = QarvdTsCfg<RS, XG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* raw_empty = raw_full + RS;
  uint64_t* xf_full = raw_empty + RS;
  uint64_t* xf_empty = xf_full + C::AS;
  uint64_t* tfull = xf_empty + C::AS;
  uint64_t* tempty = tfull + 2;
  uint64_t* out_empty = tempty + 2;
  uint64_t* drain = out_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = lane_id();
  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_y);
    for (int i = 0; i < RS; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], 1);   // the stage's MMA commit (issued after the transform read it)
    }
    for (int i = 0; i < C::AS; ++i) {
      mbar_init(&xf_full[i], 4);     // the four transform warps of the stage's group
      mbar_init(&xf_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 8);
    }
    mbar_init(out_empty, 8);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t a_slots = tmem + C::A_COL;
  pdl_wait();   // before the first global access
  // class sizes (device-resident, written by the weight preparation)
  const int k_norm_pad = p.kinfo[1];
  const int k_out_pad = p.kinfo[3];
  const int k_used = k_norm_pad + k_out_pad;
  const int num_kst = (k_used + C::BK - 1) / C::BK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        const int mb = t / p.tiles_n, nb = t - (t / p.tiles_n) * p.tiles_n;
        for (int ks = 0; ks < num_kst; ++ks, ++it) {
          const int s = it % RS;
          if (*abort_flag || !mbar_wait(&raw_empty[s], ((it / RS) & 1) ^ 1, p.wait_limit)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&raw_full[s], C::B_BYTES + C::W_BYTES);
          tma_load_2d(smem + C::OFF_B + s * C::B_BYTES, &tm_x, &raw_full[s], ks * C::BK, mb * C::BMT);
          tma_load_2d(smem + C::OFF_W + s * C::W_BYTES, &tm_w, &raw_full[s], ks * (C::BK / 2), nb * 128);
        }
      }
      if (!ok) fail_timeout(p.status, abort_flag);
      drain_loads(raw_full, it, RS, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      int it = 0, local = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++local) {
        const int acc = local & 1;
        if (*abort_flag || !mbar_wait(&tempty[acc], ((local >> 1) & 1) ^ 1, p.wait_limit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_norm = tmem + acc * C::BMT;
        const uint32_t d_out = tmem + C::ACC_OUT;
        bool started_norm = false, started_out = false;
        for (int ks = 0; ks < num_kst && ok; ++ks, ++it) {
          const int rs = it % RS, sl = it % C::AS;
          if (*abort_flag || !mbar_wait(&raw_full[rs], (it / RS) & 1, p.wait_limit) ||
              !mbar_wait(&xf_full[sl], (it / C::AS) & 1, p.wait_limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b_base = smem_u32(smem + C::OFF_B + rs * C::B_BYTES);
#pragma unroll
          for (int i = 0; i < C::BK / 32; ++i) {
            const int kk = ks * C::BK + 32 * i;
            if (kk >= k_used) break;
            const bool normal = kk < k_norm_pad;
            if (!normal && !started_out && local > 0) {
              // the previous tile's epilogue must have read the outlier accumulator
              if (!mbar_wait(out_empty, (local - 1) & 1, p.wait_limit)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            tc_mma_i8_ts(normal ? d_norm : d_out, a_slots + 32 * sl + 8 * i,
                         smem_desc(b_base + 32 * i, 0, 1024, kSwizzle128B), C::IDESC,
                         (normal ? started_norm : started_out) ? 1u : 0u);
            if (normal) started_norm = true; else started_out = true;
          }
          tc_commit(&raw_empty[rs]);
          tc_commit(&xf_empty[sl]);
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
      }
      if (!ok) fail_timeout(p.status, abort_flag);
      drain_mma(drain, p.status);
    }
  } else if (warp >= 4 && warp < C::EPI0) {
    // ------------------------------------------------------------ transform
    const uint32_t q = static_cast<uint32_t>(warp & 3);
    const uint32_t row = 32 * q + lane;
    const int group = (warp - 4) >> 2;    // widens the stages it with it % XG == group
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
      for (int ks = 0; ks < num_kst; ++ks, ++it) {
        if (it % XG != group) continue;
        const int rs = it % RS, sl = it % C::AS;
        if (!warp_wait2q(&raw_full[rs], (it / RS) & 1, &xf_empty[sl], ((it / C::AS) & 1) ^ 1, p.wait_limit,
                         abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint4* wr = reinterpret_cast<const uint4*>(smem + C::OFF_W + rs * C::W_BYTES + row * (C::BK / 2));
        uint32_t v[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {   // 16 bytes = 32 codes -> 8 words
          const uint4 r = wr[c];
          const uint32_t cw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint2 o = int4x8_to_int8_x16(cw[j]);
            v[8 * c + 2 * j] = o.x;
            v[8 * c + 2 * j + 1] = o.y;
          }
        }
        tmem_st32(a_slots + ((32 * q) << 16) + 32 * sl, v);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&xf_full[sl]);
      }
    }
    if (!ok && lane == 0) fail_timeout(p.status, abort_flag);
  } else if (warp >= C::EPI0) {
    // ------------------------------------------------------------ epilogue
    const uint32_t q = static_cast<uint32_t>(warp & 3);
    const int half = (warp - C::EPI0) >> 2;
    const float sx = ld_dep(p.g_a);
    uint8_t* stage = smem + C::OFF_C + (warp - C::EPI0) * 2 * kWarpBoxBytes;
    int next = 0, local = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++local) {
      const int mb = t / p.tiles_n, nb = t - (t / p.tiles_n) * p.tiles_n;
      const int acc = local & 1;
      const int n0 = nb * 128 + 32 * static_cast<int>(q);   // this warp's weight rows = output columns
      const int n = n0 + static_cast<int>(lane);
      const float sn = (n < p.N) ? __ldg(p.col_scale0 + n) : 0.f;
      const float so = (n < p.N) ? __ldg(p.col_scale1 + n) : 0.f;
      if (!warp_wait_uniform(&tfull[acc], (local >> 1) & 1, p.wait_limit, abort_flag, p.status)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < C::EPI_CH; ++c) {
        const int col = half * (C::BMT / 2) + 32 * c;
        const int m0 = mb * C::BMT + col;
        const bool inside = m0 < p.M && n0 < p.N;   // warp-uniform: else the box is outside Y
        uint8_t* buf = stage + next * kWarpBoxBytes;
        if (inside) {
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
        }
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(buf) + lane;
#pragma unroll
        for (int h = 0; h < 2; ++h) {   // 16 columns at a time (registers)
          uint32_t an[16], ao[16];
          tmem_ld16(tmem + ((32 * q) << 16) + acc * C::BMT + col + 16 * h, an);
          if (k_out_pad) tmem_ld16(tmem + ((32 * q) << 16) + C::ACC_OUT + col + 16 * h, ao);
          tmem_ld_wait();
          if (c == C::EPI_CH - 1 && h == 1) {   // both accumulators read: release them
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(&tempty[acc]);
              mbar_arrive(out_empty);
            }
          }
          if (!inside) continue;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            // 16 x the integer sums: the shift is exact
            const float fn = k_norm_pad ? static_cast<float>(static_cast<int32_t>(an[j]) >> 4) : 0.f;
            const float fo = k_out_pad ? static_cast<float>(static_cast<int32_t>(ao[j]) >> 4) : 0.f;
            const float v = __fadd_rn(__fmul_rn(sn, fn), __fmul_rn(so, fo));
            dst[32 * (16 * h + j)] = __float2bfloat16_rn(__fmul_rn(sx, v));
          }
        }
        if (!inside) continue;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_y, buf, n0, m0);
          bulk_commit();
        }
        next ^= 1;
      }
    }
    epilogue_warp_finish();
  }

  pdl_release();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int RS, int XG>
static ql_status launch_qarvd_ts(const void* a_codes, const float* s_x, int64_t M, const ql_weights* w, void* Y,
                                 cudaStream_t st, int* status) {
  using C = QarvdTsCfg<RS, XG>;
  const int N = w->N, Kp = w->Kp;
  CUtensorMap tx, tw, ty;
  if (!make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, Kp, M, Kp, C::BK, C::BMT,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, Kp / 2, N, Kp / 2, C::BK / 2, 128,
                    CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, N, M, static_cast<int64_t>(N) * 2, 32, 32,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
    return QL_ERR_CUDA;
  GemmArgs p{};
  fill_gemm_args(p, M, N, Kp, 128, status);
  p.tiles_m = static_cast<int32_t>((M + C::BMT - 1) / C::BMT);
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.g_a = s_x;
  p.col_scale0 = w->s_norm;
  p.col_scale1 = w->s_out;
  p.kinfo = w->kinfo;
  auto kern = k_gemm_qarvd_ts<RS, XG>;
  if (!set_smem_attr(reinterpret_cast<const void*>(kern), C::SMEM)) return QL_ERR_CUDA;
  const int grid = std::min(p.num_tiles, num_sms());
  if (launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM, st, 1, tx, tw, ty, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

ql_status launch_gemm_qarvd(const void* a_codes, const float* s_x, int64_t M, const ql_weights* w, void* Y,
                            cudaStream_t st, int* status) {
  if (M == 0) return QL_OK;
  if (w->w8 != nullptr) {
    if (M > 128) return launch_qarvd_pre<true, 4, 128, 256>(a_codes, s_x, M, w, Y, st, status);
    return launch_qarvd_pre<false, 5, 128, 128>(a_codes, s_x, M, w, Y, st, status);
  }
  return launch_qarvd_ts<6, 2>(a_codes, s_x, M, w, Y, st, status);
}

}  // namespace ql
