// Q-ARVD dual-scale W4A8 integer GEMM ("Q-ARVD: Autoregressive Video
// Diffusion Models의 양자화", Methodology and Technical details: Q_dual(W) =
// [Q_outlier(W_outliers) | Q_normal(W_normal)] with per-channel weight and
// per-tensor activation quantization).
//
// The activations arrive in the weights' channel order (normal channels,
// zero padding to 32, outlier channels, zero padding to 32), so each class
// is a contiguous, MMA-aligned K range and gets its own int32 accumulator:
//   Y[m, n] = bf16(s_x * (s_norm[n] * acc_normal[m, n] + s_out[n] * acc_outlier[m, n])).
// The MMA is tcgen05 kind::i8 (128 x 128 x 32, int32 accumulation, exact).
//
// Persistent, warp-specialized, one CTA (512 threads) per SM:
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
    const float sx = *p.g_a;
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

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 10) tmem_dealloc(tmem, 512);
}

ql_status launch_gemm_qarvd(const void* a_codes, const float* s_x, int64_t M, const ql_weights* w, void* Y,
                            cudaStream_t st, int* status) {
  if (M == 0) return QL_OK;
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
  kern<<<grid, 512, C::SMEM, st>>>(ta, tb, ty, p);
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

}  // namespace ql
