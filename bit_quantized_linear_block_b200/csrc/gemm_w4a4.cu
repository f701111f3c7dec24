// W4A4 GEMM: NVFP4 activations x NVFP4 weights -> bf16, fp32 accumulation
// in tensor memory (6Bit-Diffusion, Methodology B.1: NVFP4 weights and
// NVFP4 activations on stable blocks, targeting Blackwell's NVFP4 support).
//
// Y[m, n] = bf16(alpha * sum_k (e2m1_a * sfa)(e2m1_w * sfw)),
// alpha = g_a * g_w * alpha_mul (alpha_mul = 1/128 undoes the two Hadamard
// rotations, 1 otherwise).
//
// Persistent, warp-specialized, one CTA per SM:
//   warp 0     TMA producer: A/B FP4 tiles (128-byte swizzle) and the block
//              scales (plain bulk copies of 512-byte atoms) into a STAGES-deep
//              shared-memory ring;
//   warp 1     MMA issuer: tcgen05.cp of the stage's scales into TMEM, then
//              tcgen05.mma kind::mxf4nvf4 block16 (128 x BN x 64 each);
//   warp 2     TMEM allocator;
//   warps 4-7  epilogue: tcgen05.ld, * alpha, bf16, swizzled staging tile,
//              TMA store; ACC accumulators in TMEM let the epilogue of one
//              tile overlap the main loop of the next.
// Every mbarrier wait is bounded; on a timeout the kernel records
// QL_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#include "ql_common.cuh"
#include "gemm_common.cuh"
#include "launchers.h"

namespace ql {

template <int BN, int STAGES, int ACC>
struct W4A4Cfg {
  static constexpr int BM = 128;
  static constexpr int BKB = 128;                    // K bytes per stage = 256 FP4 values
  static constexpr int A_BYTES = BM * BKB;
  static constexpr int B_BYTES = BN * BKB;
  static constexpr int NSFB = (BN + 127) / 128;      // 128-row scale atoms per B tile
  static constexpr int SFA_BYTES = 4 * 512;
  static constexpr int SFB_BYTES = NSFB * 4 * 512;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_C = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_SFA = OFF_C + 2 * kEpiChunkBytes;
  static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
  static constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_BYTES;
  static constexpr int NBAR = 2 * STAGES + 2 * ACC + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment
  static constexpr uint32_t TM_SFA = ACC * BN;
  static constexpr uint32_t TM_SFB = TM_SFA + 16;
  static_assert(TM_SFB + 16 * NSFB <= 512, "tensor memory budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(BN % 64 == 0 && BN <= 256, "tile width");
  // Instruction descriptor (block-scaled): A/B = E2M1 (1), scale = UE4M3 (0),
  // both K-major, N >> 3 at bit 17, M >> 4 at bit 24, dense K = 64.
  static constexpr uint32_t IDESC =
      (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
};

template <int BN, int STAGES, int ACC>
__global__ void __launch_bounds__(256, 1)
    k_gemm_w4a4(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_y, const GemmArgs p) {
  using C = W4A4Cfg<BN, STAGES, ACC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + ACC;
  uint64_t* drain = tempty + ACC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_y);
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < ACC; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        const int n0 = nb * BN;
        const int ra0 = n0 >> 7;
        for (int ks = 0; ks < p.num_kst; ++ks, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (*abort_flag || !mbar_wait(&empty[s], ph ^ 1, p.wait_limit)) {
            ok = false;
            break;
          }
          const int nk = min(4, p.k_atoms - 4 * ks);
          int nsfb = 0;
#pragma unroll
          for (int r = 0; r < C::NSFB; ++r) nsfb += (ra0 + r < p.sfb_atoms);
          mbar_arrive_expect_tx(&full[s], C::A_BYTES + C::B_BYTES + nk * 512 * (1 + nsfb));
          tma_load_2d(smem + C::OFF_A + s * C::A_BYTES, &tm_a, &full[s], ks * C::BKB, mb * C::BM);
          tma_load_2d(smem + C::OFF_B + s * C::B_BYTES, &tm_b, &full[s], ks * C::BKB, n0);
          bulk_load(smem + C::OFF_SFA + s * C::SFA_BYTES,
                    p.sfa + (static_cast<size_t>(mb) * p.k_atoms + 4 * ks) * 512, nk * 512, &full[s]);
#pragma unroll
          for (int r = 0; r < C::NSFB; ++r) {
            if (ra0 + r < p.sfb_atoms)
              bulk_load(smem + C::OFF_SFB + s * C::SFB_BYTES + r * 2048,
                        p.sfb + (static_cast<size_t>(ra0 + r) * p.k_atoms + 4 * ks) * 512, nk * 512,
                        &full[s]);
          }
        }
      }
      if (!ok) fail_timeout(p.status, abort_flag);
      drain_loads(full, it, STAGES, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      int it = 0, local = 0;
      bool ok = true;
      const uint64_t sf_desc0 = smem_desc(0, 0, 128, kSwizzleNone);
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++local) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        const int acc = local % ACC;
        const uint32_t aph = (local / ACC) & 1;
        if (*abort_flag || !mbar_wait(&tempty[acc], aph ^ 1, p.wait_limit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * BN;
        const uint32_t sfb_shift = (BN % 128 != 0 && (nb & 1)) ? 2u : 0u;
        for (int ks = 0; ks < p.num_kst; ++ks, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (*abort_flag || !mbar_wait(&full[s], ph, p.wait_limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nk = min(4, p.k_atoms - 4 * ks);
          const uint32_t a_base = smem_u32(smem + C::OFF_A + s * C::A_BYTES);
          const uint32_t b_base = smem_u32(smem + C::OFF_B + s * C::B_BYTES);
          const uint32_t sfa_base = smem_u32(smem + C::OFF_SFA + s * C::SFA_BYTES);
          const uint32_t sfb_base = smem_u32(smem + C::OFF_SFB + s * C::SFB_BYTES);
          for (int i = 0; i < nk; ++i) {
            tc_cp_sf(tmem + C::TM_SFA + 4 * i, sf_desc0 | ((sfa_base + 512 * i) >> 4));
#pragma unroll
            for (int r = 0; r < C::NSFB; ++r)
              tc_cp_sf(tmem + C::TM_SFB + 4 * C::NSFB * i + 4 * r,
                       sf_desc0 | ((sfb_base + 2048 * r + 512 * i) >> 4));
          }
          for (int i = 0; i < nk; ++i) {
            const uint64_t adesc = smem_desc(a_base + 32 * i, 0, 1024, kSwizzle128B);
            const uint64_t bdesc = smem_desc(b_base + 32 * i, 0, 1024, kSwizzle128B);
            tc_mma_nvf4(d_tmem, adesc, bdesc, C::IDESC, tmem + C::TM_SFA + 4 * i,
                        tmem + C::TM_SFB + 4 * C::NSFB * i + sfb_shift, (ks > 0 || i > 0) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
      }
      if (!ok) fail_timeout(p.status, abort_flag);
      drain_mma(drain, p.status);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const float alpha = __fmul_rn(__fmul_rn(*p.g_a, *p.g_w), p.alpha_mul);
    EpilogueState es{};
    int local = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++local) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int acc = local % ACC;
      const uint32_t aph = (local / ACC) & 1;
      if (!epilogue_wait_uniform(&tfull[acc], aph, p.wait_limit, abort_flag, p.status)) break;
      tc_fence_after();
      epilogue_tile<BN>(tmem + acc * BN, &tempty[acc], smem + C::OFF_C, &tm_y, mb * C::BM, nb * BN,
                        p.N, alpha, es);
    }
    epilogue_finish(es);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
}

// --------------------------------------------------------------------------
// Host side
// --------------------------------------------------------------------------
template <int BN, int STAGES, int ACC>
static ql_status launch_w4a4_cfg(const void* a_codes, const uint8_t* a_sf, const float* g_a,
                                 int64_t M, const ql_weights* w, void* Y, cudaStream_t st,
                                 int* status) {
  using C = W4A4Cfg<BN, STAGES, ACC>;
  const int N = w->N, K = w->K;
  CUtensorMap ta, tb, ty;
  if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, K / 2, M, K / 2, 128, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, K / 2, N, K / 2, 128, BN,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, N, M, static_cast<int64_t>(N) * 2, 64,
                    128, CU_TENSOR_MAP_SWIZZLE_128B))
    return QL_ERR_CUDA;
  GemmArgs p{};
  fill_gemm_args(p, M, N, K, BN, status);
  p.num_kst = (K + 255) / 256;
  p.k_atoms = K / 64;
  p.sfb_atoms = (N + 127) / 128;
  p.sfa = a_sf;
  p.sfb = static_cast<const uint8_t*>(w->sf);
  p.g_a = g_a;
  p.g_w = w->gscale;
  p.alpha_mul = w->hadamard ? (1.0f / 128.0f) : 1.0f;
  auto kern = k_gemm_w4a4<BN, STAGES, ACC>;
  if (!set_smem_attr(reinterpret_cast<const void*>(kern), C::SMEM)) return QL_ERR_CUDA;
  const int grid = std::min(p.num_tiles, num_sms());
  kern<<<grid, 256, C::SMEM, st>>>(ta, tb, ty, p);
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

ql_status launch_gemm_w4a4(const void* a_codes, const uint8_t* a_sf, const float* g_a, int64_t M,
                           const ql_weights* w, void* Y, cudaStream_t st, int* status) {
  if (M == 0) return QL_OK;
  if (w->N % 192 == 0) return launch_w4a4_cfg<192, 4, 2>(a_codes, a_sf, g_a, M, w, Y, st, status);
  return launch_w4a4_cfg<128, 5, 2>(a_codes, a_sf, g_a, M, w, Y, st, status);
}

}  // namespace ql
