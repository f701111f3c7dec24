// W4A8 GEMM of the INT8 route: per-token INT8 activations x NVFP4 weights
// -> bf16 (6Bit-Diffusion, Methodology B.1: sensitive blocks keep INT8
// activations while all weights stay NVFP4).
//
// Y[m, n] = bf16(s_m * g_w * alpha_mul * sum_k q[m,k] * (e2m1[n,k] * sb[n,k/16]))
// with fp32 accumulation in tensor memory.  Both operands are f16, where
// every value is exact: int8 codes (|q| <= 127) and every E2M1 x E4M3
// product (at most 6 significant bits, magnitudes 2^-10 .. 2688).  The MMA
// is tcgen05 kind::f16 (128 x BN x 16).  Three forms (template flags):
//   PRE + A16  f16 weight copy (expand_f16) and f16-coded activations, both
//              by TMA straight into the MMA layout, no transform warps (the
//              form qlinear_forward takes when the copy exists);
//   PRE        f16 weight copy by TMA, int8 activations widened on chip;
//   neither    both operands widened on chip (below).
// BF16 instantiates the PRE + A16 form with bf16 operand types and no scales:
// the unquantized product X W^T of PDR's high-precision refresh.
//
// Persistent, warp-specialized, one CTA (512 threads) per SM:
//   warps 0-7   transform: raw int8 / FP4 + scale tiles -> f16 tiles in the
//               128-byte-swizzled K-major layout the MMA reads
//               (int8 via a byte-permute + f16 subtract, FP4 via the
//               hardware e2m1x2 -> f16x2 convert times the f16 block scale);
//   warp 8      TMA producer of the raw tiles (int8 A, FP4 B, B scales);
//   warp 9      MMA issuer;
//   warp 10     TMEM allocator;
//   warps 12-15 epilogue: tcgen05.ld, * s_m * g_w * alpha_mul, bf16, TMA store.
// All waits are bounded (see the W4A4 kernel for the timeout protocol).
#include <cuda_fp16.h>

#include "ql_common.cuh"
#include "gemm_common.cuh"
#include "launchers.h"

namespace ql {

template <int BN, int S, int RS, bool PRE, bool A16, bool BF16 = false>
struct W4A8Cfg {
  static_assert(!A16 || PRE, "f16 activations need pre-expanded weights");
  static constexpr bool XFORM = !(PRE && A16);   // any operand expanded on chip
  static constexpr int BM = 128;
  static constexpr int BK = 64;                        // K elements per stage
  static constexpr int CONV_A = A16 ? 0 : BM * BK * 2;    // f16, 128-byte rows
  static constexpr int CONV_B = PRE ? 0 : BN * BK * 2;
  static constexpr int RAW_A = A16 ? BM * BK * 2 : BM * BK;   // f16 (128-byte swizzle) or int8
  static constexpr int RAW_B = PRE ? BN * BK * 2 : BN * BK / 2;   // f16 (pre-expanded) or FP4
  static constexpr int NSFB = (BN + 127) / 128;
  static constexpr int RAW_SF = PRE ? 0 : NSFB * 512;   // one 4-scale column of each atom
  static constexpr int OFF_CA = 0;
  static constexpr int OFF_CB = OFF_CA + S * CONV_A;
  static constexpr int OFF_C = OFF_CB + S * CONV_B;
  static constexpr int OFF_RA = OFF_C + 2 * kEpiChunkBytes;
  static constexpr int OFF_RB = OFF_RA + RS * RAW_A;
  static constexpr int OFF_RSF = OFF_RB + RS * RAW_B;
  static constexpr int OFF_BAR = OFF_RSF + RS * RAW_SF;
  static constexpr int NBAR = 2 * RS + 2 * S + 2 * 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr int THREADS = 512;
  static constexpr int XFORM_THREADS = 256;
  static constexpr int B_CHUNKS_PER_THREAD = BN * 8 / XFORM_THREADS;
  static_assert(BN * 8 % XFORM_THREADS == 0, "B chunks per transform thread");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(2 * BN <= 512, "tensor memory budget");
  static_assert(!BF16 || (PRE && A16), "the bf16 product takes both operands by TMA");
  // kind::f16 descriptor: D = F32 (bit 4), A = B = F16 (0) or BF16 (1 at
  // bits 7 and 10; both operands always the same type), K-major, N >> 3 at
  // bit 17, M >> 4 at bit 24.
  static constexpr uint32_t IDESC = (1u << 4) | (BF16 ? ((1u << 7) | (1u << 10)) : 0u) |
                                    (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
};

// int8 x4 -> two f16x2 words holding the exact values (byte permute builds
// 1024 + (q + 128) in f16, a packed subtract removes the offset).
__device__ __forceinline__ void i8x4_to_f16(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const uint32_t a = __byte_perm(u, 0x64646464u, 0x5140u);
  const uint32_t b = __byte_perm(u, 0x64646464u, 0x5342u);
  const __half2 off = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));   // 1152
  const __half2 ra = __hsub2(*reinterpret_cast<const __half2*>(&a), off);
  const __half2 rb = __hsub2(*reinterpret_cast<const __half2*>(&b), off);
  lo = *reinterpret_cast<const uint32_t*>(&ra);
  hi = *reinterpret_cast<const uint32_t*>(&rb);
}

// Position of 16-byte chunk c of row r in a 128-byte-swizzled K-major tile.
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t c) {
  return r * 128u + ((c ^ (r & 7u)) << 4);
}

// Bounded wait decided by lane 0 and shared with the whole warp.
__device__ __forceinline__ bool warp_wait2(uint64_t* a, uint32_t pa, uint64_t* b, uint32_t pb,
                                           long long limit, volatile int* abort_flag) {
  int ok = 0;
  if (lane_id() == 0)
    ok = (*abort_flag == 0) && mbar_wait(a, pa, limit) && mbar_wait(b, pb, limit);
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

template <int BN, int S, int RS, bool PRE, bool A16, bool BF16>
__global__ void __launch_bounds__(512, 1)
    k_gemm_w4a8(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_y, const GemmArgs p) {
  using C = W4A8Cfg<BN, S, RS, PRE, A16, BF16>;
  if (p.gate != nullptr) {   // device-routed forward
    pdl_wait();
    if (gated_off(p.gate, p.gate_value)) {
      pdl_release();
      return;
    }
  }
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* raw_empty = raw_full + RS;
  uint64_t* conv_full = raw_empty + RS;
  uint64_t* conv_empty = conv_full + S;
  uint64_t* tfull = conv_empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_y);
    for (int i = 0; i < RS; ++i) {
      mbar_init(&raw_full[i], 1);
      // consumers of a raw stage: the transform warps (when they expand an
      // operand) and, when B is read in place, the MMAs' commit
      mbar_init(&raw_empty[i], (C::XFORM ? C::XFORM_THREADS / 32 : 0) + (PRE ? 1 : 0));
    }
    for (int i = 0; i < S; ++i) {
      mbar_init(&conv_full[i], C::XFORM_THREADS / 32);
      mbar_init(&conv_empty[i], 1);
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
  pdl_wait();   // everything above touched only shared and tensor memory

  if (warp < 8 && C::XFORM) {
    // ------------------------------------------------------------ transform
    const uint32_t tid = threadIdx.x;
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int n0 = nb * BN;
      const int ra0 = n0 >> 7;
      for (int ks = 0; ks < p.num_kst; ++ks, ++it) {
        const int s = it % S, rs = it % RS;
        if (!warp_wait2(&raw_full[rs], (it / RS) & 1, &conv_empty[s], ((it / S) & 1) ^ 1, p.wait_limit,
                        abort_flag)) {
          ok = false;
          break;
        }
        const uint8_t* ra = smem + C::OFF_RA + rs * C::RAW_A;
        const uint8_t* rb = smem + C::OFF_RB + rs * C::RAW_B;
        const uint8_t* rsf = smem + C::OFF_RSF + rs * C::RAW_SF;
        uint8_t* ca = smem + C::OFF_CA + s * C::CONV_A;
        uint8_t* cb = smem + C::OFF_CB + s * C::CONV_B;
        if constexpr (!A16)
#pragma unroll
        for (int i = 0; i < 4; ++i) {            // A: 128 rows x 8 chunks of 8 int8
          const uint32_t idx = tid + C::XFORM_THREADS * i;
          const uint32_t r = idx >> 3, c = idx & 7u;
          const uint2 q = *reinterpret_cast<const uint2*>(ra + idx * 8);
          uint4 o;
          i8x4_to_f16(q.x, o.x, o.y);
          i8x4_to_f16(q.y, o.z, o.w);
          *reinterpret_cast<uint4*>(ca + sw128(r, c)) = o;
        }
        if constexpr (!PRE)
#pragma unroll
        for (int i = 0; i < C::B_CHUNKS_PER_THREAD; ++i) {   // B: BN rows x 8 chunks of 8 FP4
          const uint32_t idx = tid + C::XFORM_THREADS * i;
          const uint32_t r = idx >> 3, c = idx & 7u;
          const uint32_t codes = *reinterpret_cast<const uint32_t*>(rb + idx * 4);
          const uint32_t n = static_cast<uint32_t>(n0) + r;
          const uint32_t slot = (n >> 7) - static_cast<uint32_t>(ra0);
          const uint32_t sb = rsf[slot * 512 + (n & 31u) * 16 + ((n >> 5) & 3u) * 4 + (c >> 1)];
          *reinterpret_cast<uint4*>(cb + sw128(r, c)) = fp4x8_scaled_to_f16(codes, sb);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane_id() == 0) {
          mbar_arrive(&raw_empty[rs]);
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
        const int n0 = nb * BN;
        const int ra0 = n0 >> 7;
        for (int ks = 0; ks < p.num_kst; ++ks, ++it) {
          const int s = it % RS;
          const uint32_t ph = (it / RS) & 1;
          if (*abort_flag || !mbar_wait(&raw_empty[s], ph ^ 1, p.wait_limit)) {
            ok = false;
            break;
          }
          int nsfb = 0;
#pragma unroll
          for (int r = 0; r < C::NSFB; ++r) nsfb += (ra0 + r < p.sfb_atoms);
          if (PRE) nsfb = 0;
          mbar_arrive_expect_tx(&raw_full[s], C::RAW_A + C::RAW_B + 512 * nsfb);
          tma_load_2d(smem + C::OFF_RA + s * C::RAW_A, &tm_a, &raw_full[s], ks * C::BK, mb * C::BM);
          tma_load_2d(smem + C::OFF_RB + s * C::RAW_B, &tm_b, &raw_full[s], ks * (PRE ? C::BK : C::BK / 2), n0);
#pragma unroll
          for (int r = 0; r < (PRE ? 0 : C::NSFB); ++r) {
            if (ra0 + r < p.sfb_atoms)
              bulk_load(smem + C::OFF_RSF + s * C::RAW_SF + r * 512,
                        p.sfb + (static_cast<size_t>(ra0 + r) * p.k_atoms + ks) * 512, 512, &raw_full[s]);
          }
        }
      }
      if (!ok) fail_timeout(p.status, abort_flag);
      drain_loads(raw_full, it, RS, p.status);
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
        const uint32_t d_tmem = tmem + acc * BN;
        for (int ks = 0; ks < p.num_kst; ++ks, ++it) {
          const int s = it % S, rs = it % RS;
          // expanded operands wait for the transform; operands read in place
          // (both, with A16 and PRE) wait for the raw tiles
          const bool ready = C::XFORM ? mbar_wait(&conv_full[s], (it / S) & 1, p.wait_limit)
                                      : mbar_wait(&raw_full[rs], (it / RS) & 1, p.wait_limit);
          if (*abort_flag || !ready) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = A16 ? smem_u32(smem + C::OFF_RA + rs * C::RAW_A)
                                      : smem_u32(smem + C::OFF_CA + s * C::CONV_A);
          const uint32_t b_base = PRE ? smem_u32(smem + C::OFF_RB + rs * C::RAW_B)
                                      : smem_u32(smem + C::OFF_CB + s * C::CONV_B);
#pragma unroll
          for (int i = 0; i < C::BK / 16; ++i) {
            const uint64_t adesc = smem_desc(a_base + 32 * i, 0, 1024, kSwizzle128B);
            const uint64_t bdesc = smem_desc(b_base + 32 * i, 0, 1024, kSwizzle128B);
            tc_mma_f16(d_tmem, adesc, bdesc, C::IDESC, (ks > 0 || i > 0) ? 1u : 0u);
          }
          if constexpr (C::XFORM) tc_commit(&conv_empty[s]);
          if constexpr (PRE) tc_commit(&raw_empty[rs]);   // the in-place tiles are consumed
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
      }
      if (!ok) fail_timeout(p.status, abort_flag);
      drain_mma(drain, p.status);
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ epilogue
    const float alpha = BF16 ? 1.f : __fmul_rn(ld_dep(p.g_w), p.alpha_mul);   // the bf16 product is unscaled
    EpilogueState es{};
    int local = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++local) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int acc = local & 1;
      const uint32_t aph = (local >> 1) & 1;
      if (!epilogue_wait_uniform(&tfull[acc], aph, p.wait_limit, abort_flag, p.status)) break;
      tc_fence_after();
      epilogue_tile<BN>(tmem + acc * BN, &tempty[acc], smem + C::OFF_C, &tm_y, mb * C::BM, nb * BN, p.N,
                        alpha, es, p.row_scale, p.M);
    }
    epilogue_finish(es);
  }

  pdl_release();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 10) tmem_dealloc(tmem, 512);
}

template <int BN, int S, int RS, bool PRE, bool A16, bool BF16 = false>
static ql_status launch_w4a8_cfg(const void* a_codes, const float* a_scales, int64_t M,
                                 const ql_weights* w, void* Y, cudaStream_t st, int* status, Gate gate) {
  using C = W4A8Cfg<BN, S, RS, PRE, A16, BF16>;
  const int N = w->N, K = w->K;
  const CUtensorMapDataType t16 = BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap ta, tb, ty;
  if (!(A16 ? make_tmap_2d(&ta, t16, a_codes, K, M, static_cast<int64_t>(K) * 2, C::BK,
                           C::BM, CU_TENSOR_MAP_SWIZZLE_128B)
             : make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, K, M, K, C::BK, C::BM,
                            CU_TENSOR_MAP_SWIZZLE_NONE)) ||
      !(PRE ? make_tmap_2d(&tb, t16, BF16 ? w->wbf16 : w->w16, K, N, static_cast<int64_t>(K) * 2, C::BK,
                           BN, CU_TENSOR_MAP_SWIZZLE_128B)
            : make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, K / 2, N, K / 2, C::BK / 2, BN,
                           CU_TENSOR_MAP_SWIZZLE_NONE)) ||
      !make_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, N, M, static_cast<int64_t>(N) * 2, 64,
                    128, CU_TENSOR_MAP_SWIZZLE_128B))
    return QL_ERR_CUDA;
  GemmArgs p{};
  fill_gemm_args(p, M, N, K, BN, status);
  p.num_kst = K / C::BK;
  p.k_atoms = K / 64;
  p.sfb_atoms = (N + 127) / 128;
  p.sfb = static_cast<const uint8_t*>(w->sf);
  p.g_w = w->gscale;
  p.row_scale = a_scales;
  p.alpha_mul = w->hadamard ? (1.0f / 128.0f) : 1.0f;
  p.gate = gate.route;
  p.gate_value = gate.value;
  auto kern = k_gemm_w4a8<BN, S, RS, PRE, A16, BF16>;
  if (!set_smem_attr(reinterpret_cast<const void*>(kern), C::SMEM)) return QL_ERR_CUDA;
  const int grid = std::min(p.num_tiles, num_sms());
  if (launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM, st, 1, ta, tb, ty, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

ql_status launch_gemm_w4a8(const void* a_codes, const float* a_scales, int64_t M, const ql_weights* w,
                           void* Y, cudaStream_t st, int* status, int a_f16, Gate gate) {
  if (M == 0) return QL_OK;
  const bool n192 = w->N % 192 == 0;
  if (a_f16) {   // f16 activations and pre-expanded weights: both operands by TMA
    if (w->w16 == nullptr) return QL_ERR_UNSUPPORTED_SHAPE;
    if (n192) return launch_w4a8_cfg<192, 1, 4, true, true>(a_codes, a_scales, M, w, Y, st, status, gate);
    return launch_w4a8_cfg<128, 1, 5, true, true>(a_codes, a_scales, M, w, Y, st, status, gate);
  }
  if (w->w16 != nullptr) {   // weights pre-expanded to f16 at preparation
    if (n192) return launch_w4a8_cfg<192, 2, 4, true, false>(a_codes, a_scales, M, w, Y, st, status, gate);
    return launch_w4a8_cfg<128, 2, 5, true, false>(a_codes, a_scales, M, w, Y, st, status, gate);
  }
  if (n192) return launch_w4a8_cfg<192, 2, 6, false, false>(a_codes, a_scales, M, w, Y, st, status, gate);
  return launch_w4a8_cfg<128, 2, 8, false, false>(a_codes, a_scales, M, w, Y, st, status, gate);
}

// Unquantized bf16 product Y = X W^T (fp32 accumulation) from the bf16 input
// and the kept bf16 weights: the same kernel with bf16 operand types, both
// operands by TMA, no scales.
ql_status launch_gemm_bf16(const void* X, int64_t M, const ql_weights* w, void* Y, cudaStream_t st, int* status,
                           Gate gate) {
  if (M == 0) return QL_OK;
  if (w->wbf16 == nullptr) return QL_ERR_UNSUPPORTED_SHAPE;
  if (w->N % 192 == 0) return launch_w4a8_cfg<192, 1, 4, true, true, true>(X, nullptr, M, w, Y, st, status, gate);
  return launch_w4a8_cfg<128, 1, 5, true, true, true>(X, nullptr, M, w, Y, st, status, gate);
}

}  // namespace ql
