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

// ---------------------------------------------------------------------------
// INT8 route without the f16 weight copy: the weights are the MMA's A operand
// in tensor memory, so the on-chip widening never passes through shared
// memory.  The kernel computes the transposed tile D[n, m] = sum_k
// W[n, k] q[m, k] (128 weight rows on the TMEM lanes, BMT tokens as the MMA's
// N) and writes Y[m, n] = bf16(RN(RN(g_w * alpha_mul) * s_m) * D[n, m]), the
// rounding of the other forms.
//
// Persistent, one CTA (512 to 768 threads) per SM, tiles of 128 weight rows x BMT
// tokens, weight tiles fastest (the CTAs running at once share a few token
// tiles and sweep the whole weight matrix, which stays in L2):
//   warp 0      TMA producer: the f16-coded activation tile (BMT x 64,
//               128-byte swizzle), the FP4 weight tile (128 rows x 32 bytes)
//               and its 512-byte scale column, into an RS-deep ring;
//   warp 1      TMEM allocator and MMA issuer (kind::f16, 128 x BMT x 16,
//               A from tensor memory);
//   4 XG transform warps (from warp 4), XG groups of four: group g widens
//               the stages it with it % XG == g, so a stage's widening
//               latency is spread over XG stages of MMA time.  Lane l of
//               warp w owns weight row 32 (w % 4) + l; per 64-deep K stage it
//               widens the row's 64 FP4 codes times their E4M3 scales to f16
//               (hardware e2m1x2 -> f16x2 convert, f16 multiply: exact) and
//               writes the 32 words into one of AS 32-column A slots of its
//               TMEM lane with tcgen05.st;
//   8 epilogue warps (after the transform warps): warp w reads TMEM lane
//               quarter w % 4 and half of the BMT columns, scales column m
//               by s_m, and stores 32 x 32 boxes of Y (tokens x weight rows)
//               through its own staging buffers with TMA.
// Tensor memory: two BMT-column accumulators (one for BMT = 256) and
// AS = (512 - NACC BMT) / 32 A slots.  All waits are bounded (the W4A4 kernel's timeout protocol).
// ---------------------------------------------------------------------------
template <int BMT, int RS, int XG>
struct W4A8TsCfg {
  static constexpr int BK = 64;                    // K elements per stage
  // two accumulators where they leave room for four A slots, else one
  static constexpr int NACC = (2 * BMT + 4 * 32 <= 512) ? 2 : 1;
  static constexpr int AS = (512 - NACC * BMT) / 32;  // A slots (64 f16 of K per TMEM lane)
  static constexpr int B_BYTES = BMT * BK * 2;     // f16 activation codes, 128-byte rows
  static constexpr int W_BYTES = 128 * BK / 2;     // FP4 codes, 32 bytes per weight row
  static constexpr int SF_BYTES = 512;             // the stage's column of the 128-row scale atom
  static constexpr int OFF_B = 0;
  static constexpr int OFF_W = OFF_B + RS * B_BYTES;
  static constexpr int OFF_SF = OFF_W + RS * W_BYTES;
  static constexpr int OFF_C = OFF_SF + RS * SF_BYTES;     // 8 epilogue warps x 2 staging boxes
  static constexpr int OFF_BAR = OFF_C + 8 * 2 * kWarpBoxBytes;
  static constexpr int NBAR = 2 * RS + 2 * AS + 2 * 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr int EPI0 = 4 + 4 * XG;          // first epilogue warp
  static constexpr int THREADS = (EPI0 + 8) * 32;
  static constexpr int EPI_CH = BMT / 2 / 32;      // 32-column boxes per epilogue warp and tile
  static_assert(XG >= 1 && XG <= 3, "transform warp groups");
  static_assert(AS >= 2, "tensor memory budget");
  static_assert(B_BYTES % 1024 == 0 && BMT % 64 == 0, "swizzled tiles, whole epilogue boxes");
  static_assert(SMEM <= 232448, "shared memory budget");
  // kind::f16: D = F32 (bit 4), A = B = F16, both K-major, N = BMT, M = 128
  static constexpr uint32_t IDESC = (1u << 4) | (uint32_t(BMT >> 3) << 17) | (uint32_t(128 >> 4) << 24);
};

template <int BMT, int RS, int XG>
__global__ void __launch_bounds__(W4A8TsCfg<BMT, RS, XG>::THREADS, 1)
    k_gemm_w4a8_ts(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_y, const GemmArgs p) {
  using C = W4A8TsCfg<BMT, RS, XG>;
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
  uint64_t* xf_full = raw_empty + RS;
  uint64_t* xf_empty = xf_full + C::AS;
  uint64_t* tfull = xf_empty + C::AS;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
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
      mbar_init(&tempty[i], 8);      // the eight epilogue warps
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t a_slots = tmem + C::NACC * BMT;
  pdl_wait();   // everything above touched only shared and tensor memory

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        const int mb = t / p.tiles_n, nb = t - (t / p.tiles_n) * p.tiles_n;
        for (int ks = 0; ks < p.num_kst; ++ks, ++it) {
          const int s = it % RS;
          if (*abort_flag || !mbar_wait(&raw_empty[s], ((it / RS) & 1) ^ 1, p.wait_limit)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&raw_full[s], C::B_BYTES + C::W_BYTES + C::SF_BYTES);
          tma_load_2d(smem + C::OFF_B + s * C::B_BYTES, &tm_x, &raw_full[s], ks * C::BK, mb * BMT);
          tma_load_2d(smem + C::OFF_W + s * C::W_BYTES, &tm_w, &raw_full[s], ks * (C::BK / 2), nb * 128);
          bulk_load(smem + C::OFF_SF + s * C::SF_BYTES, p.sfb + (static_cast<size_t>(nb) * p.k_atoms + ks) * 512,
                    C::SF_BYTES, &raw_full[s]);
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
        const int acc = local % C::NACC;
        if (*abort_flag || !mbar_wait(&tempty[acc], ((local / C::NACC) & 1) ^ 1, p.wait_limit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * BMT;
        for (int ks = 0; ks < p.num_kst; ++ks, ++it) {
          const int rs = it % RS, sl = it % C::AS;
          if (*abort_flag || !mbar_wait(&raw_full[rs], (it / RS) & 1, p.wait_limit) ||
              !mbar_wait(&xf_full[sl], (it / C::AS) & 1, p.wait_limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b_base = smem_u32(smem + C::OFF_B + rs * C::B_BYTES);
#pragma unroll
          for (int i = 0; i < C::BK / 16; ++i)
            tc_mma_f16_ts(d_tmem, a_slots + 32 * sl + 8 * i, smem_desc(b_base + 32 * i, 0, 1024, kSwizzle128B),
                          C::IDESC, (ks > 0 || i > 0) ? 1u : 0u);
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
    const uint32_t row = 32 * q + lane;   // weight row within the tile = TMEM lane
    const int group = (warp - 4) >> 2;    // widens the stages it with it % XG == group
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
      for (int ks = 0; ks < p.num_kst; ++ks, ++it) {
        if (it % XG != group) continue;
        const int rs = it % RS, sl = it % C::AS;
        if (!warp_wait2(&raw_full[rs], (it / RS) & 1, &xf_empty[sl], ((it / C::AS) & 1) ^ 1, p.wait_limit,
                        abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // scale atom: byte (row % 32) * 16 + (row / 32) * 4 + k16 holds the block scale of K block k16
        const uint32_t sb4 = *reinterpret_cast<const uint32_t*>(smem + C::OFF_SF + rs * C::SF_BYTES + lane * 16 + q * 4);
        const uint4* wr = reinterpret_cast<const uint4*>(smem + C::OFF_W + rs * C::W_BYTES + row * 32);
        const uint4 c0 = wr[0], c1 = wr[1];
        const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        uint32_t v[32];
#pragma unroll
        for (int w8 = 0; w8 < 8; ++w8) {   // codes 8 w8 .. 8 w8 + 7: half of block w8 / 2
          const uint4 o = fp4x8_scaled_to_f16(cw[w8], (sb4 >> (8 * (w8 >> 1))) & 0xFFu);
          v[4 * w8] = o.x;
          v[4 * w8 + 1] = o.y;
          v[4 * w8 + 2] = o.z;
          v[4 * w8 + 3] = o.w;
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
    const float alpha = __fmul_rn(ld_dep(p.g_w), p.alpha_mul);
    uint8_t* stage = smem + C::OFF_C + (warp - C::EPI0) * 2 * kWarpBoxBytes;
    int next = 0, local = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++local) {
      const int mb = t / p.tiles_n, nb = t - (t / p.tiles_n) * p.tiles_n;
      const int acc = local % C::NACC;
      if (!warp_wait_uniform(&tfull[acc], (local / C::NACC) & 1, p.wait_limit, abort_flag, p.status)) break;
      tc_fence_after();
      const int n0 = nb * 128 + 32 * static_cast<int>(q);   // this warp's weight rows = output columns
#pragma unroll 1
      for (int c = 0; c < C::EPI_CH; ++c) {
        const int col = half * (BMT / 2) + 32 * c;          // accumulator column = token offset
        const int m0 = mb * BMT + col;
        uint32_t r[32];
        tmem_ld32(tmem + ((32 * q) << 16) + acc * BMT + col, r);
        tmem_ld_wait();
        if (c == C::EPI_CH - 1) {   // the whole accumulator share is read: free it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        if (m0 >= p.M || n0 >= p.N) continue;   // warp-uniform: the box is outside Y
        const int m = m0 + static_cast<int>(lane);
        const float a_l = (m < p.M) ? __fmul_rn(alpha, ld_dep(p.row_scale + m)) : 0.f;
        uint8_t* buf = stage + next * kWarpBoxBytes;
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        // box row j = token m0 + j, column = this lane's weight row
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(buf) + lane;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          dst[32 * j] = __float2bfloat16_rn(__fmul_rn(__shfl_sync(0xffffffffu, a_l, j), __uint_as_float(r[j])));
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

template <int BMT, int RS, int XG>
static ql_status launch_w4a8_ts_cfg(const void* a_codes, const float* a_scales, int64_t M, const ql_weights* w,
                                    void* Y, cudaStream_t st, int* status, Gate gate) {
  using C = W4A8TsCfg<BMT, RS, XG>;
  const int N = w->N, K = w->K;
  CUtensorMap tx, tw, ty;
  if (!make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a_codes, K, M, static_cast<int64_t>(K) * 2, C::BK, BMT,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, K / 2, N, K / 2, C::BK / 2, 128,
                    CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, N, M, static_cast<int64_t>(N) * 2, 32, 32,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
    return QL_ERR_CUDA;
  GemmArgs p{};
  fill_gemm_args(p, M, N, K, 128, status);
  p.tiles_m = static_cast<int32_t>((M + BMT - 1) / BMT);
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.num_kst = K / C::BK;
  p.k_atoms = K / 64;
  p.sfb_atoms = (N + 127) / 128;
  p.sfb = static_cast<const uint8_t*>(w->sf);
  p.g_w = w->gscale;
  p.row_scale = a_scales;
  p.alpha_mul = w->hadamard ? (1.0f / 128.0f) : 1.0f;
  p.gate = gate.route;
  p.gate_value = gate.value;
  auto kern = k_gemm_w4a8_ts<BMT, RS, XG>;
  if (!set_smem_attr(reinterpret_cast<const void*>(kern), C::SMEM)) return QL_ERR_CUDA;
  const int grid = std::min(p.num_tiles, num_sms());
  if (launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM, st, 1, tx, tw, ty, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

ql_status launch_gemm_w4a8(const void* a_codes, const float* a_scales, int64_t M, const ql_weights* w,
                           void* Y, cudaStream_t st, int* status, int a_f16, Gate gate) {
  if (M == 0) return QL_OK;
  const bool n192 = w->N % 192 == 0;
  if (a_f16) {
    // without the weight copy: the weights widened into tensor memory
    if (w->w16 == nullptr) return launch_w4a8_ts_cfg<192, 6, 2>(a_codes, a_scales, M, w, Y, st, status, gate);
    // f16 activations and pre-expanded weights: both operands by TMA
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
