// Bandwidth-bound kernels of the activation / weight quantizers.
//
//  * block-128 Hadamard (6Bit-Diffusion, Methodology B.1: online block
//    Hadamard transform), fused into every quantizer and never stored;
//  * tensor amax pre-pass for the dynamic NVFP4 tensor scale;
//  * NVFP4 quantizer (E2M1 codes, E4M3 scale per 16 elements, fp32 tensor
//    scale), writing the block scales straight into the MMA atom layout;
//  * per-token INT8 quantizer (the route DMPQ takes for sensitive blocks);
//  * per-tensor INT8 quantizer with Q-ARVD's channel permutation
//    (Q-ARVD, Technical details: per-tensor activation quantization).
//
// Work decomposition shared by all of them: a 128-element Hadamard block is
// held by 4 consecutive lanes, 32 contiguous elements each (four 16-byte
// loads).  Butterfly distances 1..16 stay inside a lane, 32 and 64 are one
// shuffle each.  A warp covers 8 blocks = 1024 contiguous elements.
#include "ql_common.cuh"
#include "launchers.h"

namespace ql {

// 32 bf16 -> fp32 from 64 contiguous bytes.
__device__ __forceinline__ void load32(const uint4* __restrict__ src, float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 u = __ldg(src + c);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * c + 2 * i] = bf16_lo(w[i]);
      v[8 * c + 2 * i + 1] = bf16_hi(w[i]);
    }
  }
}

// Fast Walsh-Hadamard transform of one 128-block spread over 4 lanes
// (q = lane % 4 holds elements 32q .. 32q+31).  Stage distances 1, 2, ...,
// 64 in that order; the pair (i, i+s) becomes (RN(a+b), RN(a-b)).  All 32
// lanes of the warp must call this together.
__device__ __forceinline__ void fwht128(float (&v)[32], uint32_t q) {
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if ((j & s) == 0) {
        const float a = v[j], b = v[j + s];
        v[j] = __fadd_rn(a, b);
        v[j + s] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (uint32_t t = 1; t <= 2; t <<= 1) {
    const bool upper = (q & t) != 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float p = __shfl_xor_sync(0xffffffffu, v[j], t);
      v[j] = upper ? __fsub_rn(p, v[j]) : __fadd_rn(v[j], p);
    }
  }
}

__device__ __forceinline__ float warp_max(float m) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}

// ---------------------------------------------------------------------------
// amax of |H x| (or |x| when hadamard == 0) over a contiguous tensor whose
// element count is a multiple of 128.  Each CTA writes its partial max; the
// last CTA to finish (atomic ticket) folds them into *amax_out and resets
// the ticket.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreadsHbm)
    k_amax(const uint4* __restrict__ x, int64_t units, int hadamard, float* __restrict__ partials,
           unsigned int* __restrict__ ticket, float* __restrict__ amax_out) {
  const uint32_t lane = lane_id();
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t chunks = (units + 7) >> 3;
  float m = 0.f;
  for (int64_t c = warp; c < chunks; c += nwarps) {
    const int64_t u = c * 8 + (lane >> 2);
    float v[32];
    if (u < units) {
      load32(x + (c * 1024 + lane * 32) / 8, v);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0.f;
    }
    if (hadamard) fwht128(v, lane & 3);
#pragma unroll
    for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(v[j]));
  }
  m = warp_max(m);
  __shared__ float red[kThreadsHbm / 32];
  __shared__ bool s_last;
  if (lane == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = red[0];
    for (int i = 1; i < kThreadsHbm / 32; ++i) r = fmaxf(r, red[i]);
    partials[blockIdx.x] = r;
    __threadfence();
    s_last = atomicAdd(ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (s_last && threadIdx.x < 32) {
    __threadfence();
    float r = 0.f;
    const volatile float* p = partials;
    for (unsigned int i = threadIdx.x; i < gridDim.x; i += 32) r = fmaxf(r, p[i]);
    r = warp_max(r);
    if (threadIdx.x == 0) {
      *amax_out = r;
      *ticket = 0u;
    }
  }
}

// ---------------------------------------------------------------------------
// NVFP4 quantizer.  g = amax / 2688 (1 if amax == 0) from the device amax.
// Per 16-element block: sb = E4M3(RN(amax_b / RN(6 g))); if sb == 0 all
// codes are +0, else code = E2M1(RN(h * RN(1 / RN(sb * g)))).
// Rows M .. Mpad-1 (padding of the last 128-row atom) get zero scales.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreadsHbm)
    k_quant_nvfp4(const uint4* __restrict__ x, int64_t M, int32_t K, int hadamard,
                  const float* __restrict__ amax_in, uint4* __restrict__ codes,
                  uint8_t* __restrict__ sf_mma, uint8_t* __restrict__ sf_rm,
                  float* __restrict__ g_out) {
  const float amax = __ldg(amax_in);
  const float g = (amax == 0.f) ? 1.f : __fdiv_rn(amax, 2688.f);
  if (blockIdx.x == 0 && threadIdx.x == 0 && g_out != nullptr) *g_out = g;
  const float d = __fmul_rn(6.f, g);

  const uint32_t lane = lane_id();
  const int32_t upr = K >> 7;                 // Hadamard blocks per row
  const int32_t k_atoms = K >> 6;             // 4-scale groups per row
  const int64_t mpad = (M + 127) & ~int64_t(127);
  const int64_t units = M * upr, units_pad = mpad * upr;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t chunks = (units_pad + 7) >> 3;
  const uint32_t q = lane & 3;

  for (int64_t c = warp; c < chunks; c += nwarps) {
    const int64_t u = c * 8 + (lane >> 2);
    const bool real = u < units;
    float v[32];
    if (real) {
      load32(x + (u * 128 + q * 32) / 8, v);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0.f;
    }
    if (hadamard) fwht128(v, q);
    if (u >= units_pad) continue;
    const int64_t row = u / upr;
    const int32_t blk = static_cast<int32_t>(u - row * upr);
    const int32_t j0 = blk * 8 + static_cast<int32_t>(q) * 2;    // first of this lane's 2 scales
    uint32_t sb[2] = {0u, 0u};
    uint32_t packed[4] = {0u, 0u, 0u, 0u};
    if (real) {
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[16 * b + j]));
        sb[b] = e4m3_code(__fdiv_rn(amax, d));
        if (sb[b] != 0u) {
          const float inv = __frcp_rn(__fmul_rn(e4m3_value(sb[b]), g));
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t cd = e2m1_code(__fmul_rn(v[16 * b + j], inv));
            packed[2 * b + j / 8] |= cd << (4 * (j % 8));
          }
        }
      }
      codes[(u * 128 + q * 32) / 32] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      if (sf_rm != nullptr)
        *reinterpret_cast<uint16_t*>(sf_rm + row * (K >> 4) + j0) =
            static_cast<uint16_t>(sb[0] | (sb[1] << 8));
    }
    *reinterpret_cast<uint16_t*>(sf_mma + sf_mma_offset(row, j0, k_atoms)) =
        static_cast<uint16_t>(sb[0] | (sb[1] << 8));
  }
}

// ---------------------------------------------------------------------------
// Per-token INT8: one warp per row.  Pass 1: amax_m of the rotated row.
// Pass 2: recompute the rotation (the row is L1/L2 resident) and quantize
// q = clamp(rint(RN(h * RN(127 / amax_m))), -127, 127); s_m = RN(amax_m/127).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreadsHbm)
    k_quant_int8_token(const uint4* __restrict__ x, int64_t M, int32_t K, int hadamard,
                       int8_t* __restrict__ codes, float* __restrict__ scales) {
  const uint32_t lane = lane_id();
  const uint32_t q = lane & 3;
  const int32_t upr = K >> 7;
  const int32_t passes = (upr + 7) >> 3;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t row = warp; row < M; row += nwarps) {
    const uint4* xr = x + row * (K / 8);
    float m = 0.f;
    for (int p = 0; p < passes; ++p) {
      const int32_t u = p * 8 + static_cast<int32_t>(lane >> 2);
      float v[32];
      if (u < upr) {
        load32(xr + (u * 128 + q * 32) / 8, v);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.f;
      }
      if (hadamard) fwht128(v, q);
#pragma unroll
      for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(v[j]));
    }
    m = warp_max(m);
    const float inv = (m == 0.f) ? 0.f : __fdiv_rn(127.f, m);
    if (lane == 0) scales[row] = (m == 0.f) ? 0.f : __fdiv_rn(m, 127.f);
    for (int p = 0; p < passes; ++p) {
      const int32_t u = p * 8 + static_cast<int32_t>(lane >> 2);
      float v[32];
      if (u < upr) {
        load32(xr + (u * 128 + q * 32) / 8, v);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.f;
      }
      if (hadamard) fwht128(v, q);
      if (u < upr) {
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint32_t packed = 0;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            int qi = __float2int_rn(__fmul_rn(v[4 * i + b], inv));
            qi = max(-127, min(127, qi));
            packed |= (static_cast<uint32_t>(qi) & 0xFFu) << (8 * b);
          }
          w[i] = packed;
        }
        uint4* dst = reinterpret_cast<uint4*>(codes + row * K + u * 128 + q * 32);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Per-tensor INT8 in Q-ARVD channel order.  Output row = Kp bytes; slot j
// takes input channel gather[j] (or 0 for a padding slot).  The scale comes
// from the device amax of the un-rotated tensor.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreadsHbm)
    k_quant_int8_tensor_perm(const __nv_bfloat16* __restrict__ x, int64_t M, int32_t K, int32_t Kp,
                             const int32_t* __restrict__ gather, const float* __restrict__ amax_in,
                             int8_t* __restrict__ codes, float* __restrict__ scale_out) {
  extern __shared__ int32_t s_gather[];
  for (int i = threadIdx.x; i < Kp; i += blockDim.x) s_gather[i] = gather[i];
  const float amax = __ldg(amax_in);
  const float inv = (amax == 0.f) ? 0.f : __fdiv_rn(127.f, amax);
  if (blockIdx.x == 0 && threadIdx.x == 0) *scale_out = (amax == 0.f) ? 0.f : __fdiv_rn(amax, 127.f);
  __syncthreads();
  const uint32_t lane = lane_id();
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const unsigned short* xs = reinterpret_cast<const unsigned short*>(x);
  for (int64_t row = warp; row < M; row += nwarps) {
    const unsigned short* xr = xs + row * K;
    for (int32_t j0 = static_cast<int32_t>(lane) * 16; j0 < Kp; j0 += 32 * 16) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t packed = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int32_t src = s_gather[j0 + 4 * i + b];
          int qi = 0;
          if (src >= 0) {
            const float v = __uint_as_float(static_cast<uint32_t>(__ldg(xr + src)) << 16);
            qi = max(-127, min(127, __float2int_rn(__fmul_rn(v, inv))));
          }
          packed |= (static_cast<uint32_t>(qi) & 0xFFu) << (8 * b);
        }
        w[i] = packed;
      }
      *reinterpret_cast<uint4*>(codes + row * Kp + j0) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// --------------------------------------------------------------------------
// Host launchers
// --------------------------------------------------------------------------
int hbm_grid(int64_t work_items, int per_cta) {
  const int64_t want = (work_items + per_cta - 1) / per_cta;
  const int64_t cap = static_cast<int64_t>(num_sms()) * kHbmCtasPerSm;
  return static_cast<int>(std::max<int64_t>(1, std::min(want, cap)));
}

ql_status launch_amax(const void* x, int64_t M, int32_t K, int hadamard, float* amax_out, void* ws,
                      cudaStream_t st) {
  const int64_t units = M * (K / 128);
  const int grid = hbm_grid((units + 7) / 8, kThreadsHbm / 32);
  float* partials = static_cast<float*>(ws);
  unsigned int* ticket = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + kAmaxPartialBytes);
  k_amax<<<grid, kThreadsHbm, 0, st>>>(static_cast<const uint4*>(x), units, hadamard, partials, ticket,
                                       amax_out);
  return cudaPeekAtLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

ql_status launch_quant_nvfp4(const void* x, int64_t M, int32_t K, int hadamard, const float* amax_in,
                             void* codes, void* sf_mma, void* sf_rm, float* g_out, cudaStream_t st) {
  const int64_t mpad = (M + 127) / 128 * 128;
  const int grid = hbm_grid((mpad * (K / 128) + 7) / 8, kThreadsHbm / 32);
  k_quant_nvfp4<<<grid, kThreadsHbm, 0, st>>>(static_cast<const uint4*>(x), M, K, hadamard, amax_in,
                                              static_cast<uint4*>(codes), static_cast<uint8_t*>(sf_mma),
                                              static_cast<uint8_t*>(sf_rm), g_out);
  return cudaPeekAtLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

ql_status launch_quant_int8_token(const void* x, int64_t M, int32_t K, int hadamard, void* codes,
                                  float* scales, cudaStream_t st) {
  if (M == 0) return QL_OK;
  const int grid = hbm_grid(M, kThreadsHbm / 32);
  k_quant_int8_token<<<grid, kThreadsHbm, 0, st>>>(static_cast<const uint4*>(x), M, K, hadamard,
                                                   static_cast<int8_t*>(codes), scales);
  return cudaPeekAtLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

ql_status launch_quant_int8_tensor_perm(const void* x, int64_t M, int32_t K, int32_t Kp,
                                        const int32_t* gather, const float* amax_in, void* codes,
                                        float* scale_out, cudaStream_t st) {
  const int grid = M == 0 ? 1 : hbm_grid(M, kThreadsHbm / 32);
  const size_t smem = static_cast<size_t>(Kp) * sizeof(int32_t);
  if (!set_smem_attr(reinterpret_cast<const void*>(k_quant_int8_tensor_perm), static_cast<int>(smem)))
    return QL_ERR_CUDA;
  k_quant_int8_tensor_perm<<<grid, kThreadsHbm, smem, st>>>(
      static_cast<const __nv_bfloat16*>(x), M, K, Kp, gather, amax_in, static_cast<int8_t*>(codes),
      scale_out);
  return cudaPeekAtLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

}  // namespace ql
