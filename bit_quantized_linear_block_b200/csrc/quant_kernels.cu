// Bandwidth-bound kernels of the activation / weight quantizers.
//
//  * block-128 Hadamard (6Bit-Diffusion, Methodology B.1: online block
//    Hadamard transform), fused into every quantizer and never stored;
//  * tensor amax pre-pass for the dynamic NVFP4 tensor scale;
//  * NVFP4 quantizer (E2M1 codes, E4M3 scale per 16 elements, fp32 tensor
//    scale), writing the block scales straight into the MMA atom layout;
//  * the NVFP4 activation decomposition (SemanticDialect, Methodology 2.2):
//    NVFP4 of h and of its residual in one pass;
//  * per-token INT8 quantizer (the route DMPQ takes for sensitive blocks),
//    also with 6-bit codes (W4A6);
//  * per-tensor INT8 / INT6 quantizer with Q-ARVD's channel permutation
//    (Q-ARVD, Technical details: per-tensor activation quantization).
//
// Work decomposition of the rotated kernels: a 128-element Hadamard block is
// held by 2 lanes, 64 contiguous elements (one 128-byte row) each, in pair
// registers (x_j, x_{j+32}).  Butterfly distances 1..16 are packed f32x2
// operations inside a lane, 32 is inside each pair, 64 is one shuffle
// between the two lanes.  A warp covers 16 blocks = 2048 contiguous
// elements per chunk.
#include "ql_common.cuh"
#include "gemm_common.cuh"
#include "launchers.h"

namespace ql {

__device__ __forceinline__ float warp_max(float m) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}

// ---------------------------------------------------------------------------
// Streaming front end shared by the amax and NVFP4 kernels: half a Hadamard
// block (64 bf16 = 128 bytes) per lane, the two halves of a block in lanes
// 2i and 2i+1.
//
// A warp walks the flat tensor in chunks of 16 blocks (4 KB) with a
// kRing-deep ring of 4 KB slots in shared memory, each filled by ONE TMA
// load issued by the warp's first lane and tracked by the slot's mbarrier.
// The tensor map views the input as rows of 128 bytes (one lane's half
// block) with a 32-row box and the 128-byte swizzle, so 16-byte piece s of
// lane l's row lands at s ^ (l % 8): the read-back, where every lane reads
// its own row piece by piece, is free of bank conflicts.  Slots start on
// 1024-byte boundaries (the swizzle's period).  Rows past the end read as
// zeros.
// ---------------------------------------------------------------------------
constexpr int kRing = 3;                         // stages per warp
constexpr int kLaneBytes = 128;                  // 64 bf16
constexpr int kChunkBytes = 32 * kLaneBytes;     // 16 blocks of 128 bf16
constexpr int kWarpsPerCta = kThreadsHbm / 32;                         // amax: 2 CTAs/SM
constexpr int kRingBytesPerCta = kWarpsPerCta * kRing * kChunkBytes;   // 96 KB
constexpr int kRingCtasPerSm = 2;
constexpr int kQuantThreads = 384;                                     // NVFP4: 1 CTA/SM
constexpr int kQuantWarps = kQuantThreads / 32;
constexpr int kQuantRingBytes = kQuantWarps * kRing * kChunkBytes;     // 144 KB
constexpr int kRingAlignPad = 1024;                                    // for the 1024-byte aligned base

__device__ __forceinline__ uint8_t* ring_base(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + (((a + 1023u) & ~1023u) - a);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// This lane's 64 elements of a landed slot, in pair registers
// P[j] = (x_j, x_{j+32}), j = 0..31 (indices within the lane's half block).
__device__ __forceinline__ void read_half(const uint8_t* slot_ptr, float2 (&P)[32]) {
  const uint32_t lane = lane_id();
  const uint8_t* my = slot_ptr + lane * kLaneBytes;
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const uint4 a = *reinterpret_cast<const uint4*>(my + ((s ^ (lane & 7u)) << 4));        // x_{8s..8s+7}
    const uint4 b = *reinterpret_cast<const uint4*>(my + (((s + 4) ^ (lane & 7u)) << 4));  // x_{32+8s..}
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w};
    const uint32_t wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      P[8 * s + 2 * i] = make_float2(bf16_lo(wa[i]), bf16_lo(wb[i]));
      P[8 * s + 2 * i + 1] = make_float2(bf16_hi(wa[i]), bf16_hi(wb[i]));
    }
  }
}

// Block-128 FWHT with the block split over lanes 2i (elements 0..63) and 2i+1
// (64..127).  Distances 1..16 are butterflies between pairs (packed f32x2),
// 32 is inside each pair, 64 goes across the lane pair.  Each butterfly
// (a, b) -> (RN(a + b), RN(a - b)); a - b is computed as fma(b, -1, a),
// which rounds the same exact value once.  All lanes must call this.
__device__ __forceinline__ void fwht128_half(float2 (&P)[32]) {
  const float2 m1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if ((j & s) == 0) {
        const float2 a = P[j], b = P[j + s];
        P[j] = __fadd2_rn(a, b);
        P[j + s] = __ffma2_rn(b, m1, a);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float a = P[j].x, b = P[j].y;
    P[j] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
  }
  const float sg = (lane_id() & 1u) ? -1.f : 1.f;
  const float2 sg2 = make_float2(sg, sg);
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    float2 p;
    p.x = __shfl_xor_sync(0xffffffffu, P[j].x, 1);
    p.y = __shfl_xor_sync(0xffffffffu, P[j].y, 1);
    P[j] = __ffma2_rn(P[j], sg2, p);   // lower half: x + p, upper half: p - x
  }
}

// Per-warp ring driver: calls body(P, half_index) for each half block this
// lane owns (half_index = 2 * block + (lane & 1)).  `bars` holds kRing
// mbarriers per warp.  A wait that runs out of its cycle budget records
// QL_ERR_TIMEOUT, waits (bounded) for the warp's loads still in flight and
// ends the warp's walk.  REVERSE walks each warp's chunks from the last to
// the first (the grid sweeps the tensor from its end): a pass that follows a
// front-to-back pass over the same tensor meets the most recently read part,
// the part most likely still in L2, first.
template <int WARPS, bool REVERSE = false, class Body>
__device__ __forceinline__ void stream_blocks(const CUtensorMap* tm, int64_t total_bytes, int hadamard,
                                              uint8_t* ring_all, uint64_t* bars, int* status, Body body) {
  const int wid = threadIdx.x >> 5;
  uint8_t* ring_g = ring_all + wid * kRing * kChunkBytes;
  uint64_t* bar = bars + wid * kRing;
  const bool leader = lane_id() == 0;
  const int64_t nchunks = (total_bytes + kChunkBytes - 1) / kChunkBytes;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * WARPS + wid;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * WARPS;
  const int64_t mine = (gw < nchunks) ? (nchunks - gw + nw - 1) / nw : 0;
  if (leader) {
#pragma unroll
    for (int i = 0; i < kRing; ++i) mbar_init(&bar[i], 1);
    fence_mbar_init();
  }
  __syncwarp();
  auto chunk = [&](int64_t k) { return gw + (REVERSE ? (mine - 1 - k) : k) * nw; };   // k-th chunk walked
  auto issue = [&](int64_t k) {   // chunk k of this warp's walk into slot k % kRing
    if (leader) {
      const int slot = static_cast<int>(k % kRing);
      mbar_arrive_expect_tx(&bar[slot], kChunkBytes);
      tma_load_2d(ring_g + slot * kChunkBytes, tm, &bar[slot], 0, static_cast<int32_t>(chunk(k) * 32));
    }
  };
  for (int64_t i = 0; i < kRing - 1 && i < mine; ++i) issue(i);
  int64_t k = 0;
  for (; k < mine; ++k) {
    // the slot refilled here was read in the previous iteration, before its
    // closing __syncwarp
    if (k + kRing - 1 < mine) issue(k + kRing - 1);
    const int slot = static_cast<int>(k % kRing);
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar[slot], static_cast<uint32_t>((k / kRing) & 1),
                                                      kDrainLimit));
    if (!ok) break;
    float2 P[32];
    read_half(ring_g + slot * kChunkBytes, P);
    __syncwarp();
    if (hadamard) fwht128_half(P);
    body(P, chunk(k) * 32 + lane_id());
  }
  if (k < mine && leader) {   // timed out: let the loads in flight land before the CTA may exit
    record_error(status, QL_ERR_TIMEOUT);
    for (int64_t j = k; j < mine && j < k + kRing; ++j)   // chunks k .. k + kRing - 1 were issued
      (void)mbar_wait(&bar[j % kRing], static_cast<uint32_t>((j / kRing) & 1), kDrainLimit);
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// amax of |H x| (or |x| when hadamard == 0) over a contiguous tensor whose
// element count is a multiple of 128.  Each CTA writes its partial max; the
// last CTA to finish (atomic ticket) folds them into *amax_out and resets
// the ticket.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreadsHbm, kRingCtasPerSm)
    k_amax(const __grid_constant__ CUtensorMap tm_x, int64_t total_bytes, int hadamard,
           float* __restrict__ partials, unsigned int* __restrict__ ticket, float* __restrict__ amax_out,
           int* status, const int32_t* gate, int32_t gate_value) {
  extern __shared__ uint8_t ring_raw[];
  __shared__ uint64_t bars[kWarpsPerCta * kRing];
  uint8_t* ring_all = ring_base(ring_raw);
  const uint32_t lane = lane_id();
  pdl_wait();
  if (gated_off(gate, gate_value)) {
    pdl_release();
    return;
  }
  float m = 0.f;
  stream_blocks<kWarpsPerCta>(&tm_x, total_bytes, hadamard, ring_all, bars, status, [&](float2 (&P)[32], int64_t) {
    float2 mm = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      mm.x = fmax3(mm.x, fabsf(P[j].x), fabsf(P[j + 1].x));
      mm.y = fmax3(mm.y, fabsf(P[j].y), fabsf(P[j + 1].y));
    }
    m = fmax3(m, mm.x, mm.y);   // blocks past the end hold zeros
  });
  pdl_release();
  m = warp_max(m);
  __shared__ float red[kWarpsPerCta];
  __shared__ bool s_last;
  if (lane == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = red[0];
    for (int i = 1; i < kWarpsPerCta; ++i) r = fmaxf(r, red[i]);
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

// Eight E2M1 codes (hardware RN-even, saturating convert), element 0 in
// bits 0-3 ... element 7 in bits 28-31.  Each convert packs its second
// source operand in the low nibble and its first in the high nibble.
__device__ __forceinline__ uint32_t e2m1x8(float a0, float a1, float a2, float a3, float a4, float a5,
                                           float a6, float a7) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(a0), "f"(a1), "f"(a2), "f"(a3), "f"(a4), "f"(a5), "f"(a6), "f"(a7));
  return r;
}

// Two E2M1 codes (bits 0-7 of `byte`: the first element in the low nibble)
// -> their values {0, 0.5, 1, 1.5, 2, 3, 4, 6} with the sign (code 8 is -0),
// by the hardware convert to f16x2 (exact: every E2M1 value is an f16).
__device__ __forceinline__ float2 e2m1x2_to_f32x2(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(r) : "r"(byte));
  return __half22float2(*reinterpret_cast<const __half2*>(&r));
}

// Correctly rounded a / d for a >= 0 from r = RN(1 / d): Markstein's
// correction step (P. Markstein, "Computation of elementary functions on
// the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990):
// q0 = RN(a r) is within one ulp of a / d, so the remainder a - q0 d is
// exact in one fma, and RN(q0 + (a - q0 d) r) is the correctly rounded
// quotient when r is within half an ulp of 1 / d (no over- or underflow).
// The caller takes __fdiv_rn instead when d is outside [2^-100, 2^100].
__device__ __forceinline__ float div_rn_by(float a, float d, float r) {
  const float q0 = __fmul_rn(a, r);
  const float e = __fmaf_rn(-q0, d, a);
  return __fmaf_rn(e, r, q0);
}

// Per-launch tables of the NVFP4 block-scale arithmetic for the 128
// non-negative E4M3 codes: den[c] = RN(E4M3(c) g), inv[c] = RN(1 / den[c])
// (0 for c = 0).  The same operations the per-block code would run.
struct Nvfp4Tables {
  float den[128];
  float inv[128];
};

__device__ __forceinline__ void nvfp4_tables_fill(Nvfp4Tables* t, float g) {
  for (int c = threadIdx.x; c < 128; c += blockDim.x) {
    const float dn = __fmul_rn(e4m3_value(static_cast<uint32_t>(c)), g);
    t->den[c] = dn;
    t->inv[c] = c ? __frcp_rn(dn) : 0.f;
  }
}

// Block scale code of a block with absolute maximum a: E4M3(RN(a / d)).
struct Nvfp4ScaleDiv {
  float d, r;
  bool fast;
  __device__ __forceinline__ explicit Nvfp4ScaleDiv(float d_) {
    d = d_;
    r = __frcp_rn(d_);
    fast = d_ >= 7.8886091e-31f && d_ <= 1.2676506e30f;   // [2^-100, 2^100]
  }
  __device__ __forceinline__ uint32_t code(float a) const {
    return e4m3_code(fast ? div_rn_by(a, d, r) : __fdiv_rn(a, d));
  }
};

// NVFP4 of one half block (64 values in the pair layout: 16-element blocks
// b = 0, 1 in P[16b..16b+15].x, b = 2, 3 in the .y halves).  Writes the four
// E4M3 scales, the codes (cw[i]: elements 8i .. 8i+7 of the half) and each
// block's RN(E4M3 value * g) (den[b] for blocks b and b + 2).
__device__ __forceinline__ void nvfp4_half(const float2 (&P)[32], const Nvfp4ScaleDiv& sd,
                                           const Nvfp4Tables* tab, uint32_t (&sb)[4], uint32_t (&cw)[8],
                                           float2 (&den)[2]) {
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    float2 a = make_float2(0.f, 0.f);
#pragma unroll
    for (int t = 0; t < 16; t += 2) {
      a.x = fmax3(a.x, fabsf(P[16 * b + t].x), fabsf(P[16 * b + t + 1].x));
      a.y = fmax3(a.y, fabsf(P[16 * b + t].y), fabsf(P[16 * b + t + 1].y));
    }
    sb[b] = sd.code(a.x);
    sb[b + 2] = sd.code(a.y);
    den[b] = make_float2(tab->den[sb[b]], tab->den[sb[b + 2]]);
    const float2 inv = make_float2(tab->inv[sb[b]], tab->inv[sb[b + 2]]);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = 16 * b + 8 * h;
      float2 y[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) y[t] = __fmul2_rn(P[j + t], inv);
      const uint32_t lo = e2m1x8(y[0].x, y[1].x, y[2].x, y[3].x, y[4].x, y[5].x, y[6].x, y[7].x);
      const uint32_t hi = e2m1x8(y[0].y, y[1].y, y[2].y, y[3].y, y[4].y, y[5].y, y[6].y, y[7].y);
      cw[2 * b + h] = sb[b] ? lo : 0u;           // all-zero block -> +0 codes
      cw[4 + 2 * b + h] = sb[b + 2] ? hi : 0u;
    }
  }
}

// ---------------------------------------------------------------------------
// NVFP4 quantizer.  g = amax / 2688 (1 if amax == 0) from the device amax.
// Per 16-element block: sb = E4M3(RN(amax_b / RN(6 g))); if sb == 0 all
// codes are +0, else code = E2M1(RN(h * RN(1 / RN(sb * g)))).
// In the pair layout each lane holds four 16-element blocks, two in the .x
// and two in the .y halves of its registers, so two blocks are scaled by one
// packed multiply.  Rows M .. Mpad-1 (padding of the last
// 128-row atom) get zero scales.
//
// DECOMP (activation decomposition, SemanticDialect, Methodology 2.2): the
// residual r = RN(h - RN(e2m1(q1) * RN(sb1 * g))) is quantized again with
// the same g; a row of the output holds [q1 | q2] (K/2 bytes each) and its
// scales cover K' = 2K (q1's at scale indices 0 .. K/16-1, q2's after them),
// the operand of a W4A4 GEMM over K' against the weights repeated along K.
// ---------------------------------------------------------------------------
template <bool DECOMP>
__global__ void __launch_bounds__(kQuantThreads, 1)
    k_quant_nvfp4(const __grid_constant__ CUtensorMap tm_x, int64_t M, int32_t K, int hadamard,
                  const float* amax_in, uint8_t* __restrict__ codes,
                  uint8_t* __restrict__ sf_mma, uint8_t* __restrict__ sf_rm,
                  float* __restrict__ g_out, int* status, const int32_t* gate, int32_t gate_value) {
  extern __shared__ uint8_t ring_raw[];
  __shared__ Nvfp4Tables tab;
  __shared__ uint64_t bars[kQuantWarps * kRing];
  uint8_t* ring_all = ring_base(ring_raw);
  pdl_wait();
  if (gated_off(gate, gate_value)) {
    pdl_release();
    return;
  }
  const float amax_t = ld_dep(amax_in);
  const float g = (amax_t == 0.f) ? 1.f : __fdiv_rn(amax_t, 2688.f);
  if (blockIdx.x == 0 && threadIdx.x == 0 && g_out != nullptr) *g_out = g;
  const Nvfp4ScaleDiv sd(__fmul_rn(6.f, g));
  nvfp4_tables_fill(&tab, g);
  __syncthreads();
  const uint32_t upr = static_cast<uint32_t>(K >> 7);
  const int32_t kq = DECOMP ? 2 * K : K;           // K of the quantized operand
  const int32_t k_atoms = kq >> 6;
  const int64_t row_bytes = kq >> 1;
  const int64_t units = M * upr;
  const int64_t halves = 2 * units;
  stream_blocks<kQuantWarps, true>(&tm_x, M * K * 2, hadamard, ring_all, bars, status, [&](float2 (&P)[32], int64_t hu) {
    if (hu >= halves) return;
    // half index -> (row, first scale index, first code byte); 32-bit division (units < 2^32)
    const uint32_t u = static_cast<uint32_t>(hu >> 1);
    const uint32_t row = u / upr;
    const uint32_t j0 = (u - row * upr) * 8 + (static_cast<uint32_t>(hu) & 1u) * 4;
    uint8_t* cdst = codes + static_cast<int64_t>(row) * row_bytes + j0 * 8;
    uint32_t sb[4], cw[8];
    float2 den[2];
    nvfp4_half(P, sd, &tab, sb, cw, den);
    auto store = [&](int part) {
      uint4* dst = reinterpret_cast<uint4*>(cdst + part * (K >> 1));
      dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
      dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
      const uint32_t j = j0 + part * (K >> 4);
      const uint32_t sw = sb[0] | (sb[1] << 8) | (sb[2] << 16) | (sb[3] << 24);
      *reinterpret_cast<uint32_t*>(sf_mma + sf_mma_offset(row, j, k_atoms)) = sw;
      if (sf_rm != nullptr) *reinterpret_cast<uint32_t*>(sf_rm + static_cast<size_t>(row) * (kq >> 4) + j) = sw;
    };
    store(0);
    if constexpr (DECOMP) {
      // residual in place: P <- RN(P - RN(e2m1(q1) * den))
#pragma unroll
      for (int b = 0; b < 2; ++b) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int j = 16 * b + 8 * h;
          const uint32_t lo = cw[2 * b + h], hi = cw[4 + 2 * b + h];
#pragma unroll
          for (int t = 0; t < 4; ++t) {   // elements 2t, 2t+1 of the group
            const float2 vx = e2m1x2_to_f32x2(lo >> (8 * t)), vy = e2m1x2_to_f32x2(hi >> (8 * t));
            P[j + 2 * t].x = __fsub_rn(P[j + 2 * t].x, __fmul_rn(vx.x, den[b].x));
            P[j + 2 * t + 1].x = __fsub_rn(P[j + 2 * t + 1].x, __fmul_rn(vx.y, den[b].x));
            P[j + 2 * t].y = __fsub_rn(P[j + 2 * t].y, __fmul_rn(vy.x, den[b].y));
            P[j + 2 * t + 1].y = __fsub_rn(P[j + 2 * t + 1].y, __fmul_rn(vy.y, den[b].y));
          }
        }
      }
      nvfp4_half(P, sd, &tab, sb, cw, den);
      store(1);
    }
  });
  pdl_release();
  // zero scales of the padding rows of the last 128-row atom
  const int64_t mpad = (M + 127) & ~int64_t(127);
  const int64_t pad_words = (mpad - M) * k_atoms;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < pad_words;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = M + i / k_atoms;
    const int32_t j = static_cast<int32_t>(i % k_atoms) * 4;
    *reinterpret_cast<uint32_t*>(sf_mma + sf_mma_offset(row, j, k_atoms)) = 0u;
  }
}

// ---------------------------------------------------------------------------
// Per-token INT8: one warp per row.  The bf16 row comes into one of the
// warp's two 1024-byte aligned shared-memory buffers by TMA (the streaming
// kernels' 128-byte-row view and swizzle; the next row's load is in flight
// while this one is quantized), lane l takes half blocks 32 p + l (p = 0, 1, ...) with the same
// half-block FWHT as the NVFP4 path.  amax_m = max |h| over the row,
// q = clamp(rint(RN(h * RN(127 / amax_m))), -127, 127), s_m = RN(amax_m/127).
// A row of at most 2048 elements is rotated once and stays in registers;
// longer rows are rotated again, from shared memory, for the second pass.
// ---------------------------------------------------------------------------
// F16 = true writes each code as the equal f16 value (an integer in
// [-127, 127], exact), the operand layout of the f16 MMA.
//
// No clamp is needed: with inv = RN(qmax / amax) and |h| <= amax,
// |RN(h * inv)| <= qmax (1 + 2^-24)^2 < qmax + 1/2, so the rounded code
// never leaves [-qmax, qmax].  The int8 path keeps each code's low byte
// (two's complement) and packs four with byte permutes; the f16 path
// rounds in fp32 (rint), turns -0 into +0 (the code 0 is stored as +0) and
// converts two codes per instruction.  The rounding is a conversion of the
// rounded product, never an addition after it: the compiler may fuse a
// product and a following addition into one FMA, which rounds once.
// rint(RN(x * inv)) in the low byte of the result, for |RN(x * inv)| < 2^22:
// RN(y + 1.5 * 2^23) holds rint(y) (RN to even) in its low mantissa bits.
// __fmul_rn and __fadd_rn are never contracted into one FMA (which would
// round x * inv + 1.5 * 2^23 once and differ where RN(x * inv) is a
// half-integer); the packed f32x2 forms gave exactly that difference.
__device__ __forceinline__ int rint_low_byte(float x, float inv) {
  return static_cast<int>(__float_as_uint(__fadd_rn(__fmul_rn(x, inv), 12582912.0f)));
}

__device__ __forceinline__ uint32_t pack4_s8(int a0, int a1, int a2, int a3) {
  const uint32_t t01 = __byte_perm(static_cast<uint32_t>(a0), static_cast<uint32_t>(a1), 0x0040);
  const uint32_t t23 = __byte_perm(static_cast<uint32_t>(a2), static_cast<uint32_t>(a3), 0x0040);
  return __byte_perm(t01, t23, 0x5410);
}

template <bool F16>
__device__ __forceinline__ void quant_int8_half(const float2 (&P)[32], float inv, uint8_t* dst) {
  if constexpr (F16) {
    uint32_t w[32];   // element pairs (2i, 2i+1) and (32+2i, 32+2i+1) -> f16 words
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 a = __fmul2_rn(P[2 * i], make_float2(inv, inv));       // (x_2i, x_32+2i)
      const float2 c = __fmul2_rn(P[2 * i + 1], make_float2(inv, inv));   // (x_2i+1, x_32+2i+1)
      const float l0 = __fadd_rn(rintf(a.x), 0.f), l1 = __fadd_rn(rintf(c.x), 0.f);
      const float h0 = __fadd_rn(rintf(a.y), 0.f), h1 = __fadd_rn(rintf(c.y), 0.f);
      const __half2 lo = __floats2half2_rn(l0, l1);
      const __half2 hi = __floats2half2_rn(h0, h1);
      w[i] = *reinterpret_cast<const uint32_t*>(&lo);          // elements 2i, 2i+1
      w[16 + i] = *reinterpret_cast<const uint32_t*>(&hi);     // elements 32+2i, 32+2i+1
    }
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int i = 0; i < 8; ++i) d[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  } else {
    uint32_t w[16];
    const float2 inv2 = make_float2(inv, inv);
#pragma unroll
    for (int i = 0; i < 8; ++i) {   // elements 4i..4i+3 (.x halves) and 32+4i.. (.y halves)
      const float2 y0 = __fmul2_rn(P[4 * i], inv2), y1 = __fmul2_rn(P[4 * i + 1], inv2);
      const float2 y2 = __fmul2_rn(P[4 * i + 2], inv2), y3 = __fmul2_rn(P[4 * i + 3], inv2);
      w[i] = pack4_s8(__float2int_rn(y0.x), __float2int_rn(y1.x), __float2int_rn(y2.x), __float2int_rn(y3.x));
      w[8 + i] = pack4_s8(__float2int_rn(y0.y), __float2int_rn(y1.y), __float2int_rn(y2.y), __float2int_rn(y3.y));
    }
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) d[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  }
}

template <bool F16>
__global__ void __launch_bounds__(kThreadsHbm)
    k_quant_int8_token(const __grid_constant__ CUtensorMap tm_x, int64_t M, int32_t K, int hadamard,
                       int32_t buf_bytes, int32_t box_rows, int qmax, uint8_t* __restrict__ codes,
                       float* __restrict__ scales, int* status, const int32_t* gate, int32_t gate_value) {
  extern __shared__ uint8_t s_raw[];
  __shared__ uint64_t bars[2 * (kThreadsHbm / 32)];
  uint8_t* s_rows = ring_base(s_raw);
  pdl_wait();
  if (gated_off(gate, gate_value)) {
    pdl_release();
    return;
  }
  const uint32_t lane = lane_id();
  const int wid = threadIdx.x >> 5;
  const int32_t halves = K >> 6;                 // 64-element half blocks (128-byte rows) per token row
  const int32_t passes = (halves + 31) >> 5;
  uint8_t* const rows0 = s_rows + (2 * wid) * buf_bytes;   // the warp's two row buffers
  auto rows = [&](int b) { return rows0 + b * buf_bytes; };
  uint64_t* bar = bars + 2 * wid;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + wid;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  if (lane == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncwarp();
  auto issue_row = [&](int64_t r, int b) {   // token row r into buffer b: halves / box_rows boxes
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar[b], static_cast<uint32_t>(halves) * kLaneBytes);
      for (int32_t y = 0; y < halves; y += box_rows)
        tma_load_2d(rows(b) + y * kLaneBytes, &tm_x, &bar[b], 0, static_cast<int32_t>(r * halves + y));
    }
  };
  auto load_half = [&](const uint8_t* row, int p, float2 (&P)[32]) {
    if (32 * p + static_cast<int32_t>(lane) < halves) {
      read_half(row + p * kChunkBytes, P);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) P[j] = make_float2(0.f, 0.f);
    }
    if (hadamard) fwht128_half(P);   // all lanes (pair shuffles)
  };
  if (gw < M) issue_row(gw, 0);
  int k = 0;
  bool ok = true;
  for (int64_t r = gw; r < M; r += nw, ++k) {
    // the buffer refilled here was read in the previous iteration, before its closing __syncwarp
    if (r + nw < M) issue_row(r + nw, (k + 1) & 1);
    ok = __all_sync(0xffffffffu, mbar_wait(&bar[k & 1], static_cast<uint32_t>((k >> 1) & 1), kDrainLimit));
    if (!ok) break;
    const uint8_t* row = rows(k & 1);
    float2 P[32];
    float m = 0.f;
    for (int p = 0; p < passes; ++p) {
      load_half(row, p, P);
#pragma unroll
      for (int j = 0; j < 32; j += 2)
        m = fmax3(m, fmax3(fabsf(P[j].x), fabsf(P[j].y), fabsf(P[j + 1].x)), fabsf(P[j + 1].y));
    }
    m = warp_max(m);
    const float fq = static_cast<float>(qmax);
    const float inv = (m == 0.f) ? 0.f : __fdiv_rn(fq, m);
    if (lane == 0) scales[r] = (m == 0.f) ? 0.f : __fdiv_rn(m, fq);
    constexpr int kElemBytes = F16 ? 2 : 1;
    uint8_t* crow = codes + r * K * kElemBytes;
    for (int p = 0; p < passes; ++p) {
      if (passes > 1) load_half(row, p, P);    // one pass: P still holds the rotated half
      const int32_t hb = 32 * p + static_cast<int32_t>(lane);
      if (hb < halves) quant_int8_half<F16>(P, inv, crow + 64 * kElemBytes * hb);
    }
    __syncwarp();
  }
  pdl_release();
  if (!ok && lane == 0) {   // timed out at iteration k: let this row's and the next row's loads land
    record_error(status, QL_ERR_TIMEOUT);
    const int64_t r = gw + static_cast<int64_t>(k) * nw;
    (void)mbar_wait(&bar[k & 1], static_cast<uint32_t>((k >> 1) & 1), kDrainLimit);
    if (r + nw < M) (void)mbar_wait(&bar[(k + 1) & 1], static_cast<uint32_t>(((k + 1) >> 1) & 1), kDrainLimit);
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// Per-tensor INT8 in Q-ARVD channel order.  Output row = Kp bytes; slot j
// takes input channel gather[j] (or 0 for a padding slot).  The scale comes
// from the device amax of the un-rotated tensor.
//
// A CTA walks groups of G consecutive rows (G from the host: about 12 KB of
// bf16 per group) through a ring of R group buffers (R from the host, 2 to
// 4: the depth that keeps the most groups in flight per SM at the occupancy
// it allows), R - 1 groups in flight while one is read.  Thread 0 brings each row of
// a group into its own shared-memory buffer by one bulk copy; each buffer
// ends with 16 zero bytes, and the gather table (uint16 in shared memory)
// sends padding slots to that zero element, so every slot is one table
// read, one row read and no branch.  The warps work independently: each
// waits on the group's mbarrier, takes whole 512-slot units (lane l: slots
// 4l + 128s + c, s, c < 4; consecutive lanes read neighbouring channels),
// writes four codes per lane and step as one coalesced word, and arrives on
// the group's release barrier; thread 0 refills a buffer once every warp has
// released it.  Units are numbered across groups and dealt to the warps
// round-robin, so a group's ragged unit count does not load one warp more
// than the others.
//
// Codes: rint(RN(x * RN(qmax / amax))) by rint_low_byte, low bytes packed
// by byte permutes; no clamp is needed, as in the per-token quantizer
// (|y| < qmax + 1/2).
// ---------------------------------------------------------------------------
constexpr int kPermMaxRing = 4;
constexpr int kPermThreads = 256;
constexpr int kPermWarps = kPermThreads / 32;
constexpr int kPermUnit = 512;   // slots per warp unit
struct PermLayout {
  int32_t G, row_stride, group_bytes, table_bytes, ring;
  PermLayout(int32_t K, int32_t Kp, int32_t R)
      : G(std::max(1, 12288 / (2 * K))), row_stride(2 * K + 16), group_bytes(G * (2 * K + 16)),
        table_bytes((2 * Kp + 15) / 16 * 16), ring(R) {}
  int32_t total() const { return table_bytes + ring * group_bytes; }
};

__global__ void __launch_bounds__(kPermThreads)
    k_quant_int8_tensor_perm(const uint8_t* __restrict__ x, int64_t M, int32_t K, int32_t Kp,
                             const int32_t* __restrict__ gather, const float* amax_in, int qmax,
                             int8_t* __restrict__ codes, float* __restrict__ scale_out, int* status,
                             int32_t G, int32_t row_stride, int32_t group_bytes, int32_t table_bytes, int32_t R) {
  extern __shared__ __align__(16) uint8_t s_perm[];
  __shared__ uint64_t full[kPermMaxRing], release[kPermMaxRing];
  __shared__ int s_fail;
  uint16_t* s_gather = reinterpret_cast<uint16_t*>(s_perm);
  uint8_t* ring = s_perm + table_bytes;
  const int64_t ngroups = (M + G - 1) / G;
  const int warp = threadIdx.x >> 5;
  const uint32_t lane = lane_id();
  if (threadIdx.x == 0) {
    for (int i = 0; i < R; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&release[i], kPermWarps);
    }
    fence_mbar_init();
    s_fail = 0;
  }
  for (int i = threadIdx.x; i < R * G; i += kPermThreads)   // the zero element after each row buffer
    *reinterpret_cast<uint4*>(ring + (i / G) * group_bytes + (i % G) * row_stride + 2 * K) = make_uint4(0, 0, 0, 0);
  __syncthreads();
  pdl_wait();
  const int64_t first = blockIdx.x, step = gridDim.x;
  auto issue = [&](int64_t grp, int slot) {   // thread 0 only
    const int32_t rows = static_cast<int32_t>(M - grp * G < G ? M - grp * G : G);
    mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(rows) * 2u * static_cast<uint32_t>(K));
    for (int32_t r = 0; r < rows; ++r)
      bulk_load(ring + slot * group_bytes + r * row_stride, x + (grp * G + r) * 2 * K, 2u * static_cast<uint32_t>(K),
                &full[slot]);
  };
  int issued = 0;   // groups issued by thread 0 (iterations 0 .. issued - 1)
  if (threadIdx.x == 0)
    for (; issued < R && first + issued * step < ngroups; ++issued) issue(first + issued * step, issued);
  for (int i = threadIdx.x; i < Kp; i += kPermThreads) {   // padding slots (-1) read the zero element
    const int32_t g = gather[i];
    s_gather[i] = static_cast<uint16_t>(g < 0 ? K : g);
  }
  const float amax = ld_dep(amax_in);
  const float fq = static_cast<float>(qmax);
  const float inv = (amax == 0.f) ? 0.f : __fdiv_rn(fq, amax);
  if (blockIdx.x == 0 && threadIdx.x == 0) *scale_out = (amax == 0.f) ? 0.f : __fdiv_rn(amax, fq);
  __syncthreads();   // gather table complete
  const int32_t upr = (Kp + kPermUnit - 1) / kPermUnit;   // units per row
  int32_t deal = 0;                                       // units dealt before this group, mod kPermWarps
  int k = 0;
  bool ok = true;
  for (int64_t grp = first; grp < ngroups; grp += step, ++k) {
    const int slot = k % R;
    if (threadIdx.x == 0 && k > 0 && first + static_cast<int64_t>(k - 1 + R) * step < ngroups) {
      // refill the buffer of iteration k - 1 with iteration k - 1 + R's rows
      // once every warp has released it
      const int prev = (k - 1) % R;
      if (!mbar_wait(&release[prev], static_cast<uint32_t>(((k - 1) / R) & 1), kDrainLimit)) {
        s_fail = 1;
        record_error(status, QL_ERR_TIMEOUT);
      } else {
        issue(first + static_cast<int64_t>(k - 1 + R) * step, prev);
        ++issued;
      }
    }
    int w_ok = 1;
    if (lane == 0)
      w_ok = *reinterpret_cast<volatile int*>(&s_fail) == 0 &&
             mbar_wait(&full[slot], static_cast<uint32_t>((k / R) & 1), kDrainLimit);
    if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
      if (lane == 0 && !s_fail) {
        s_fail = 1;
        record_error(status, QL_ERR_TIMEOUT);
      }
      ok = false;
      break;
    }
    const int32_t rows = static_cast<int32_t>(M - grp * G < G ? M - grp * G : G);
    const int32_t units = rows * upr;
    const uint8_t* buf = ring + slot * group_bytes;
    for (int32_t u = (warp - deal + kPermWarps) % kPermWarps; u < units; u += kPermWarps) {
      const int32_t r = u / upr;
      const int32_t j0 = (u - r * upr) * kPermUnit + 4 * static_cast<int32_t>(lane);
      const unsigned short* xr = reinterpret_cast<const unsigned short*>(buf + r * row_stride);
      int8_t* dst = codes + (grp * G + r) * Kp;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const int32_t j = j0 + 128 * s;
        if (j < Kp) {   // Kp is a multiple of 32: four slots are all in or all out
          const uint2 gi = *reinterpret_cast<const uint2*>(s_gather + j);
          const float2 v01 = make_float2(__uint_as_float(static_cast<uint32_t>(xr[gi.x & 0xFFFFu]) << 16),
                                         __uint_as_float(static_cast<uint32_t>(xr[gi.x >> 16]) << 16));
          const float2 v23 = make_float2(__uint_as_float(static_cast<uint32_t>(xr[gi.y & 0xFFFFu]) << 16),
                                         __uint_as_float(static_cast<uint32_t>(xr[gi.y >> 16]) << 16));
          *reinterpret_cast<uint32_t*>(dst + j) =
              pack4_s8(rint_low_byte(v01.x, inv), rint_low_byte(v01.y, inv), rint_low_byte(v23.x, inv),
                       rint_low_byte(v23.y, inv));
        }
      }
    }
    deal = (deal + units) % kPermWarps;
    __syncwarp();
    if (lane == 0) mbar_arrive(&release[slot]);
  }
  pdl_release();
  if (threadIdx.x == 0) {
    // every copy issued must land before the CTA exits; after a normal walk
    // each was consumed, after a failure wait for the rest with a bounded budget
    // (only the last R issued can be in flight: a buffer is refilled
    // after every warp consumed its previous copy)
    if (!ok || *reinterpret_cast<volatile int*>(&s_fail))
      for (int j = issued > R ? issued - R : 0; j < issued; ++j)
        (void)mbar_wait(&full[j % R], static_cast<uint32_t>((j / R) & 1), kDrainLimit);
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// f16 expansion of NVFP4 weights for the INT8 route's GEMM: out[n, k] =
// e2m1(code[n, k]) * e4m3(sb[n, k/16]) (without the tensor scale), exact in
// f16 (at most 6 significant bits, magnitudes 2^-10 .. 2688).  A thread
// expands 8 consecutive codes (one 32-bit word, half a scale block).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreadsHbm)
    k_expand_nvfp4_f16(const uint32_t* __restrict__ codes, const uint8_t* __restrict__ sf, int32_t N, int32_t K,
                       uint4* __restrict__ out) {
  const int64_t words = static_cast<int64_t>(N) * (K / 8);
  const int32_t wpr = K / 8, k_atoms = K / 64;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < words;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = i / wpr;
    const int32_t c8 = static_cast<int32_t>(i - n * wpr);
    const uint32_t sb = sf[sf_mma_offset(n, c8 >> 1, k_atoms)];
    out[i] = fp4x8_scaled_to_f16(__ldg(codes + i), sb);
  }
}

// Test hook: counts the dividends a (fp32 bit patterns a_begin ..
// a_begin + count - 1, non-negative and finite) where the quantizer's
// block-scale division differs from __fdiv_rn(a, d).
__global__ void k_debug_div_check(float d, uint32_t a_begin, uint64_t count,
                                  unsigned long long* mismatches) {
  const Nvfp4ScaleDiv sd(d);
  unsigned long long bad = 0;
  for (uint64_t i = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
    const float a = __uint_as_float(a_begin + static_cast<uint32_t>(i));
    const float q = sd.fast ? div_rn_by(a, sd.d, sd.r) : __fdiv_rn(a, d);
    bad += __float_as_uint(q) != __float_as_uint(__fdiv_rn(a, d));
  }
  for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
  if ((threadIdx.x & 31) == 0 && bad) atomicAdd(mismatches, bad);
}

// --------------------------------------------------------------------------
// Host launchers
// --------------------------------------------------------------------------
// The streaming kernels' view of a contiguous bf16 tensor: rows of 128 bytes
// (half a Hadamard block), a box of 32 rows (one warp's 4 KB chunk), 128-byte
// swizzle.  total_bytes is a multiple of 256.
static bool make_stream_tmap(CUtensorMap* tm, const void* x, int64_t total_bytes, uint32_t box_rows = 32) {
  if (total_bytes / kLaneBytes >= (int64_t(1) << 31)) return false;   // row coordinates are 32-bit
  return make_tmap_2d(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, x, kLaneBytes, total_bytes / kLaneBytes, kLaneBytes,
                      kLaneBytes, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

ql_status launch_debug_div_check(float d, uint32_t a_begin, uint64_t count, unsigned long long* mismatches,
                                 cudaStream_t st) {
  const int grid = num_sms() * 8;
  k_debug_div_check<<<grid, 256, 0, st>>>(d, a_begin, count, mismatches);
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

int hbm_grid(int64_t work_items, int per_cta) {
  const int64_t want = (work_items + per_cta - 1) / per_cta;
  const int64_t cap = static_cast<int64_t>(num_sms()) * kHbmCtasPerSm;
  return static_cast<int>(std::max<int64_t>(1, std::min(want, cap)));
}

// Streaming kernels with the cp.async ring: 96 KB of shared memory and at
// most 128 registers per thread, two resident CTAs per SM.
static int ring_grid(int64_t nchunks) {
  const int64_t want = (nchunks + kWarpsPerCta - 1) / kWarpsPerCta;
  return static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>(want, static_cast<int64_t>(num_sms()) * kRingCtasPerSm)));
}

ql_status launch_amax(const void* x, int64_t M, int32_t K, int hadamard, float* amax_out, void* ws,
                      cudaStream_t st, Gate gate) {
  const int64_t units = M * (K / 128);
  if (units == 0) return cudaMemsetAsync(amax_out, 0, sizeof(float), st) == cudaSuccess ? QL_OK : QL_ERR_CUDA;
  const int grid = ring_grid((units * 256 + kChunkBytes - 1) / kChunkBytes);
  float* partials = static_cast<float*>(ws);
  unsigned int* ticket = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + kAmaxPartialBytes);
  CUtensorMap tm;
  if (!make_stream_tmap(&tm, x, units * 256)) return QL_ERR_CUDA;
  if (!set_smem_attr(reinterpret_cast<const void*>(k_amax), kRingBytesPerCta + kRingAlignPad)) return QL_ERR_CUDA;
  if (launch_pdl(k_amax, dim3(grid), dim3(kThreadsHbm), kRingBytesPerCta + kRingAlignPad, st, 1, tm, units * 256,
                 hadamard, partials, ticket, amax_out, status_word(), gate.route, gate.value) != cudaSuccess) {
    (void)cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

ql_status launch_quant_nvfp4(const void* x, int64_t M, int32_t K, int hadamard, const float* amax_in,
                             void* codes, void* sf_mma, void* sf_rm, float* g_out, cudaStream_t st, int decomp,
                             Gate gate) {
  if (M == 0) return QL_OK;
  const int64_t nchunks = (M * K * 2 + kChunkBytes - 1) / kChunkBytes;
  const int grid = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>((nchunks + kQuantWarps - 1) / kQuantWarps, num_sms())));
  auto kern = decomp ? k_quant_nvfp4<true> : k_quant_nvfp4<false>;
  CUtensorMap tm;
  if (!make_stream_tmap(&tm, x, M * K * 2)) return QL_ERR_CUDA;
  if (!set_smem_attr(reinterpret_cast<const void*>(kern), kQuantRingBytes + kRingAlignPad)) return QL_ERR_CUDA;
  if (launch_pdl(kern, dim3(grid), dim3(kQuantThreads), kQuantRingBytes + kRingAlignPad, st, 1, tm, M, K, hadamard,
                 amax_in, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(sf_mma), static_cast<uint8_t*>(sf_rm),
                 g_out, status_word(), gate.route, gate.value) != cudaSuccess) {
    (void)cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

ql_status launch_expand_nvfp4_f16(const void* codes, const void* sf, int32_t N, int32_t K, void* out,
                                  cudaStream_t st) {
  const int grid = hbm_grid(static_cast<int64_t>(N) * (K / 8), kThreadsHbm);
  k_expand_nvfp4_f16<<<grid, kThreadsHbm, 0, st>>>(static_cast<const uint32_t*>(codes),
                                                   static_cast<const uint8_t*>(sf), N, K, static_cast<uint4*>(out));
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

ql_status launch_quant_int8_token(const void* x, int64_t M, int32_t K, int hadamard, void* codes,
                                  float* scales, cudaStream_t st, int f16_codes, int qmax, Gate gate) {
  if (M == 0) return QL_OK;
  // a token row is K/64 rows of 128 bytes; TMA boxes of at most 256 rows that tile it exactly
  const int32_t halves = K / 64;
  int32_t box_rows = std::min<int32_t>(halves, 256);
  while (halves % box_rows != 0) --box_rows;
  const int64_t buf = (static_cast<int64_t>(halves) * kLaneBytes + 1023) / 1024 * 1024;   // 1024-byte aligned
  const int64_t per_warp = 2 * buf;                                                        // two row buffers
  if (per_warp > 200 * 1024) return QL_ERR_UNSUPPORTED_SHAPE;
  const int warps = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(kThreadsHbm / 32, (200 * 1024) / per_warp)));
  const size_t smem = static_cast<size_t>(warps) * per_warp + kRingAlignPad;
  const int per_sm = std::max(1, std::min(4, static_cast<int>((227 * 1024) / smem)));
  const int64_t want = (M + warps - 1) / warps;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, static_cast<int64_t>(per_sm) * num_sms())));
  CUtensorMap tm;
  if (!make_stream_tmap(&tm, x, M * K * 2, static_cast<uint32_t>(box_rows))) return QL_ERR_CUDA;
  auto kern = f16_codes ? k_quant_int8_token<true> : k_quant_int8_token<false>;
  if (!set_smem_attr(reinterpret_cast<const void*>(kern), static_cast<int>(smem))) return QL_ERR_CUDA;
  if (launch_pdl(kern, dim3(grid), dim3(32 * warps), smem, st, 1, tm, M, K, hadamard, static_cast<int32_t>(buf),
                 box_rows, qmax, static_cast<uint8_t*>(codes), scales, status_word(), gate.route,
                 gate.value) != cudaSuccess) {
    (void)cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

ql_status launch_quant_int8_tensor_perm(const void* x, int64_t M, int32_t K, int32_t Kp,
                                        const int32_t* gather, const float* amax_in, void* codes,
                                        float* scale_out, cudaStream_t st, int qmax) {
  if (K > 65535) return QL_ERR_UNSUPPORTED_SHAPE;   // uint16 gather table
  // ring depth: the most groups in flight per SM ((depth - 1) per resident
  // CTA, the one being read aside), fewer slots where that fits more CTAs
  PermLayout L(K, Kp, 0);
  int best = 0, best_flight = 0;
  for (int R = kPermMaxRing; R >= 2; --R) {
    L.ring = R;
    if (L.total() > 220 * 1024) continue;
    if (!set_smem_attr(reinterpret_cast<const void*>(k_quant_int8_tensor_perm), L.total())) return QL_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_quant_int8_tensor_perm, kPermThreads,
                                                      L.total()) != cudaSuccess)
      return QL_ERR_CUDA;
    if (per_sm * (R - 1) > best_flight) {
      best_flight = per_sm * (R - 1);
      best = R;
    }
  }
  if (best == 0) return QL_ERR_UNSUPPORTED_SHAPE;   // not even two row groups fit in shared memory
  L.ring = best;
  if (!set_smem_attr(reinterpret_cast<const void*>(k_quant_int8_tensor_perm), L.total())) return QL_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_quant_int8_tensor_perm, kPermThreads, L.total()) !=
          cudaSuccess ||
      per_sm < 1)
    return QL_ERR_CUDA;
  // as many CTAs as can be resident at once: each walks row groups
  // blockIdx.x, blockIdx.x + gridDim.x, ..., so a CTA that waited for a free
  // SM would start its rows late
  const int64_t ngroups = (M + L.G - 1) / L.G;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(ngroups, static_cast<int64_t>(per_sm) * num_sms())));
  if (launch_pdl(k_quant_int8_tensor_perm, dim3(grid), dim3(kPermThreads), L.total(), st, 1,
                 static_cast<const uint8_t*>(x), M, K, Kp, gather, amax_in, qmax, static_cast<int8_t*>(codes),
                 scale_out, status_word(), L.G, L.row_stride, L.group_bytes, L.table_bytes, L.ring) != cudaSuccess) {
    (void)cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

}  // namespace ql
