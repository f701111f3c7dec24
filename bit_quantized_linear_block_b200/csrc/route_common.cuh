// Device pieces of the DMPQ router shared by qlinear_route,
// qlinear_route_noalloc and the token-split form (qlinear_gamma_sums,
// qlinear_route_from_sums) (6Bit-Diffusion, Methodology A.1 / B.1):
// Gamma = sum |out - in| / sum |in| with fp32 differences and fp64 sums.
#pragma once

#include "ql_common.cuh"

namespace ql {

constexpr int kRouteUnroll = 4;   // 16-byte vectors of each tensor in flight per thread

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// fp64 sums of |y - x| (s1) and |x| (s0) over the 8 bf16 pairs of one
// 16-byte vector of each tensor.
__device__ __forceinline__ void gamma_accumulate(const uint4& a, const uint4& b, double& s1, double& s0) {
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w};
  const uint32_t wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float x0 = bf16_lo(wa[k]), x1 = bf16_hi(wa[k]);
    const float y0 = bf16_lo(wb[k]), y1 = bf16_hi(wb[k]);
    s1 += static_cast<double>(fabsf(__fsub_rn(y0, x0)));
    s1 += static_cast<double>(fabsf(__fsub_rn(y1, x1)));
    s0 += static_cast<double>(fabsf(x0));
    s0 += static_cast<double>(fabsf(x1));
  }
}

// This thread's share of both sums: grid-stride over 16-byte vectors with
// kRouteUnroll vectors of each tensor loaded before any is used (enough
// bytes in flight to cover HBM latency), the < 8-element tail by the first
// threads.
__device__ __forceinline__ void gamma_thread_sums(const uint4* __restrict__ in, const uint4* __restrict__ out,
                                                  int64_t numel, double& s1, double& s0) {
  const int64_t nvec = numel >> 3;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthr = static_cast<int64_t>(gridDim.x) * blockDim.x;
  double a1 = 0.0, a0 = 0.0, b1 = 0.0, b0 = 0.0;
  int64_t i = tid;
  for (; i + (kRouteUnroll - 1) * nthr < nvec; i += kRouteUnroll * nthr) {
    uint4 va[kRouteUnroll], vb[kRouteUnroll];
#pragma unroll
    for (int u = 0; u < kRouteUnroll; ++u) {
      va[u] = __ldcs(in + i + u * nthr);
      vb[u] = __ldcs(out + i + u * nthr);
    }
#pragma unroll
    for (int u = 0; u < kRouteUnroll; u += 2) {
      gamma_accumulate(va[u], vb[u], a1, a0);
      gamma_accumulate(va[u + 1], vb[u + 1], b1, b0);
    }
  }
  for (; i < nvec; i += nthr) gamma_accumulate(__ldcs(in + i), __ldcs(out + i), a1, a0);
  if (tid < (numel & 7)) {
    const unsigned short* ia = reinterpret_cast<const unsigned short*>(in) + (nvec << 3) + tid;
    const unsigned short* ib = reinterpret_cast<const unsigned short*>(out) + (nvec << 3) + tid;
    const float x = __uint_as_float(static_cast<uint32_t>(*ia) << 16);
    const float y = __uint_as_float(static_cast<uint32_t>(*ib) << 16);
    a1 += static_cast<double>(fabsf(__fsub_rn(y, x)));
    a0 += static_cast<double>(fabsf(x));
  }
  s1 = a1 + b1;
  s0 = a0 + b0;
}

// Block-wide sums of (s1, s0) into thread 0's return values (blockDim.x a
// multiple of 32, at most 1024).
__device__ __forceinline__ void gamma_block_sums(double& s1, double& s0) {
  __shared__ double red[2][32];
  s1 = warp_sum_f64(s1);
  s0 = warp_sum_f64(s0);
  const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (lane_id() == 0) {
    red[0][w] = s1;
    red[1][w] = s0;
  }
  __syncthreads();
  if (w == 0) {
    s1 = lane_id() < nw ? red[0][lane_id()] : 0.0;
    s0 = lane_id() < nw ? red[1][lane_id()] : 0.0;
    s1 = warp_sum_f64(s1);
    s0 = warp_sum_f64(s0);
  }
  __syncthreads();
}

// Per-CTA partials, then the last CTA to finish (atomic ticket) adds all
// partials with the whole block.  Returns true in thread 0 of that CTA only,
// with the totals in (s1, s0); the ticket is reset for the next call.
__device__ __forceinline__ bool gamma_total(double& s1, double& s0, double* partials, unsigned int* ticket) {
  __shared__ bool s_last;
  gamma_block_sums(s1, s0);
  if (threadIdx.x == 0) {
    partials[2 * blockIdx.x] = s1;
    partials[2 * blockIdx.x + 1] = s0;
    __threadfence();
    s_last = atomicAdd(ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return false;
  __threadfence();
  double a = 0.0, b = 0.0;
  const volatile double* p = partials;
  for (unsigned int i = threadIdx.x; i < gridDim.x; i += blockDim.x) {
    a += p[2 * i];
    b += p[2 * i + 1];
  }
  gamma_block_sums(a, b);
  if (threadIdx.x != 0) return false;
  s1 = a;
  s0 = b;
  *ticket = 0u;
  return true;
}

// Gamma = s1 / s0 (+inf when s0 is 0); route = 1 (INT8) if Gamma > threshold.
__device__ __forceinline__ void gamma_decide(double s1, double s0, float threshold, double* gamma_out,
                                             int32_t* route_out) {
  const double gamma = (s0 == 0.0) ? __longlong_as_double(0x7ff0000000000000ll) : s1 / s0;
  *gamma_out = gamma;
  *route_out = (gamma > static_cast<double>(threshold)) ? 1 : 0;
}

__device__ __forceinline__ void gamma_finish(double s1, double s0, double* partials, unsigned int* ticket,
                                             float threshold, double* gamma_out, int32_t* route_out) {
  if (gamma_total(s1, s0, partials, ticket)) gamma_decide(s1, s0, threshold, gamma_out, route_out);
}

}  // namespace ql
