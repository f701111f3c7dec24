// DMPQ router and Q-ARVD weight-preparation kernels.
//
// Router (6Bit-Diffusion, Methodology A.1 / B.1): Gamma = ||out - in||_1 /
// ||in||_1 of one transformer block; INT8 activations when Gamma exceeds
// the threshold, NVFP4 otherwise.  One launch: grid-stride 16-byte loads of
// both tensors, fp32 differences, fp64 per-thread sums, per-CTA partials,
// and the last CTA to finish (atomic ticket) adds the partials and writes
// Gamma and the route.  With the block's tokens split across ranks, each
// rank writes its two sums instead (k_gamma_sums), the ranks add them, and
// a one-thread kernel (k_route_from_sums) makes the same decision.
//
// Q-ARVD (Methodology / Formula and operation flow): input-channel L2 norms
// of W, median and MAD, modified z-score M_k = (v_k - median)/MAD, outlier
// iff M_k > tau and v_k > alpha * median; normal channels then outlier
// channels, each class padded to 32; per output row one INT4 scale per
// class.
#include "ql_common.cuh"
#include "route_common.cuh"
#include "gemm_common.cuh"
#include "launchers.h"

namespace ql {


// ---------------------------------------------------------------------------
// Gamma / route
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreadsHbm)
    k_gamma_route(const uint4* __restrict__ in, const uint4* __restrict__ out, int64_t numel,
                  double* __restrict__ partials, unsigned int* __restrict__ ticket, float threshold,
                  double* __restrict__ gamma_out, int32_t* __restrict__ route_out) {
  pdl_wait();
  double s1, s0;
  gamma_thread_sums(in, out, numel, s1, s0);
  pdl_release();
  gamma_finish(s1, s0, partials, ticket, threshold, gamma_out, route_out);
}

// Token-split form: this rank's two sums only (sums_out[0] = sum |out - in|,
// sums_out[1] = sum |in|); the ranks add them and k_route_from_sums decides.
__global__ void __launch_bounds__(kThreadsHbm)
    k_gamma_sums(const uint4* __restrict__ in, const uint4* __restrict__ out, int64_t numel,
                 double* __restrict__ partials, unsigned int* __restrict__ ticket, double* __restrict__ sums_out) {
  pdl_wait();
  double s1, s0;
  gamma_thread_sums(in, out, numel, s1, s0);
  pdl_release();
  if (gamma_total(s1, s0, partials, ticket)) {
    sums_out[0] = s1;
    sums_out[1] = s0;
  }
}

__global__ void k_route_from_sums(const double* __restrict__ sums, float threshold, double* __restrict__ gamma_out,
                                  int32_t* __restrict__ route_out) {
  pdl_wait();
  if (threadIdx.x == 0) gamma_decide(sums[0], sums[1], threshold, gamma_out, route_out);
}

// ---------------------------------------------------------------------------
// Q-ARVD: partial column sums of squares.  Thread = one pair of adjacent
// columns; blockIdx.y = one slice of rows.  partial[slice][k].
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreadsHbm)
    k_colnorm_partial(const uint32_t* __restrict__ w, int32_t N, int32_t K, int32_t rows_per_slice,
                      double* __restrict__ partial) {
  const int32_t pair = blockIdx.x * blockDim.x + threadIdx.x;
  if (pair >= K / 2) return;
  const int32_t r0 = blockIdx.y * rows_per_slice;
  const int32_t r1 = min(N, r0 + rows_per_slice);
  double a = 0.0, b = 0.0;
  for (int32_t r = r0; r < r1; ++r) {
    const uint32_t v = __ldg(w + static_cast<int64_t>(r) * (K / 2) + pair);
    const double x = static_cast<double>(bf16_lo(v)), y = static_cast<double>(bf16_hi(v));
    a += x * x;
    b += y * y;
  }
  partial[static_cast<int64_t>(blockIdx.y) * K + 2 * pair] = a;
  partial[static_cast<int64_t>(blockIdx.y) * K + 2 * pair + 1] = b;
}

// Ascending bitonic sort of n (power of two) doubles in shared memory.
__device__ void bitonic_sort(double* s, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool up = (i & size) == 0;
          const double a = s[i], b = s[j];
          if ((a > b) == up) {
            s[i] = b;
            s[j] = a;
          }
        }
      }
    }
  }
  __syncthreads();
}

__device__ __forceinline__ double median_of_sorted(const double* s, int n) {
  return (n & 1) ? s[n / 2] : (s[n / 2 - 1] + s[n / 2]) / 2.0;
}

// Single CTA.  Dynamic shared memory: npow2 doubles (sort buffer) + K ints.
__global__ void __launch_bounds__(1024)
    k_qarvd_select(const double* __restrict__ partial, int32_t slices, int32_t K, int32_t npow2,
                   float tau, float alpha, int32_t Kp, double* __restrict__ norms,
                   uint8_t* __restrict__ mask, int32_t* __restrict__ perm,
                   int32_t* __restrict__ gather, int32_t* __restrict__ kinfo) {
  extern __shared__ double s_buf[];
  int32_t* s_flag = reinterpret_cast<int32_t*>(s_buf + npow2);
  __shared__ double s_med, s_mad;
  __shared__ int32_t s_scan[1024 + 1];
  const double inf = __longlong_as_double(0x7ff0000000000000ll);
  for (int k = threadIdx.x; k < npow2; k += blockDim.x) {
    double v = inf;
    if (k < K) {
      double acc = 0.0;
      for (int s = 0; s < slices; ++s) acc += partial[static_cast<int64_t>(s) * K + k];
      v = sqrt(acc);
      norms[k] = v;
    }
    s_buf[k] = v;
  }
  bitonic_sort(s_buf, npow2);
  if (threadIdx.x == 0) s_med = median_of_sorted(s_buf, K);
  __syncthreads();
  const double med = s_med;
  for (int k = threadIdx.x; k < npow2; k += blockDim.x) s_buf[k] = (k < K) ? fabs(norms[k] - med) : inf;
  bitonic_sort(s_buf, npow2);
  if (threadIdx.x == 0) s_mad = median_of_sorted(s_buf, K);
  __syncthreads();
  const double mad = s_mad;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const double v = norms[k];
    const double z = (v - med) / mad;   // IEEE: MAD == 0 gives +-inf or NaN
    const int32_t o = (z > static_cast<double>(tau)) && (v > static_cast<double>(alpha) * med);
    s_flag[k] = o;
    mask[k] = static_cast<uint8_t>(o);
  }
  __syncthreads();
  // Stable partition: each thread owns a contiguous run of channels.
  const int per = (K + blockDim.x - 1) / blockDim.x;
  const int k0 = threadIdx.x * per, k1 = min(K, k0 + per);
  int cnt = 0;
  for (int k = k0; k < k1; ++k) cnt += s_flag[k];
  s_scan[threadIdx.x + 1] = cnt;
  if (threadIdx.x == 0) s_scan[0] = 0;
  __syncthreads();
  if (threadIdx.x == 0)
    for (int i = 1; i <= static_cast<int>(blockDim.x); ++i) s_scan[i] += s_scan[i - 1];
  __syncthreads();
  const int n_out = s_scan[blockDim.x];
  const int k_norm = K - n_out;
  const int k_norm_pad = (k_norm + 31) & ~31;
  const int k_out_pad = (n_out + 31) & ~31;
  int o_rank = s_scan[threadIdx.x];     // outliers before k0
  int n_rank = k0 - o_rank;             // normal channels before k0 (k0 <= K)
  if (k0 >= K) n_rank = 0;
  for (int k = k0; k < k1; ++k) {
    if (s_flag[k]) {
      perm[k_norm + o_rank] = k;
      gather[k_norm_pad + o_rank] = k;
      ++o_rank;
    } else {
      perm[n_rank] = k;
      gather[n_rank] = k;
      ++n_rank;
    }
  }
  for (int j = threadIdx.x; j < Kp; j += blockDim.x) {
    const bool pad = (j >= k_norm && j < k_norm_pad) || (j >= k_norm_pad + n_out);
    if (pad) gather[j] = -1;
  }
  if (threadIdx.x == 0) {
    kinfo[0] = k_norm;
    kinfo[1] = k_norm_pad;
    kinfo[2] = n_out;
    kinfo[3] = k_out_pad;
  }
}

// Per output row (one warp): class amaxes, scales s = RN(amax/7), codes
// clamp(rint(RN(w * RN(7/amax))), -7, 7) as two's-complement nibbles in
// class order.  Dynamic shared memory: Kp gather entries.
__global__ void __launch_bounds__(kThreadsHbm)
    k_qarvd_pack(const __nv_bfloat16* __restrict__ w, int32_t N, int32_t K, int32_t Kp,
                 const uint8_t* __restrict__ mask, const int32_t* __restrict__ gather,
                 const int32_t* __restrict__ kinfo, uint8_t* __restrict__ codes,
                 float* __restrict__ s_norm, float* __restrict__ s_out) {
  extern __shared__ int32_t s_gather[];
  for (int i = threadIdx.x; i < Kp; i += blockDim.x) s_gather[i] = gather[i];
  __syncthreads();
  const int32_t k_norm_pad = kinfo[1];
  const uint32_t lane = lane_id();
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const unsigned short* ws = reinterpret_cast<const unsigned short*>(w);
  for (int64_t n = warp; n < N; n += nwarps) {
    const unsigned short* wr = ws + n * K;
    float an = 0.f, ao = 0.f;
    for (int32_t k = lane; k < K; k += 32) {
      const float v = fabsf(__uint_as_float(static_cast<uint32_t>(__ldg(wr + k)) << 16));
      if (__ldg(mask + k)) ao = fmaxf(ao, v); else an = fmaxf(an, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      an = fmaxf(an, __shfl_xor_sync(0xffffffffu, an, o));
      ao = fmaxf(ao, __shfl_xor_sync(0xffffffffu, ao, o));
    }
    const float inv_n = (an == 0.f) ? 0.f : __fdiv_rn(7.f, an);
    const float inv_o = (ao == 0.f) ? 0.f : __fdiv_rn(7.f, ao);
    if (lane == 0) {
      s_norm[n] = (an == 0.f) ? 0.f : __fdiv_rn(an, 7.f);
      s_out[n] = (ao == 0.f) ? 0.f : __fdiv_rn(ao, 7.f);
    }
    uint8_t* cr = codes + n * (Kp / 2);
    for (int32_t j0 = static_cast<int32_t>(lane) * 8; j0 < Kp; j0 += 32 * 8) {
      uint32_t packed = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int32_t j = j0 + i;
        const int32_t src = s_gather[j];
        int qi = 0;
        if (src >= 0) {
          const float v = __uint_as_float(static_cast<uint32_t>(__ldg(wr + src)) << 16);
          const float inv = (j < k_norm_pad) ? inv_n : inv_o;
          qi = max(-7, min(7, __float2int_rn(__fmul_rn(v, inv))));
        }
        packed |= (static_cast<uint32_t>(qi) & 0xFu) << (4 * i);
      }
      *reinterpret_cast<uint32_t*>(cr + j0 / 2) = packed;
    }
  }
}

// --------------------------------------------------------------------------
// Host launchers
// --------------------------------------------------------------------------
ql_status launch_gamma_route(const void* in, const void* out, int64_t numel, float threshold,
                             double* gamma, int32_t* route, void* ws, cudaStream_t st) {
  const int grid = hbm_grid(std::max<int64_t>(1, (numel / 8 + kThreadsHbm - 1) / kThreadsHbm), 1);
  double* partials = static_cast<double*>(ws);
  unsigned int* ticket = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + kRoutePartialBytes);
  if (launch_pdl(k_gamma_route, dim3(grid), dim3(kThreadsHbm), 0, st, 1, static_cast<const uint4*>(in),
                 static_cast<const uint4*>(out), numel, partials, ticket, threshold, gamma, route) != cudaSuccess) {
    (void)cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

ql_status launch_gamma_sums(const void* in, const void* out, int64_t numel, double* sums, void* ws,
                            cudaStream_t st) {
  const int grid = hbm_grid(std::max<int64_t>(1, (numel / 8 + kThreadsHbm - 1) / kThreadsHbm), 1);
  double* partials = static_cast<double*>(ws);
  unsigned int* ticket = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + kRoutePartialBytes);
  if (launch_pdl(k_gamma_sums, dim3(grid), dim3(kThreadsHbm), 0, st, 1, static_cast<const uint4*>(in),
                 static_cast<const uint4*>(out), numel, partials, ticket, sums) != cudaSuccess) {
    (void)cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

ql_status launch_route_from_sums(const double* sums, float threshold, double* gamma, int32_t* route,
                                 cudaStream_t st) {
  if (launch_pdl(k_route_from_sums, dim3(1), dim3(32), 0, st, 1, sums, threshold, gamma, route) != cudaSuccess) {
    (void)cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

int qarvd_slices(int32_t N) { return std::max(1, std::min(64, N / 64)); }

ql_status launch_qarvd_prepare(const void* W, int32_t N, int32_t K, float tau, float alpha,
                               const ql_weights* w, void* ws, cudaStream_t st) {
  const int slices = qarvd_slices(N);
  const int rows_per_slice = (N + slices - 1) / slices;
  double* partial = static_cast<double*>(ws);
  dim3 g1((K / 2 + kThreadsHbm - 1) / kThreadsHbm, slices);
  k_colnorm_partial<<<g1, kThreadsHbm, 0, st>>>(static_cast<const uint32_t*>(W), N, K,
                                                rows_per_slice, partial);
  if (cudaGetLastError() != cudaSuccess) return QL_ERR_CUDA;
  int npow2 = 1;
  while (npow2 < K) npow2 <<= 1;
  const size_t smem_sel = static_cast<size_t>(npow2) * sizeof(double) + static_cast<size_t>(K) * 4;
  if (!set_smem_attr(reinterpret_cast<const void*>(k_qarvd_select), static_cast<int>(smem_sel)))
    return QL_ERR_CUDA;
  k_qarvd_select<<<1, 1024, smem_sel, st>>>(partial, slices, K, npow2, tau, alpha, w->Kp, w->norms,
                                            w->outlier_mask, w->perm, w->gather, w->kinfo);
  if (cudaGetLastError() != cudaSuccess) return QL_ERR_CUDA;
  const size_t smem_pack = static_cast<size_t>(w->Kp) * sizeof(int32_t);
  if (!set_smem_attr(reinterpret_cast<const void*>(k_qarvd_pack), static_cast<int>(smem_pack)))
    return QL_ERR_CUDA;
  const int grid = hbm_grid(N, kThreadsHbm / 32);
  k_qarvd_pack<<<grid, kThreadsHbm, smem_pack, st>>>(
      static_cast<const __nv_bfloat16*>(W), N, K, w->Kp, w->outlier_mask, w->gather, w->kinfo,
      static_cast<uint8_t*>(w->codes), w->s_norm, w->s_out);
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

}  // namespace ql
