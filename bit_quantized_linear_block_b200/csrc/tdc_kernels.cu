// Temporal delta cache ("6Bit-Diffusion", Methodology A.2 and B.2 TDC) with
// PDR's forced INT8 after a skip and its BF16 refresh on an outlier-heavy
// input (B.3).
//
// A transformer block's residual delta Delta_t = output - input changes
// little between adjacent timesteps.  The cache keeps the block's latest two
// computed deltas (bf16, two caller-owned slots), E = the relative L1
// distance between them, and the current run of skips.  Per timestep the
// caller either
//   * computes the block and calls qlinear_tdc_refresh, ONE pass over the
//     block input, the block output and the latest delta that writes the new
//     delta into the other slot and reduces, in fp64,
//       Gamma = sum |out - in| / sum |in|            (the DMPQ router's input)
//       E     = sum |D_new - D_prev| / sum |D_prev|  (the skip criterion), or
//   * skips the block with qlinear_tdc_skip: out = bf16(in + D_latest).
// The kernel that finishes a step (the refresh's last CTA, or the skip
// kernel's first thread) also writes the decision for the next step into the
// device state:
//   skip  iff two deltas are cached, E < eps_threshold,
//         acc + E <= acc_max and skips < max_skips
//   route BF16 when the last refresh saw an outlier-block ratio rho >
//         rho_max (PDR's high-precision refresh), else INT8 when the step
//         just taken was a skip (no fresh Gamma: PDR) or Gamma >
//         gamma_threshold, else NVFP4.
// rho is the fraction of the input's whole 16-element blocks whose largest
// magnitude a exceeds kappa times the mean of the other 15 elements:
// RN(15 a) > RN(kappa RN(s - a)), s the fp32 sum of |x| taken as two
// sequential halves of 8 and then their sum.  The refresh walks the tensors
// a block (two 16-byte vectors of each) at a time so one thread sees it all.
// Arithmetic: fp32 differences of the bf16 values (RN), bf16 rounding RN-even,
// fp64 sums (their order differs from a sequential sum only by rounding).
#include "ql_common.cuh"
#include "route_common.cuh"
#include "gemm_common.cuh"
#include "launchers.h"

namespace ql {

struct TdcSums {
  double d, x, e, p;   // sum |out - in|, sum |in|, sum |D_new - D_prev|, sum |D_prev|
  unsigned long long nflag;   // outlier blocks of the input
};

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ double inf_f64() { return __longlong_as_double(0x7ff0000000000000ll); }

// One bf16 pair: the new delta's two values (returned packed) and the sums.
template <bool PREV>
__device__ __forceinline__ uint32_t tdc_pair(uint32_t xw, uint32_t yw, uint32_t pw, TdcSums& s) {
  const float x0 = bf16_lo(xw), x1 = bf16_hi(xw);
  const float d0 = __fsub_rn(bf16_lo(yw), x0), d1 = __fsub_rn(bf16_hi(yw), x1);
  s.d += static_cast<double>(fabsf(d0));
  s.d += static_cast<double>(fabsf(d1));
  s.x += static_cast<double>(fabsf(x0));
  s.x += static_cast<double>(fabsf(x1));
  const uint32_t dn = bf16x2_rn(d0, d1);
  if constexpr (PREV) {
    const float p0 = bf16_lo(pw), p1 = bf16_hi(pw);
    s.e += static_cast<double>(fabsf(__fsub_rn(bf16_lo(dn), p0)));
    s.e += static_cast<double>(fabsf(__fsub_rn(bf16_hi(dn), p1)));
    s.p += static_cast<double>(fabsf(p0));
    s.p += static_cast<double>(fabsf(p1));
  }
  return dn;
}

template <bool PREV>
__device__ __forceinline__ uint4 tdc_vec(const uint4& xi, const uint4& yo, const uint4& pv, TdcSums& s) {
  uint4 r;
  r.x = tdc_pair<PREV>(xi.x, yo.x, pv.x, s);
  r.y = tdc_pair<PREV>(xi.y, yo.y, pv.y, s);
  r.z = tdc_pair<PREV>(xi.z, yo.z, pv.z, s);
  r.w = tdc_pair<PREV>(xi.w, yo.w, pv.w, s);
  return r;
}

// |x| of one 16-byte vector in element order: sequential fp32 sum and max.
__device__ __forceinline__ void abs_half(const uint4& v, float& sum, float& mx) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float a0 = fabsf(bf16_lo(w[k])), a1 = fabsf(bf16_hi(w[k]));
    sum = __fadd_rn(__fadd_rn(sum, a0), a1);
    mx = fmax3(mx, a0, a1);
  }
}

// One 16-element block: the new delta's two vectors, the sums and the
// outlier test on the input.
template <bool PREV>
__device__ __forceinline__ void tdc_block(const uint4 (&xi)[2], const uint4 (&yo)[2], const uint4 (&pv)[2],
                                          uint4 (&dn)[2], float kappa, TdcSums& s) {
  float h0 = 0.f, h1 = 0.f, a = 0.f;
  dn[0] = tdc_vec<PREV>(xi[0], yo[0], pv[0], s);
  dn[1] = tdc_vec<PREV>(xi[1], yo[1], pv[1], s);
  abs_half(xi[0], h0, a);
  abs_half(xi[1], h1, a);
  const float others = __fsub_rn(__fadd_rn(h0, h1), a);
  s.nflag += (__fmul_rn(a, 15.f) > __fmul_rn(kappa, others)) ? 1ull : 0ull;
}

// This thread's share: grid-stride over 16-element blocks, two blocks of
// every tensor loaded before either is used; the < 16-element tail (outside
// the outlier test) by the first threads as bf16 scalars.
template <bool PREV>
__device__ __forceinline__ void tdc_thread(const uint4* __restrict__ in, const uint4* __restrict__ out,
                                           const uint4* __restrict__ prev, uint4* __restrict__ dst,
                                           int64_t numel, float kappa, TdcSums& s) {
  const int64_t nblk = numel >> 4;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthr = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const uint4 z = make_uint4(0, 0, 0, 0);
  int64_t b = tid;
  for (; b + nthr < nblk; b += 2 * nthr) {
    uint4 x[2][2], y[2][2], p[2][2], d[2][2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t v = 2 * (b + u * nthr);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        x[u][h] = __ldcs(in + v + h);
        y[u][h] = __ldcs(out + v + h);
        p[u][h] = PREV ? __ldcs(prev + v + h) : z;
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      tdc_block<PREV>(x[u], y[u], p[u], d[u], kappa, s);
      const int64_t v = 2 * (b + u * nthr);
      dst[v] = d[u][0];
      dst[v + 1] = d[u][1];
    }
  }
  for (; b < nblk; b += nthr) {
    uint4 x[2], y[2], p[2], d[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      x[h] = __ldcs(in + 2 * b + h);
      y[h] = __ldcs(out + 2 * b + h);
      p[h] = PREV ? __ldcs(prev + 2 * b + h) : z;
    }
    tdc_block<PREV>(x, y, p, d, kappa, s);
    dst[2 * b] = d[0];
    dst[2 * b + 1] = d[1];
  }
  if (tid < (numel & 15)) {
    const int64_t e = (nblk << 4) + tid;
    const uint32_t xv = reinterpret_cast<const unsigned short*>(in)[e];
    const uint32_t yv = reinterpret_cast<const unsigned short*>(out)[e];
    const uint32_t pv = PREV ? reinterpret_cast<const unsigned short*>(prev)[e] : 0u;
    const uint32_t dn = tdc_pair<PREV>(xv, yv, pv, s);   // low halves carry the element; the high halves are 0
    reinterpret_cast<unsigned short*>(dst)[e] = static_cast<unsigned short>(dn & 0xFFFFu);
  }
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void block_sum4(TdcSums& s) {
  __shared__ double red[4][32];
  __shared__ unsigned long long redn[32];
  s.d = warp_sum_f64(s.d);
  s.x = warp_sum_f64(s.x);
  s.e = warp_sum_f64(s.e);
  s.p = warp_sum_f64(s.p);
  s.nflag = warp_sum_u64(s.nflag);
  const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (lane_id() == 0) {
    red[0][w] = s.d;
    red[1][w] = s.x;
    red[2][w] = s.e;
    red[3][w] = s.p;
    redn[w] = s.nflag;
  }
  __syncthreads();
  if (w == 0) {
    const bool in = lane_id() < nw;
    s.d = warp_sum_f64(in ? red[0][lane_id()] : 0.0);
    s.x = warp_sum_f64(in ? red[1][lane_id()] : 0.0);
    s.e = warp_sum_f64(in ? red[2][lane_id()] : 0.0);
    s.p = warp_sum_f64(in ? red[3][lane_id()] : 0.0);
    s.nflag = warp_sum_u64(in ? redn[lane_id()] : 0ull);
  }
  __syncthreads();
}

// Decision for the next step from the state of the step just taken.
__device__ __forceinline__ void tdc_decide(ql_tdc_state* st, const ql_tdc_params& prm) {
  st->next_skip = (st->n_delta == 2 && st->eps < static_cast<double>(prm.eps_threshold) &&
                   st->acc + st->eps <= static_cast<double>(prm.acc_max) && st->skips < prm.max_skips)
                      ? 1
                      : 0;
  st->next_route = (st->rho > static_cast<double>(prm.rho_max)) ? QL_ROUTE_BF16
                   : (st->last_skipped != 0 || st->gamma > static_cast<double>(prm.gamma_threshold))
                       ? QL_ROUTE_INT8
                       : QL_ROUTE_NVFP4;
}

__global__ void k_tdc_init(ql_tdc_state* st) {
  st->gamma = inf_f64();   // no Gamma yet: the first step runs INT8
  st->eps = inf_f64();
  st->acc = 0.0;
  st->rho = 0.0;
  st->n_delta = 0;
  st->cur = 1;             // the first delta goes to slot 0
  st->skips = 0;
  st->last_skipped = 0;
  st->next_skip = 0;
  st->next_route = QL_ROUTE_INT8;
  st->steps = 0;
  st->reserved = 0;
}

// The slots are read from the state once, at the start: the state is
// rewritten only by the last CTA, after every CTA has taken its ticket.
__global__ void __launch_bounds__(kThreadsHbm)
    k_tdc_refresh(const uint4* __restrict__ in, const uint4* __restrict__ out, int64_t numel, uint4* slot0,
                  uint4* slot1, ql_tdc_state* st, const ql_tdc_params prm, double* __restrict__ partials,
                  unsigned int* __restrict__ ticket) {
  pdl_wait();
  const int cur = st->cur;
  const int n_delta = st->n_delta;
  const bool has_prev = n_delta >= 1;
  const uint4* prev = cur ? slot1 : slot0;
  uint4* dst = cur ? slot0 : slot1;
  TdcSums s{0.0, 0.0, 0.0, 0.0, 0ull};
  if (has_prev)
    tdc_thread<true>(in, out, prev, dst, numel, prm.kappa, s);
  else
    tdc_thread<false>(in, out, prev, dst, numel, prm.kappa, s);
  pdl_release();
  __shared__ bool s_last;
  block_sum4(s);
  if (threadIdx.x == 0) {
    partials[5 * blockIdx.x + 0] = s.d;
    partials[5 * blockIdx.x + 1] = s.x;
    partials[5 * blockIdx.x + 2] = s.e;
    partials[5 * blockIdx.x + 3] = s.p;
    partials[5 * blockIdx.x + 4] = __longlong_as_double(static_cast<long long>(s.nflag));   // bit pattern
    __threadfence();
    s_last = atomicAdd(ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  TdcSums t{0.0, 0.0, 0.0, 0.0, 0ull};
  const volatile double* pp = partials;
  for (unsigned int b = threadIdx.x; b < gridDim.x; b += blockDim.x) {
    t.d += pp[5 * b + 0];
    t.x += pp[5 * b + 1];
    t.e += pp[5 * b + 2];
    t.p += pp[5 * b + 3];
    t.nflag += static_cast<unsigned long long>(__double_as_longlong(pp[5 * b + 4]));
  }
  block_sum4(t);
  if (threadIdx.x == 0) {
    st->gamma = (t.x == 0.0) ? inf_f64() : t.d / t.x;
    st->eps = (!has_prev || t.p == 0.0) ? inf_f64() : t.e / t.p;
    const int64_t nblk = numel >> 4;
    st->rho = nblk ? static_cast<double>(t.nflag) / static_cast<double>(nblk) : 0.0;
    st->n_delta = min(n_delta + 1, 2);
    st->cur = 1 - cur;
    st->acc = 0.0;
    st->skips = 0;
    st->last_skipped = 0;
    st->steps += 1;
    tdc_decide(st, prm);
    *ticket = 0u;
  }
}

// out = bf16(RN(in + D_latest)).  The state update touches neither the slot
// index nor the delta count, which the other CTAs read.
__global__ void __launch_bounds__(kThreadsHbm)
    k_tdc_skip(const uint4* __restrict__ in, int64_t numel, const uint4* slot0, const uint4* slot1,
               ql_tdc_state* st, const ql_tdc_params prm, uint4* __restrict__ out, int* status) {
  pdl_wait();
  const int cur = st->cur;
  if (st->n_delta < 1) {   // nothing cached: the caller skipped without a delta
    if (blockIdx.x == 0 && threadIdx.x == 0) record_error(status, QL_ERR_INVALID_ARG);
    return;
  }
  const uint4* dl = cur ? slot1 : slot0;
  const int64_t nvec = numel >> 3;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthr = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = tid; i < nvec; i += nthr) {
    const uint4 a = __ldcs(in + i), d = __ldcs(dl + i);
    uint4 r;
    r.x = bf16x2_rn(__fadd_rn(bf16_lo(a.x), bf16_lo(d.x)), __fadd_rn(bf16_hi(a.x), bf16_hi(d.x)));
    r.y = bf16x2_rn(__fadd_rn(bf16_lo(a.y), bf16_lo(d.y)), __fadd_rn(bf16_hi(a.y), bf16_hi(d.y)));
    r.z = bf16x2_rn(__fadd_rn(bf16_lo(a.z), bf16_lo(d.z)), __fadd_rn(bf16_hi(a.z), bf16_hi(d.z)));
    r.w = bf16x2_rn(__fadd_rn(bf16_lo(a.w), bf16_lo(d.w)), __fadd_rn(bf16_hi(a.w), bf16_hi(d.w)));
    __stcs(out + i, r);
  }
  if (tid < (numel & 7)) {
    const int64_t e = (nvec << 3) + tid;
    const float x = __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const unsigned short*>(in)[e]) << 16);
    const float d = __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const unsigned short*>(dl)[e]) << 16);
    reinterpret_cast<unsigned short*>(out)[e] = static_cast<unsigned short>(bf16x2_rn(__fadd_rn(x, d), 0.f) & 0xFFFFu);
  }
  pdl_release();
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    st->acc += st->eps;
    st->skips += 1;
    st->last_skipped = 1;
    st->steps += 1;
    tdc_decide(st, prm);
  }
}

// --------------------------------------------------------------------------
// Host launchers
// --------------------------------------------------------------------------
ql_status launch_tdc_init(ql_tdc_state* st, cudaStream_t s) {
  k_tdc_init<<<1, 1, 0, s>>>(st);
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

ql_status launch_tdc_refresh(const void* in, const void* out, int64_t numel, void* slot0, void* slot1,
                             ql_tdc_state* st, const ql_tdc_params& prm, void* ws, cudaStream_t s) {
  const int grid = hbm_grid(std::max<int64_t>(1, (numel / 16 + kThreadsHbm - 1) / kThreadsHbm), 1);
  double* partials = static_cast<double*>(ws);
  unsigned int* ticket = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + kTdcPartialBytes);
  if (launch_pdl(k_tdc_refresh, dim3(grid), dim3(kThreadsHbm), 0, s, 1, static_cast<const uint4*>(in),
                 static_cast<const uint4*>(out), numel, static_cast<uint4*>(slot0), static_cast<uint4*>(slot1), st, prm,
                 partials, ticket) != cudaSuccess) {
    (void)cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

ql_status launch_tdc_skip(const void* in, int64_t numel, const void* slot0, const void* slot1,
                          ql_tdc_state* st, const ql_tdc_params& prm, void* out, int* status, cudaStream_t s) {
  const int grid = hbm_grid(std::max<int64_t>(1, (numel / 8 + kThreadsHbm - 1) / kThreadsHbm), 1);
  if (launch_pdl(k_tdc_skip, dim3(grid), dim3(kThreadsHbm), 0, s, 1, static_cast<const uint4*>(in), numel,
                 static_cast<const uint4*>(slot0), static_cast<const uint4*>(slot1), st, prm, static_cast<uint4*>(out),
                 status) != cudaSuccess) {
    (void)cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

}  // namespace ql
