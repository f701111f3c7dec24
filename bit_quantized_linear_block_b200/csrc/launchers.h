// Host-side launch functions of the kernels, one translation unit each,
// called by the C-ABI layer (capi.cu).
#pragma once

#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/qlinear.h"

namespace ql {

constexpr int kHbmCtasPerSm = 4;                 // 256-thread CTAs per SM for streaming kernels
constexpr int kMaxPartials = 4096;               // upper bound of any streaming grid
constexpr size_t kAmaxPartialBytes = kMaxPartials * sizeof(float);
constexpr size_t kAmaxWsBytes = kAmaxPartialBytes + 256;   // partials + ticket
constexpr size_t kRoutePartialBytes = 2 * kMaxPartials * sizeof(double);
constexpr size_t kTdcPartialBytes = 5 * kMaxPartials * sizeof(double);

// Device-routed forward: a launch runs only when *route == value (null
// route: always).
struct Gate {
  const int32_t* route = nullptr;
  int32_t value = 0;
};

int num_sms();
int* status_word();   // device status word of the current device (see qlinear_device_status)
bool set_smem_attr(const void* kernel, int bytes);
int hbm_grid(int64_t work_items, int per_cta);
int qarvd_slices(int32_t N);

// Tensor amax (rotated when hadamard != 0) into *amax_out; ws needs
// kAmaxWsBytes (partials + ticket).
ql_status launch_amax(const void* x, int64_t M, int32_t K, int hadamard, float* amax_out, void* ws,
                      cudaStream_t st, Gate gate = {});
// decomp = 1: activation decomposition, codes [M, K] bytes = [q1 | q2] per
// row and scales over K' = 2K.
ql_status launch_quant_nvfp4(const void* x, int64_t M, int32_t K, int hadamard, const float* amax_in,
                             void* codes, void* sf_mma, void* sf_rm, float* g_out, cudaStream_t st,
                             int decomp = 0, Gate gate = {});
// f16 copy [N, K] of NVFP4 weights without the tensor scale (INT8 route).
ql_status launch_expand_nvfp4_f16(const void* codes, const void* sf, int32_t N, int32_t K, void* out,
                                  cudaStream_t st);
// f16_codes = 1 writes each INT8 code as the equal f16 value ([M, K] f16).
// qmax: 127 (INT8) or 31 (INT6 codes in int8 / f16 containers).
ql_status launch_quant_int8_token(const void* x, int64_t M, int32_t K, int hadamard, void* codes,
                                  float* scales, cudaStream_t st, int f16_codes = 0, int qmax = 127,
                                  Gate gate = {});
ql_status launch_quant_int8_tensor_perm(const void* x, int64_t M, int32_t K, int32_t Kp,
                                        const int32_t* gather, const float* amax_in, void* codes,
                                        float* scale_out, cudaStream_t st, int qmax = 127);
ql_status launch_gamma_route(const void* in, const void* out, int64_t numel, float threshold,
                             double* gamma, int32_t* route, void* ws, cudaStream_t st);
// sums[0] = sum |out - in|, sums[1] = sum |in| (fp64); ws as for launch_gamma_route.
ql_status launch_gamma_sums(const void* in, const void* out, int64_t numel, double* sums, void* ws,
                            cudaStream_t st);
ql_status launch_route_from_sums(const double* sums, float threshold, double* gamma, int32_t* route,
                                 cudaStream_t st);
ql_status launch_qarvd_prepare(const void* W, int32_t N, int32_t K, float tau, float alpha,
                               const ql_weights* w, void* ws, cudaStream_t st);

ql_status launch_debug_div_check(float d, uint32_t a_begin, uint64_t count, unsigned long long* mismatches,
                                 cudaStream_t st);
ql_status launch_tdc_init(ql_tdc_state* st, cudaStream_t s);
ql_status launch_tdc_refresh(const void* in, const void* out, int64_t numel, void* slot0, void* slot1,
                             ql_tdc_state* st, const ql_tdc_params& prm, void* ws, cudaStream_t s);
ql_status launch_tdc_skip(const void* in, int64_t numel, const void* slot0, const void* slot1,
                          ql_tdc_state* st, const ql_tdc_params& prm, void* out, int* status, cudaStream_t s);

ql_status launch_gemm_w4a4(const void* a_codes, const uint8_t* a_sf, const float* g_a, int64_t M,
                           const ql_weights* w, void* Y, cudaStream_t st, int* status, Gate gate = {});
// a_f16 = 1: activations are f16 [M, K] holding the INT8 codes (needs
// weights prepared with expand_f16).
ql_status launch_gemm_w4a8(const void* a_codes, const float* a_scales, int64_t M,
                           const ql_weights* w, void* Y, cudaStream_t st, int* status, int a_f16 = 0,
                           Gate gate = {});
// int8 copy [N, Kp] of the Q-ARVD INT4 codes (sign-extended).
ql_status launch_expand_int4_i8(const void* codes, int32_t N, int32_t Kp, void* out, cudaStream_t st);
// Uses the int8 weight copy (w->w8) when the weights carry one.
// Unquantized bf16 product from weights prepared with keep_bf16.
ql_status launch_gemm_bf16(const void* X, int64_t M, const ql_weights* w, void* Y, cudaStream_t st, int* status,
                           Gate gate = {});
ql_status launch_gemm_qarvd(const void* a_codes, const float* s_x, int64_t M, const ql_weights* w,
                            void* Y, cudaStream_t st, int* status);

}  // namespace ql
