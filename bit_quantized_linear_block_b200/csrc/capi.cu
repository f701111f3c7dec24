// C ABI of the qlinear library: argument checks, workspace layout, tensor
// maps and kernel sequencing.  Every entry point validates on the host
// before touching CUDA, so a bad call enqueues nothing.
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "ql_common.cuh"
#include "gemm_common.cuh"
#include "launchers.h"

// Device status word of each device (see qlinear_device_status).
__device__ int g_ql_device_status = 0;

namespace ql {
namespace {

constexpr int kMaxDevices = 64;
constexpr long long kDefaultWaitLimit = 2000000000ll;   // ~1 s of SM clock

std::mutex g_mu;
int g_sms[kMaxDevices] = {0};
int* g_status[kMaxDevices] = {nullptr};
bool g_checked[kMaxDevices] = {false};
bool g_ok_arch[kMaxDevices] = {false};
std::unordered_map<const void*, int> g_smem_set[kMaxDevices];
std::atomic<long long> g_wait_limit{kDefaultWaitLimit};

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                              CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                              CUtensorMapFloatOOBfill);
EncodeFn g_encode = nullptr;

int current_device() {
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return -1;
  return d;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

// Device checks: an sm_100 GPU must be current.  Cached per device.
ql_status device_ready() {
  const int d = current_device();
  if (d < 0) return QL_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_checked[d]) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, d) != cudaSuccess) return QL_ERR_NO_DEVICE;
    g_ok_arch[d] = (prop.major == 10 && prop.minor == 0);
    g_sms[d] = prop.multiProcessorCount;
    void* sp = nullptr;
    if (cudaGetSymbolAddress(&sp, g_ql_device_status) != cudaSuccess) return QL_ERR_CUDA;
    g_status[d] = static_cast<int*>(sp);
    g_checked[d] = true;
  }
  return g_ok_arch[d] ? QL_OK : QL_ERR_NO_DEVICE;
}

int num_sms() {
  const int d = current_device();
  return (d >= 0 && g_sms[d] > 0) ? g_sms[d] : 148;
}

int* status_word() {
  const int d = current_device();
  return d >= 0 ? g_status[d] : nullptr;
}

bool set_smem_attr(const void* kernel, int bytes) {
  const int d = current_device();
  if (d < 0) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_smem_set[d].find(kernel);
  if (it != g_smem_set[d].end() && it->second >= bytes) return true;
  // Opt in whenever dynamic shared memory is used: static shared memory
  // counts against the same 48 KB default.
  if (bytes > 0 &&
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  g_smem_set[d][kernel] = bytes;
  return true;
}

bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int64_t inner,
                  int64_t outer, int64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                  CUtensorMapSwizzle swizzle) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return false;
      g_encode = reinterpret_cast<EncodeFn>(fn);
    }
  }
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_stride_bytes)};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int64_t d0, int64_t d1,
                  int64_t d2, int64_t stride1_bytes, int64_t stride2_bytes, uint32_t b0, uint32_t b1,
                  uint32_t b2) {
  CUtensorMap dummy;
  if (!make_tmap_2d(&dummy, dtype, base, d0, d1, stride1_bytes, b0, b1, CU_TENSOR_MAP_SWIZZLE_NONE))
    return false;   // also resolves the encoder
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d0), static_cast<cuuint64_t>(d1),
                              static_cast<cuuint64_t>(d2)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(stride1_bytes), static_cast<cuuint64_t>(stride2_bytes)};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_sf_tmap(CUtensorMap* map, const void* base, int64_t rows, int K, uint32_t box_k) {
  const int64_t groups = (rows + 127) / 128;
  const int64_t k_atoms = K / 64;
  return make_tmap_3d(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, base, 128, k_atoms, groups, 512, k_atoms * 512, 128,
                      box_k, 1);
}

void fill_gemm_args(GemmArgs& p, int64_t M, int N, int K, int BN, int* status) {
  p.M = static_cast<int32_t>(M);
  p.N = N;
  p.K = K;
  p.tiles_m = static_cast<int32_t>((M + 127) / 128);
  p.tiles_n = (N + BN - 1) / BN;
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.group_m = 8;
  p.wait_limit = g_wait_limit.load(std::memory_order_relaxed);
  p.status = status;
}

int32_t qarvd_kp(int32_t K) { return ((K + 31) / 32) * 32 + 32; }

}  // namespace ql

using namespace ql;

namespace {

// Shape rules shared by every entry point.
ql_status check_k(int64_t K) {
  if (K <= 0 || K % 128 != 0 || K > (1 << 20)) return QL_ERR_UNSUPPORTED_SHAPE;
  return QL_OK;
}
ql_status check_m(int64_t M) {
  if (M < 0) return QL_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 31) - 128) return QL_ERR_UNSUPPORTED_SHAPE;
  return QL_OK;
}
// Streaming kernels index 128-element blocks with 32-bit integers and
// address the input as 128-byte TMA rows with 32-bit row coordinates.
ql_status check_mk(int64_t M, int64_t K) {
  if ((M + 127) / 128 * 128 * (K / 128) >= (int64_t(1) << 32)) return QL_ERR_UNSUPPORTED_SHAPE;
  if (M * K >= (int64_t(1) << 37)) return QL_ERR_UNSUPPORTED_SHAPE;
  return QL_OK;
}
// The GEMMs count output tiles of 128 x 128 (or wider) in 32 bits.
ql_status check_mn(int64_t M, int64_t N) {
  if ((M + 127) / 128 * ((N + 127) / 128) >= (int64_t(1) << 31)) return QL_ERR_UNSUPPORTED_SHAPE;
  return QL_OK;
}
ql_status check_w(const ql_weights* w) {
  if (w == nullptr || w->codes == nullptr) return QL_ERR_INVALID_ARG;
  if (w->fmt != QL_W_NVFP4 && w->fmt != QL_W_QARVD_INT4 && w->fmt != QL_W_NVFP4_DECOMP) return QL_ERR_INVALID_ARG;
  if (check_k(w->K) != QL_OK || w->N <= 0 || w->N % 16 != 0) return QL_ERR_UNSUPPORTED_SHAPE;
  if ((w->fmt == QL_W_NVFP4 || w->fmt == QL_W_NVFP4_DECOMP) && (w->sf == nullptr || w->gscale == nullptr))
    return QL_ERR_INVALID_ARG;
  if (w->fmt == QL_W_NVFP4_DECOMP && check_k(2 * w->K) != QL_OK) return QL_ERR_UNSUPPORTED_SHAPE;
  if (w->fmt == QL_W_QARVD_INT4 &&
      (w->gather == nullptr || w->kinfo == nullptr || w->s_norm == nullptr || w->s_out == nullptr ||
       w->Kp != qarvd_kp(w->K)))
    return QL_ERR_INVALID_ARG;
  return QL_OK;
}

#define QL_TRY(expr)                 \
  do {                               \
    const ql_status _s = (expr);     \
    if (_s != QL_OK) return _s;      \
  } while (0)

struct Carver {  // sequential 256-byte aligned sub-buffers of one allocation
  uint8_t* base;
  size_t off = 0;
  template <class T>
  T* take(size_t bytes) {
    T* p = reinterpret_cast<T*>(base + off);
    off += align256(bytes);
    return p;
  }
};

// W4A6: the INT6 formats are the INT8 formats with codes in [-31, 31].
int32_t int_base_fmt(int32_t f) {
  return f == QL_ROUTE_INT6 ? int32_t(QL_ROUTE_INT8)
         : f == QL_ACT_INT6_F16 ? int32_t(QL_ACT_INT8_F16)
         : f == QL_ACT_INT6_TENSOR ? int32_t(QL_ACT_INT8_TENSOR) : f;
}
int act_qmax(int32_t f) {
  return (f == QL_ROUTE_INT6 || f == QL_ACT_INT6_F16 || f == QL_ACT_INT6_TENSOR) ? 31 : 127;
}

// f16_codes: the INT8 route keeps its codes as f16 values (weights with an
// f16 copy), 2 bytes per element.
size_t forward_act_bytes(int64_t M, int32_t K, int32_t Kp, int32_t fmt, bool f16_codes = false) {
  if (fmt == QL_ROUTE_NVFP4 || fmt == QL_ACT_NVFP4_DECOMP) {
    const int32_t kq = fmt == QL_ACT_NVFP4_DECOMP ? 2 * K : K;
    return kAmaxWsBytes + 256 + 256 + align256(static_cast<size_t>(M) * kq / 2) +
           align256(qlinear_sf_bytes(M, kq));
  }
  if (fmt == QL_ROUTE_INT8)
    return align256(static_cast<size_t>(M) * K * (f16_codes ? 2 : 1)) + align256(4 * static_cast<size_t>(M));
  return kAmaxWsBytes + 256 + 256 + align256(static_cast<size_t>(M) * Kp);
}

}  // namespace

extern "C" {

int qlinear_abi_version(void) { return QLINEAR_ABI_VERSION; }

const char* qlinear_status_string(int s) {
  switch (s) {
    case QL_OK: return "ok";
    case QL_ERR_INVALID_ARG: return "invalid argument";
    case QL_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case QL_ERR_ALIGNMENT: return "misaligned pointer";
    case QL_ERR_CUDA: return "CUDA runtime error";
    case QL_ERR_TIMEOUT: return "device wait timed out";
    case QL_ERR_WORKSPACE: return "workspace too small";
    case QL_ERR_NO_DEVICE: return "no sm_100 device";
    default: return "unknown status";
  }
}

void qlinear_debug_set_wait_limit(long long cycles) {
  g_wait_limit.store(cycles < 0 ? kDefaultWaitLimit : cycles, std::memory_order_relaxed);
}

ql_status qlinear_debug_div_check(float d, uint32_t a_begin, uint64_t count, unsigned long long* mismatches_dev,
                                  void* stream) {
  if (mismatches_dev == nullptr || !(d > 0.f) || d > 3.4028235e38f) return QL_ERR_INVALID_ARG;
  if (a_begin >= 0x7F800000u || count > 0x7F800000ull - a_begin) return QL_ERR_INVALID_ARG;
  if (!aligned(mismatches_dev, 8)) return QL_ERR_ALIGNMENT;
  QL_TRY(device_ready());
  return launch_debug_div_check(d, a_begin, count, mismatches_dev, static_cast<cudaStream_t>(stream));
}

ql_status qlinear_device_status(void* stream, int32_t* status_out) {
  if (status_out == nullptr) return QL_ERR_INVALID_ARG;
  QL_TRY(device_ready());
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return QL_ERR_CUDA;
  int v = 0;
  int* p = status_word();
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return QL_ERR_CUDA;
  if (cudaMemset(p, 0, sizeof(int)) != cudaSuccess) return QL_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return QL_ERR_CUDA;
  *status_out = v;
  return QL_OK;
}

size_t qlinear_sf_bytes(int64_t rows, int32_t K) {
  if (rows < 0 || K <= 0 || K % 64 != 0) return 0;
  return static_cast<size_t>((rows + 127) / 128) * 128 * (K / 16);
}

// ---------------------------------------------------------------- weights
size_t qlinear_weights_bytes(int32_t N, int32_t K, const ql_weight_cfg* cfg) {
  if (cfg == nullptr || N <= 0 || check_k(K) != QL_OK) return 0;
  const size_t n = N, k = K;
  if (cfg->fmt == QL_W_NVFP4)
    return align256(n * k / 2) + align256(qlinear_sf_bytes(N, K)) + 256 + (cfg->expand_f16 ? align256(n * k * 2) : 0) +
           (cfg->keep_bf16 ? align256(n * k * 2) : 0);
  if (cfg->fmt == QL_W_NVFP4_DECOMP) return align256(n * k) + align256(qlinear_sf_bytes(N, 2 * K)) + 256;
  if (cfg->fmt == QL_W_QARVD_INT4) {
    const size_t kp = qarvd_kp(K);
    return align256(n * kp / 2) + align256(k) + align256(4 * k) + align256(4 * kp) + 256 +
           2 * align256(4 * n) + align256(8 * k) + (cfg->expand_i8 ? align256(n * kp) : 0);
  }
  return 0;
}

size_t qlinear_prepare_ws_bytes(int32_t N, int32_t K, const ql_weight_cfg* cfg) {
  if (cfg == nullptr || N <= 0 || check_k(K) != QL_OK) return 0;
  if (cfg->fmt == QL_W_NVFP4) return kAmaxWsBytes + 256;
  if (cfg->fmt == QL_W_NVFP4_DECOMP)   // + the codes and scales of one copy before the repeat
    return kAmaxWsBytes + 256 + align256(static_cast<size_t>(N) * K / 2) + align256(qlinear_sf_bytes(N, K));
  if (cfg->fmt == QL_W_QARVD_INT4) return align256(static_cast<size_t>(qarvd_slices(N)) * K * 8);
  return 0;
}

ql_status qlinear_prepare_weights(const void* W, int32_t N, int32_t K, const ql_weight_cfg* cfg,
                                  void* wbuf, size_t wbuf_bytes, ql_weights* out, void* ws,
                                  size_t ws_bytes, void* stream) {
  if (W == nullptr || cfg == nullptr || wbuf == nullptr || out == nullptr || ws == nullptr)
    return QL_ERR_INVALID_ARG;
  if (cfg->fmt != QL_W_NVFP4 && cfg->fmt != QL_W_QARVD_INT4 && cfg->fmt != QL_W_NVFP4_DECOMP)
    return QL_ERR_INVALID_ARG;
  if (cfg->fmt != QL_W_NVFP4 && cfg->expand_f16 != 0) return QL_ERR_INVALID_ARG;
  if (cfg->fmt != QL_W_QARVD_INT4 && cfg->expand_i8 != 0) return QL_ERR_INVALID_ARG;
  if (cfg->fmt != QL_W_NVFP4 && cfg->keep_bf16 != 0) return QL_ERR_INVALID_ARG;
  if (cfg->fmt == QL_W_NVFP4_DECOMP && check_k(2 * K) != QL_OK) return QL_ERR_UNSUPPORTED_SHAPE;
  QL_TRY(check_k(K));
  if (N <= 0 || N % 16 != 0 || N > (1 << 24)) return QL_ERR_UNSUPPORTED_SHAPE;
  QL_TRY(check_mk(N, K));
  if (cfg->fmt == QL_W_QARVD_INT4 && (cfg->hadamard != 0 || K > 16384 || !(cfg->tau > 0.f) ||
                                      !(cfg->alpha >= 0.f)))
    return QL_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(wbuf, 256) || !aligned(ws, 256)) return QL_ERR_ALIGNMENT;
  if (wbuf_bytes < qlinear_weights_bytes(N, K, cfg) || ws_bytes < qlinear_prepare_ws_bytes(N, K, cfg))
    return QL_ERR_WORKSPACE;
  QL_TRY(device_ready());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ql_weights w;
  std::memset(&w, 0, sizeof(w));
  w.fmt = cfg->fmt;
  w.N = N;
  w.K = K;
  Carver c{static_cast<uint8_t*>(wbuf)};
  if (cfg->fmt == QL_W_NVFP4_DECOMP) {
    // quantize once into the workspace, then repeat along K: codes [c | c]
    // per row; per 128-row group the scale atoms of K twice in a row
    w.hadamard = cfg->hadamard ? 1 : 0;
    w.codes = c.take<uint8_t>(static_cast<size_t>(N) * K);
    w.sf = c.take<uint8_t>(qlinear_sf_bytes(N, 2 * K));
    w.gscale = c.take<float>(256);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    float* amax = reinterpret_cast<float*>(wsb + kAmaxWsBytes);
    uint8_t* tcodes = wsb + kAmaxWsBytes + 256;
    uint8_t* tsf = tcodes + align256(static_cast<size_t>(N) * K / 2);
    QL_TRY(launch_amax(W, N, K, w.hadamard, amax, ws, st));
    QL_TRY(launch_quant_nvfp4(W, N, K, w.hadamard, amax, tcodes, tsf, nullptr, w.gscale, st));
    const size_t half = static_cast<size_t>(K) / 2, group = static_cast<size_t>(K / 64) * 512;
    const size_t groups = (static_cast<size_t>(N) + 127) / 128;
    uint8_t* wc = static_cast<uint8_t*>(w.codes);
    uint8_t* wf = static_cast<uint8_t*>(w.sf);
    for (int part = 0; part < 2; ++part) {
      if (cudaMemcpy2DAsync(wc + part * half, 2 * half, tcodes, half, half, N, cudaMemcpyDeviceToDevice, st) !=
              cudaSuccess ||
          cudaMemcpy2DAsync(wf + part * group, 2 * group, tsf, group, group, groups, cudaMemcpyDeviceToDevice,
                            st) != cudaSuccess)
        return QL_ERR_CUDA;
    }
  } else if (cfg->fmt == QL_W_NVFP4) {
    w.hadamard = cfg->hadamard ? 1 : 0;
    w.codes = c.take<uint8_t>(static_cast<size_t>(N) * K / 2);
    w.sf = c.take<uint8_t>(qlinear_sf_bytes(N, K));
    w.gscale = c.take<float>(256);
    float* amax = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kAmaxWsBytes);
    QL_TRY(launch_amax(W, N, K, w.hadamard, amax, ws, st));
    QL_TRY(launch_quant_nvfp4(W, N, K, w.hadamard, amax, w.codes, w.sf, nullptr, w.gscale, st));
    if (cfg->expand_f16) {
      w.w16 = c.take<uint16_t>(static_cast<size_t>(N) * K * 2);
      QL_TRY(launch_expand_nvfp4_f16(w.codes, w.sf, N, K, w.w16, st));
    }
    if (cfg->keep_bf16) {   // the weights as given, for the unquantized product
      w.wbf16 = c.take<uint16_t>(static_cast<size_t>(N) * K * 2);
      if (cudaMemcpyAsync(w.wbf16, W, static_cast<size_t>(N) * K * 2, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return QL_ERR_CUDA;
    }
  } else {
    w.Kp = qarvd_kp(K);
    w.codes = c.take<uint8_t>(static_cast<size_t>(N) * w.Kp / 2);
    w.outlier_mask = c.take<uint8_t>(K);
    w.perm = c.take<int32_t>(4 * static_cast<size_t>(K));
    w.gather = c.take<int32_t>(4 * static_cast<size_t>(w.Kp));
    w.kinfo = c.take<int32_t>(256);
    w.s_norm = c.take<float>(4 * static_cast<size_t>(N));
    w.s_out = c.take<float>(4 * static_cast<size_t>(N));
    w.norms = c.take<double>(8 * static_cast<size_t>(K));
    QL_TRY(launch_qarvd_prepare(W, N, K, cfg->tau, cfg->alpha, &w, ws, st));
    if (cfg->expand_i8) {
      w.w8 = c.take<int8_t>(static_cast<size_t>(N) * w.Kp);
      QL_TRY(launch_expand_int4_i8(w.codes, N, w.Kp, w.w8, st));
    }
  }
  *out = w;
  return QL_OK;
}

// ---------------------------------------------------------------- router
size_t qlinear_route_ws_bytes(int64_t numel) {
  if (numel < 0) return 0;
  return kRoutePartialBytes + 256;
}

ql_status qlinear_route(const void* in, const void* out, int64_t numel, float threshold,
                        double* gamma_dev, int32_t* route_dev, void* ws, size_t ws_bytes,
                        void* stream) {
  if (numel < 0 || gamma_dev == nullptr || route_dev == nullptr || ws == nullptr)
    return QL_ERR_INVALID_ARG;
  if (numel > 0 && (in == nullptr || out == nullptr)) return QL_ERR_INVALID_ARG;
  if (!(threshold == threshold)) return QL_ERR_INVALID_ARG;
  if (!aligned(in, 16) || !aligned(out, 16) || !aligned(ws, 256) || !aligned(gamma_dev, 8) ||
      !aligned(route_dev, 4))
    return QL_ERR_ALIGNMENT;
  if (ws_bytes < qlinear_route_ws_bytes(numel)) return QL_ERR_WORKSPACE;
  QL_TRY(device_ready());
  return launch_gamma_route(in, out, numel, threshold, gamma_dev, route_dev, ws,
                            static_cast<cudaStream_t>(stream));
}

ql_status qlinear_gamma_sums(const void* in, const void* out, int64_t numel, double* sums_dev, void* ws,
                             size_t ws_bytes, void* stream) {
  if (numel < 0 || sums_dev == nullptr || ws == nullptr) return QL_ERR_INVALID_ARG;
  if (numel > 0 && (in == nullptr || out == nullptr)) return QL_ERR_INVALID_ARG;
  if (!aligned(in, 16) || !aligned(out, 16) || !aligned(ws, 256) || !aligned(sums_dev, 8))
    return QL_ERR_ALIGNMENT;
  if (ws_bytes < qlinear_route_ws_bytes(numel)) return QL_ERR_WORKSPACE;
  QL_TRY(device_ready());
  return launch_gamma_sums(in, out, numel, sums_dev, ws, static_cast<cudaStream_t>(stream));
}

ql_status qlinear_route_from_sums(const double* sums_dev, float threshold, double* gamma_dev, int32_t* route_dev,
                                  void* stream) {
  if (sums_dev == nullptr || gamma_dev == nullptr || route_dev == nullptr) return QL_ERR_INVALID_ARG;
  if (!(threshold == threshold)) return QL_ERR_INVALID_ARG;
  if (!aligned(sums_dev, 8) || !aligned(gamma_dev, 8) || !aligned(route_dev, 4)) return QL_ERR_ALIGNMENT;
  QL_TRY(device_ready());
  return launch_route_from_sums(sums_dev, threshold, gamma_dev, route_dev, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- temporal delta cache
namespace {
bool tdc_params_ok(const ql_tdc_params* p) {
  return p != nullptr && p->gamma_threshold == p->gamma_threshold && p->eps_threshold == p->eps_threshold &&
         p->acc_max == p->acc_max && p->kappa == p->kappa && p->rho_max == p->rho_max && p->max_skips >= 0;
}
}  // namespace

ql_status qlinear_tdc_init(ql_tdc_state* state_dev, void* stream) {
  if (state_dev == nullptr) return QL_ERR_INVALID_ARG;
  if (!aligned(state_dev, 8)) return QL_ERR_ALIGNMENT;
  QL_TRY(device_ready());
  return launch_tdc_init(state_dev, static_cast<cudaStream_t>(stream));
}

size_t qlinear_tdc_ws_bytes(int64_t numel) {
  if (numel < 0) return 0;
  return kTdcPartialBytes + 256;
}

ql_status qlinear_tdc_refresh(const void* in, const void* out, int64_t numel, void* delta0, void* delta1,
                              ql_tdc_state* state_dev, const ql_tdc_params* params, void* ws, size_t ws_bytes,
                              void* stream) {
  if (numel < 0 || state_dev == nullptr || ws == nullptr || !tdc_params_ok(params)) return QL_ERR_INVALID_ARG;
  if (numel > 0 && (in == nullptr || out == nullptr || delta0 == nullptr || delta1 == nullptr))
    return QL_ERR_INVALID_ARG;
  if (!aligned(in, 16) || !aligned(out, 16) || !aligned(delta0, 16) || !aligned(delta1, 16) ||
      !aligned(state_dev, 8) || !aligned(ws, 256))
    return QL_ERR_ALIGNMENT;
  if (ws_bytes < qlinear_tdc_ws_bytes(numel)) return QL_ERR_WORKSPACE;
  QL_TRY(device_ready());
  return launch_tdc_refresh(in, out, numel, delta0, delta1, state_dev, *params, ws,
                            static_cast<cudaStream_t>(stream));
}

ql_status qlinear_tdc_skip(const void* in, int64_t numel, const void* delta0, const void* delta1,
                           ql_tdc_state* state_dev, const ql_tdc_params* params, void* out, void* stream) {
  if (numel < 0 || state_dev == nullptr || !tdc_params_ok(params)) return QL_ERR_INVALID_ARG;
  if (numel > 0 && (in == nullptr || out == nullptr || delta0 == nullptr || delta1 == nullptr))
    return QL_ERR_INVALID_ARG;
  if (!aligned(in, 16) || !aligned(out, 16) || !aligned(delta0, 16) || !aligned(delta1, 16) ||
      !aligned(state_dev, 8))
    return QL_ERR_ALIGNMENT;
  QL_TRY(device_ready());
  return launch_tdc_skip(in, numel, delta0, delta1, state_dev, *params, out, status_word(),
                         static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- activations
size_t qlinear_quantize_ws_bytes(int64_t M, int32_t K, int32_t act_fmt) {
  if (M < 0 || check_k(K) != QL_OK) return 0;
  act_fmt = int_base_fmt(act_fmt);
  if (act_fmt != QL_ROUTE_NVFP4 && act_fmt != QL_ROUTE_INT8 && act_fmt != QL_ACT_INT8_TENSOR &&
      act_fmt != QL_ACT_INT8_F16 && act_fmt != QL_ACT_NVFP4_DECOMP)
    return 0;
  return kAmaxWsBytes + 256;
}

ql_status qlinear_tensor_amax(const void* X, int64_t M, int32_t K, int32_t hadamard, float* amax_out,
                              void* ws, size_t ws_bytes, void* stream) {
  QL_TRY(check_m(M));
  QL_TRY(check_k(K));
  QL_TRY(check_mk(M, K));
  if (amax_out == nullptr || ws == nullptr || (M > 0 && X == nullptr)) return QL_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(amax_out, 4) || !aligned(ws, 256)) return QL_ERR_ALIGNMENT;
  if (ws_bytes < qlinear_quantize_ws_bytes(M, K, QL_ROUTE_NVFP4)) return QL_ERR_WORKSPACE;
  QL_TRY(device_ready());
  return launch_amax(X, M, K, hadamard ? 1 : 0, amax_out, ws, static_cast<cudaStream_t>(stream));
}

ql_status qlinear_quantize_act(const void* X, int64_t M, int32_t K, int32_t act_fmt, int32_t hadamard,
                               const ql_weights* w, const float* amax_in, void* codes, void* sf_mma,
                               void* sf_rowmajor, float* scales, void* ws, size_t ws_bytes,
                               void* stream) {
  QL_TRY(check_m(M));
  QL_TRY(check_k(K));
  QL_TRY(check_mk(M, K));
  if (codes == nullptr || scales == nullptr || ws == nullptr || (M > 0 && X == nullptr))
    return QL_ERR_INVALID_ARG;
  const int qmax = act_qmax(act_fmt);
  act_fmt = int_base_fmt(act_fmt);
  if (act_fmt == QL_ROUTE_NVFP4 || act_fmt == QL_ACT_NVFP4_DECOMP) {
    if (sf_mma == nullptr) return QL_ERR_INVALID_ARG;
  } else if (act_fmt == QL_ACT_INT8_TENSOR) {
    QL_TRY(check_w(w));
    if (w->fmt != QL_W_QARVD_INT4 || w->K != K || hadamard != 0) return QL_ERR_INVALID_ARG;
  } else if (act_fmt != QL_ROUTE_INT8 && act_fmt != QL_ACT_INT8_F16) {
    return QL_ERR_INVALID_ARG;
  }
  if (!aligned(X, 16) || !aligned(codes, 16) || !aligned(sf_mma, 16) || !aligned(sf_rowmajor, 16) ||
      !aligned(scales, 4) || !aligned(ws, 256) || !aligned(amax_in, 4))
    return QL_ERR_ALIGNMENT;
  if (ws_bytes < qlinear_quantize_ws_bytes(M, K, act_fmt)) return QL_ERR_WORKSPACE;
  QL_TRY(device_ready());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int had = hadamard ? 1 : 0;
  if (act_fmt == QL_ROUTE_INT8) return launch_quant_int8_token(X, M, K, had, codes, scales, st, 0, qmax);
  if (act_fmt == QL_ACT_INT8_F16) return launch_quant_int8_token(X, M, K, had, codes, scales, st, 1, qmax);
  const float* amax = amax_in;
  if (amax == nullptr) {
    float* slot = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kAmaxWsBytes);
    QL_TRY(launch_amax(X, M, K, had, slot, ws, st));
    amax = slot;
  }
  if (act_fmt == QL_ROUTE_NVFP4 || act_fmt == QL_ACT_NVFP4_DECOMP)
    return launch_quant_nvfp4(X, M, K, had, amax, codes, sf_mma, sf_rowmajor, scales, st,
                              act_fmt == QL_ACT_NVFP4_DECOMP ? 1 : 0);
  return launch_quant_int8_tensor_perm(X, M, K, w->Kp, w->gather, amax, codes, scales, st, qmax);
}

// ---------------------------------------------------------------- GEMM
ql_status qlinear_gemm(int32_t act_fmt, const void* a_codes, const void* a_sf, const float* a_scales,
                       int64_t M, const ql_weights* w, void* Y, void* stream) {
  QL_TRY(check_m(M));
  QL_TRY(check_w(w));
  QL_TRY(check_mn(M, w->N));
  if (M > 0 && (a_codes == nullptr || (a_scales == nullptr && act_fmt != QL_ROUTE_BF16) || Y == nullptr))
    return QL_ERR_INVALID_ARG;
  act_fmt = int_base_fmt(act_fmt);   // INT6 codes run through the INT8 GEMMs unchanged
  if (act_fmt == QL_ROUTE_BF16) {      // a_codes: the bf16 input [M, K]; no scales
    if (w->fmt != QL_W_NVFP4 || w->wbf16 == nullptr || (M > 0 && a_codes == nullptr)) return QL_ERR_INVALID_ARG;
    if (!aligned(a_codes, 16) || !aligned(Y, 16)) return QL_ERR_ALIGNMENT;
    QL_TRY(device_ready());
    return launch_gemm_bf16(a_codes, M, w, Y, static_cast<cudaStream_t>(stream), status_word());
  }
  if (act_fmt == QL_ROUTE_NVFP4 || act_fmt == QL_ROUTE_INT8 || act_fmt == QL_ACT_INT8_F16) {
    if (w->fmt != QL_W_NVFP4) return QL_ERR_INVALID_ARG;
    if (act_fmt == QL_ROUTE_NVFP4 && M > 0 && a_sf == nullptr) return QL_ERR_INVALID_ARG;
  } else if (act_fmt == QL_ACT_INT8_TENSOR) {
    if (w->fmt != QL_W_QARVD_INT4) return QL_ERR_INVALID_ARG;
  } else if (act_fmt == QL_ACT_NVFP4_DECOMP) {
    if (w->fmt != QL_W_NVFP4_DECOMP || (M > 0 && a_sf == nullptr)) return QL_ERR_INVALID_ARG;
  } else {
    return QL_ERR_INVALID_ARG;
  }
  if (!aligned(a_codes, 16) || !aligned(a_sf, 16) || !aligned(Y, 16) || !aligned(a_scales, 4))
    return QL_ERR_ALIGNMENT;
  QL_TRY(device_ready());
  if (M == 0) return QL_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* status = status_word();
  if (act_fmt == QL_ROUTE_NVFP4)
    return launch_gemm_w4a4(a_codes, static_cast<const uint8_t*>(a_sf), a_scales, M, w, Y, st, status);
  if (act_fmt == QL_ACT_NVFP4_DECOMP) {   // one W4A4 contraction over K' = 2K
    ql_weights w2 = *w;
    w2.K = 2 * w->K;
    return launch_gemm_w4a4(a_codes, static_cast<const uint8_t*>(a_sf), a_scales, M, &w2, Y, st, status);
  }
  if (act_fmt == QL_ROUTE_INT8) return launch_gemm_w4a8(a_codes, a_scales, M, w, Y, st, status);
  if (act_fmt == QL_ACT_INT8_F16) return launch_gemm_w4a8(a_codes, a_scales, M, w, Y, st, status, 1);
  return launch_gemm_qarvd(a_codes, a_scales, M, w, Y, st, status);
}

// ---------------------------------------------------------------- forward
size_t qlinear_forward_ws_bytes(int64_t M, const ql_weights* w, int32_t route) {
  if (M < 0 || check_w(w) != QL_OK) return 0;
  if (w->fmt == QL_W_QARVD_INT4) return forward_act_bytes(M, w->K, w->Kp, QL_ACT_INT8_TENSOR);
  if (w->fmt == QL_W_NVFP4_DECOMP)
    return route == QL_ROUTE_NVFP4 ? forward_act_bytes(M, w->K, 0, QL_ACT_NVFP4_DECOMP) : 0;
  if (route == QL_ROUTE_BF16) return w->wbf16 != nullptr ? 256 : 0;
  route = int_base_fmt(route);
  if (route != QL_ROUTE_NVFP4 && route != QL_ROUTE_INT8) return 0;
  return forward_act_bytes(M, w->K, 0, route, true);
}

ql_status qlinear_forward(const void* X, int64_t M, const ql_weights* w, int32_t route, void* Y,
                          void* ws, size_t ws_bytes, void* stream) {
  QL_TRY(check_m(M));
  QL_TRY(check_w(w));
  QL_TRY(check_mk(M, w->K));
  QL_TRY(check_mn(M, w->N));
  if (ws == nullptr || (M > 0 && (X == nullptr || Y == nullptr))) return QL_ERR_INVALID_ARG;
  if (w->fmt == QL_W_NVFP4_DECOMP && route != QL_ROUTE_NVFP4) return QL_ERR_INVALID_ARG;
  if (route == QL_ROUTE_BF16) {   // PDR's high-precision refresh: the input as it is
    if (w->fmt != QL_W_NVFP4 || w->wbf16 == nullptr) return QL_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(ws, 256)) return QL_ERR_ALIGNMENT;
    QL_TRY(device_ready());
    return launch_gemm_bf16(X, M, w, Y, static_cast<cudaStream_t>(stream), status_word());
  }
  // W4A6: route QL_ROUTE_INT6 (or QL_ACT_INT6_TENSOR for Q-ARVD weights)
  const int qmax = (route == QL_ROUTE_INT6 || route == QL_ACT_INT6_TENSOR) ? 31 : 127;
  if (w->fmt == QL_W_NVFP4 && route == QL_ACT_INT6_TENSOR) return QL_ERR_INVALID_ARG;
  const int32_t fmt = (w->fmt == QL_W_QARVD_INT4)     ? int32_t(QL_ACT_INT8_TENSOR)
                      : (w->fmt == QL_W_NVFP4_DECOMP) ? int32_t(QL_ACT_NVFP4_DECOMP)
                                                      : int_base_fmt(route);
  if (fmt != QL_ROUTE_NVFP4 && fmt != QL_ROUTE_INT8 && fmt != QL_ACT_INT8_TENSOR && fmt != QL_ACT_NVFP4_DECOMP)
    return QL_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(ws, 256)) return QL_ERR_ALIGNMENT;
  if (ws_bytes < qlinear_forward_ws_bytes(M, w, route)) return QL_ERR_WORKSPACE;
  QL_TRY(device_ready());
  if (M == 0) return QL_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int K = w->K;
  Carver c{static_cast<uint8_t*>(ws)};
  int* status = status_word();
  if (fmt == QL_ROUTE_NVFP4 || fmt == QL_ACT_NVFP4_DECOMP) {
    const int decomp = fmt == QL_ACT_NVFP4_DECOMP ? 1 : 0;
    const int kq = decomp ? 2 * K : K;
    void* aws = c.take<uint8_t>(kAmaxWsBytes);
    float* amax = c.take<float>(256);
    float* g = c.take<float>(256);
    uint8_t* codes = c.take<uint8_t>(static_cast<size_t>(M) * kq / 2);
    uint8_t* sf = c.take<uint8_t>(qlinear_sf_bytes(M, kq));
    QL_TRY(launch_amax(X, M, K, w->hadamard, amax, aws, st));
    QL_TRY(launch_quant_nvfp4(X, M, K, w->hadamard, amax, codes, sf, nullptr, g, st, decomp));
    ql_weights w2 = *w;
    w2.K = kq;
    return launch_gemm_w4a4(codes, sf, g, M, &w2, Y, st, status);
  }
  if (fmt == QL_ROUTE_INT8) {
    // codes as f16 values: the f16 MMA's operand type (weights from their f16
    // copy, or widened into tensor memory without one)
    uint8_t* codes = c.take<uint8_t>(static_cast<size_t>(M) * K * 2);
    float* s = c.take<float>(4 * static_cast<size_t>(M));
    QL_TRY(launch_quant_int8_token(X, M, K, w->hadamard, codes, s, st, 1, qmax));
    return launch_gemm_w4a8(codes, s, M, w, Y, st, status, 1);
  }
  void* aws = c.take<uint8_t>(kAmaxWsBytes);
  float* amax = c.take<float>(256);
  float* sx = c.take<float>(256);
  int8_t* codes = c.take<int8_t>(static_cast<size_t>(M) * w->Kp);
  QL_TRY(launch_amax(X, M, K, 0, amax, aws, st));
  QL_TRY(launch_quant_int8_tensor_perm(X, M, K, w->Kp, w->gather, amax, codes, sx, st, qmax));
  return launch_gemm_qarvd(codes, sx, M, w, Y, st, status);
}

// ---------------------------------------------------------------- forward, device route
size_t qlinear_forward_routed_ws_bytes(int64_t M, const ql_weights* w) {
  if (M < 0 || check_w(w) != QL_OK || w->fmt != QL_W_NVFP4) return 0;
  return forward_act_bytes(M, w->K, 0, QL_ROUTE_NVFP4) +
         forward_act_bytes(M, w->K, 0, QL_ROUTE_INT8, true);
}

ql_status qlinear_forward_routed(const void* X, int64_t M, const ql_weights* w, const int32_t* route_dev, void* Y,
                                 void* ws, size_t ws_bytes, void* stream) {
  QL_TRY(check_m(M));
  QL_TRY(check_w(w));
  QL_TRY(check_mk(M, w->K));
  QL_TRY(check_mn(M, w->N));
  if (w->fmt != QL_W_NVFP4 || route_dev == nullptr || ws == nullptr || (M > 0 && (X == nullptr || Y == nullptr)))
    return QL_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(ws, 256) || !aligned(route_dev, 4)) return QL_ERR_ALIGNMENT;
  if (ws_bytes < qlinear_forward_routed_ws_bytes(M, w)) return QL_ERR_WORKSPACE;
  QL_TRY(device_ready());
  if (M == 0) return QL_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int K = w->K;
  Carver c{static_cast<uint8_t*>(ws)};
  int* status = status_word();
  const Gate g_fp4{route_dev, QL_ROUTE_NVFP4}, g_int8{route_dev, QL_ROUTE_INT8}, g_bf16{route_dev, QL_ROUTE_BF16};
  // NVFP4 route
  void* aws = c.take<uint8_t>(kAmaxWsBytes);
  float* amax = c.take<float>(256);
  float* g = c.take<float>(256);
  uint8_t* codes4 = c.take<uint8_t>(static_cast<size_t>(M) * K / 2);
  uint8_t* sf = c.take<uint8_t>(qlinear_sf_bytes(M, K));
  QL_TRY(launch_amax(X, M, K, w->hadamard, amax, aws, st, g_fp4));
  QL_TRY(launch_quant_nvfp4(X, M, K, w->hadamard, amax, codes4, sf, nullptr, g, st, 0, g_fp4));
  QL_TRY(launch_gemm_w4a4(codes4, sf, g, M, w, Y, st, status, g_fp4));
  // INT8 route
  uint8_t* codes8 = c.take<uint8_t>(static_cast<size_t>(M) * K * 2);
  float* s8 = c.take<float>(4 * static_cast<size_t>(M));
  QL_TRY(launch_quant_int8_token(X, M, K, w->hadamard, codes8, s8, st, 1, 127, g_int8));
  QL_TRY(launch_gemm_w4a8(codes8, s8, M, w, Y, st, status, 1, g_int8));
  // BF16 (PDR's refresh) when the weights were kept
  if (w->wbf16 != nullptr) QL_TRY(launch_gemm_bf16(X, M, w, Y, st, status, g_bf16));
  return QL_OK;
}

}  // extern "C"
