// Allocation-free DMPQ router.
//
// Same Gamma / route computation as qlinear_route, but its scratch (per-CTA
// fp64 partial sums and a finished-CTA counter) lives in a file-scope device
// array instead of a caller-provided workspace, so a caller that cannot
// allocate device memory can still run the router.  The array is sized for
// kNoAllocMaxCtas CTAs; every device that loads the library keeps it until
// the process exits.
#include <mutex>

#include "ql_common.cuh"
#include "route_common.cuh"
#include "launchers.h"

namespace {

constexpr int kNoAllocMaxCtas = 1024;
constexpr size_t kTicketOffset = kNoAllocMaxCtas * 2 * sizeof(double);   // after the partials
constexpr size_t kNoAllocScratchBytes = kTicketOffset + 256;              // 16640 bytes
constexpr int kMaxDev = 64;

// In host code this name is only a stand-in for the device array; the host
// passes the address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDev] = {nullptr};

// Gamma = sum|out - in| / sum|in| (fp32 differences, fp64 sums) with the
// scratch at `scratch`: partials [2 * gridDim.x] doubles, then the counter.
__global__ void __launch_bounds__(ql::kThreadsHbm)
    k_gamma_route_static(const uint4* __restrict__ in, const uint4* __restrict__ out, int64_t numel,
                         unsigned char* __restrict__ scratch, float threshold,
                         double* __restrict__ gamma_out, int32_t* __restrict__ route_out) {
  double* partials = reinterpret_cast<double*>(scratch);
  unsigned int* ticket = reinterpret_cast<unsigned int*>(scratch + kTicketOffset);
  double s1, s0;
  ql::gamma_thread_sums(in, out, numel, s1, s0);
  ql::gamma_finish(s1, s0, partials, ticket, threshold, gamma_out, route_out);
}

bool is_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" ql_status qlinear_route_noalloc(const void* in, const void* out, int64_t numel,
                                           float threshold, double* gamma_dev, int32_t* route_dev,
                                           void* stream) {
  if (numel < 0 || gamma_dev == nullptr || route_dev == nullptr) return QL_ERR_INVALID_ARG;
  if (numel > 0 && (in == nullptr || out == nullptr)) return QL_ERR_INVALID_ARG;
  if (!(threshold == threshold)) return QL_ERR_INVALID_ARG;
  if (!is_aligned(in, 16) || !is_aligned(out, 16) || !is_aligned(gamma_dev, 8) ||
      !is_aligned(route_dev, 4))
    return QL_ERR_ALIGNMENT;
  int dev = -1, major = 0, minor = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return QL_ERR_NO_DEVICE;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return QL_ERR_NO_DEVICE;
  if (major != 10 || minor != 0) return QL_ERR_NO_DEVICE;
  // Set-up, once per device with that device current: the device address of
  // the scratch array.
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_setup_mu);
    if (g_scratch_addr[dev] == nullptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr) return QL_ERR_CUDA;
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }
  const int64_t want = (numel / 8 + ql::kThreadsHbm - 1) / ql::kThreadsHbm;
  const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(want, static_cast<int64_t>(sms) * ql::kHbmCtasPerSm));
  if (grid > kNoAllocMaxCtas) return QL_ERR_UNSUPPORTED_SHAPE;   // would overrun the scratch array
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents: the counter must start at 0.
  if (cudaMemsetAsync(static_cast<unsigned char*>(scratch) + kTicketOffset, 0, sizeof(unsigned int), st) !=
      cudaSuccess)
    return QL_ERR_CUDA;
  // The launch's own return code decides success: an error left pending by
  // an unrelated earlier call is not this call's failure.
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned int>(grid));
  cfg.blockDim = dim3(ql::kThreadsHbm);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k_gamma_route_static, static_cast<const uint4*>(in),
                                           static_cast<const uint4*>(out), numel,
                                           static_cast<unsigned char*>(scratch), threshold, gamma_dev,
                                           route_dev);
  return e == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}
