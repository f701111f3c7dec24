// Pieces shared by the tcgen05 GEMM kernels: arguments, tile order, bounded
// teardown, the bf16 epilogue and host-side tensor-map creation.
#pragma once

#include <algorithm>
#include <utility>
#include "ql_common.cuh"

namespace ql {

constexpr int kEpiChunkCols = 64;                        // bf16 columns per TMA store
constexpr int kEpiChunkBytes = 128 * kEpiChunkCols * 2;  // 16 KB staging tile
constexpr long long kDrainLimit = 4000000000ll;          // cycles for teardown waits

struct GemmArgs {
  int32_t M, N, K;
  int32_t tiles_m, tiles_n, num_tiles;
  int32_t num_kst;      // K stages of the main loop
  int32_t k_atoms;      // NVFP4: K / 64 (4-scale groups per row)
  int32_t sfb_atoms;    // NVFP4: 128-row scale atoms of the weights
  int32_t group_m;      // tile raster: m-blocks per group
  const uint8_t* sfa;   // NVFP4 activation scales (MMA layout)
  const uint8_t* sfb;   // NVFP4 weight scales (MMA layout)
  const float* g_a;     // activation tensor scale (NVFP4 / per-tensor INT8)
  const float* g_w;     // weight tensor scale (NVFP4)
  const float* row_scale;  // per-token activation scales (INT8 route)
  const float* col_scale0; // Q-ARVD s_norm
  const float* col_scale1; // Q-ARVD s_out
  const int32_t* kinfo;    // Q-ARVD class sizes
  float alpha_mul;
  long long wait_limit;
  int* status;             // device status word
  const int32_t* gate;     // device-routed forward: the route in device memory (or null)
  int32_t gate_value;      // this launch's route
};

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + (((a + 1023u) & ~1023u) - a);
}

// Tile t -> (m-block, n-block).  Groups of `group_m` m-blocks sweep all
// n-blocks together so that concurrently running CTAs share A and B tiles
// in L2.
__device__ __forceinline__ void tile_coords(int t, const GemmArgs& p, int& mb, int& nb) {
  const int per_group = p.group_m * p.tiles_n;
  const int g = t / per_group;
  const int first_m = g * p.group_m;
  const int gm = min(p.group_m, p.tiles_m - first_m);
  const int r = t - g * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

__device__ __forceinline__ void fail_timeout(int* status, volatile int* abort_flag) {
  record_error(status, QL_ERR_TIMEOUT);
  *abort_flag = 1;
}

// Accumulator-ready wait of the 128 epilogue threads (one 128-aligned group
// of four warps) with ONE decision for all of them: the group's first thread
// does the bounded wait and publishes the outcome
// through shared memory behind a named barrier, so no epilogue thread can
// leave the tile loop while another one waits at a later named barrier.
// The flag slot sits right after the abort flag.
__device__ __forceinline__ bool epilogue_wait_uniform(uint64_t* bar, uint32_t parity, long long limit,
                                                      volatile int* abort_flag, int* status) {
  volatile int* slot = abort_flag + 1;
  if ((threadIdx.x & 127) == 0) {
    const bool ok = (*abort_flag == 0) && mbar_wait(bar, parity, limit);
    if (!ok) fail_timeout(status, abort_flag);
    *slot = ok ? 1 : 0;
  }
  named_bar_sync(1, 128);
  return *slot != 0;
}

// Wait for the last (up to) `stages` loads this producer issued, so that no
// copy is still writing shared memory when the CTA retires.
__device__ __forceinline__ void drain_loads(uint64_t* full, int issued, int stages, int* status) {
  for (int j = max(0, issued - stages); j < issued; ++j) {
    if (!mbar_wait(&full[j % stages], (j / stages) & 1, kDrainLimit))
      record_error(status, QL_ERR_TIMEOUT);
  }
}

// Wait until every tcgen05 operation issued by this thread has completed.
__device__ __forceinline__ void drain_mma(uint64_t* bar, int* status) {
  tc_commit(bar);
  if (!mbar_wait(bar, 0, kDrainLimit)) record_error(status, QL_ERR_TIMEOUT);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

struct EpilogueState {
  uint32_t buf;
};

// Store one 64-column chunk (this thread's row `row`, values v[0..63]) via
// the swizzled staging buffer and a TMA store.  Called by all 128 epilogue
// threads (a 128-aligned group of four warps); its first thread issues the
// bulk operations.
__device__ __forceinline__ void epilogue_store_chunk(const uint32_t (&packed)[32], uint8_t* sC,
                                                     const CUtensorMap* tm_y, int c0, int r0,
                                                     EpilogueState& es) {
  const int row = threadIdx.x & 127;
  const bool leader = row == 0;
  if (leader) bulk_wait_read<1>();
  named_bar_sync(1, 128);
  uint8_t* dst = sC + es.buf * kEpiChunkBytes + row * 128;
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<uint4*>(dst + ((q ^ (row & 7)) << 4)) =
        make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
  fence_proxy_async_smem();
  named_bar_sync(1, 128);
  if (leader) {
    tma_store_2d(tm_y, sC + es.buf * kEpiChunkBytes, c0, r0);
    bulk_commit();
  }
  es.buf ^= 1;
}

// bf16 epilogue of one BM x BN fp32 accumulator: y = alpha * acc, with
// alpha multiplied by row_scale[row] when row_scale is given (rows past
// the end of the operand read no scale).  Frees the accumulator (arrive on
// `tempty`) as soon as the last columns are in registers.
template <int BN>
__device__ __forceinline__ void epilogue_tile(uint32_t acc_tmem, uint64_t* tempty, uint8_t* sC,
                                              const CUtensorMap* tm_y, int m0, int n0, int N,
                                              float alpha, EpilogueState& es,
                                              const float* row_scale = nullptr, int M = 0) {
  const int ew = (threadIdx.x >> 5) & 3;
  const int lane = threadIdx.x & 31;
  constexpr int CH = BN / kEpiChunkCols;
  if (row_scale != nullptr) {
    const int m = m0 + (threadIdx.x & 127);
    alpha = (m < M) ? __fmul_rn(alpha, ld_dep(row_scale + m)) : 0.f;
  }
#pragma unroll 1
  for (int c = 0; c < CH; ++c) {
    uint32_t r0[32], r1[32];
    const uint32_t taddr = acc_tmem + (static_cast<uint32_t>(ew * 32) << 16) + c * kEpiChunkCols;
    tmem_ld32(taddr, r0);
    tmem_ld32(taddr + 32, r1);
    tmem_ld_wait();
    if (c == CH - 1) {
      tc_fence_before();
      if (lane == 0) mbar_arrive(tempty);
    }
    if (n0 + c * kEpiChunkCols >= N) continue;   // same for all 128 threads
    uint32_t packed[32];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      packed[j] = pack_bf16x2(__fmul_rn(alpha, __uint_as_float(r0[2 * j])),
                              __fmul_rn(alpha, __uint_as_float(r0[2 * j + 1])));
      packed[16 + j] = pack_bf16x2(__fmul_rn(alpha, __uint_as_float(r1[2 * j])),
                                   __fmul_rn(alpha, __uint_as_float(r1[2 * j + 1])));
    }
    epilogue_store_chunk(packed, sC, tm_y, n0 + c * kEpiChunkCols, m0, es);
  }
}

__device__ __forceinline__ void epilogue_finish(EpilogueState&) {
  if ((threadIdx.x & 127) == 0) bulk_wait_all();
}

// ---------------------------------------------------------------------------
// Per-warp epilogue.  A warp reads 32 TMEM lanes (its lane quarter) of the
// accumulator and owns those 32 output rows; it stores them in boxes of
// 32 rows x 32 bf16 columns through its own staging buffers (2 KB each,
// 64-byte swizzle) with TMA stores, so epilogue warps never wait for each
// other.  The output tensor map has box {32, 32} and SWIZZLE_64B.
// ---------------------------------------------------------------------------
constexpr int kWarpBoxCols = 32;
constexpr int kWarpBoxBytes = 32 * kWarpBoxCols * 2;   // 2 KB

struct WarpStoreState {
  int next;   // staging buffer for the next box
};

// Accumulator-ready wait of one warp: lane 0 does the bounded wait and the
// outcome is broadcast, so the whole warp takes the same branch.
__device__ __forceinline__ bool warp_wait_uniform(uint64_t* bar, uint32_t parity, long long limit,
                                                  volatile int* abort_flag, int* status) {
  int ok = 0;
  if (lane_id() == 0) {
    ok = (*abort_flag == 0) && mbar_wait(bar, parity, limit);
    if (!ok) fail_timeout(status, abort_flag);
  }
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// One warp's share of an accumulator tile: NCH boxes of 32 columns starting
// at TMEM address `taddr` (lane quarter already folded in) and at output
// column `col0`; output row of lane i = row0 + i.  y = bf16(alpha * acc),
// alpha times row_scale[row] when row_scale is given.  After the TMEM reads
// the warp arrives once on the mbarrier at `release` (a shared::cluster
// address: this CTA's barrier or the pair leader's).  Boxes entirely past M
// or N are skipped; TMA clips partial ones.
template <int NCH, int NBUF>
__device__ __forceinline__ void epilogue_warp_tile(uint32_t taddr, uint32_t release, uint8_t* stage,
                                                   const CUtensorMap* tm_y, int row0, int col0, int M,
                                                   int N, float alpha, WarpStoreState& ws,
                                                   const float* row_scale = nullptr) {
  const int lane = lane_id();
  uint32_t r[NCH][32];
#pragma unroll
  for (int c = 0; c < NCH; ++c) tmem_ld32(taddr + kWarpBoxCols * c, r[c]);
  tmem_ld_wait();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive_cluster(release);
  if (row_scale != nullptr) {
    const int row = row0 + lane;
    alpha = (row < M) ? __fmul_rn(alpha, ld_dep(row_scale + row)) : 0.f;
  }
  if (row0 >= M) return;   // warp-uniform
  const uint32_t swz = (lane >> 1) & 3;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int col = col0 + kWarpBoxCols * c;
    if (col >= N) break;   // warp-uniform
    uint8_t* buf = stage + ws.next * kWarpBoxBytes;
    if (lane == 0) bulk_wait_read<NBUF - 1>();
    __syncwarp();
    uint8_t* dst = buf + lane * 64;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 v;
      v.x = pack_bf16x2(__fmul_rn(alpha, __uint_as_float(r[c][8 * q + 0])),
                        __fmul_rn(alpha, __uint_as_float(r[c][8 * q + 1])));
      v.y = pack_bf16x2(__fmul_rn(alpha, __uint_as_float(r[c][8 * q + 2])),
                        __fmul_rn(alpha, __uint_as_float(r[c][8 * q + 3])));
      v.z = pack_bf16x2(__fmul_rn(alpha, __uint_as_float(r[c][8 * q + 4])),
                        __fmul_rn(alpha, __uint_as_float(r[c][8 * q + 5])));
      v.w = pack_bf16x2(__fmul_rn(alpha, __uint_as_float(r[c][8 * q + 6])),
                        __fmul_rn(alpha, __uint_as_float(r[c][8 * q + 7])));
      *reinterpret_cast<uint4*>(dst + ((q ^ swz) << 4)) = v;
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tm_y, buf, col, row0);
      bulk_commit();
    }
    ws.next = (ws.next + 1 == NBUF) ? 0 : ws.next + 1;
  }
}

__device__ __forceinline__ void epilogue_warp_finish() {
  if (lane_id() == 0) bulk_wait_all();
  __syncwarp();
}

// ---------------------------------------------------------------------------
// Host helpers (defined in capi.cu)
// ---------------------------------------------------------------------------
bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int64_t inner,
                  int64_t outer, int64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                  CUtensorMapSwizzle swizzle);
bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int64_t d0, int64_t d1,
                  int64_t d2, int64_t stride1_bytes, int64_t stride2_bytes, uint32_t b0, uint32_t b1,
                  uint32_t b2);
// Block scales in the MMA layout as a 3-D tensor of 32-bit words
// (128 words of a 512-byte atom, K/64 atoms of a 128-row group, row groups);
// one box is box_k atoms (4 = one 256-value K stage) of one group.
bool make_sf_tmap(CUtensorMap* map, const void* base, int64_t rows, int K, uint32_t box_k);
int num_sms();
bool set_smem_attr(const void* kernel, int bytes);

// Launch with programmatic stream serialization (the kernel calls
// pdl_wait_then_release before touching global memory) and, when
// cluster_x > 1, a cluster of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
void fill_gemm_args(GemmArgs& p, int64_t M, int N, int K, int BN, int* status);

}  // namespace ql
