// W4A4 GEMM: NVFP4 activations x NVFP4 weights -> bf16, fp32 accumulation
// in tensor memory (6Bit-Diffusion, Methodology B.1: NVFP4 weights and
// NVFP4 activations on stable blocks, targeting Blackwell's NVFP4 support).
//
// Y[m, n] = bf16(alpha * sum_k (e2m1_a * sfa)(e2m1_w * sfw)),
// alpha = g_a * g_w * alpha_mul (alpha_mul = 1/128 undoes the two Hadamard
// rotations, 1 otherwise).
//
// Persistent and warp-specialized, 384 threads per CTA, one CTA per SM.
//   PAIR = true   two SMs of a cluster share each 256 x BN tile through
//                 tcgen05 cta_group::2: each CTA holds its 128 rows of A and
//                 half of the BN rows of B; the leader (cluster rank 0)
//                 issues the MMAs, which write each CTA's 128 x BN
//                 accumulator into that CTA's tensor memory.
//   PAIR = false  one SM per 128 x BN tile (used when M <= 128).
// Roles:
//   warp 0      TMA producer: A/B FP4 tiles (128-byte swizzle) and the
//               block scales into a STAGES-deep shared-memory ring;
//   warp 1      MMA issuer: tcgen05.cp of block scales into tensor memory
//               and tcgen05.mma kind::mxf4nvf4 block16 (BM x BN x 64);
//   warp 2      tensor-memory allocation;
//   warps 4-11  epilogue, two warps per TMEM lane quarter, each with half of
//               the tile's columns: tcgen05.ld, * alpha, bf16, TMA store of
//               32 x 32 boxes from per-warp staging buffers.  With two
//               accumulators the epilogue of one tile overlaps the main
//               loop of the next.
//
// Measured on this GPU, the tensor pipe runs block-scaled MMAs at their
// math rate (N / 2 cycles per 64-deep K step of a CTA pair) whatever the
// number of scale copies issued beside them, and is not slowed by
// concurrent shared-memory, tensor-memory or bulk-copy traffic.  The main
// loop is bound by the latency of its operand loads instead: a stage of
// TMA loads takes about 1500-2000 cycles to land, and shared memory holds
// only four to six stages, so the deeper the ring (in MMA cycles per byte
// of shared memory), the faster the loop.  Scale feeding:
//   RES = true    (K <= 64 * kResKSteps) the activation scales of a
//                 128-row block for the whole K range stay resident in
//                 tensor memory while the unit walks the N tiles of that
//                 row block (tiles are handed out in contiguous row-major
//                 ranges); the B scales of each K step go to one of
//                 SFB_SLOTS small slots.
//     APANEL      additionally keeps the row block's A tiles for the whole K
//                 range in shared memory, so only B and its scales stream
//                 through the ring (half the bytes per stage); the panel is
//                 reloaded chunk by chunk, each chunk as soon as the MMAs of
//                 the row block's last tile have read it.
//   RES = false   the A and B scales of each stage are copied per stage into
//                 one of SF_SLOTS slots (rotating per stage).
// The tensor pipe runs the copies and MMAs of one issuing thread in issue
// order, so a copy into a scale slot follows the MMAs issued before it.
// Every mbarrier wait is bounded; on a timeout the kernel records
// QL_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#include "ql_common.cuh"
#include "gemm_common.cuh"
#include "launchers.h"

namespace ql {

constexpr int kResKSteps = 30;   // K steps (64 wide) of resident activation scales

template <int BN, int STAGES, bool PAIR, int ACC_, int EPI_BUF, bool RES, int BKB_ = 128, bool APANEL = false>
struct W4A4Cfg {
  static constexpr int CTAS = PAIR ? 2 : 1;
  static constexpr int BM = 128;                     // rows per CTA
  static constexpr int BKB = BKB_;                   // K bytes per stage (2 FP4 values a byte)
  static constexpr int KC = BKB / 128;               // 128-byte K chunks (one swizzle span each)
  static constexpr int KSTEPS = BKB / 32;            // 64-wide MMA K steps (scale atoms) per stage
  static constexpr int BNL = BN / CTAS;              // B rows held by each CTA
  static constexpr int A_CHUNK = BM * 128;
  static constexpr int B_CHUNK = BNL * 128;
  static constexpr int A_BYTES = KC * A_CHUNK;
  static constexpr int B_BYTES = KC * B_CHUNK;
  // APANEL: the A tiles of the current row block for the whole K range stay
  // in shared memory (one chunk of A_CHUNK bytes per K stage) while the unit
  // walks that row block's N tiles, so only B streams through the ring.
  static constexpr int APCH = APANEL ? (kResKSteps + KSTEPS - 1) / KSTEPS : 0;   // panel chunks
  static constexpr int A_RING = APANEL ? APCH * A_CHUNK : STAGES * A_BYTES;
  // 128-row scale atoms per B tile.  Each CTA of a pair holds the weight
  // scales of all BN rows: each SM's MMA reads every B row's scales from its
  // own tensor memory.
  static constexpr int NSFB = (BN + 127) / 128;
  static constexpr int SFA_BYTES = RES ? 0 : KSTEPS * 512;      // per stage
  static constexpr int SFB_GROUP = KSTEPS * 512;                // one 128-row atom column per stage
  static constexpr int SFB_BYTES = NSFB * SFB_GROUP;            // per stage
  static constexpr int SFA_RES_BYTES = RES ? kResKSteps * 512 : 0;
  static constexpr int ACC = ACC_;
  static constexpr int EPI_WARPS = 8;
  static constexpr int EPI_CH = BN / 2 / kWarpBoxCols;   // boxes per epilogue warp per tile
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + A_RING;
  static constexpr int OFF_SFB = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_SFA = OFF_SFB + STAGES * SFB_BYTES;
  static constexpr int OFF_SFA_RES = OFF_SFA + STAGES * SFA_BYTES;
  static constexpr int OFF_C = OFF_SFA_RES + ((SFA_RES_BYTES + 1023) / 1024) * 1024;
  static constexpr int OFF_BAR = OFF_C + EPI_WARPS * EPI_BUF * kWarpBoxBytes;
  static constexpr int NBAR = 2 * STAGES + 2 * ACC + 1 + 2 + 2 * APCH;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment
  // Tensor memory: ACC accumulators of BN columns, then the scales.
  static constexpr uint32_t TM_SF = ACC * BN;
  //   RES: resident A scales (4 columns per K step), then SFB_SLOTS slots of
  //        4 * NSFB columns (the B scales of one K step).
  static constexpr uint32_t TM_SFB_RES = TM_SF + 4 * kResKSteps;
  static constexpr uint32_t SFB_KCOLS = 4 * NSFB;
  static constexpr int SFB_SLOTS_FIT = RES ? static_cast<int>((512 - TM_SFB_RES) / SFB_KCOLS) : 1;
  static constexpr int SFB_SLOTS = SFB_SLOTS_FIT < 4 ? SFB_SLOTS_FIT : 4;
  //   streaming: SF_SLOTS slots of one stage's A and B scales.
  static constexpr uint32_t SF_COLS = 16 + 16 * NSFB;
  static constexpr int SF_SLOTS_FIT = RES ? 2 : static_cast<int>((512 - TM_SF) / SF_COLS);
  static constexpr int SF_SLOTS = SF_SLOTS_FIT < 4 ? SF_SLOTS_FIT : 4;
  static_assert(RES ? SFB_SLOTS >= 1 : (SF_SLOTS >= 2 && SF_SLOTS < STAGES), "scale slots");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(BN % 64 == 0 && BN <= 256 && BNL % 16 == 0, "tile width");
  static_assert(A_CHUNK % 1024 == 0 && B_CHUNK % 1024 == 0, "1024-byte aligned chunks");
  static_assert(BKB % 128 == 0 && (RES || BKB == 128), "streamed scales take 128-byte stages");
  static_assert(EPI_BUF >= 1 && EPI_BUF <= EPI_CH, "staging buffers");
  static_assert(!APANEL || (RES && KC == 1), "the A panel goes with resident scales and 128-byte stages");
  // Instruction descriptor (block-scaled): A/B = E2M1 (1), scale = UE4M3 (0),
  // both K-major, N >> 3 at bit 17, M >> 4 at bit 24, dense K = 64.
  static constexpr uint32_t IDESC =
      (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t((BM * CTAS) >> 4) << 24);
};

// The tiles of one processing unit: contiguous row-major ranges (so the N
// tiles of a row block follow each other) or a strided walk over the
// grouped raster of tile_coords.
struct TileWalk {
  int begin, end, step;
  bool contiguous;
  __device__ __forceinline__ TileWalk(const GemmArgs& p, int unit, int nunits, bool contig) : contiguous(contig) {
    if (contig) {
      begin = static_cast<int>(static_cast<int64_t>(unit) * p.num_tiles / nunits);
      end = static_cast<int>(static_cast<int64_t>(unit + 1) * p.num_tiles / nunits);
      step = 1;
    } else {
      begin = unit;
      end = p.num_tiles;
      step = nunits;
    }
  }
  __device__ __forceinline__ void coords(int t, const GemmArgs& p, int& mb, int& nb) const {
    if (contiguous) {
      mb = t / p.tiles_n;
      nb = t - mb * p.tiles_n;
    } else {
      tile_coords(t, p, mb, nb);
    }
  }
};

template <int BN, int STAGES, bool PAIR, int ACC_, int EPI_BUF, bool RES, int BKB_, bool APANEL>
__global__ void __launch_bounds__(384, 1)
    k_gemm_w4a4(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                const __grid_constant__ CUtensorMap tm_y, const GemmArgs p) {
  using C = W4A4Cfg<BN, STAGES, PAIR, ACC_, EPI_BUF, RES, BKB_, APANEL>;
  if (p.gate != nullptr) {   // device-routed forward: both CTAs of a pair read the same route
    pdl_wait();
    if (gated_off(p.gate, p.gate_value)) {
      pdl_release();
      return;
    }
  }
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);   // pair: the leader's is used
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + C::ACC;                                // pair: the leader's is used
  uint64_t* drain = tempty + C::ACC;
  uint64_t* sfa_full = drain + 1;                                   // RES: pair: the leader's is used
  uint64_t* sfa_empty = sfa_full + 1;
  uint64_t* a_full = sfa_empty + 1;                                 // APANEL: per chunk; pair: the leader's
  uint64_t* a_empty = a_full + C::APCH;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5;
  const int unit = PAIR ? (blockIdx.x >> 1) : blockIdx.x;       // tile-processing unit
  const int nunits = PAIR ? (gridDim.x >> 1) : gridDim.x;
  const TileWalk walk(p, unit, nunits, RES);

  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_sfa);
    prefetch_tmap(&tm_sfb);
    prefetch_tmap(&tm_y);
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < C::ACC; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], C::EPI_WARPS * C::CTAS);
    }
    mbar_init(drain, 1);
    mbar_init(sfa_full, 1);
    mbar_init(sfa_empty, 1);
    for (int i = 0; i < C::APCH; ++i) {
      mbar_init(&a_full[i], 1);
      mbar_init(&a_empty[i], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if constexpr (PAIR) cluster_sync();   // both CTAs' barriers exist before any remote use
  if (warp == 2) {
    if constexpr (PAIR)
      tmem_alloc_pair(tmem_slot, 512);
    else
      tmem_alloc(tmem_slot, 512);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();   // everything above touched only shared and tensor memory

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      int it = 0, nsfa = 0, cur_mb = -1, a_issued = 0;
      bool ok = true;
      for (int t = walk.begin; t < walk.end && ok; t += walk.step) {
        int mb, nb;
        walk.coords(t, p, mb, nb);
        const bool newrb = mb != cur_mb;   // first tile of a row block (RES walks)
        const int n0 = nb * BN;
        const int ra0 = n0 >> 7;
        const int a_row = mb * C::BM * C::CTAS + static_cast<int>(rank) * C::BM;
        const int b_row = n0 + static_cast<int>(rank) * C::BNL;
        const int sfa_group = mb * C::CTAS + static_cast<int>(rank);
        if constexpr (RES) {
          if (mb != cur_mb) {
            // A scales of the whole K range for this row block
            if (nsfa > 0 && (*abort_flag || !mbar_wait(sfa_empty, (nsfa - 1) & 1, p.wait_limit))) {
              ok = false;
              break;
            }
            uint8_t* dst = smem + C::OFF_SFA_RES;
            const uint32_t bytes = 512u * p.k_atoms;
            if constexpr (PAIR) {
              if (leader) mbar_arrive_expect_tx(sfa_full, 2 * bytes);
              tma_load_3d_pair(dst, &tm_sfa, map_to_rank(smem_u32(sfa_full), 0), 0, 0, sfa_group);
            } else {
              mbar_arrive_expect_tx(sfa_full, bytes);
              tma_load_3d(dst, &tm_sfa, sfa_full, 0, 0, sfa_group);
            }
            cur_mb = mb;
            ++nsfa;
          }
        }
        int nsfb = 0;
#pragma unroll
        for (int r = 0; r < C::NSFB; ++r) nsfb += (ra0 + r < p.sfb_atoms);
        const uint32_t tx = (APANEL ? 0u : C::A_BYTES) + C::B_BYTES + C::SFA_BYTES + nsfb * C::SFB_GROUP;
        if (APANEL && newrb) a_issued = 0;
        for (int ks = 0; ks < p.num_kst; ++ks, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if constexpr (APANEL) {
            if (newrb) {
              // Chunk ks of the new row block's A panel, once the MMAs of the
              // previous row block's last tile have read the old chunk.
              const int gen = nsfa - 1;
              if (gen > 0 && (*abort_flag || !mbar_wait(&a_empty[ks], (gen - 1) & 1, p.wait_limit))) {
                ok = false;
                break;
              }
              uint8_t* pa = smem + C::OFF_A + ks * C::A_CHUNK;
              if constexpr (PAIR) {
                if (leader) mbar_arrive_expect_tx(&a_full[ks], 2 * C::A_CHUNK);
                tma_load_2d_pair(pa, &tm_a, map_to_rank(smem_u32(&a_full[ks]), 0), ks * C::BKB, a_row);
              } else {
                mbar_arrive_expect_tx(&a_full[ks], C::A_CHUNK);
                tma_load_2d(pa, &tm_a, &a_full[ks], ks * C::BKB, a_row);
              }
              a_issued = ks + 1;
            }
          }
          if (*abort_flag || !mbar_wait(&empty[s], ph ^ 1, p.wait_limit)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + C::OFF_A + s * C::A_BYTES;
          uint8_t* sb = smem + C::OFF_B + s * C::B_BYTES;
          uint8_t* ssfa = smem + C::OFF_SFA + s * C::SFA_BYTES;
          uint8_t* ssfb = smem + C::OFF_SFB + s * C::SFB_BYTES;
          if constexpr (PAIR) {
            // Both CTAs' bytes complete on the leader's barrier.
            if (leader) mbar_arrive_expect_tx(&full[s], 2 * tx);
            const uint32_t bar = map_to_rank(smem_u32(&full[s]), 0);
#pragma unroll
            for (int c = 0; c < C::KC; ++c) {
              if constexpr (!APANEL) tma_load_2d_pair(sa + c * C::A_CHUNK, &tm_a, bar, ks * C::BKB + 128 * c, a_row);
              tma_load_2d_pair(sb + c * C::B_CHUNK, &tm_b, bar, ks * C::BKB + 128 * c, b_row);
            }
            if constexpr (!RES) tma_load_3d_pair(ssfa, &tm_sfa, bar, 0, C::KSTEPS * ks, sfa_group);
#pragma unroll
            for (int r = 0; r < C::NSFB; ++r)
              if (ra0 + r < p.sfb_atoms)
                tma_load_3d_pair(ssfb + r * C::SFB_GROUP, &tm_sfb, bar, 0, C::KSTEPS * ks, ra0 + r);
          } else {
            mbar_arrive_expect_tx(&full[s], tx);
#pragma unroll
            for (int c = 0; c < C::KC; ++c) {
              if constexpr (!APANEL) tma_load_2d(sa + c * C::A_CHUNK, &tm_a, &full[s], ks * C::BKB + 128 * c, a_row);
              tma_load_2d(sb + c * C::B_CHUNK, &tm_b, &full[s], ks * C::BKB + 128 * c, b_row);
            }
            if constexpr (!RES) tma_load_3d(ssfa, &tm_sfa, &full[s], 0, C::KSTEPS * ks, sfa_group);
#pragma unroll
            for (int r = 0; r < C::NSFB; ++r)
              if (ra0 + r < p.sfb_atoms)
                tma_load_3d(ssfb + r * C::SFB_GROUP, &tm_sfb, &full[s], 0, C::KSTEPS * ks, ra0 + r);
          }
        }
      }
      if (!ok) fail_timeout(p.status, abort_flag);
      if (leader) {
        drain_loads(full, it, STAGES, p.status);   // pair: covers both CTAs' bytes
        if (RES && nsfa > 0 && !mbar_wait(sfa_full, (nsfa - 1) & 1, kDrainLimit)) record_error(p.status, QL_ERR_TIMEOUT);
        if (APANEL)   // the last panel's chunks have landed
          for (int c = 0; c < a_issued; ++c)
            if (!mbar_wait(&a_full[c], (nsfa - 1) & 1, kDrainLimit)) record_error(p.status, QL_ERR_TIMEOUT);
      } else {
        // The peer's loads complete on the leader's barriers; the leader frees
        // each stage (empty) only after the MMAs consumed both halves.
        for (int j = max(0, it - STAGES); j < it; ++j)
          if (!mbar_wait(&empty[j % STAGES], (j / STAGES) & 1, kDrainLimit)) record_error(p.status, QL_ERR_TIMEOUT);
        if (RES && nsfa > 0 && !mbar_wait(sfa_empty, (nsfa - 1) & 1, kDrainLimit)) record_error(p.status, QL_ERR_TIMEOUT);
        if (APANEL)   // ... and each panel chunk after the last tile's MMAs read it
          for (int c = 0; c < a_issued; ++c)
            if (!mbar_wait(&a_empty[c], (nsfa - 1) & 1, kDrainLimit)) record_error(p.status, QL_ERR_TIMEOUT);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (leader && elect_one()) {
      int it = 0, local = 0, gk = 0, nsfa = 0, cur_mb = -1;
      bool ok = true;
      const uint64_t sf_desc0 = smem_desc(0, 0, 128, kSwizzleNone);
      auto commit_to = [&](uint64_t* bar) {
        if constexpr (PAIR) {
          tc_commit_pair(map_to_rank(smem_u32(bar), 0));
          tc_commit_pair(map_to_rank(smem_u32(bar), 1));
        } else {
          tc_commit(bar);
        }
      };
      auto cp_sf = [&](uint32_t taddr, uint32_t saddr) {
        if constexpr (PAIR) tc_cp_sf_pair(taddr, sf_desc0 | (saddr >> 4));
        else tc_cp_sf(taddr, sf_desc0 | (saddr >> 4));
      };
      for (int t = walk.begin; t < walk.end && ok; t += walk.step, ++local) {
        int mb, nb;
        walk.coords(t, p, mb, nb);
        const bool newrb = mb != cur_mb;
        bool lastrb = true;   // the unit's last tile of this row block: it releases the A panel
        if (t + walk.step < walk.end) {
          int mb2, nb2;
          walk.coords(t + walk.step, p, mb2, nb2);
          lastrb = mb2 != mb;
        }
        if constexpr (RES) {
          if (mb != cur_mb) {
            if (*abort_flag || !mbar_wait(sfa_full, nsfa & 1, p.wait_limit)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t src = smem_u32(smem + C::OFF_SFA_RES);
            for (int kk = 0; kk < p.k_atoms; ++kk) cp_sf(tmem + C::TM_SF + 4 * kk, src + 512 * kk);
            commit_to(sfa_empty);
            cur_mb = mb;
            ++nsfa;
          }
        }
        const int acc = local % C::ACC;
        const uint32_t aph = (local / C::ACC) & 1;
        if (*abort_flag || !mbar_wait(&tempty[acc], aph ^ 1, p.wait_limit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * BN;
        // A 192-wide tile at an odd index starts 64 rows into a scale atom.
        const uint32_t sfb_shift = (BN % 128 != 0 && (nb & 1)) ? 2u : 0u;
        for (int ks = 0; ks < p.num_kst; ++ks, ++it) {
          const int s = it % STAGES;
          if (*abort_flag || !mbar_wait(&full[s], (it / STAGES) & 1, p.wait_limit)) {
            ok = false;
            break;
          }
          if constexpr (APANEL) {
            if (newrb && (*abort_flag || !mbar_wait(&a_full[ks], (nsfa - 1) & 1, p.wait_limit))) {
              ok = false;
              break;
            }
          }
          tc_fence_after();
          const int nk = min(C::KSTEPS, p.k_atoms - C::KSTEPS * ks);
          const uint32_t a_base = APANEL ? smem_u32(smem + C::OFF_A + ks * C::A_CHUNK)
                                         : smem_u32(smem + C::OFF_A + s * C::A_BYTES);
          const uint32_t b_base = smem_u32(smem + C::OFF_B + s * C::B_BYTES);
          const uint32_t sfa_base = smem_u32(smem + C::OFF_SFA + s * C::SFA_BYTES);
          const uint32_t sfb_base = smem_u32(smem + C::OFF_SFB + s * C::SFB_BYTES);
          const uint32_t t_slot = tmem + C::TM_SF + (it % C::SF_SLOTS) * C::SF_COLS;   // streaming
#pragma unroll
          for (int i = 0; i < C::KSTEPS; ++i) {
            if (i >= nk) break;
            uint32_t t_sfa, t_sfb;
            if constexpr (RES) {
              t_sfa = tmem + C::TM_SF + 4 * (C::KSTEPS * ks + i);
              t_sfb = tmem + C::TM_SFB_RES + (gk % C::SFB_SLOTS) * C::SFB_KCOLS;
              ++gk;
            } else {
              t_sfa = t_slot + 4 * i;
              t_sfb = t_slot + 16 + C::SFB_KCOLS * i;
              cp_sf(t_sfa, sfa_base + 512 * i);
            }
#pragma unroll
            for (int r = 0; r < C::NSFB; ++r) cp_sf(t_sfb + 4 * r, sfb_base + C::SFB_GROUP * r + 512 * i);
            const uint32_t koff = 32 * (i & 3);
            const uint64_t adesc = smem_desc(a_base + (i >> 2) * C::A_CHUNK + koff, 0, 1024, kSwizzle128B);
            const uint64_t bdesc = smem_desc(b_base + (i >> 2) * C::B_CHUNK + koff, 0, 1024, kSwizzle128B);
            const uint32_t accum = (ks > 0 || i > 0) ? 1u : 0u;
            if constexpr (PAIR)
              tc_mma_nvf4_pair(d_tmem, adesc, bdesc, C::IDESC, t_sfa, t_sfb + sfb_shift, accum);
            else
              tc_mma_nvf4(d_tmem, adesc, bdesc, C::IDESC, t_sfa, t_sfb + sfb_shift, accum);
          }
          commit_to(&empty[s]);
          if (APANEL && lastrb) commit_to(&a_empty[ks]);
        }
        if (!ok) break;
        commit_to(&tfull[acc]);
      }
      if (!ok) fail_timeout(p.status, abort_flag);
      if constexpr (PAIR) {
        tc_commit_pair(map_to_rank(smem_u32(drain), 0));
        if (!mbar_wait(drain, 0, kDrainLimit)) record_error(p.status, QL_ERR_TIMEOUT);
      } else {
        drain_mma(drain, p.status);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const float alpha = __fmul_rn(__fmul_rn(ld_dep(p.g_a), ld_dep(p.g_w)), p.alpha_mul);
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    uint8_t* stage = smem + C::OFF_C + (warp - 4) * EPI_BUF * kWarpBoxBytes;
    WarpStoreState ws{0};
    int local = 0;
    for (int t = walk.begin; t < walk.end; t += walk.step, ++local) {
      int mb, nb;
      walk.coords(t, p, mb, nb);
      const int acc = local % C::ACC;
      if (!warp_wait_uniform(&tfull[acc], (local / C::ACC) & 1, p.wait_limit, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t release = PAIR ? map_to_rank(smem_u32(&tempty[acc]), 0) : smem_u32(&tempty[acc]);
      const int row0 = mb * C::BM * C::CTAS + static_cast<int>(rank) * C::BM + 32 * quarter;
      const int c_off = half * (BN / 2);
      const uint32_t taddr = tmem + acc * BN + c_off + (static_cast<uint32_t>(32 * quarter) << 16);
      epilogue_warp_tile<C::EPI_CH, EPI_BUF>(taddr, release, stage, &tm_y, row0, nb * BN + c_off, p.M, p.N,
                                             alpha, ws);
    }
    epilogue_warp_finish();
  }

  pdl_release();
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();   // no CTA leaves while its peer may still signal it
  tc_fence_after();
  if (warp == 2) {
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem, 512);
    else
      tmem_dealloc(tmem, 512);
  }
}

// --------------------------------------------------------------------------
// Host side
// --------------------------------------------------------------------------
template <int BN, int STAGES, bool PAIR, int ACC_, int EPI_BUF, bool RES, int BKB_ = 128, bool APANEL = false>
static ql_status launch_w4a4_cfg(const void* a_codes, const uint8_t* a_sf, const float* g_a,
                                 int64_t M, const ql_weights* w, void* Y, cudaStream_t st,
                                 int* status, Gate gate) {
  using C = W4A4Cfg<BN, STAGES, PAIR, ACC_, EPI_BUF, RES, BKB_, APANEL>;
  const int N = w->N, K = w->K;
  if (RES && K / 64 > kResKSteps) return QL_ERR_UNSUPPORTED_SHAPE;
  CUtensorMap ta, tb, tsa, tsb, ty;
  if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, K / 2, M, K / 2, 128, C::BM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, K / 2, N, K / 2, 128, C::BNL,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_sf_tmap(&tsa, a_sf, M, K, RES ? K / 64 : C::KSTEPS) || !make_sf_tmap(&tsb, w->sf, N, K, C::KSTEPS) ||
      !make_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, N, M, static_cast<int64_t>(N) * 2,
                    kWarpBoxCols, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return QL_ERR_CUDA;
  GemmArgs p{};
  fill_gemm_args(p, M, N, K, BN, status);
  p.tiles_m = static_cast<int32_t>((M + C::BM * C::CTAS - 1) / (C::BM * C::CTAS));
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.num_kst = (K + 2 * C::BKB - 1) / (2 * C::BKB);
  p.k_atoms = K / 64;
  p.sfb_atoms = (N + 127) / 128;
  p.g_a = g_a;
  p.g_w = w->gscale;
  p.alpha_mul = w->hadamard ? (1.0f / 128.0f) : 1.0f;
  p.gate = gate.route;
  p.gate_value = gate.value;
  auto kern = k_gemm_w4a4<BN, STAGES, PAIR, ACC_, EPI_BUF, RES, BKB_, APANEL>;
  if (!set_smem_attr(reinterpret_cast<const void*>(kern), C::SMEM)) return QL_ERR_CUDA;
  const int units = std::min(p.num_tiles, num_sms() / C::CTAS);
  if (launch_pdl(kern, dim3(static_cast<unsigned>(units * C::CTAS)), dim3(384), C::SMEM, st, C::CTAS, ta, tb,
                 tsa, tsb, ty, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return QL_OK;
}

ql_status launch_gemm_w4a4(const void* a_codes, const uint8_t* a_sf, const float* g_a, int64_t M,
                           const ql_weights* w, void* Y, cudaStream_t st, int* status, Gate gate) {
  if (M == 0) return QL_OK;
  const bool res = w->K / 64 <= kResKSteps;
  const int64_t N = w->N;
  // 192-wide tiles spend fewer tensor-pipe instructions per output column
  // than 128-wide ones (measured 1.4x on the 5120-column Wan-14B FFN-down);
  // a ragged last tile reads zero weight rows past N (TMA fill, zero scales
  // in the padded scale rows) and stores no column past N.  128-wide tiles
  // remain for N <= 128 and where the last 192-wide tile would waste more
  // than 30% of the columns.
  const int64_t n192 = (N + 191) / 192 * 192, n256 = (N + 255) / 256 * 256;
  const bool wide = N > 128 && 10 * n192 <= 13 * N;
  if (M > 128) {   // CTA pairs on 256-row tiles
    if (res) {
      // K <= 1920: the activation scales of a row block stay in tensor
      // memory while the unit walks the row block's N tiles.  With many N
      // tiles per row block the A tiles stay in shared memory too and only
      // the weights stream (half the L2 reads; measured 4-5% faster on the
      // 5760- and 7680-column linears).  With few, each unit reloads the
      // panel about once per ten tiles and the streamed form is faster.
      const int64_t tiles_n = wide ? n192 / 192 : (N + 127) / 128;
      if (tiles_n >= 16) {
        if (wide)
          return launch_w4a4_cfg<192, 4, true, 2, 1, true, 128, true>(a_codes, a_sf, g_a, M, w, Y, st, status, gate);
        return launch_w4a4_cfg<128, 5, true, 2, 1, true, 128, true>(a_codes, a_sf, g_a, M, w, Y, st, status, gate);
      }
      if (wide) return launch_w4a4_cfg<192, 5, true, 2, 3, true>(a_codes, a_sf, g_a, M, w, Y, st, status, gate);
      return launch_w4a4_cfg<128, 6, true, 2, 2, true>(a_codes, a_sf, g_a, M, w, Y, st, status, gate);
    }
    // Longer K: A and its scales stream with B.  256-wide tiles load the
    // fewest operand bytes per MMA cycle; their single accumulator costs an
    // epilogue bubble per tile that long K amortizes.
    if (N > 192 && 10 * n256 <= 13 * N)
      return launch_w4a4_cfg<256, 5, true, 1, 2, false>(a_codes, a_sf, g_a, M, w, Y, st, status, gate);
    if (wide) return launch_w4a4_cfg<192, 5, true, 2, 3, false>(a_codes, a_sf, g_a, M, w, Y, st, status, gate);
    return launch_w4a4_cfg<128, 6, true, 2, 2, false>(a_codes, a_sf, g_a, M, w, Y, st, status, gate);
  }
  if (wide) {
    if (res) return launch_w4a4_cfg<192, 4, false, 2, 2, true>(a_codes, a_sf, g_a, M, w, Y, st, status, gate);
    return launch_w4a4_cfg<192, 4, false, 2, 2, false>(a_codes, a_sf, g_a, M, w, Y, st, status, gate);
  }
  if (res) return launch_w4a4_cfg<128, 5, false, 2, 2, true>(a_codes, a_sf, g_a, M, w, Y, st, status, gate);
  return launch_w4a4_cfg<128, 5, false, 2, 2, false>(a_codes, a_sf, g_a, M, w, Y, st, status, gate);
}

}  // namespace ql
