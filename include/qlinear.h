/*
 * qlinear.h -- C ABI of the B200 (sm_100a) quantized linear layer.
 *
 * The layer follows two web pages on video-diffusion-transformer
 * quantization:
 *   "6Bit-Diffusion" (gist.science 2603.18742), Methodology B.1 (DMPQ):
 *     an online block Hadamard transform on the activations, activations
 *     routed per transformer block to INT8 (sensitive blocks) or NVFP4
 *     (stable blocks) by the block's input/output relative L1 distance
 *     Gamma, and all weights quantized offline to NVFP4;
 *   "Q-ARVD: Autoregressive Video Diffusion Models의 양자화", Methodology
 *     and Formula/operation flow: outlier input channels found from the
 *     channel L2 norms by a median/MAD modified z-score with threshold tau
 *     and minimum magnitude alpha, separate per-output-channel scales for
 *     the outlier and normal channel classes, per-tensor INT8 activations.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers on the current CUDA device,
 *     allocated and owned by the caller.  The library never allocates device
 *     memory; scratch space is a caller-provided workspace whose size the
 *     matching *_ws_bytes() query returns.  Pointers must be 16-byte aligned
 *     (256-byte for workspaces and weight buffers).
 *   - A workspace must be zero-filled before its first use.  Kernels that
 *     count finished CTAs in it put the counter back to zero, so a workspace
 *     stays usable for later calls on the same stream; two calls in flight
 *     at once need two workspaces.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy stream).
 *     Calls enqueue work and return; they never synchronize, except where a
 *     comment says so.
 *   - Calls return a ql_status and never throw or abort.  Shape and pointer
 *     checks run on the host before anything is enqueued; a failed check
 *     enqueues nothing.
 *   - Matrices are row-major.  X is [M, K] (tokens x in-features), W is
 *     [N, K] (nn.Linear layout), Y = X W^T is [M, N], all bf16.
 *   - K must be a multiple of 128 (the Hadamard block), at most 2^20, and N
 *     a multiple of 16, at most 2^24.  M may be any value from 0 to
 *     2^31 - 128, with ceil(M/128) * K < 2^32 and M * K < 2^37 (the
 *     streaming kernels index 128-element blocks in 32 bits and read the
 *     input as 128-byte rows with 32-bit coordinates) and, for the GEMMs,
 *     ceil(M/128) * ceil(N/128) < 2^31 (output tiles).  A call beyond these
 *     limits returns QL_ERR_UNSUPPORTED_SHAPE.
 *   - Non-finite inputs give unspecified (but memory-safe) results.
 *
 * Data layouts:
 *   NVFP4 codes   uint8 [rows, K/2]; byte j holds element 2j in its low
 *                 nibble and 2j+1 in its high nibble; E2M1 code = sign bit 3,
 *                 magnitude bits 0-2 indexing {0,.5,1,1.5,2,3,4,6}.
 *   NVFP4 scales  one E4M3 byte per 16 elements along K.  "MMA layout":
 *                 rows padded to a multiple of 128 (padding scales are 0);
 *                 512-byte atoms, atom (r/128, j/4) at byte offset
 *                 ((r/128) * (K/64) + j/4) * 512; inside an atom, scale j of
 *                 row r sits at (r%32)*16 + ((r/32)%4)*4 + j%4.
 *                 "Row-major": uint8 [rows, K/16].
 *   Tensor scale  fp32 g = amax(rotated tensor) / 2688 (1 if amax is 0);
 *                 dequantized value = e2m1 * e4m3 * g.
 *   INT8 token    int8 [M, K] and fp32 [M] scales s_m = amax_m / 127.
 */
#ifndef QLINEAR_H
#define QLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QLINEAR_ABI_VERSION 7

#if defined(__GNUC__)
#define QL_API __attribute__((visibility("default")))
#else
#define QL_API
#endif

typedef enum {
  QL_OK = 0,
  QL_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, negative size      */
  QL_ERR_UNSUPPORTED_SHAPE = 2, /* K % 128, N % 16, or a size beyond limits   */
  QL_ERR_ALIGNMENT = 3,         /* pointer not aligned as required            */
  QL_ERR_CUDA = 4,              /* a CUDA runtime call failed                 */
  QL_ERR_TIMEOUT = 5,           /* a device-side wait hit its limit           */
  QL_ERR_WORKSPACE = 6,         /* workspace or buffer smaller than required  */
  QL_ERR_NO_DEVICE = 7          /* no usable sm_100 device                    */
} ql_status;

/* Weight formats. */
typedef enum {
  QL_W_NVFP4 = 0,       /* NVFP4 (E2M1 + E4M3/16 + fp32), optional Hadamard  */
  QL_W_QARVD_INT4 = 2,  /* Q-ARVD dual-scale signed INT4, K permuted         */
  QL_W_NVFP4_DECOMP = 3 /* NVFP4 repeated along K for decomposed activations:
                           codes [N, K] bytes = [c | c] per row, scales over
                           2K; pairs only with QL_ACT_NVFP4_DECOMP           */
} ql_weight_format;

/* Activation routes / formats. */
typedef enum {
  QL_ROUTE_NVFP4 = 0,       /* W4A4: NVFP4 activations                       */
  QL_ROUTE_INT8 = 1,        /* W4A8: per-token INT8 activations              */
  QL_ACT_INT8_TENSOR = 2,   /* Q-ARVD: per-tensor INT8, permuted K           */
  QL_ACT_INT8_F16 = 3,      /* W4A8: per-token INT8 codes stored as the equal
                               f16 values, f16 [M, K] (the operand type of
                               the f16 MMA)                                  */
  QL_ACT_NVFP4_DECOMP = 4,  /* activation decomposition (SemanticDialect,
                               Methodology 2.2): NVFP4 of h, then NVFP4 of the
                               residual r = RN(h - RN(e2m1(q1) RN(sb1 g))) with
                               the same tensor scale g; codes [M, K] bytes =
                               [q1 | q2] per row, scales over K' = 2K (q1's
                               first); the GEMM needs QL_W_NVFP4_DECOMP      */
  /* W4A6: 6-bit signed integer activations, symmetric [-31, 31], the INT8
     recipes with 31 in place of 127, in 8-bit (or f16) containers that the
     integer GEMMs multiply exactly. */
  QL_ROUTE_INT6 = 5,        /* per-token INT6 (int8 [M, K] + fp32 [M]); also
                               a qlinear_forward route                        */
  QL_ACT_INT6_F16 = 6,      /* per-token INT6 codes as f16 values           */
  QL_ACT_INT6_TENSOR = 7,   /* Q-ARVD per-tensor INT6 in the permuted K order  */
  QL_ROUTE_BF16 = 8         /* unquantized bf16 product X W^T (PDR's
                               high-precision refresh); the activations are
                               the bf16 input itself; needs weights prepared
                               with keep_bf16                                 */
} ql_act_format;

typedef struct {
  int32_t fmt;       /* ql_weight_format                                       */
  int32_t hadamard;  /* NVFP4: 1 = rotate K by blockdiag(H_128) (must match the
                        activations' setting); Q-ARVD: must be 0              */
  float tau;         /* Q-ARVD modified z-score threshold (3.5)                */
  float alpha;       /* Q-ARVD minimum magnitude factor (2.0)                  */
  int32_t expand_f16;/* NVFP4: 1 = also keep an f16 copy of the dequantized
                        weights (E2M1 x E4M3, without g_w; exact in f16) for
                        the INT8 route's GEMM, which then reads it directly
                        instead of expanding the FP4 codes on chip.  Costs
                        2 bytes per weight in the weight buffer.              */
  int32_t expand_i8; /* Q-ARVD: 1 = also keep the INT4 codes sign-extended to
                        int8 ([N, Kp], exact) for the GEMM, which then loads
                        both operands by TMA instead of widening the weights
                        on chip.  Costs 1 byte per code in the weight buffer. */
  int32_t keep_bf16; /* NVFP4: 1 = also keep the bf16 weights [N, K] for the
                        QL_ROUTE_BF16 product.  2 bytes per weight.          */
  int32_t reserved;  /* 0                                                      */
} ql_weight_cfg;

/* Packed weights.  Filled by qlinear_prepare_weights(); every pointer points
   into the caller's weight buffer.  Treat as read-only. */
typedef struct {
  int32_t fmt, N, K, hadamard;
  int32_t Kp;            /* Q-ARVD: padded permuted K of codes/activations     */
  int32_t reserved0;
  void* codes;           /* NVFP4 [N, K/2]; Q-ARVD INT4 nibbles [N, Kp/2]       */
  void* sf;              /* NVFP4 block scales, MMA layout                      */
  float* gscale;         /* NVFP4 fp32 tensor scale g_w (1 value)               */
  uint8_t* outlier_mask; /* Q-ARVD [K], 1 = outlier channel                     */
  int32_t* perm;         /* Q-ARVD [K] channels in class order                  */
  int32_t* gather;       /* Q-ARVD [Kp] source channel of each slot, -1 = pad   */
  int32_t* kinfo;        /* Q-ARVD [4] k_norm, k_norm_pad, n_out, k_out_pad     */
  float* s_norm;         /* Q-ARVD [N] scale of the normal channels             */
  float* s_out;          /* Q-ARVD [N] scale of the outlier channels            */
  double* norms;         /* Q-ARVD [K] input-channel L2 norms                   */
  void* w16;             /* NVFP4 with expand_f16: f16 [N, K] = E2M1 x E4M3
                            (no g_w); NULL otherwise                            */
  void* w8;              /* Q-ARVD with expand_i8: int8 [N, Kp] = the INT4
                            codes sign-extended; NULL otherwise                 */
  void* wbf16;           /* NVFP4 with keep_bf16: the bf16 weights [N, K] as
                            given (not rotated); NULL otherwise                 */
} ql_weights;

/* ---- library ------------------------------------------------------------ */

QL_API int qlinear_abi_version(void);
QL_API const char* qlinear_status_string(int status);

/* Reads and clears the device status word of the current device, which the
   kernels set when a bounded wait times out (QL_ERR_TIMEOUT) .  Synchronizes
   `stream` first.  *status_out receives QL_OK or the first error recorded. */
QL_API ql_status qlinear_device_status(void* stream, int32_t* status_out);

/* Test hook: the cycle budget of every pipeline wait in the GEMM kernels
   (default about one second).  0 makes the first wait that is not already
   satisfied time out, so a test can exercise the timeout path; the kernel
   then drains its in-flight copies with a separate, generous budget and
   returns.  Negative restores the default.  Host-global, not thread-safe. */
QL_API void qlinear_debug_set_wait_limit(long long cycles);

/* Test hook: adds to *mismatches_dev (device, 8-byte aligned) the number of
   dividends a with fp32 bit patterns a_begin .. a_begin + count - 1 (must
   stay non-negative and finite) for which the NVFP4 quantizer's block-scale
   division by d differs from the correctly rounded a / d. */
QL_API ql_status qlinear_debug_div_check(float d, uint32_t a_begin, uint64_t count,
                                         unsigned long long* mismatches_dev, void* stream);

/* ---- sizes ---------------------------------------------------------------- */

/* Bytes of NVFP4 block scales in the MMA layout for a [rows, K] tensor. */
QL_API size_t qlinear_sf_bytes(int64_t rows, int32_t K);

/* ---- weights: offline preparation ----------------------------------------
   NVFP4 (6Bit-Diffusion, Methodology B.1): W -> (Hadamard) -> NVFP4 with a
   tensor scale from amax of the rotated W.
   Q-ARVD (Q-ARVD, Methodology / Formula and operation flow): channel norms,
   median/MAD z-score mask, class-ordered permutation, per-row dual INT4
   scales, INT4 codes.  The weight buffer (qlinear_weights_bytes) holds every
   output; `ws` is scratch (qlinear_prepare_ws_bytes).  Asynchronous.
   Q-ARVD weights need hadamard = 0, tau > 0, alpha >= 0 and K <= 16384 (one
   CTA sorts all channel norms in shared memory); otherwise the call returns
   QL_ERR_INVALID_ARG.  The per-tensor Q-ARVD activation quantizer stages a
   row in shared memory and returns QL_ERR_UNSUPPORTED_SHAPE when that does
   not fit (about K > 22000). */
QL_API size_t qlinear_weights_bytes(int32_t N, int32_t K, const ql_weight_cfg* cfg);
QL_API size_t qlinear_prepare_ws_bytes(int32_t N, int32_t K, const ql_weight_cfg* cfg);
QL_API ql_status qlinear_prepare_weights(const void* W_bf16, int32_t N, int32_t K,
                                  const ql_weight_cfg* cfg,
                                  void* wbuf, size_t wbuf_bytes, ql_weights* out,
                                  void* ws, size_t ws_bytes, void* stream);

/* ---- DMPQ router (6Bit-Diffusion, Methodology A.1 and B.1) ----------------
   Gamma = sum|out - in| / sum|in| over `numel` bf16 elements (fp32
   differences, fp64 sums); *route_dev = 1 (INT8) if Gamma > threshold else
   0 (NVFP4); Gamma = +inf (route INT8) when sum|in| is 0.  gamma_dev and
   route_dev are device pointers. */
QL_API size_t qlinear_route_ws_bytes(int64_t numel);
QL_API ql_status qlinear_route(const void* in_bf16, const void* out_bf16, int64_t numel,
                        float threshold, double* gamma_dev, int32_t* route_dev,
                        void* ws, size_t ws_bytes, void* stream);

/* ---- router with the block's tokens split across ranks -----------------------
   The same Gamma when each rank holds some rows of the block: each rank
   calls qlinear_gamma_sums on its own rows, the ranks add the two sums
   (one all-reduce of 2 doubles), and each calls qlinear_route_from_sums.
   Only the order of the fp64 additions differs from qlinear_route on the
   whole block.
   qlinear_gamma_sums: sums_dev[0] = sum|out - in|, sums_dev[1] = sum|in|
   over this rank's numel elements (fp64, device, 8-byte aligned).  ws as
   for qlinear_route (qlinear_route_ws_bytes(numel) bytes, 256-byte aligned,
   zero-filled before its first use; calls sharing one must not overlap).
   qlinear_route_from_sums: *gamma_dev = sums_dev[0] / sums_dev[1] (+inf
   when sums_dev[1] is 0), *route_dev = 1 (INT8) if Gamma > threshold. */
QL_API ql_status qlinear_gamma_sums(const void* in_bf16, const void* out_bf16, int64_t numel,
                                    double* sums_dev, void* ws, size_t ws_bytes, void* stream);
QL_API ql_status qlinear_route_from_sums(const double* sums_dev, float threshold, double* gamma_dev,
                                         int32_t* route_dev, void* stream);

/* ---- router without a workspace (no counterpart on the pages) --------------
   Same Gamma and route as qlinear_route, for callers that cannot allocate
   device memory or hand over a workspace: code that runs where another
   component owns every device allocation (an inference engine or plugin host
   with its own memory pool and budget), or a latency-critical loop that must
   not call cudaMalloc, which can block and synchronize the device.  The
   caller still passes the inputs and the two outputs.
   Scratch: a file-scope device array of 16640 bytes (fp64 partial sums of
   up to 1024 CTAs plus a finished-CTA counter); every GPU that loads this
   library holds it until the process exits.  The first call on a device
   looks up the array's device address with cudaGetSymbolAddress and caches
   it, so make that first call before any stream capture.  All calls share
   the one array and it keeps the last call's contents; each call zeroes the
   counter before its kernel runs.  Calls that overlap on the GPU (two
   streams, two host threads) race on the array: serialize them.  A call
   that would need more than 1024 CTAs of scratch returns
   QL_ERR_UNSUPPORTED_SHAPE (on a 148-SM B200 the grid is at most 592). */
QL_API ql_status qlinear_route_noalloc(const void* in_bf16, const void* out_bf16, int64_t numel,
                                       float threshold, double* gamma_dev, int32_t* route_dev,
                                       void* stream);

/* ---- tensor amax ------------------------------------------------------------
   *amax_out (device fp32) = max |H x| over the whole [M, K] tensor (|x| when
   hadamard is 0): the input of the dynamic NVFP4 tensor scale
   g = amax / (6 * 448) and of the per-tensor INT8 / INT6 scale amax / 127
   (amax / 31).  One launch; ws needs qlinear_quantize_ws_bytes(M, K,
   QL_ROUTE_NVFP4) bytes. */
QL_API ql_status qlinear_tensor_amax(const void* X_bf16, int64_t M, int32_t K, int32_t hadamard,
                                     float* amax_out, void* ws, size_t ws_bytes, void* stream);

/* ---- activation quantization (inspection entry point) ---------------------
   QL_ROUTE_NVFP4:     codes uint8 [M, K/2]; sf_mma (MMA layout, required);
                       sf_rowmajor [M, K/16] (optional, may be NULL);
                       scales = fp32[1] tensor scale g_x.
   QL_ROUTE_INT8:      codes int8 [M, K]; scales = fp32 [M]; sf_* unused.
   QL_ACT_INT8_F16:    as QL_ROUTE_INT8, codes f16 [M, K] (exact integers).
   QL_ACT_INT8_TENSOR: needs Q-ARVD weights `w`; codes int8 [M, w->Kp] in the
                       weights' channel order with zero padding; scales =
                       fp32[1]; hadamard must be 0.
   QL_ACT_NVFP4_DECOMP: codes uint8 [M, K] = [q1 | q2] per row; sf_mma over
                       2K (q1's scales first, required); sf_rowmajor [M, K/8]
                       (optional); scales = fp32[1] tensor scale g_x.
   QL_ROUTE_INT6, QL_ACT_INT6_F16, QL_ACT_INT6_TENSOR: as the INT8 formats,
                       codes in [-31, 31], scales amax / 31.
   `hadamard` = 1 rotates each 128-block of K first (NVFP4 / INT8 routes).
   amax_in: optional device fp32 tensor amax (NVFP4 and per-tensor INT8),
   e.g. from qlinear_tensor_amax or a calibrated static value; NULL makes the
   call compute the dynamic amax itself (one extra launch).
   The per-token formats keep two token rows per warp in shared memory:
   K > 51200 returns QL_ERR_UNSUPPORTED_SHAPE there (and on the INT8 / INT6
   routes of qlinear_forward). */
QL_API size_t qlinear_quantize_ws_bytes(int64_t M, int32_t K, int32_t act_fmt);
QL_API ql_status qlinear_quantize_act(const void* X_bf16, int64_t M, int32_t K,
                                      int32_t act_fmt, int32_t hadamard, const ql_weights* w,
                                      const float* amax_in, void* codes, void* sf_mma,
                                      void* sf_rowmajor, float* scales,
                                      void* ws, size_t ws_bytes, void* stream);

/* ---- GEMM on quantized activations ----------------------------------------
   Y[m, n] = bf16(alpha_m * sum_k a[m,k] w[n,k]) with fp32 accumulation:
   QL_ROUTE_NVFP4:     tcgen05 block-scaled FP4 MMA; alpha = g_x g_w / 128 if
                       the weights are rotated, else g_x g_w.
   QL_ROUTE_INT8:      INT8 x NVFP4 weights (their f16 copy when prepared with
                       expand_f16, else expanded on chip to f16);
                       alpha_m = s_m g_w (/128 if rotated).
   QL_ACT_INT8_F16:    as QL_ROUTE_INT8 with f16 codes: with the f16 copy both
                       operands go straight to the f16 MMA; without it the
                       FP4 weights are widened into tensor memory and fed to
                       the MMA from there (same results).
   QL_ACT_INT8_TENSOR: INT8 x INT4 integer MMA, two class accumulators;
                       y = s_x (s_norm[n] acc_normal + s_out[n] acc_outlier).
   QL_ACT_NVFP4_DECOMP: the W4A4 GEMM over K' = 2K ([q1 | q2] x [W | W]).
   QL_ROUTE_INT6, QL_ACT_INT6_F16, QL_ACT_INT6_TENSOR: as the INT8 formats
                       (the codes are integers in [-31, 31]).
   Operands are the outputs of qlinear_quantize_act for the same format. */
QL_API ql_status qlinear_gemm(int32_t act_fmt, const void* a_codes, const void* a_sf,
                       const float* a_scales, int64_t M, const ql_weights* w,
                       void* Y_bf16, void* stream);

/* ---- forward: quantize + GEMM ----------------------------------------------
   route: QL_ROUTE_NVFP4, QL_ROUTE_INT8 or QL_ROUTE_INT6 for NVFP4 weights
   (the activation rotation follows w->hadamard); for Q-ARVD weights
   QL_ROUTE_INT6 or QL_ACT_INT6_TENSOR selects per-tensor INT6 activations,
   any other value per-tensor INT8; QL_ROUTE_NVFP4 only for
   QL_W_NVFP4_DECOMP weights.  Scratch for the quantized activations lives
   in `ws`.  On the INT8 route the codes are kept as the equal f16 values
   (2 bytes each, QL_ACT_INT8_F16), the f16 MMA's operand type. */
QL_API size_t qlinear_forward_ws_bytes(int64_t M, const ql_weights* w, int32_t route);
QL_API ql_status qlinear_forward(const void* X_bf16, int64_t M, const ql_weights* w,
                          int32_t route, void* Y_bf16,
                          void* ws, size_t ws_bytes, void* stream);

/* ---- forward with the route in device memory ----------------------------
   DMPQ routes a block from the previous step's Gamma, which the router (or
   a TDC state's next_route) leaves in device memory.  This forward enqueues
   the kernels of every route the weights support -- NVFP4, INT8 (f16-coded)
   and, with keep_bf16, BF16 -- and each kernel
   waits for its predecessor, reads *route_dev and returns at once unless
   the route is its own.  So the call never synchronizes with the host and
   a whole step can be captured in one CUDA graph.  Weights: QL_W_NVFP4.
   route_dev: device int32, 4-byte aligned, written earlier in the same
   stream; a value no enqueued route has leaves Y unwritten.  ws:
   qlinear_forward_routed_ws_bytes bytes, 256-byte aligned. */
QL_API size_t qlinear_forward_routed_ws_bytes(int64_t M, const ql_weights* w);
QL_API ql_status qlinear_forward_routed(const void* X_bf16, int64_t M, const ql_weights* w,
                                        const int32_t* route_dev, void* Y_bf16, void* ws,
                                        size_t ws_bytes, void* stream);

/* ---- temporal delta cache ------------------------------------------------
   "6Bit-Diffusion", Methodology A.2 / B.2 (TDC) and B.3 (PDR).  A block's
   residual delta D = bf16(out - in) changes little between adjacent
   timesteps; a block whose last two computed deltas are close is skipped
   and reuses the latest delta.  The caller owns, per transformer block, two
   bf16 delta slots of the block's activation size and one ql_tdc_state in
   device memory.  Each step it reads next_skip (and next_route) from the
   state -- written by the previous step's kernel -- and either computes
   the block and calls qlinear_tdc_refresh, or calls qlinear_tdc_skip.

   Definitions (fp32 differences of bf16 values, RN; fp64 sums):
     Gamma = sum |out - in| / sum |in|                  (+inf if sum |in| = 0)
     E     = sum |D_new - D_prev| / sum |D_prev|        (+inf with < 2 deltas
                                                          or sum |D_prev| = 0)
     skip next   iff n_delta == 2, E < eps_threshold, acc + E <= acc_max and
                 skips < max_skips  (acc sums E over the current run of skips)
     next_route  BF16 if the last refresh saw rho > rho_max; else INT8 if
                 the step just taken was a skip or Gamma > gamma_threshold
                 (strict), else NVFP4; INT8 before any Gamma.
     rho         (PDR) fraction of the input's whole 16-element blocks whose
                 largest magnitude a exceeds kappa times the mean of the
                 other 15: RN(a 15) > RN(kappa RN(s - a)), s the fp32 sum
                 of |x| (two sequential halves of 8, then their sum).       */
typedef struct {
  double gamma;          /* Gamma of the last computed step                   */
  double eps;            /* E between the two cached deltas                   */
  double acc;            /* summed E over the current run of skips            */
  double rho;            /* outlier-block ratio of the last refreshed input   */
  int32_t n_delta;       /* cached deltas, 0..2                               */
  int32_t cur;           /* slot (0 or 1) holding the latest delta            */
  int32_t skips;         /* consecutive skips so far                          */
  int32_t last_skipped;  /* 1 when the last step was a skip                   */
  int32_t next_skip;     /* decision for the next step: 1 = skip              */
  int32_t next_route;    /* QL_ROUTE_* of the next step if it is computed     */
  int32_t steps;         /* steps taken since qlinear_tdc_init                */
  int32_t reserved;
} ql_tdc_state;

typedef struct {
  float gamma_threshold; /* DMPQ route threshold (0.05)                       */
  float eps_threshold;   /* skip while E is below this                        */
  float acc_max;         /* cap on the summed E of one run of skips           */
  int32_t max_skips;     /* cap on consecutive skips (>= 0)                   */
  float kappa;           /* outlier block: largest magnitude > kappa x mean of
                            the rest (8)                                       */
  float rho_max;         /* BF16 when rho exceeds this (>= 1: never)           */
} ql_tdc_params;
/* A NaN in any float field of ql_tdc_params, or max_skips < 0, makes the
   TDC calls return QL_ERR_INVALID_ARG before any CUDA call. */

/* Reset a block's cache state (device pointer, 8-byte aligned): no deltas,
   Gamma = E = +inf, next step computed on the INT8 route. */
QL_API ql_status qlinear_tdc_init(ql_tdc_state* state_dev, void* stream);
QL_API size_t qlinear_tdc_ws_bytes(int64_t numel);
/* After computing the block: one pass over in, out [numel] bf16 and the
   latest delta; writes D_new = bf16(RN(out - in)) into the other slot, then
   Gamma, E, the state and the next decision.  delta0/delta1: the block's two
   slots (bf16 [numel] each, 16-byte aligned).  ws: zero-filled before first
   use, qlinear_tdc_ws_bytes(numel) bytes, 256-byte aligned; calls that share
   a workspace must not overlap on the GPU. */
QL_API ql_status qlinear_tdc_refresh(const void* in_bf16, const void* out_bf16, int64_t numel,
                                     void* delta0, void* delta1, ql_tdc_state* state_dev,
                                     const ql_tdc_params* params, void* ws, size_t ws_bytes,
                                     void* stream);
/* Skip the block: out = bf16(RN(in + D_latest)), then acc += E, skips += 1
   and the next decision (route INT8).  Skipping with no cached delta writes
   nothing and records QL_ERR_INVALID_ARG in the device status word. */
QL_API ql_status qlinear_tdc_skip(const void* in_bf16, int64_t numel, const void* delta0,
                                  const void* delta1, ql_tdc_state* state_dev,
                                  const ql_tdc_params* params, void* out_bf16, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* QLINEAR_H */
