"""Plain CPU oracle for the quantized linear layer (TEST INFRASTRUCTURE ONLY).

This module is the slow, obviously-correct restatement of what the GPU path
computes.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import it; the product path never does, and it shares no
code, table or helper with the CUDA library.

Sources (web pages, cited by title and section):
  * "6Bit-Diffusion" (gist.science 2603.18742), Methodology, B.1 DMPQ:
    routed activations (INT8 for sensitive blocks, NVFP4 otherwise), all
    weights offline in NVFP4, an online block Hadamard transform against
    outliers, and the block input/output relative L1 distance Gamma that
    drives the route.
  * "Q-ARVD: Autoregressive Video Diffusion Models의 양자화", Methodology,
    Formula/operation flow and Technical details: channel L2 norms, the
    median/MAD modified z-score M_i = (v_i - median)/MAD, the threshold tau
    and the minimum-magnitude factor alpha, Q_dual(W) = [Q_outlier | Q_normal],
    per-channel weights and per-tensor activations.
  * Number formats (the pages only name NVFP4): E2M1 and E4M3 as defined by
    the OCP Microscaling Formats specification; NVFP4 = E2M1 values with one
    E4M3 scale per 16 contiguous elements and one fp32 tensor scale.

Arithmetic conventions (readings of points the pages leave open):
  * every "RN" below is IEEE binary32 round-to-nearest-even; numpy float32
    ufuncs give exactly that, with no fused multiply-add;
  * reductions that only take a max are exact; sums that feed Gamma and the
    channel norms are fp64;
  * the GEMM reference is an fp64 product of dequantized values.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, format definitions, library routines or brute force.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32
HADAMARD_N = 128          # block size of the online rotation
NVFP4_BLOCK = 16          # elements per E4M3 block scale
E2M1_MAX = 6.0
E4M3_MAX = 448.0
INT8_QMAX = 127
INT4_QMAX = 7
QARVD_K_ALIGN = 32        # each Q-ARVD channel class is zero-padded to this


# ---------------------------------------------------------------------------
# Number formats (OCP MX definitions).  Both encoders are "nearest grid value,
# ties to the even code, clamp to the largest finite value".
# ---------------------------------------------------------------------------

def e2m1_magnitudes() -> np.ndarray:
    """Magnitudes of the eight E2M1 codes 0..7 (1 sign, 2 exponent bits with
    bias 1, 1 mantissa bit; exponent field 0 is subnormal)."""
    vals = []
    for code in range(8):
        e, m = code >> 1, code & 1
        if e == 0:
            vals.append(m * 0.5)
        else:
            vals.append((1.0 + m / 2.0) * 2.0 ** (e - 1))
    return np.array(vals, dtype=np.float64)


def e4m3_magnitudes() -> np.ndarray:
    """Magnitudes of E4M3 codes 0..126 (bias 7, 3 mantissa bits, exponent
    field 0 subnormal, code 127 = NaN and therefore excluded)."""
    vals = []
    for code in range(127):
        e, m = code >> 3, code & 7
        if e == 0:
            vals.append(m / 8.0 * 2.0 ** -6)
        else:
            vals.append((1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals, dtype=np.float64)


def _nearest_code_ties_even(mag: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the grid value nearest to each |x|; on an exact tie the even
    index wins; values beyond the last grid point clamp to it."""
    mag = np.asarray(mag, dtype=np.float64)
    hi = np.searchsorted(grid, mag, side="left")          # grid[hi-1] < mag <= grid[hi]
    hi = np.clip(hi, 0, len(grid) - 1)
    lo = np.clip(hi - 1, 0, len(grid) - 1)
    d_lo = np.abs(mag - grid[lo])
    d_hi = np.abs(grid[hi] - mag)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(mag >= grid[-1], len(grid) - 1, idx)
    return idx.astype(np.int64)


def e4m3_encode(x) -> np.ndarray:
    """Non-negative fp32 -> E4M3 code (uint8), RN-even, saturating at 448.
    Block scales are never negative, so the sign bit is always 0."""
    x = np.asarray(x, dtype=np.float32)
    if np.any(x < 0) or np.any(~np.isfinite(x)):
        raise ValueError("E4M3 scale inputs must be finite and >= 0")
    return _nearest_code_ties_even(x.astype(np.float64), e4m3_magnitudes()).astype(np.uint8)


def e4m3_decode(code) -> np.ndarray:
    code = np.asarray(code, dtype=np.int64)
    return e4m3_magnitudes()[code & 0x7F].astype(np.float32)


def e2m1_encode(y) -> np.ndarray:
    """fp32 -> 4-bit E2M1 code (uint8 0..15): bit 3 is the sign of y (so -0.0
    and small negatives give 0x8), bits 0-2 the nearest magnitude code with
    ties to even, |y| > 6 saturating to 6."""
    y = np.asarray(y, dtype=np.float32)
    mag_code = _nearest_code_ties_even(np.abs(y).astype(np.float64), e2m1_magnitudes())
    sign = np.signbit(y).astype(np.int64)
    return (mag_code | (sign << 3)).astype(np.uint8)


def e2m1_decode(code) -> np.ndarray:
    code = np.asarray(code, dtype=np.int64)
    mag = e2m1_magnitudes()[code & 7]
    return np.where(code & 8, -mag, mag)


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[R, K] 4-bit codes -> [R, K/2] bytes; even column in the low nibble."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def bf16_bits_to_f32(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> the exactly equal fp32 values."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------
# a1: online block Hadamard (6Bit-Diffusion, Methodology B.1).  Sylvester
# matrix in natural order, +-1 entries, no normalisation; the rotation is
# undone by the 1/128 folded into the GEMM scale because weights receive the
# same rotation and H H^T = 128 I.
# ---------------------------------------------------------------------------

def sylvester_hadamard(n: int) -> np.ndarray:
    """H[i, j] = (-1)^popcount(i & j), the natural-order Sylvester matrix."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    bits = np.bitwise_and(i, j)
    pop = np.zeros_like(bits)
    while np.any(bits):
        pop += bits & 1
        bits >>= 1
    return np.where(pop % 2 == 0, 1, -1).astype(np.int64)


def block_hadamard(x32: np.ndarray) -> np.ndarray:
    """Rotate each contiguous 128-element block of every row by H_128.

    Fast Walsh-Hadamard butterflies in fp32, stage distances 1, 2, 4, ..., 64
    in that order; each pair (i, i+s) with bit s of i clear becomes
    (RN(a + b), RN(a - b)).  The result equals x @ H in exact arithmetic."""
    x32 = np.asarray(x32, dtype=np.float32)
    rows, k = x32.shape
    if k % HADAMARD_N:
        raise ValueError("K must be a multiple of 128 for the block Hadamard")
    h = x32.reshape(rows, k // HADAMARD_N, HADAMARD_N).copy()
    s = 1
    while s < HADAMARD_N:
        v = h.reshape(rows, k // HADAMARD_N, HADAMARD_N // (2 * s), 2, s)
        a = v[:, :, :, 0, :].copy()
        b = v[:, :, :, 1, :].copy()
        v[:, :, :, 0, :] = a + b
        v[:, :, :, 1, :] = a - b
        s *= 2
    return h.reshape(rows, k)


# ---------------------------------------------------------------------------
# a2 + a3 (+ a6 for weights): NVFP4 quantisation with a dynamic fp32 tensor
# scale (6Bit-Diffusion, Methodology B.1: NVFP4 for stable blocks and for all
# weights).  Two-level recipe: g = amax / (6 * 448); per 16-element block an
# E4M3 scale sb ~ amax_b / (6 g); codes = E2M1(h / (sb g)).
# ---------------------------------------------------------------------------

def nvfp4_tensor_scale(h: np.ndarray) -> np.float32:
    a_t = np.float32(np.max(np.abs(h))) if h.size else np.float32(0)
    if a_t == 0:
        return np.float32(1.0)
    return np.float32(a_t / np.float32(E2M1_MAX * E4M3_MAX))


def nvfp4_quantize(h: np.ndarray, g: np.float32 | None = None):
    """h: fp32 [R, K] (K % 16 == 0).  Returns (packed codes uint8 [R, K/2],
    block scales uint8 [R, K/16] row-major, tensor scale g as np.float32)."""
    h = np.asarray(h, dtype=np.float32)
    rows, k = h.shape
    if k % NVFP4_BLOCK:
        raise ValueError("K must be a multiple of 16")
    g = nvfp4_tensor_scale(h) if g is None else np.float32(g)
    blocks = h.reshape(rows, k // NVFP4_BLOCK, NVFP4_BLOCK)
    a_b = np.max(np.abs(blocks), axis=2)                       # exact
    d = np.float32(np.float32(E2M1_MAX) * g)                    # RN(6 g)
    sf = (a_b / d).astype(np.float32)                           # RN(a_b / d)
    sb = e4m3_encode(sf)
    denom = (e4m3_decode(sb) * g).astype(np.float32)            # RN(sb * g)
    nz = sb != 0
    inv = np.zeros_like(denom)
    inv[nz] = np.float32(1.0) / denom[nz]                       # RN(1 / (sb g))
    y = (blocks * inv[:, :, None]).astype(np.float32)           # RN(h * inv)
    q = e2m1_encode(y)
    q[~nz] = 0                                                  # all-zero block -> +0 codes
    return pack_nibbles(q.reshape(rows, k)), sb, g


def nvfp4_dequantize(packed: np.ndarray, sb: np.ndarray) -> np.ndarray:
    """fp64 [R, K] = e2m1 value * E4M3 block scale (tensor scale excluded)."""
    q = unpack_nibbles(packed)
    rows, k = q.shape
    vals = e2m1_decode(q).reshape(rows, k // NVFP4_BLOCK, NVFP4_BLOCK)
    scales = e4m3_decode(sb).astype(np.float64)
    return (vals * scales[:, :, None]).reshape(rows, k)


# ---------------------------------------------------------------------------
# Activation decomposition (SemanticDialect, Methodology 2.2 "Activation
# Decomposition": the activation is quantized, the quantization error -- the
# residual -- is quantized again, and its product is added to the output).
# Readings of what the page leaves open:
#   * both parts are NVFP4 with the SAME fp32 tensor scale g (the tensor
#     amax of h); the residual's own 16-element E4M3 block scales follow its
#     smaller magnitude.  With one g the layer's product is one contraction
#     over the K-concatenated pair [q1 | q2] against [W | W];
#   * the residual is taken against the value the GEMM multiplies:
#     v1 = RN(e2m1(q1) * RN(E4M3(sb1) * g)), r = RN(h - v1);
#   * every token is decomposed (the page's attention-based salient-token
#     selection needs attention maps and is not part of this layer).
# ---------------------------------------------------------------------------

def nvfp4_values(packed: np.ndarray, sb: np.ndarray, g) -> np.ndarray:
    """fp32 [R, K]: RN(e2m1 value * RN(E4M3 block scale * g)) per element."""
    q = unpack_nibbles(packed)
    rows, k = q.shape
    s = (e4m3_decode(sb) * np.float32(g)).astype(np.float32)            # RN(sb * g)
    v = e2m1_decode(q).astype(np.float32).reshape(rows, k // NVFP4_BLOCK, NVFP4_BLOCK)
    return (v * s[:, :, None]).astype(np.float32).reshape(rows, k)      # RN(value * s)


def nvfp4_decompose(h: np.ndarray, g: np.float32 | None = None):
    """h: fp32 [R, K].  Returns (packed uint8 [R, K] = [q1 (K/2 bytes) | q2
    (K/2 bytes)], block scales uint8 [R, K/8] = [sb1 | sb2], g)."""
    h = np.asarray(h, dtype=np.float32)
    g = nvfp4_tensor_scale(h) if g is None else np.float32(g)
    p1, s1, g = nvfp4_quantize(h, g)
    r = (h - nvfp4_values(p1, s1, g)).astype(np.float32)               # RN(h - v1)
    p2, s2, _ = nvfp4_quantize(r, g)
    return np.concatenate([p1, p2], axis=1), np.concatenate([s1, s2], axis=1), g


def decompose_weights(wq: dict) -> dict:
    """NVFP4 weights repeated along K ([W | W]) to pair with decomposed activations."""
    return dict(packed=np.concatenate([wq["packed"], wq["packed"]], axis=1),
                sb=np.concatenate([wq["sb"], wq["sb"]], axis=1), g=wq["g"])


# ---------------------------------------------------------------------------
# a4: per-token INT8 (6Bit-Diffusion, Methodology B.1: INT8 for the blocks the
# router marks sensitive; per-token granularity and symmetric +-127 range
# are readings).  a10 activations: per-tensor INT8 (Q-ARVD, Technical
# details: per-tensor activation quantisation).
# ---------------------------------------------------------------------------

def _int8_from_amax(x: np.ndarray, amax: np.ndarray, qmax: int = INT8_QMAX):
    """Symmetric integer codes in [-qmax, qmax] (int8 containers): scale =
    RN(amax / qmax), q = clamp(rint(RN(x * RN(qmax / amax)))), 0 where amax = 0."""
    amax = np.asarray(amax, dtype=np.float32)
    nz = amax != 0
    scale = np.where(nz, (amax / np.float32(qmax)).astype(np.float32), np.float32(0))
    inv = np.zeros_like(amax)
    inv[nz] = np.float32(qmax) / amax[nz]                       # RN(qmax / amax)
    y = (x * inv).astype(np.float32)                            # RN(x * inv)
    q = np.clip(np.rint(y), -qmax, qmax).astype(np.int8)        # ties to even
    return q, scale.astype(np.float32)


def int8_per_token(h: np.ndarray, qmax: int = INT8_QMAX):
    """h: fp32 [R, K] -> (int8 [R, K], fp32 [R] scales s_m = amax_m / qmax)."""
    h = np.asarray(h, dtype=np.float32)
    amax = np.max(np.abs(h), axis=1) if h.shape[1] else np.zeros(h.shape[0], np.float32)
    q, s = _int8_from_amax(h, amax[:, None], qmax)
    return q, s[:, 0]


def int8_per_tensor(x: np.ndarray, qmax: int = INT8_QMAX):
    """x: fp32 [R, K] -> (int8 [R, K], fp32 scale s = amax / qmax)."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    q, s = _int8_from_amax(x, np.array([[amax]], dtype=np.float32), qmax)
    return q, np.float32(s[0, 0])


# W4A6 (S2Q-VDiT and Q-ARVD report W4A6 results; 6Bit-Diffusion's average
# activation width is about 6 bits).  Reading: 6-bit signed integer
# activations, symmetric [-31, 31], the same per-token / per-tensor recipes
# as INT8 with 31 in place of 127, carried in int8 containers so the exact
# integer products of the existing GEMMs apply unchanged.
INT6_QMAX = 31


# ---------------------------------------------------------------------------
# a5: DMPQ router (6Bit-Diffusion, Methodology A.1 and B.1).  Gamma is the
# relative L1 distance between a transformer block's output and input; a
# block whose Gamma exceeds the threshold runs INT8 activations, otherwise
# NVFP4.  The pre-learned linear model of the page has positive slope, so
# thresholding its prediction is thresholding Gamma.
# ---------------------------------------------------------------------------

ROUTE_NVFP4 = 0
ROUTE_INT8 = 1


def dmpq_gamma(inp_bits: np.ndarray, out_bits: np.ndarray) -> float:
    """inp/out: bf16 bit patterns of equal shape.  d_i = RN(out_i - in_i) in
    fp32; Gamma = sum|d_i| / sum|in_i| with both sums in fp64."""
    x = bf16_bits_to_f32(inp_bits).ravel()
    y = bf16_bits_to_f32(out_bits).ravel()
    d = (y - x).astype(np.float32)
    s1 = float(np.sum(np.abs(d).astype(np.float64)))
    s0 = float(np.sum(np.abs(x).astype(np.float64)))
    if s0 == 0.0:
        return float("inf")
    return s1 / s0


def dmpq_route(gamma: float, threshold: float) -> int:
    """Strictly greater than the threshold -> INT8, else NVFP4."""
    return ROUTE_INT8 if gamma > threshold else ROUTE_NVFP4


# ---------------------------------------------------------------------------
# a7: Q-ARVD outlier-aware dual-scale weight quantiser (Q-ARVD, Methodology
# and Formula/operation flow).  Input-channel L2 norms v_k; modified z-score
# M_k = (v_k - median(v)) / MAD with MAD = median(|v - median(v)|); channel
# k is an outlier iff M_k > tau and v_k > alpha * median(v).  Each output row
# gets one symmetric INT4 scale over its normal channels and another over its
# outlier channels.
# ---------------------------------------------------------------------------

def median_sorted(v: np.ndarray) -> float:
    """Median by full sort; even length -> mean of the two middle values."""
    s = np.sort(np.asarray(v, dtype=np.float64))
    n = len(s)
    if n == 0:
        raise ValueError("median of an empty vector")
    if n % 2:
        return float(s[n // 2])
    return float((s[n // 2 - 1] + s[n // 2]) / 2.0)


def qarvd_channel_norms(w_bits: np.ndarray) -> np.ndarray:
    """v_k = sqrt(sum_n w[n,k]^2), weights exact from bf16, fp64 throughout."""
    w = bf16_bits_to_f32(w_bits).astype(np.float64)
    return np.sqrt(np.sum(w * w, axis=0))


def qarvd_outlier_mask(v: np.ndarray, tau: float, alpha: float):
    """Returns (mask bool [K], modified z-scores M [K], median, MAD).  With
    MAD == 0 the IEEE quotient makes every channel above the median an
    outlier candidate (+inf > tau) and every other channel not."""
    v = np.asarray(v, dtype=np.float64)
    med = median_sorted(v)
    mad = median_sorted(np.abs(v - med))
    with np.errstate(divide="ignore", invalid="ignore"):
        m = (v - med) / mad
    mask = (m > tau) & (v > alpha * med)
    return mask, m, med, mad


def qarvd_layout(mask: np.ndarray):
    """Channel order and padded sizes of the dual-scale layout: normal
    channels ascending, then outlier channels ascending; each class padded
    with zero channels to a multiple of 32.  Returns (perm int32 [K],
    k_norm, k_norm_pad, n_out, k_out_pad)."""
    mask = np.asarray(mask, dtype=bool)
    normal = np.nonzero(~mask)[0]
    outl = np.nonzero(mask)[0]
    perm = np.concatenate([normal, outl]).astype(np.int32)
    k_norm, n_out = len(normal), len(outl)
    pad = lambda n: -(-n // QARVD_K_ALIGN) * QARVD_K_ALIGN
    return perm, k_norm, pad(k_norm), n_out, pad(n_out)


def _int4_row_quant(w: np.ndarray):
    """Per-row symmetric INT4 of one channel class: s = RN(amax / 7);
    q = clamp(rint(RN(w * RN(7 / amax))), -7, 7); empty or zero class -> s = 0."""
    rows = w.shape[0]
    if w.shape[1] == 0:
        return np.zeros((rows, 0), np.int8), np.zeros(rows, np.float32)
    amax = np.max(np.abs(w), axis=1).astype(np.float32)
    nz = amax != 0
    s = np.where(nz, (amax / np.float32(INT4_QMAX)).astype(np.float32), np.float32(0))
    inv = np.zeros_like(amax)
    inv[nz] = np.float32(INT4_QMAX) / amax[nz]
    y = (w * inv[:, None]).astype(np.float32)
    q = np.clip(np.rint(y), -INT4_QMAX, INT4_QMAX).astype(np.int8)
    return q, s.astype(np.float32)


def qarvd_pack(w_bits: np.ndarray, tau: float = 3.5, alpha: float = 2.0):
    """Full dual-scale weight preparation.  Returns a dict with mask, perm,
    the class sizes, s_norm [N], s_out [N] and the INT4 codes [N, Kp] (int8
    values in -7..7, permuted and zero-padded; Kp = k_norm_pad + k_out_pad)."""
    w = bf16_bits_to_f32(w_bits)
    v = qarvd_channel_norms(w_bits)
    mask, m, med, mad = qarvd_outlier_mask(v, tau, alpha)
    perm, k_norm, k_norm_pad, n_out, k_out_pad = qarvd_layout(mask)
    q_n, s_norm = _int4_row_quant(w[:, perm[:k_norm]])
    q_o, s_out = _int4_row_quant(w[:, perm[k_norm:]])
    n = w.shape[0]
    codes = np.zeros((n, k_norm_pad + k_out_pad), dtype=np.int8)
    codes[:, :k_norm] = q_n
    codes[:, k_norm_pad:k_norm_pad + n_out] = q_o
    return dict(norms=v, zscore=m, median=med, mad=mad, mask=mask, perm=perm,
                k_norm=k_norm, k_norm_pad=k_norm_pad, n_out=n_out, k_out_pad=k_out_pad,
                s_norm=s_norm, s_out=s_out, codes=codes)


def qarvd_permute_activations(q: np.ndarray, perm: np.ndarray, k_norm: int,
                              k_norm_pad: int, n_out: int, k_out_pad: int) -> np.ndarray:
    """Lay int8 activation codes out in the weights' channel order, padded."""
    rows = q.shape[0]
    out = np.zeros((rows, k_norm_pad + k_out_pad), dtype=np.int8)
    out[:, :k_norm] = q[:, perm[:k_norm]]
    out[:, k_norm_pad:k_norm_pad + n_out] = q[:, perm[k_norm:]]
    return out


def pack_int4(codes: np.ndarray) -> np.ndarray:
    """int8 values in -7..7 [R, K] -> two's-complement nibbles, [R, K/2]."""
    return pack_nibbles((np.asarray(codes, dtype=np.int8).view(np.uint8)) & 0xF)


# ---------------------------------------------------------------------------
# a8 / a9 / a10: reference GEMMs.  fp64 products of dequantized operands, the
# fp32 scales applied in fp64 at the end.  Y = X W^T with W in nn.Linear
# layout [N, K].
# ---------------------------------------------------------------------------

def gemm_w4a4(a_packed, a_sb, g_x, w_packed, w_sb, g_w, rows=None) -> np.ndarray:
    """R[m, n] = g_x g_w / 128 * sum_k dq_x[m,k] dq_w[n,k]  (fp64)."""
    dq_x = nvfp4_dequantize(a_packed if rows is None else a_packed[rows],
                            a_sb if rows is None else a_sb[rows])
    dq_w = nvfp4_dequantize(w_packed, w_sb)
    alpha = float(np.float64(g_x) * np.float64(g_w) / HADAMARD_N)
    return (dq_x @ dq_w.T) * alpha


def gemm_w4a8_token(q_x, s_x, w_packed, w_sb, g_w, hadamard=True, rows=None) -> np.ndarray:
    """INT8-route product: R[m, n] = s_m g_w / c * sum_k q_x[m,k] dq_w[n,k]
    with c = 128 when the operands were rotated, else 1."""
    q = np.asarray(q_x if rows is None else q_x[rows], dtype=np.float64)
    s = np.asarray(s_x if rows is None else s_x[rows], dtype=np.float64)
    dq_w = nvfp4_dequantize(w_packed, w_sb)
    c = HADAMARD_N if hadamard else 1
    return (q @ dq_w.T) * (s[:, None] * np.float64(g_w) / c)


def gemm_bf16(x_bits, w_bits, rows=None) -> np.ndarray:
    """Unquantized product of the bf16 operands, exact in fp64 (PDR's
    high-precision path): R = X W^T."""
    x = bf16_bits_to_f32(x_bits if rows is None else x_bits[rows]).astype(np.float64)
    return x @ bf16_bits_to_f32(w_bits).astype(np.float64).T


def gemm_qarvd(q_x_perm, s_x, codes, s_norm, s_out, k_norm_pad, rows=None) -> np.ndarray:
    """Dual-scale integer product: exact int64 class sums, then
    R[m, n] = s_x (s_norm[n] acc_normal + s_out[n] acc_outlier) in fp64."""
    qx = np.asarray(q_x_perm if rows is None else q_x_perm[rows], dtype=np.int64)
    qw = np.asarray(codes, dtype=np.int64)
    acc_n = qx[:, :k_norm_pad] @ qw[:, :k_norm_pad].T
    acc_o = qx[:, k_norm_pad:] @ qw[:, k_norm_pad:].T
    sx = np.float64(s_x)
    return sx * (acc_n.astype(np.float64) * np.asarray(s_norm, np.float64)[None, :]
                 + acc_o.astype(np.float64) * np.asarray(s_out, np.float64)[None, :])


# ---------------------------------------------------------------------------
# The composed path, as the library's forward runs it.
# ---------------------------------------------------------------------------

def prepare_weights_nvfp4(w_bits: np.ndarray, hadamard: bool = True):
    w = bf16_bits_to_f32(w_bits)
    hw = block_hadamard(w) if hadamard else w
    packed, sb, g = nvfp4_quantize(hw)
    return dict(packed=packed, sb=sb, g=g)


ROUTE_NVFP4_DECOMP = 4   # NVFP4 activations with the residual decomposition


def quantize_activations(x_bits: np.ndarray, route: int, hadamard: bool = True):
    x = bf16_bits_to_f32(x_bits)
    h = block_hadamard(x) if hadamard else x
    if route == ROUTE_NVFP4_DECOMP:
        packed, sb, g = nvfp4_decompose(h)
        return dict(packed=packed, sb=sb, g=g)
    if route == ROUTE_NVFP4:
        packed, sb, g = nvfp4_quantize(h)
        return dict(packed=packed, sb=sb, g=g)
    q, s = int8_per_token(h)
    return dict(q=q, s=s)


def forward(x_bits, wq: dict, route: int, hadamard: bool = True, rows=None) -> np.ndarray:
    """Quantize the activations on the given route and multiply (fp64)."""
    aq = quantize_activations(x_bits, route, hadamard)
    if route == ROUTE_NVFP4_DECOMP:
        wd = decompose_weights(wq)
        return gemm_w4a4(aq["packed"], aq["sb"], aq["g"], wd["packed"], wd["sb"], wd["g"], rows)
    if route == ROUTE_NVFP4:
        return gemm_w4a4(aq["packed"], aq["sb"], aq["g"], wq["packed"], wq["sb"], wq["g"], rows)
    return gemm_w4a8_token(aq["q"], aq["s"], wq["packed"], wq["sb"], wq["g"], hadamard, rows)
