"""Pins for the oracle's Hadamard rotation and quantizers."""
import numpy as np
import pytest
import scipy.linalg

from oracle import qlinear_oracle as O


# ---- a1 block Hadamard ------------------------------------------------------

def test_sylvester_matrix_is_scipy_hadamard_and_orthogonal():
    h = O.sylvester_hadamard(128)
    assert np.array_equal(h, scipy.linalg.hadamard(128))
    assert np.array_equal(h @ h.T, 128 * np.eye(128, dtype=np.int64))


def test_fwht_exact_on_integer_inputs():
    rng = np.random.default_rng(0)
    x = rng.integers(-1000, 1000, size=(5, 384)).astype(np.float32)
    got = O.block_hadamard(x)
    h = scipy.linalg.hadamard(128).astype(np.float64)
    want = np.concatenate([x[:, i:i + 128].astype(np.float64) @ h for i in range(0, 384, 128)], 1)
    assert np.array_equal(got.astype(np.float64), want)


def test_fwht_rounding_bound_on_real_inputs():
    """Seven fp32 butterfly levels: |err| <= 7 u sum|x| per output."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((8, 256)).astype(np.float32) * 37
    got = O.block_hadamard(x).astype(np.float64)
    h = scipy.linalg.hadamard(128).astype(np.float64)
    for b in range(2):
        blk = x[:, b * 128:(b + 1) * 128].astype(np.float64)
        exact = blk @ h
        bound = 7 * 2.0 ** -24 * np.abs(blk).sum(1, keepdims=True) * 1.01
        assert np.all(np.abs(got[:, b * 128:(b + 1) * 128] - exact) <= bound)


def test_fwht_first_stage_pairs_neighbours():
    """A unit impulse at index 1 gives row 1 of H: (+1, -1, +1, -1, ...)."""
    x = np.zeros((1, 128), np.float32)
    x[0, 1] = 1
    assert np.array_equal(O.block_hadamard(x)[0], scipy.linalg.hadamard(128)[1].astype(np.float32))


# ---- a2/a3 NVFP4 -------------------------------------------------------------

def _nvfp4_roundtrip_case(rng, rows=6, k=64):
    """Activations built from chosen codes and scales with tensor scale 1:
    every block's amax is 6*sb (one element has magnitude code 7) and one
    block has sb = 448, so the tensor amax is 2688."""
    codes = rng.integers(0, 16, size=(rows, k)).astype(np.uint8)
    sb = rng.integers(1, 127, size=(rows, k // 16)).astype(np.uint8)
    codes[:, ::16] = 7 | (codes[:, ::16] & 8)          # a +-6 in every block
    sb[0, 0] = 0x7E
    vals = O.e2m1_decode(codes).reshape(rows, k // 16, 16) * O.e4m3_decode(sb)[:, :, None]
    x = vals.reshape(rows, k).astype(np.float32)
    x[O.e2m1_decode(codes) == 0] = 0.0
    neg0 = (codes == 8)
    x[neg0] = np.float32(-0.0)
    return x, codes, sb


def test_nvfp4_exact_roundtrip():
    rng = np.random.default_rng(2)
    for _ in range(5):
        x, codes, sb = _nvfp4_roundtrip_case(rng)
        packed, sb2, g = O.nvfp4_quantize(x)
        assert g == np.float32(1.0)
        assert np.array_equal(sb2, sb)
        assert np.array_equal(O.unpack_nibbles(packed), codes)


def test_nvfp4_zero_blocks_and_zero_tensor():
    x = np.zeros((2, 32), np.float32)
    packed, sb, g = O.nvfp4_quantize(x)
    assert g == 1.0 and not sb.any() and not packed.any()
    x[1, 16:] = -np.float32(0.0)
    x[0, 0] = 3.0
    packed, sb, g = O.nvfp4_quantize(x)
    assert sb[1, 1] == 0 and not packed[1].any()        # negative zeros -> +0 codes


def test_nvfp4_subnormal_block_scale():
    x = np.zeros((1, 32), np.float32)
    x[0, 0] = 2688.0                                     # g = 1
    x[0, 16] = 6 * 2.0 ** -8                             # sb = 2^-8 (subnormal code 2)
    x[0, 17] = 2.0 ** -8
    packed, sb, g = O.nvfp4_quantize(x)
    assert sb[0, 1] == 2
    dq = O.nvfp4_dequantize(packed, sb) * float(g)
    assert dq[0, 16] == x[0, 16] and dq[0, 17] == x[0, 17]


def test_nvfp4_tensor_scale_takes_the_largest_magnitude():
    """The tensor scale follows the largest MAGNITUDE, here a negative
    value: g = 5376 / (6 * 448) = 2 exactly, its block scale is 448 and the
    element itself is the code for -6."""
    x = np.zeros((1, 32), np.float32)
    x[0, 3] = -5376.0
    x[0, 20] = 1.0
    packed, sb, g = O.nvfp4_quantize(x)
    assert g == np.float32(2.0)
    assert sb[0, 0] == 0x7E
    assert O.unpack_nibbles(packed)[0, 3] == 0xF


def test_nvfp4_static_scale_saturates():
    x = np.full((1, 16), 100.0, np.float32)
    packed, sb, g = O.nvfp4_quantize(x, g=np.float32(0.01))
    assert sb[0, 0] == 0x7E                              # 100/(0.06) > 448 -> 448
    assert np.all(O.unpack_nibbles(packed) == 7)         # 100/4.48 > 6 -> 6


def test_nvfp4_codes_are_nearest_after_scaling():
    """Definition check on random data: each code is the E2M1 encoding of
    RN(h * RN(1 / RN(sb * g))) with sb the E4M3 of RN(amax_b / RN(6 g))."""
    rng = np.random.default_rng(3)
    h = (rng.standard_normal((4, 128)) * rng.uniform(0.01, 10, (4, 1))).astype(np.float32)
    packed, sb, g = O.nvfp4_quantize(h)
    assert g == np.float32(np.abs(h).max() / np.float32(2688))
    codes = O.unpack_nibbles(packed)
    for r in range(4):
        for b in range(8):
            blk = h[r, b * 16:(b + 1) * 16]
            sf = np.float32(np.abs(blk).max() / np.float32(np.float32(6) * g))
            assert sb[r, b] == O.e4m3_encode(sf)
            inv = np.float32(1) / np.float32(O.e4m3_decode(sb[r, b]) * g)
            for j in range(16):
                y = np.float32(blk[j] * inv)
                assert codes[r, b * 16 + j] == O.e2m1_encode(y)
                assert abs(abs(float(O.e2m1_decode(codes[r, b * 16 + j]))) - min(abs(float(y)), 6.0)) <= 1.0


# ---- a4 / a10 INT8 -----------------------------------------------------------

def test_int8_per_token_integer_rows_roundtrip():
    rng = np.random.default_rng(4)
    q = rng.integers(-127, 128, size=(6, 64)).astype(np.float32)
    q[:, 0] = 127
    got, s = O.int8_per_token(q)
    assert np.all(s == 1.0) and np.array_equal(got.astype(np.float32), q)


def test_int8_per_token_brute_force():
    rng = np.random.default_rng(5)
    h = rng.standard_normal((7, 48)).astype(np.float32)
    h[3] = 0
    q, s = O.int8_per_token(h)
    for r in range(7):
        a = max(abs(float(v)) for v in h[r])
        if a == 0:
            assert s[r] == 0 and not q[r].any()
            continue
        assert s[r] == np.float32(np.float32(a) / np.float32(127))
        inv = np.float32(np.float32(127) / np.float32(a))
        for j in range(48):
            y = float(np.float32(h[r, j] * inv))
            assert q[r, j] == max(-127, min(127, round(y)))   # Python round: ties to even


def test_int8_per_tensor():
    x = np.array([[1.0, -2.0], [0.5, 254.0]], np.float32)
    q, s = O.int8_per_tensor(x)
    assert s == np.float32(2.0)
    assert q.tolist() == [[0, -1], [0, 127]]             # 0.5 and -1 -> ties to even 0, -1


def test_int6_brute_force_and_range():
    """W4A6: the INT8 recipe with qmax = 31 (codes within [-31, 31])."""
    rng = np.random.default_rng(8)
    h = rng.standard_normal((5, 40)).astype(np.float32)
    h[2, 7] = 40.0
    q, s = O.int8_per_token(h, O.INT6_QMAX)
    assert np.abs(q.astype(int)).max() == 31
    for r in range(5):
        a = max(abs(float(v)) for v in h[r])
        assert s[r] == np.float32(np.float32(a) / np.float32(31))
        inv = np.float32(np.float32(31) / np.float32(a))
        for j in range(40):
            assert q[r, j] == max(-31, min(31, round(float(np.float32(h[r, j] * inv)))))
    qt, st = O.int8_per_tensor(np.array([[1.0, -62.0], [0.5, 31.0]], np.float32), O.INT6_QMAX)
    assert st == np.float32(2.0) and qt.tolist() == [[0, -31], [0, 16]]   # 0.5 -> 0 and 15.5 -> 16 (ties to even)


def test_int6_integer_rows_roundtrip():
    rng = np.random.default_rng(9)
    q = rng.integers(-31, 32, size=(4, 64)).astype(np.float32)
    q[:, 5] = -31
    got, s = O.int8_per_token(q, O.INT6_QMAX)
    assert np.all(s == 1.0) and np.array_equal(got.astype(np.float32), q)


# ---- a7 Q-ARVD ---------------------------------------------------------------

def test_qarvd_golden_zscore_cases(golden):
    for line in golden("qarvd_zscore_cases.txt"):
        head, norms, want = [p.strip() for p in line.split("|")]
        tau, alpha = map(float, head.split())
        v = np.array([float(t) for t in norms.split()])
        mask, _, _, _ = O.qarvd_outlier_mask(v, tau, alpha)
        expect = [] if want == "-" else [int(t) for t in want.split()]
        assert np.nonzero(mask)[0].tolist() == expect, line


def test_median_matches_numpy_and_selection():
    rng = np.random.default_rng(6)
    for n in (1, 2, 7, 100, 3073):
        v = rng.standard_normal(n)
        assert O.median_sorted(v) == pytest.approx(float(np.median(v)), abs=0, rel=1e-15)
        if n % 2:
            assert O.median_sorted(v) == np.partition(v, n // 2)[n // 2]


def test_qarvd_channel_norms_closed_form():
    """v_k is the L2 norm of input channel k (a column of W [N, K]):
    columns (3, 4), (1, 0), (0, 2) give 5, 1, 2."""
    w = np.array([[3.0, 1.0, 0.0], [4.0, 0.0, 2.0]], np.float32)
    bits = (w.view(np.uint32) >> 16).astype(np.uint16)        # exact in bf16
    assert O.qarvd_channel_norms(bits).tolist() == [5.0, 1.0, 2.0]


def test_qarvd_layout_and_int4():
    rng = np.random.default_rng(7)
    mask = np.zeros(70, bool)
    mask[[3, 40, 69]] = True
    perm, k_norm, k_norm_pad, n_out, k_out_pad = O.qarvd_layout(mask)
    assert sorted(perm.tolist()) == list(range(70))
    assert perm[-3:].tolist() == [3, 40, 69] and np.all(np.diff(perm[:67]) > 0)
    assert (k_norm, k_norm_pad, n_out, k_out_pad) == (67, 96, 3, 32)
    w = rng.standard_normal((5, 9)).astype(np.float32)
    q, s = O._int4_row_quant(w)
    for r in range(5):
        a = np.float32(np.abs(w[r]).max())
        assert s[r] == np.float32(a / np.float32(7))
        inv = np.float32(np.float32(7) / a)
        assert q[r].tolist() == [max(-7, min(7, round(float(np.float32(v * inv))))) for v in w[r]]


def test_qarvd_planted_channels_detected():
    """Weights N(0, 0.02) with 2% of input channels x20: every planted
    channel is found and nothing else (norm ~20x the median)."""
    from bit_quantized_linear_block_b200 import synthetic as S
    rng = np.random.default_rng([3, 30])
    w = S.weights(1024, 3072, 0.02, 3, 30, outlier_frac=0.02, outlier_scale=20.0)
    rng.standard_normal(size=(1024, 3072), dtype=np.float32)
    planted = set(rng.choice(3072, size=61, replace=False).tolist())
    bits = S.bf16_bits(w)
    mask, m, med, mad = O.qarvd_outlier_mask(O.qarvd_channel_norms(bits), 3.5, 2.0)
    assert set(np.nonzero(mask)[0].tolist()) == planted
