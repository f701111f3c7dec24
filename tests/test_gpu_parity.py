"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on
identical seeded bf16 inputs.  Quantized codes, scales, masks and routes
must match bit for bit; GEMM outputs within the stated tolerances."""
import numpy as np
import pytest
import torch

from oracle import qlinear_oracle as O
from bit_quantized_linear_block_b200 import synthetic as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ql():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from bit_quantized_linear_block_b200 import qlinear
    return qlinear


def _np(t):
    return t.detach().cpu().numpy()


def _x(m, k, seed, outliers=8, scale=50.0):
    return S.activations_fixed_outliers(m, k, outliers, scale, seed, 1)


def normwise_err(y, r):
    return float(np.abs(y - r).max() / max(np.abs(r).max(), 1e-30))


def excess_err(y, r):
    """Error beyond the round-to-nearest bf16 rounding of the output: bf16
    keeps 8 significant bits, so that rounding alone moves a value by up to
    2^-8 of its magnitude."""
    ex = np.maximum(0.0, np.abs(y - r) - 2.0 ** -8 * np.maximum(np.abs(y), np.abs(r)))
    return float(ex.max() / max(np.abs(r).max(), 1e-30))


# ---------------------------------------------------------------- quantizers

SHAPES = [(1, 128), (77, 384), (256, 1920), (300, 640), (129, 1024)]


@pytest.mark.parametrize("m,k", SHAPES)
@pytest.mark.parametrize("hadamard", [True, False])
def test_nvfp4_quantize_bit_exact(ql, m, k, hadamard):
    x = _x(m, k, seed=m + k)
    xb = S.bf16_bits(x)
    h = O.block_hadamard(O.bf16_bits_to_f32(xb)) if hadamard else O.bf16_bits_to_f32(xb)
    packed, sb, g = O.nvfp4_quantize(h)
    q = ql.qlinear_quantize_act(x.cuda(), ql.QL_ROUTE_NVFP4, hadamard=hadamard)
    torch.cuda.synchronize()
    assert _np(q["scales"])[0] == g
    assert np.array_equal(_np(q["sf_rowmajor"]), sb)
    assert np.array_equal(_np(ql.sf_mma_to_rowmajor(q["sf_mma"], m, k)), sb)
    mpad = (m + 127) // 128 * 128
    assert not _np(ql.sf_mma_to_rowmajor(q["sf_mma"], mpad, k))[m:].any()   # padding rows
    assert np.array_equal(_np(q["codes"]), packed)


def test_block_scale_division_is_correctly_rounded(ql):
    """The quantizer divides each block maximum a by d = RN(6 g) with a
    reciprocal and one Markstein correction.  Against the correctly rounded
    quotient, for every fp32 dividend from d 2^-12 (below, the E4M3 code is 0
    whatever the rounding) to 450 d (block maxima never exceed 448 d (1 +
    2^-22)), for divisors from random, tiny, huge and edge tensor scales."""
    rng = np.random.default_rng(0)
    gs = ([1.0, 1.0 / 3.0, 0.1, 7.0, 2.0 ** -20, 2.0 ** 20, 1e-33, 1e33]
          + list(rng.uniform(1e-3, 10.0, 16)) + list(10.0 ** rng.uniform(-30, 30, 16)))
    bits = lambda v: int(np.array(v, np.float32).view(np.uint32))
    for g in gs:
        d = np.float32(np.float32(6.0) * np.float32(g))
        lo = bits(d * np.float32(2.0 ** -12))
        hi = bits(min(np.float32(d) * np.float32(450.0), np.float32(3.0e38)))
        assert ql.qlinear_debug_div_check(float(d), lo, hi - lo + 1) == 0, float(d)


def test_nvfp4_quantize_zero_and_tiny_blocks(ql):
    x = np.zeros((130, 256), np.float32)
    x[0, 0] = 3000.0
    x[5, 16:32] = 1e-3          # subnormal E4M3 block scale
    x[7, 32:48] = -1e-6         # scale rounds to 0 -> all +0 codes
    x[9, 64:80] = -0.0
    xt = S.to_bf16(x)
    packed, sb, g = O.nvfp4_quantize(O.bf16_bits_to_f32(S.bf16_bits(xt)))
    q = ql.qlinear_quantize_act(xt.cuda(), ql.QL_ROUTE_NVFP4, hadamard=False)
    torch.cuda.synchronize()
    assert _np(q["scales"])[0] == g
    assert np.array_equal(_np(q["sf_rowmajor"]), sb)
    assert np.array_equal(_np(q["codes"]), packed)


@pytest.mark.parametrize("m,k", SHAPES)
@pytest.mark.parametrize("hadamard", [True, False])
def test_int8_token_quantize_bit_exact(ql, m, k, hadamard):
    x = _x(m, k, seed=3 * m + k)
    xb = S.bf16_bits(x)
    h = O.block_hadamard(O.bf16_bits_to_f32(xb)) if hadamard else O.bf16_bits_to_f32(xb)
    qo, so = O.int8_per_token(h)
    q = ql.qlinear_quantize_act(x.cuda(), ql.QL_ROUTE_INT8, hadamard=hadamard)
    torch.cuda.synchronize()
    assert np.array_equal(_np(q["scales"])[:m], so)
    assert np.array_equal(_np(q["codes"]), qo)


def test_int8_token_zero_row(ql):
    x = np.zeros((3, 128), np.float32)
    x[1] = np.arange(128) - 64
    xt = S.to_bf16(x)
    qo, so = O.int8_per_token(O.block_hadamard(O.bf16_bits_to_f32(S.bf16_bits(xt))))
    q = ql.qlinear_quantize_act(xt.cuda(), ql.QL_ROUTE_INT8, hadamard=True)
    torch.cuda.synchronize()
    assert np.array_equal(_np(q["scales"]), so) and np.array_equal(_np(q["codes"]), qo)


# ---------------------------------------------------------------- router

@pytest.mark.parametrize("numel", [0, 5, 1920, 256 * 1920 + 3])
def test_route_gamma(ql, numel):
    rng = np.random.default_rng(numel)
    x = rng.standard_normal(numel).astype(np.float32)
    y = x + rng.standard_normal(numel).astype(np.float32) * 0.04
    xt, yt = S.to_bf16(x), S.to_bf16(y)
    g_ref = O.dmpq_gamma(S.bf16_bits(xt), S.bf16_bits(yt))
    g, r = ql.qlinear_route(xt.cuda(), yt.cuda(), 0.05)
    torch.cuda.synchronize()
    g, r = float(_np(g)[0]), int(_np(r)[0])
    if numel == 0:
        assert g == float("inf") and r == 1
    else:
        assert g == pytest.approx(g_ref, rel=1e-12)
        assert r == O.dmpq_route(g_ref, 0.05)


def test_route_closed_forms(ql):
    rng = np.random.default_rng(9)
    x = rng.integers(-15, 16, size=4096).astype(np.float32) / 16
    xt = S.to_bf16(x)
    for y, want in [(x, 0.0), (x * np.float32(1.125), 0.125), (-x, 2.0)]:
        g, r = ql.qlinear_route(xt.cuda(), S.to_bf16(y).cuda(), 0.125)
        torch.cuda.synchronize()
        assert float(_np(g)[0]) == want
        assert int(_np(r)[0]) == (1 if want > 0.125 else 0)


def test_route_sweep_blocks_match_oracle(ql):
    """The routing sweep's blocks at a reduced token count: identical routes."""
    for b in range(30):
        x, y, sigma = S.dmpq_block_pair(b, m=512)
        g_ref = O.dmpq_gamma(S.bf16_bits(x), S.bf16_bits(y))
        assert abs(g_ref - 0.05) / 0.05 > 1e-9
        g, r = ql.qlinear_route(x.cuda(), y.cuda(), 0.05)
        torch.cuda.synchronize()
        assert float(_np(g)[0]) == pytest.approx(g_ref, rel=1e-12)
        assert int(_np(r)[0]) == O.dmpq_route(g_ref, 0.05)


# ---------------------------------------------------------------- weights

@pytest.mark.parametrize("n,k", [(1920, 1920), (640, 384), (16, 128)])
def test_prepare_weights_nvfp4_bit_exact(ql, n, k):
    w = S.weights(n, k, 0.02, 5, n + k)
    ref = O.prepare_weights_nvfp4(S.bf16_bits(w), hadamard=True)
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4, hadamard=True)
    torch.cuda.synchronize()
    codes = _np(pw.view("codes", torch.uint8, n * k // 2)).reshape(n, k // 2)
    sf = pw.view("sf", torch.uint8, ql.lib.qlinear_sf_bytes(n, k))
    assert _np(pw.view("gscale", torch.float32, 1))[0] == ref["g"]
    assert np.array_equal(_np(ql.sf_mma_to_rowmajor(sf, n, k)), ref["sb"])
    assert np.array_equal(codes, ref["packed"])


# ---------------------------------------------------------------- W4A4 GEMM

W4A4_CASES = [
    (256, 1920, 1920),   # the single-linear workload
    (300, 384, 640),     # ragged M, two 192-wide tiles, half-full last K stage
    (129, 640, 384),     # N not a multiple of 192 -> 128-wide tiles
    (1, 192, 128),
    (1000, 5760, 1920),  # many tiles per CTA (persistent loop, both accumulators)
    (300, 1040, 640),    # ragged last 192-wide tile, N not a multiple of 128 (padded scale rows)
    (520, 5120, 2048),   # ragged 192-wide tiles with streamed scales (the Wan-14B FFN-down form)
    (100, 1040, 2048),   # one SM per tile (M <= 128), ragged, streamed scales
    (2048, 384, 1920),   # two N tiles per row block: the resident A panel reloaded many times per unit
    (4000, 192, 256),    # one N tile per row block, ragged M, one K chunk
    (600, 1920, 7680),   # streamed 256-wide tiles, ragged last tile (N = 7.5 tiles), long K
]


@pytest.mark.parametrize("m,n,k", W4A4_CASES)
def test_forward_w4a4_parity(ql, m, n, k):
    x = _x(m, k, seed=m * 7 + n)
    w = S.weights(n, k, 0.02, 6, m + n + k)
    xb, wb = S.bf16_bits(x), S.bf16_bits(w)
    wq = O.prepare_weights_nvfp4(wb)
    rows = np.arange(m) if m <= 512 else np.unique(np.r_[np.random.default_rng(0).choice(m, 256, replace=False), m - 1])
    ref = O.forward(xb, wq, O.ROUTE_NVFP4, rows=rows)
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4, hadamard=True)
    y = ql.qlinear_forward(x.cuda(), pw, ql.QL_ROUTE_NVFP4)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    yn = _np(y.float())[rows].astype(np.float64)
    assert np.isfinite(yn).all()
    assert normwise_err(yn, ref) <= 1e-2
    # the operands' products are exact and the accumulation is fp32, so every
    # output is the exact product up to its bf16 rounding (measured: no excess)
    assert excess_err(yn, ref) <= 1e-5


def test_gemm_timeout_path_reports_and_recovers(ql):
    """A zero wait budget makes the GEMM's first unsatisfied wait time out:
    the kernel records QL_ERR_TIMEOUT, drains and returns; the context stays
    usable and the next call with the default budget is correct."""
    m, n, k = 256, 384, 1920
    x = _x(m, k, seed=11)
    w = S.weights(n, k, 0.02, 6, 11)
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4, hadamard=True)
    xc = x.cuda()
    assert ql.qlinear_device_status() == 0
    ql.qlinear_debug_set_wait_limit(0)
    try:
        ql.qlinear_forward(xc, pw, ql.QL_ROUTE_NVFP4)
        st = ql.qlinear_device_status()
    finally:
        ql.qlinear_debug_set_wait_limit(-1)
    assert st == 5
    y = ql.qlinear_forward(xc, pw, ql.QL_ROUTE_NVFP4)
    assert ql.qlinear_device_status() == 0
    ref = O.forward(S.bf16_bits(x), O.prepare_weights_nvfp4(S.bf16_bits(w)), O.ROUTE_NVFP4)
    assert normwise_err(_np(y.float()).astype(np.float64), ref) <= 1e-2


# ---------------------------------------------------------------- W4A8 (INT8 route)

W4A8_CASES = [(256, 1920, 1920), (300, 384, 640), (129, 640, 384), (1000, 5760, 1920), (1, 192, 128),
              (2048, 576, 1024),   # several tiles per CTA (persistent loop over both accumulators)
              (700, 320, 256)]     # 128-wide tiles, the last one half past N


@pytest.mark.parametrize("expand", [False, True])
@pytest.mark.parametrize("m,n,k", W4A8_CASES)
def test_forward_w4a8_int8_route_parity(ql, m, n, k, expand):
    x = _x(m, k, seed=m * 3 + n)
    w = S.weights(n, k, 0.02, 7, m + n + k)
    xb, wb = S.bf16_bits(x), S.bf16_bits(w)
    wq = O.prepare_weights_nvfp4(wb)
    rows = np.arange(m) if m <= 512 else np.unique(np.r_[np.random.default_rng(1).choice(m, 256, replace=False), m - 1])
    ref = O.forward(xb, wq, O.ROUTE_INT8, rows=rows)
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4, hadamard=True, expand_f16=expand)
    if expand:   # the f16 copy is E2M1 x E4M3 exactly (no tensor scale)
        w16 = _np(pw.view("w16", torch.float16, n * k).reshape(n, k).float()).astype(np.float64)
        deq = (O.e2m1_decode(O.unpack_nibbles(wq["packed"])).astype(np.float64)
               * np.repeat(O.e4m3_decode(wq["sb"]).astype(np.float64), 16, axis=1))
        assert np.array_equal(w16, deq)
    y = ql.qlinear_forward(x.cuda(), pw, ql.QL_ROUTE_INT8)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    yn = _np(y.float())[rows].astype(np.float64)
    assert np.isfinite(yn).all()
    assert excess_err(yn, ref) <= 1e-5
    # int8 codes through qlinear_gemm: both operands widened on chip (no copy)
    # or the activations widened next to the f16 weight copy
    q = ql.qlinear_quantize_act(x.cuda(), ql.QL_ROUTE_INT8, hadamard=True)
    y2 = ql.qlinear_gemm(ql.QL_ROUTE_INT8, q, m, pw)
    # the same codes stored as f16 values: with the copy both operands by TMA,
    # without it the weights widened into tensor memory (the MMA's A operand)
    q3 = ql.qlinear_quantize_act(x.cuda(), ql.QL_ACT_INT8_F16, hadamard=True)
    y3 = ql.qlinear_gemm(ql.QL_ACT_INT8_F16, q3, m, pw)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    assert np.array_equal(_np(q3["codes"].float()), _np(q["codes"].float()))
    assert np.array_equal(_np(q3["scales"]), _np(q["scales"]))
    assert excess_err(_np(y2.float())[rows].astype(np.float64), ref) <= 1e-5
    assert excess_err(_np(y3.float())[rows].astype(np.float64), ref) <= 1e-5
    assert torch.equal(y3, y)   # the forward takes the f16-coded form


@pytest.mark.parametrize("m,n,k", [(300, 384, 640), (1, 320, 256), (700, 1040, 1024), (2000, 1920, 1920),
                                   (193, 128, 7680)])
def test_w4a8_forms_agree(ql, m, n, k):
    """The four INT8-route GEMM forms multiply the same exact f16 values with
    fp32 accumulation: weights widened into tensor memory (f16 codes, no
    copy), both operands widened on chip (int8 codes, no copy), and the f16
    weight copy with f16 or int8 codes.  Each is held to the oracle's product
    and all four must give the same bits.  Shapes: ragged token tiles (193,
    300, 700, 2000 rows against 192-row tiles), weight tiles past N (320,
    1040), one K stage per scale atom up to K = 7680."""
    x = _x(m, k, seed=m + 5 * n + k)
    w = S.weights(n, k, 0.02, 8, m + 2 * n + k)
    xb, wb = S.bf16_bits(x), S.bf16_bits(w)
    wq = O.prepare_weights_nvfp4(wb)
    rows = np.arange(m) if m <= 512 else np.unique(np.r_[np.random.default_rng(2).choice(m, 256, replace=False), m - 1])
    ref = O.forward(xb, wq, O.ROUTE_INT8, rows=rows)
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4, hadamard=True)
    pwx = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4, hadamard=True, expand_f16=True)
    xc = x.cuda()
    q8 = ql.qlinear_quantize_act(xc, ql.QL_ROUTE_INT8, hadamard=True)
    q16 = ql.qlinear_quantize_act(xc, ql.QL_ACT_INT8_F16, hadamard=True)
    ys = {"tmem": ql.qlinear_gemm(ql.QL_ACT_INT8_F16, q16, m, pw),
          "onchip": ql.qlinear_gemm(ql.QL_ROUTE_INT8, q8, m, pw),
          "copy_f16": ql.qlinear_gemm(ql.QL_ACT_INT8_F16, q16, m, pwx),
          "copy_int8": ql.qlinear_gemm(ql.QL_ROUTE_INT8, q8, m, pwx)}
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    for name, y in ys.items():
        yn = _np(y.float())[rows].astype(np.float64)
        assert np.isfinite(yn).all(), name
        assert excess_err(yn, ref) <= 1e-5, name
    for name, y in ys.items():
        assert torch.equal(y, ys["copy_f16"]), name


# ---------------------------------------------------------------- Q-ARVD

def _qarvd_weights(n, k, seed, frac=0.05, scale=20.0):
    return S.weights(n, k, 0.02, seed, 77, outlier_frac=frac, outlier_scale=scale)


def _assert_guard_band(pk, tau=3.5, alpha=2.0):
    """Mask decisions are bit-exact only away from the boundaries."""
    m = pk["zscore"][np.isfinite(pk["zscore"])]
    assert np.all(np.abs(m - tau) > 1e-9 * tau)
    assert np.all(np.abs(pk["norms"] - alpha * pk["median"]) > 1e-9 * max(pk["median"], 1e-30))


@pytest.mark.parametrize("n,k,frac", [(384, 640, 0.05), (256, 3072, 0.02), (64, 128, 0.0), (160, 1024, 0.3)])
def test_prepare_weights_qarvd_bit_exact(ql, n, k, frac):
    w = _qarvd_weights(n, k, seed=n + k, frac=frac)
    wb = S.bf16_bits(w)
    pk = O.qarvd_pack(wb, 3.5, 2.0)
    _assert_guard_band(pk)
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_QARVD_INT4, hadamard=False, tau=3.5, alpha=2.0)
    torch.cuda.synchronize()
    kp = pw.desc.Kp
    norms = _np(pw.view("norms", torch.float64, k))
    assert np.allclose(norms, pk["norms"], rtol=1e-13, atol=0)
    assert np.array_equal(_np(pw.view("outlier_mask", torch.uint8, k)).astype(bool), pk["mask"])
    assert np.array_equal(_np(pw.view("perm", torch.int32, k)), pk["perm"])
    kinfo = _np(pw.view("kinfo", torch.int32, 4)).tolist()
    assert kinfo == [pk["k_norm"], pk["k_norm_pad"], pk["n_out"], pk["k_out_pad"]]
    assert np.array_equal(_np(pw.view("s_norm", torch.float32, n)), pk["s_norm"])
    assert np.array_equal(_np(pw.view("s_out", torch.float32, n)), pk["s_out"])
    want = np.zeros((n, kp), np.int8)
    want[:, :pk["codes"].shape[1]] = pk["codes"]
    got = _np(pw.view("codes", torch.uint8, n * kp // 2)).reshape(n, kp // 2)
    assert np.array_equal(got, O.pack_int4(want))


@pytest.mark.parametrize("expand", [False, True])
@pytest.mark.parametrize("m,n,k,frac", [(300, 384, 640, 0.05), (256, 256, 3072, 0.05), (77, 128, 128, 0.05),
                                        (513, 200 - 8, 1024, 0.0), (130, 64, 512, 0.3),
                                        (2048, 1920, 512, 0.05)])   # several tiles per SM pair
def test_qarvd_activation_quant_and_forward_parity(ql, m, n, k, frac, expand):
    w = _qarvd_weights(n, k, seed=m + n, frac=frac)
    pk = O.qarvd_pack(S.bf16_bits(w), 3.5, 2.0)
    _assert_guard_band(pk)
    x = _x(m, k, seed=m + 5 * k)
    xb = S.bf16_bits(x)
    qx, sx = O.int8_per_tensor(O.bf16_bits_to_f32(xb))
    qxp = O.qarvd_permute_activations(qx, pk["perm"], pk["k_norm"], pk["k_norm_pad"], pk["n_out"], pk["k_out_pad"])
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_QARVD_INT4, hadamard=False, expand_i8=expand)
    xc = x.cuda()
    q = ql.qlinear_quantize_act(xc, ql.QL_ACT_INT8_TENSOR, hadamard=False, w=pw)
    y = ql.qlinear_forward(xc, pw)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    kp = pw.desc.Kp
    assert (pw.desc.w8 is not None) == expand
    if expand:   # the int8 copy is the INT4 codes sign-extended, zero in the padding
        want_w = np.zeros((n, kp), np.int8)
        want_w[:, :pk["codes"].shape[1]] = pk["codes"]
        assert np.array_equal(_np(pw.view("w8", torch.int8, n * kp)).reshape(n, kp), want_w)
    want = np.zeros((m, kp), np.int8)
    want[:, :qxp.shape[1]] = qxp
    assert _np(q["scales"])[0] == sx
    assert np.array_equal(_np(q["codes"]), want)
    ref = O.gemm_qarvd(qxp, sx, pk["codes"], pk["s_norm"], pk["s_out"], pk["k_norm_pad"])
    assert excess_err(_np(y.float()).astype(np.float64), ref) <= 1e-5


@pytest.mark.parametrize("m,n,k,frac,seed", [(300, 384, 384, 0.05, 3), (77, 128, 128, 0.05, 4),
                                             (700, 640, 3072, 0.02, 5), (256, 256, 640, 0.0, 5),
                                             (1000, 208, 1024, 0.05, 6)])
def test_qarvd_forms_agree(ql, m, n, k, frac, seed):
    """The INT4 weights widened on chip into tensor memory and the int8
    weight copy multiply the same integers with exact int32 accumulation and
    the same epilogue rounding: identical outputs, each held to the oracle.
    Shapes: ragged 128-token tiles (77, 300, 700, 1000), weight tiles past N
    (208), a weight set without outlier channels (frac 0: the outlier
    class is empty), and an outlier class that follows a partial K stage."""
    w = S.weights(n, k, 0.02, seed, 77, outlier_frac=frac, outlier_scale=20.0)
    pk = O.qarvd_pack(S.bf16_bits(w), 3.5, 2.0)
    _assert_guard_band(pk)
    if frac == 0.0:
        assert pk["n_out"] == 0
    x = _x(m, k, seed=m + 3 * k)
    qx, sx = O.int8_per_tensor(O.bf16_bits_to_f32(S.bf16_bits(x)))
    qxp = O.qarvd_permute_activations(qx, pk["perm"], pk["k_norm"], pk["k_norm_pad"], pk["n_out"], pk["k_out_pad"])
    ref = O.gemm_qarvd(qxp, sx, pk["codes"], pk["s_norm"], pk["s_out"], pk["k_norm_pad"])
    wc = w.cuda()
    pw = ql.qlinear_prepare_weights(wc, ql.QL_W_QARVD_INT4, hadamard=False)
    pw8 = ql.qlinear_prepare_weights(wc, ql.QL_W_QARVD_INT4, hadamard=False, expand_i8=True)
    xc = x.cuda()
    y_tmem = ql.qlinear_forward(xc, pw)
    y_copy = ql.qlinear_forward(xc, pw8)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    for y in (y_tmem, y_copy):
        yn = _np(y.float()).astype(np.float64)
        assert np.isfinite(yn).all()
        assert excess_err(yn, ref) <= 1e-5
    assert torch.equal(y_tmem, y_copy)


# ---------------------------------------------------------------- W4A6 (INT6 activations)

@pytest.mark.parametrize("expand", [False, True])
@pytest.mark.parametrize("m,n,k", [(300, 384, 640), (129, 1920, 1920), (1, 192, 128)])
def test_w4a6_token_route_parity(ql, m, n, k, expand):
    """6-bit signed integer activations per token (codes in [-31, 31]) into
    the INT8-route GEMM: codes and scales bit-exact, product within the INT8
    tolerance against the oracle's INT6 product."""
    x = _x(m, k, seed=m + 11 * k)
    w = S.weights(n, k, 0.02, 7, m + n)
    xb, wb = S.bf16_bits(x), S.bf16_bits(w)
    q6, s6 = O.int8_per_token(O.block_hadamard(O.bf16_bits_to_f32(xb)), O.INT6_QMAX)
    wq = O.prepare_weights_nvfp4(wb)
    ref = O.gemm_w4a8_token(q6, s6, wq["packed"], wq["sb"], wq["g"])
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4, hadamard=True, expand_f16=expand)
    xc = x.cuda()
    q = ql.qlinear_quantize_act(xc, ql.QL_ROUTE_INT6, hadamard=True)
    y = ql.qlinear_forward(xc, pw, ql.QL_ROUTE_INT6)
    y2 = ql.qlinear_gemm(ql.QL_ROUTE_INT6, q, m, pw)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    assert np.array_equal(_np(q["codes"]), q6) and np.array_equal(_np(q["scales"])[:m], s6)
    assert np.abs(q6.astype(int)).max() <= 31
    assert excess_err(_np(y.float()).astype(np.float64), ref) <= 1e-5
    assert excess_err(_np(y2.float()).astype(np.float64), ref) <= 1e-5
    qf = ql.qlinear_quantize_act(xc, ql.QL_ACT_INT6_F16, hadamard=True)
    y3 = ql.qlinear_gemm(ql.QL_ACT_INT6_F16, qf, m, pw)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    assert np.array_equal(_np(qf["codes"].float()), q6.astype(np.float32))
    assert excess_err(_np(y3.float()).astype(np.float64), ref) <= 1e-5
    assert torch.equal(y3, y)   # the forward quantizes to f16-coded INT6


@pytest.mark.parametrize("expand", [False, True])
@pytest.mark.parametrize("m,n,k", [(300, 384, 640), (77, 128, 128), (600, 576, 1024)])
def test_w4a6_qarvd_parity(ql, m, n, k, expand):
    """Q-ARVD with per-tensor INT6 activations (its W4A6 setting)."""
    w = _qarvd_weights(n, k, seed=m + n + 1)
    pk = O.qarvd_pack(S.bf16_bits(w), 3.5, 2.0)
    _assert_guard_band(pk)
    x = _x(m, k, seed=m + 3 * k)
    qx, sx = O.int8_per_tensor(O.bf16_bits_to_f32(S.bf16_bits(x)), O.INT6_QMAX)
    qxp = O.qarvd_permute_activations(qx, pk["perm"], pk["k_norm"], pk["k_norm_pad"], pk["n_out"], pk["k_out_pad"])
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_QARVD_INT4, hadamard=False, expand_i8=expand)
    xc = x.cuda()
    q = ql.qlinear_quantize_act(xc, ql.QL_ACT_INT6_TENSOR, hadamard=False, w=pw)
    y = ql.qlinear_forward(xc, pw, ql.QL_ROUTE_INT6)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    kp = pw.desc.Kp
    want = np.zeros((m, kp), np.int8)
    want[:, :qxp.shape[1]] = qxp
    assert _np(q["scales"])[0] == sx and np.array_equal(_np(q["codes"]), want)
    ref = O.gemm_qarvd(qxp, sx, pk["codes"], pk["s_norm"], pk["s_out"], pk["k_norm_pad"])
    assert excess_err(_np(y.float()).astype(np.float64), ref) <= 1e-5



# ---------------------------------------------------------------- BF16 (PDR's refresh)

@pytest.mark.parametrize("m,n,k", [(300, 384, 640), (129, 1920, 1920), (1, 640, 128), (1000, 5760, 1920)])
def test_bf16_route_parity(ql, m, n, k):
    """The unquantized product X W^T from the kept bf16 weights (fp32
    accumulation, bf16 out) against the exact fp64 product."""
    x = _x(m, k, seed=m + 13 * k)
    w = S.weights(n, k, 0.02, 9, m + n)
    xb, wb = S.bf16_bits(x), S.bf16_bits(w)
    rows = np.arange(m) if m <= 512 else np.unique(np.r_[np.random.default_rng(2).choice(m, 256, replace=False), m - 1])
    ref = O.gemm_bf16(xb, wb, rows=rows)
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4, hadamard=True, keep_bf16=True)
    xc = x.cuda()
    y = ql.qlinear_forward(xc, pw, ql.QL_ROUTE_BF16)
    y2 = ql.qlinear_gemm(ql.QL_ROUTE_BF16, {"codes": xc, "scales": None}, m, pw)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    assert torch.equal(pw.view("wbf16", torch.bfloat16, n * k).reshape(n, k).cpu(), w)   # kept as given
    yn = _np(y.float())[rows].astype(np.float64)
    assert excess_err(yn, ref) <= 1e-5
    assert torch.equal(y, y2)


def test_bf16_route_needs_kept_weights(ql):
    w = S.weights(64, 128, 0.02, 9, 3)
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4, hadamard=True)
    with pytest.raises(ql.QLinearError):
        ql.qlinear_forward(_x(8, 128, seed=1).cuda(), pw, ql.QL_ROUTE_BF16)
