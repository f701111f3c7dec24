"""Pins for the oracle's DMPQ Gamma/route and its reference GEMMs."""
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import qlinear_oracle as O


def _bits(x32):
    return torch.from_numpy(np.asarray(x32, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ---- a5 Gamma and route ------------------------------------------------------

def test_gamma_closed_form_power_of_two_scaling():
    """out = (1 + c) in with c = 2^-3 and inputs of <= 4 significant bits:
    every difference is exact, so Gamma = c exactly."""
    rng = np.random.default_rng(0)
    x = rng.integers(-15, 16, size=(64, 32)).astype(np.float32) * np.float32(2.0 ** -4)
    y = x * np.float32(1.125)
    assert O.dmpq_gamma(_bits(x), _bits(y)) == 0.125
    assert O.dmpq_gamma(_bits(x), _bits(-x)) == 2.0
    assert O.dmpq_gamma(_bits(x), _bits(x)) == 0.0


def test_gamma_brute_force_small():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 5)).astype(np.float32)
    y = x + rng.standard_normal((3, 5)).astype(np.float32) * 0.1
    xb, yb = _bits(x), _bits(y)
    xf, yf = O.bf16_bits_to_f32(xb).ravel(), O.bf16_bits_to_f32(yb).ravel()
    num = sum(Fraction(float(abs(np.float32(b - a)))) for a, b in zip(xf, yf))
    den = sum(Fraction(float(abs(a))) for a in xf)
    assert O.dmpq_gamma(xb, yb) == pytest.approx(float(num / den), rel=1e-15)


def test_route_threshold_is_strict_and_zero_input_is_int8():
    assert O.dmpq_route(0.05, 0.05) == O.ROUTE_NVFP4
    assert O.dmpq_route(0.0500001, 0.05) == O.ROUTE_INT8
    z = np.zeros((2, 2), np.uint16)
    g = O.dmpq_gamma(z, z)
    assert g == float("inf") and O.dmpq_route(g, 0.05) == O.ROUTE_INT8


def test_gamma_tracks_sigma_on_sweep_block():
    """For in ~ N(0,1) and out = in + N(0, s): E|d| / E|x| = s (sanity band)."""
    from bit_quantized_linear_block_b200 import synthetic as S
    x, y, sigma = S.dmpq_block_pair(0, m=256, k=1920)
    g = O.dmpq_gamma(S.bf16_bits(x), S.bf16_bits(y))
    assert abs(g / sigma - 1) < 0.05 or sigma < 5e-3


# ---- a8 / a9 / a10 GEMMs -----------------------------------------------------

def _exact_w4a4(a_packed, a_sb, g_x, w_packed, w_sb, g_w):
    qa, qw = O.unpack_nibbles(a_packed), O.unpack_nibbles(w_packed)
    mags = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2),
            Fraction(3), Fraction(4), Fraction(6)]
    val = lambda c: -mags[c & 7] if c & 8 else mags[c & 7]
    e4 = lambda c: Fraction(float(O.e4m3_magnitudes()[c]))
    m, k = qa.shape
    n = qw.shape[0]
    alpha = Fraction(float(g_x)) * Fraction(float(g_w)) / 128
    out = np.zeros((m, n))
    for i in range(m):
        for j in range(n):
            s = sum(val(int(qa[i, t])) * e4(int(a_sb[i, t // 16])) *
                    val(int(qw[j, t])) * e4(int(w_sb[j, t // 16])) for t in range(k))
            out[i, j] = float(s * alpha)
    return out


def test_w4a4_gemm_equals_exact_rational_sum():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((3, 128)) * 3).astype(np.float32)
    w = (rng.standard_normal((4, 128)) * 0.02).astype(np.float32)
    hx, hw = O.block_hadamard(x), O.block_hadamard(w)
    ap, asb, gx = O.nvfp4_quantize(hx)
    wp, wsb, gw = O.nvfp4_quantize(hw)
    got = O.gemm_w4a4(ap, asb, gx, wp, wsb, gw)
    want = _exact_w4a4(ap, asb, gx, wp, wsb, gw)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("hadamard", [True, False])
def test_w4a8_token_gemm_brute_force(hadamard):
    """With rotated operands the product carries the 1/128 of H H^T = 128 I;
    without rotation it does not."""
    rng = np.random.default_rng(3)
    rot = O.block_hadamard if hadamard else (lambda v: v)
    h = rot((rng.standard_normal((2, 128)) * 2).astype(np.float32))
    q, s = O.int8_per_token(h)
    wp, wsb, gw = O.nvfp4_quantize(rot(rng.standard_normal((3, 128)).astype(np.float32)))
    got = O.gemm_w4a8_token(q, s, wp, wsb, gw, hadamard=hadamard)
    dq = O.nvfp4_dequantize(wp, wsb)
    c = 128 if hadamard else 1
    for i in range(2):
        for j in range(3):
            acc = sum(Fraction(int(q[i, t])) * Fraction(float(dq[j, t])) for t in range(128))
            want = acc * Fraction(float(s[i])) * Fraction(float(gw)) / c
            assert got[i, j] == pytest.approx(float(want), rel=1e-15)


def test_qarvd_gemm_integer_brute_force():
    rng = np.random.default_rng(4)
    w = (rng.standard_normal((5, 70)) * 0.02).astype(np.float32)
    w[:, [2, 50]] *= 20
    pk = O.qarvd_pack(_bits(w))
    assert pk["mask"][[2, 50]].all() and pk["mask"].sum() == 2
    x = rng.standard_normal((3, 70)).astype(np.float32)
    qx, sx = O.int8_per_tensor(x)
    qxp = O.qarvd_permute_activations(qx, pk["perm"], pk["k_norm"], pk["k_norm_pad"],
                                      pk["n_out"], pk["k_out_pad"])
    got = O.gemm_qarvd(qxp, sx, pk["codes"], pk["s_norm"], pk["s_out"], pk["k_norm_pad"])
    for i in range(3):
        for j in range(5):
            acc_n = sum(int(qx[i, c]) * int(pk["codes"][j, p]) for p, c in enumerate(pk["perm"][:pk["k_norm"]]))
            acc_o = sum(int(qx[i, c]) * int(pk["codes"][j, pk["k_norm_pad"] + p])
                        for p, c in enumerate(pk["perm"][pk["k_norm"]:]))
            want = float(sx) * (float(pk["s_norm"][j]) * acc_n + float(pk["s_out"][j]) * acc_o)
            assert got[i, j] == pytest.approx(want, rel=1e-15)


def test_hadamard_invariance_unquantized():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, 256))
    w = rng.standard_normal((6, 256))
    h = scipy.linalg.hadamard(128).astype(np.float64)
    bh = np.kron(np.eye(2), h)
    assert np.allclose((x @ bh) @ (w @ bh).T / 128, x @ w.T, rtol=0, atol=1e-12)


def test_quantized_product_close_to_float_product():
    """Informative bound: W4A4 with Hadamard stays within a few percent of
    the unquantized product on outlier-heavy activations."""
    from bit_quantized_linear_block_b200 import synthetic as S
    x, w = S.single_linear()
    xb, wb = S.bf16_bits(x)[:32], S.bf16_bits(w)[:64]
    wq = O.prepare_weights_nvfp4(wb)
    r = O.forward(xb, wq, O.ROUTE_NVFP4)
    exact = O.bf16_bits_to_f32(xb).astype(np.float64) @ O.bf16_bits_to_f32(wb).astype(np.float64).T
    assert np.abs(r - exact).max() / np.abs(exact).max() < 0.2
    r8 = O.forward(xb, wq, O.ROUTE_INT8)
    assert np.abs(r8 - exact).max() / np.abs(exact).max() < np.abs(r - exact).max() / np.abs(exact).max()
