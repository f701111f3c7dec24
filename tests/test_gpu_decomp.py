"""GPU parity of the activation decomposition (SemanticDialect, Methodology
2.2): NVFP4 codes and scales of h and of its residual bit-exact against the
oracle, the weights repeated along K bit-exact, and the decomposed forward
within the W4A4 tolerance (and closer to the exact product than plain NVFP4)."""
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


def _x(m, k, seed):
    return S.activations_fixed_outliers(m, k, 8, 50.0, seed, 1)


def normwise_err(y, r):
    return float(np.abs(y - r).max() / max(np.abs(r).max(), 1e-30))


@pytest.mark.parametrize("m,k", [(1, 128), (77, 384), (256, 1920), (300, 640), (129, 1024)])
@pytest.mark.parametrize("hadamard", [True, False])
def test_decomposed_quantize_bit_exact(ql, m, k, hadamard):
    x = _x(m, k, seed=m + 3 * k)
    xb = S.bf16_bits(x)
    h = O.block_hadamard(O.bf16_bits_to_f32(xb)) if hadamard else O.bf16_bits_to_f32(xb)
    packed, sb, g = O.nvfp4_decompose(h)
    q = ql.qlinear_quantize_act(x.cuda(), ql.QL_ACT_NVFP4_DECOMP, hadamard=hadamard)
    torch.cuda.synchronize()
    assert _np(q["scales"])[0] == g
    assert np.array_equal(_np(q["sf_rowmajor"]), sb)
    assert np.array_equal(_np(ql.sf_mma_to_rowmajor(q["sf_mma"], m, 2 * k)), sb)
    mpad = (m + 127) // 128 * 128
    assert not _np(ql.sf_mma_to_rowmajor(q["sf_mma"], mpad, 2 * k))[m:].any()
    assert np.array_equal(_np(q["codes"]), packed)
    # the first half is the plain NVFP4 quantization
    q1 = ql.qlinear_quantize_act(x.cuda(), ql.QL_ROUTE_NVFP4, hadamard=hadamard)
    assert np.array_equal(_np(q1["codes"]), _np(q["codes"])[:, :k // 2])


def test_decomposed_quantize_zero_and_exact_blocks(ql):
    """All-zero rows, a subnormal-scale block and blocks exact at level one
    (zero residual: +0 codes and zero scales in the second half)."""
    x = np.zeros((130, 256), np.float32)
    x[0, 0] = 2688.0                                                # tensor amax 6 * 448: g = 1
    x[3, :16] = np.array([6, 4, -3, 2, 1.5, -1, 0.5, 0] * 2, np.float32) * 2.0 ** 3   # exact at level one
    x[5, 16:32] = 1e-3
    x[9, 64:80] = -0.0
    xt = S.to_bf16(x)
    packed, sb, g = O.nvfp4_decompose(O.bf16_bits_to_f32(S.bf16_bits(xt)))
    q = ql.qlinear_quantize_act(xt.cuda(), ql.QL_ACT_NVFP4_DECOMP, hadamard=False)
    torch.cuda.synchronize()
    assert _np(q["scales"])[0] == g
    assert np.array_equal(_np(q["sf_rowmajor"]), sb)
    assert np.array_equal(_np(q["codes"]), packed)
    assert not packed[3, 128:].any() and not sb[3, 16:].any()    # zero residual where level one is exact


@pytest.mark.parametrize("n,k", [(1920, 1920), (640, 384), (16, 128)])
def test_prepare_weights_decomp_bit_exact(ql, n, k):
    w = S.weights(n, k, 0.02, 5, n + k)
    ref = O.decompose_weights(O.prepare_weights_nvfp4(S.bf16_bits(w), hadamard=True))
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4_DECOMP, hadamard=True)
    torch.cuda.synchronize()
    codes = _np(pw.view("codes", torch.uint8, n * k)).reshape(n, k)
    sf = pw.view("sf", torch.uint8, ql.lib.qlinear_sf_bytes(n, 2 * k))
    assert _np(pw.view("gscale", torch.float32, 1))[0] == ref["g"]
    assert np.array_equal(_np(ql.sf_mma_to_rowmajor(sf, n, 2 * k)), ref["sb"])
    assert np.array_equal(codes, ref["packed"])


@pytest.mark.parametrize("m,n,k", [(256, 1920, 1920), (300, 384, 640), (129, 640, 384), (1, 192, 128),
                                   (1000, 5760, 1920)])
def test_forward_decomposed_parity(ql, m, n, k):
    x = _x(m, k, seed=m * 5 + n)
    w = S.weights(n, k, 0.02, 6, m + n + k)
    xb, wb = S.bf16_bits(x), S.bf16_bits(w)
    wq = O.prepare_weights_nvfp4(wb)
    rows = np.arange(m) if m <= 512 else np.unique(np.r_[np.random.default_rng(1).choice(m, 256, replace=False), m - 1])
    ref = O.forward(xb, wq, O.ROUTE_NVFP4_DECOMP, rows=rows)
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4_DECOMP, hadamard=True)
    xc = x.cuda()
    y = ql.qlinear_forward(xc, pw, ql.QL_ROUTE_NVFP4)
    q = ql.qlinear_quantize_act(xc, ql.QL_ACT_NVFP4_DECOMP, hadamard=True)
    y2 = ql.qlinear_gemm(ql.QL_ACT_NVFP4_DECOMP, q, m, pw)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    yn = _np(y.float())[rows].astype(np.float64)
    assert np.isfinite(yn).all()
    assert normwise_err(yn, ref) <= 1e-2
    assert torch.equal(y, y2)
    exact = O.bf16_bits_to_f32(xb)[rows].astype(np.float64) @ O.bf16_bits_to_f32(wb).astype(np.float64).T
    plain = O.forward(xb, wq, O.ROUTE_NVFP4, rows=rows)
    assert normwise_err(yn, exact) < normwise_err(plain, exact)     # the residual pays off


def test_decomposed_weights_reject_other_routes(ql):
    w = S.weights(64, 128, 0.02, 6, 1)
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4_DECOMP, hadamard=True)
    x = _x(8, 128, seed=2).cuda()
    with pytest.raises(ql.QLinearError):
        ql.qlinear_forward(x, pw, ql.QL_ROUTE_INT8)
    q = ql.qlinear_quantize_act(x, ql.QL_ROUTE_NVFP4, hadamard=True)
    with pytest.raises(ql.QLinearError):
        ql.qlinear_gemm(ql.QL_ROUTE_NVFP4, q, 8, pw)
