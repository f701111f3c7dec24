"""GPU parity at the full workload sizes: the single linear, the
CogVideoX-2B block linears, the DMPQ routing sweep, the CogVideoX-5B Q-ARVD
linears and the Wan-14B linears.  Quantized codes, scales, masks and routes
are compared in full (the oracle runs over row chunks with the tensor scale
of the whole tensor); GEMM outputs on 1024 seeded sample rows that include
the last (ragged) M tile."""
import functools

import numpy as np
import pytest
import torch

from oracle import qlinear_oracle as O
from bit_quantized_linear_block_b200 import synthetic as S

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

CHUNK = 4096


@pytest.fixture(scope="module")
def ql():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from bit_quantized_linear_block_b200 import qlinear
    return qlinear


def _np(t):
    return t.detach().cpu().numpy()


def sample_rows(m, n=1024, seed=0):
    rng = np.random.default_rng(seed)
    base = rng.choice(m, size=min(n, m), replace=False)
    tail = np.arange(max(0, m - 120), m)          # rows of the last, partial 128-row tile
    return np.unique(np.concatenate([base, tail]))


def normwise_err(y, r):
    return float(np.abs(y - r).max() / max(np.abs(r).max(), 1e-30))


def excess_err(y, r):
    ex = np.maximum(0.0, np.abs(y - r) - 2.0 ** -8 * np.maximum(np.abs(y), np.abs(r)))
    return float(ex.max() / max(np.abs(r).max(), 1e-30))


def oracle_rotated_amax(bits, hadamard=True):
    amax = np.float32(0)
    for i in range(0, bits.shape[0], CHUNK):
        x = O.bf16_bits_to_f32(bits[i:i + CHUNK])
        h = O.block_hadamard(x) if hadamard else x
        amax = max(amax, np.float32(np.max(np.abs(h))))
    return amax


def check_nvfp4_quant_full(ql, x, hadamard=True):
    """GPU activation quantizer vs the oracle over all rows; returns the
    oracle's (packed, sb, g) of the sampled rows for the GEMM check."""
    bits = S.bf16_bits(x)
    m, k = bits.shape
    g = O.nvfp4_tensor_scale(np.array([oracle_rotated_amax(bits, hadamard)], np.float32))
    q = ql.qlinear_quantize_act(x.cuda(), ql.QL_ROUTE_NVFP4, hadamard=hadamard)
    torch.cuda.synchronize()
    assert _np(q["scales"])[0] == g
    codes, sfr = _np(q["codes"]), _np(q["sf_rowmajor"])
    sfm = _np(ql.sf_mma_to_rowmajor(q["sf_mma"], m, k))
    for i in range(0, m, CHUNK):
        x32 = O.bf16_bits_to_f32(bits[i:i + CHUNK])
        packed, sb, _ = O.nvfp4_quantize(O.block_hadamard(x32) if hadamard else x32, g)
        assert np.array_equal(codes[i:i + CHUNK], packed), f"codes differ in rows {i}.."
        assert np.array_equal(sfr[i:i + CHUNK], sb) and np.array_equal(sfm[i:i + CHUNK], sb)
    return g


def check_nvfp4_weights(ql, w, hadamard=True):
    n, k = w.shape
    ref = O.prepare_weights_nvfp4(S.bf16_bits(w), hadamard=hadamard)
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4, hadamard=hadamard)
    torch.cuda.synchronize()
    assert _np(pw.view("gscale", torch.float32, 1))[0] == ref["g"]
    codes = _np(pw.view("codes", torch.uint8, n * k // 2)).reshape(n, k // 2)
    assert np.array_equal(codes, ref["packed"])
    sf = pw.view("sf", torch.uint8, ql.lib.qlinear_sf_bytes(n, k))
    assert np.array_equal(_np(ql.sf_mma_to_rowmajor(sf, n, k)), ref["sb"])
    return pw, ref


def w4a4_reference_rows(xbits, g_x, wref, rows, hadamard=True):
    x32 = O.bf16_bits_to_f32(xbits[rows])
    packed, sb, _ = O.nvfp4_quantize(O.block_hadamard(x32) if hadamard else x32, g_x)
    return O.gemm_w4a4(packed, sb, g_x, wref["packed"], wref["sb"], wref["g"])


def run_w4a4_linear(ql, x, w, seed):
    g_x = check_nvfp4_quant_full(ql, x)
    pw, wref = check_nvfp4_weights(ql, w)
    y = ql.qlinear_forward(x.cuda(), pw, ql.QL_ROUTE_NVFP4)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    rows = sample_rows(x.shape[0], seed=seed)
    ref = w4a4_reference_rows(S.bf16_bits(x), g_x, wref, rows)
    yn = _np(y.float())[rows].astype(np.float64)
    assert np.isfinite(yn).all()
    err = normwise_err(yn, ref)
    assert err <= 1e-2, err
    return err


# ---------------------------------------------------------------- configs

def test_single_linear_full_output(ql):
    x, w = S.single_linear(seed=0)
    xb, wb = S.bf16_bits(x), S.bf16_bits(w)
    ref = O.forward(xb, O.prepare_weights_nvfp4(wb), O.ROUTE_NVFP4)
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4, hadamard=True)
    y = ql.qlinear_forward(x.cuda(), pw, ql.QL_ROUTE_NVFP4)
    torch.cuda.synchronize()
    assert normwise_err(_np(y.float()).astype(np.float64), ref) <= 1e-2


@pytest.mark.parametrize("name", [l.name for l in S.COGVIDEOX_2B])
def test_cogvideox2b_block_linear(ql, name):
    lin = [l for l in S.COGVIDEOX_2B if l.name == name][0]
    x, w = S.cogvideox2b_linear(lin)
    run_w4a4_linear(ql, x, w, seed=1)


def test_dmpq_routing_sweep_and_routed_ffn_up(ql):
    w = S.dmpq_ffn_up_weights()
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4, hadamard=True)
    wref = O.prepare_weights_nvfp4(S.bf16_bits(w))
    routes = []
    checked = set()
    for b in range(30):
        x, y, sigma = S.dmpq_block_pair(b)
        xb, yb = S.bf16_bits(x), S.bf16_bits(y)
        g_ref = O.dmpq_gamma(xb, yb)
        assert abs(g_ref - 0.05) / 0.05 > 1e-9
        xd = x.cuda()
        g, r = ql.qlinear_route(xd, y.cuda(), 0.05)
        torch.cuda.synchronize()
        assert float(g.item()) == pytest.approx(g_ref, rel=1e-12)
        route = int(r.item())
        assert route == O.dmpq_route(g_ref, 0.05)
        routes.append(route)
        if route in checked:
            continue
        checked.add(route)
        # the routed FFN up-projection of this block's input, full size
        out = ql.qlinear_forward(xd, pw, route)
        torch.cuda.synchronize()
        assert ql.qlinear_device_status() == 0
        rows = sample_rows(x.shape[0], seed=b)
        ref = O.forward(xb, wref, route, rows=rows)
        yn = _np(out.float())[rows].astype(np.float64)
        if route == O.ROUTE_INT8:
            q = ql.qlinear_quantize_act(xd, ql.QL_ROUTE_INT8, hadamard=True)
            codes, scales = _np(q["codes"]), _np(q["scales"])
            for i in range(0, x.shape[0], CHUNK):      # every code and token scale
                qo, so = O.int8_per_token(O.block_hadamard(O.bf16_bits_to_f32(xb[i:i + CHUNK])))
                assert np.array_equal(codes[i:i + CHUNK], qo) and np.array_equal(scales[i:i + CHUNK], so)
            assert excess_err(yn, ref) <= 1e-5
        else:
            check_nvfp4_quant_full(ql, x)
            assert normwise_err(yn, ref) <= 1e-2
            assert excess_err(yn, ref) <= 1e-5
    assert checked == {0, 1}, routes       # the sweep exercises both routes


@functools.lru_cache(maxsize=1)
def _cogvideox5b_case(name):
    """Inputs and the oracle's packed weights of one linear (shared by both weight forms)."""
    lin = [l for l in S.COGVIDEOX_5B if l.name == name][0]
    x, w = S.cogvideox5b_qarvd_linear(lin)
    return lin, x, w, O.qarvd_pack(S.bf16_bits(w), 3.5, 2.0)


@pytest.mark.parametrize("name", [l.name for l in S.COGVIDEOX_5B])
@pytest.mark.parametrize("expand", [False, True])
def test_cogvideox5b_qarvd_linear(ql, name, expand):
    lin, x, w, pk = _cogvideox5b_case(name)
    zs = pk["zscore"][np.isfinite(pk["zscore"])]
    assert np.all(np.abs(zs - 3.5) > 3.5e-9)
    assert np.all(np.abs(pk["norms"] - 2.0 * pk["median"]) > 1e-9 * pk["median"])
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_QARVD_INT4, hadamard=False, expand_i8=expand)
    torch.cuda.synchronize()
    n, k, kp = lin.n, lin.k, pw.desc.Kp
    assert np.array_equal(_np(pw.view("outlier_mask", torch.uint8, k)).astype(bool), pk["mask"])
    assert np.array_equal(_np(pw.view("perm", torch.int32, k)), pk["perm"])
    assert np.array_equal(_np(pw.view("s_norm", torch.float32, n)), pk["s_norm"])
    assert np.array_equal(_np(pw.view("s_out", torch.float32, n)), pk["s_out"])
    want = np.zeros((n, kp), np.int8)
    want[:, :pk["codes"].shape[1]] = pk["codes"]
    got = _np(pw.view("codes", torch.uint8, n * kp // 2)).reshape(n, kp // 2)
    assert np.array_equal(got, O.pack_int4(want))
    if expand:
        assert np.array_equal(_np(pw.view("w8", torch.int8, n * kp)).reshape(n, kp), want)
    xb = S.bf16_bits(x)
    xd = x.cuda()
    q = ql.qlinear_quantize_act(xd, ql.QL_ACT_INT8_TENSOR, hadamard=False, w=pw)
    y = ql.qlinear_forward(xd, pw)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    amax = oracle_rotated_amax(xb, hadamard=False)
    _, sx = O.int8_per_tensor(np.array([[amax]], np.float32))
    assert _np(q["scales"])[0] == sx
    codes = _np(q["codes"])
    lay = (pk["perm"], pk["k_norm"], pk["k_norm_pad"], pk["n_out"], pk["k_out_pad"])
    # every activation code, in row chunks (the quantizer does not depend on
    # the weight form, so the int8-copy variant checks the GEMM only)
    for i in (range(0, x.shape[0], CHUNK) if not expand else ()):
        qx, _ = O._int8_from_amax(O.bf16_bits_to_f32(xb[i:i + CHUNK]), np.array([[amax]], np.float32))
        qxp = O.qarvd_permute_activations(qx, *lay)
        assert np.array_equal(codes[i:i + CHUNK, :qxp.shape[1]], qxp)
        assert not codes[i:i + CHUNK, qxp.shape[1]:].any()
    rows = sample_rows(x.shape[0], seed=3)
    qx, _ = O._int8_from_amax(O.bf16_bits_to_f32(xb[rows]), np.array([[amax]], np.float32))
    qxp = O.qarvd_permute_activations(qx, *lay)
    ref = O.gemm_qarvd(qxp, sx, pk["codes"], pk["s_norm"], pk["s_out"], pk["k_norm_pad"])
    assert excess_err(_np(y.float())[rows].astype(np.float64), ref) <= 1e-5


@pytest.mark.parametrize("name", [l.name for l in S.WAN_14B])
def test_wan14b_linear(ql, name):
    lin = [l for l in S.WAN_14B if l.name == name][0]
    x, w = S.wan14b_linear(lin)
    run_w4a4_linear(ql, x, w, seed=4)


def test_cogvideox2b_ffn_down_decomposed(ql):
    """Activation decomposition (SemanticDialect, Methodology 2.2) on the
    CogVideoX-2B FFN-down linear ([17776, 7680] -> 1920, K' = 15360): every
    code and scale of both levels bit-exact over all rows, the product on
    sampled rows within the W4A4 tolerance."""
    lin = [l for l in S.COGVIDEOX_2B if l.name == "ffn_down"][0]
    x, w = S.cogvideox2b_linear(lin)
    bits = S.bf16_bits(x)
    m, k = bits.shape
    g = O.nvfp4_tensor_scale(np.array([oracle_rotated_amax(bits)], np.float32))
    xd = x.cuda()
    q = ql.qlinear_quantize_act(xd, ql.QL_ACT_NVFP4_DECOMP, hadamard=True)
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4_DECOMP, hadamard=True)
    y = ql.qlinear_forward(xd, pw, ql.QL_ROUTE_NVFP4)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    assert _np(q["scales"])[0] == g
    codes, sfr = _np(q["codes"]), _np(q["sf_rowmajor"])
    for i in range(0, m, CHUNK):
        packed, sb, _ = O.nvfp4_decompose(O.block_hadamard(O.bf16_bits_to_f32(bits[i:i + CHUNK])), g)
        assert np.array_equal(codes[i:i + CHUNK], packed), f"codes differ in rows {i}.."
        assert np.array_equal(sfr[i:i + CHUNK], sb)
    wref = O.decompose_weights(O.prepare_weights_nvfp4(S.bf16_bits(w)))
    rows = sample_rows(m, seed=7)
    packed, sb, _ = O.nvfp4_decompose(O.block_hadamard(O.bf16_bits_to_f32(bits[rows])), g)
    ref = O.gemm_w4a4(packed, sb, g, wref["packed"], wref["sb"], wref["g"])
    yn = _np(y.float())[rows].astype(np.float64)
    assert np.isfinite(yn).all() and normwise_err(yn, ref) <= 1e-2
