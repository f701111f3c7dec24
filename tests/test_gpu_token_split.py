"""GPU parity of the token-split layer (a block's rows split across ranks).

The ranks are emulated on one GPU by contiguous row slices of one block,
run one after another, so no kernel waits on another; the exchange step
(an all-reduce over ranks) is the elementwise sum or max over the slices'
scalars, taken on the device.  The split must reproduce the unsplit block:
the same tensor amax, bit-identical quantized codes and scales, the same
route with Gamma equal to fp64 rounding, and output rows within one bf16
unit in the last place of the unsplit output."""
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


@pytest.fixture(scope="module")
def SH(ql):
    from bit_quantized_linear_block_b200 import sharded
    return sharded


def _np(t):
    return t.detach().cpu().numpy()


def _within_one_bf16_ulp(a, b):
    """bf16 keeps 8 significant bits: one unit in the last place is at most
    2^-7 of the magnitude."""
    a, b = a.float(), b.float()
    return bool(((a - b).abs() <= 2.0 ** -7 * torch.maximum(a.abs(), b.abs())).all())


# ---------------------------------------------------------------- Gamma and the route

@pytest.mark.parametrize("m,k,world", [(301, 1920, 2), (301, 1920, 3), (3, 384, 5), (1000, 640, 8)])
def test_token_split_gamma_matches_unsplit(ql, SH, m, k, world):
    rng = np.random.default_rng(m + world)
    x = rng.standard_normal((m, k)).astype(np.float32)
    y = x + rng.standard_normal((m, k)).astype(np.float32) * 0.04
    xt, yt = S.to_bf16(x), S.to_bf16(y)
    xc, yc = xt.cuda(), yt.cuda()
    g_full, r_full = ql.qlinear_route(xc, yc, 0.05)
    parts = [ql.qlinear_gamma_sums(xc[lo:hi], yc[lo:hi])
             for lo, hi in (SH.shard_rows(m, world, r) for r in range(world))]
    sums = torch.stack(parts).sum(0).contiguous()          # the all-reduce(sum)
    g, r = ql.qlinear_route_from_sums(sums, 0.05)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    g_ref = O.dmpq_gamma(S.bf16_bits(xt), S.bf16_bits(yt))
    assert float(_np(g)[0]) == pytest.approx(float(_np(g_full)[0]), rel=1e-12)
    assert float(_np(g)[0]) == pytest.approx(g_ref, rel=1e-12)
    assert int(_np(r)[0]) == int(_np(r_full)[0]) == O.dmpq_route(g_ref, 0.05)


def test_token_split_gamma_closed_forms(ql, SH):
    """Values on a 1/16 grid: every fp64 partial sum is exact, so Gamma is
    exact under any split; an all-zero input gives +inf and INT8."""
    rng = np.random.default_rng(11)
    x = rng.integers(-15, 16, size=(64, 128)).astype(np.float32) / 16
    xc = S.to_bf16(x).cuda()
    for y, want in [(x, 0.0), (x * np.float32(1.125), 0.125), (-x, 2.0)]:
        yc = S.to_bf16(y).cuda()
        sums = (ql.qlinear_gamma_sums(xc[:23], yc[:23]) + ql.qlinear_gamma_sums(xc[23:], yc[23:])).contiguous()
        g, r = ql.qlinear_route_from_sums(sums, 0.125)
        torch.cuda.synchronize()
        assert float(_np(g)[0]) == want
        assert int(_np(r)[0]) == (1 if want > 0.125 else 0)
    z = torch.zeros((8, 128), dtype=torch.bfloat16, device="cuda")
    g, r = ql.qlinear_route_from_sums(ql.qlinear_gamma_sums(z, z), 0.05)
    torch.cuda.synchronize()
    assert float(_np(g)[0]) == float("inf") and int(_np(r)[0]) == 1


def test_token_split_route_without_a_process_group(ql, SH):
    x, y, _ = S.dmpq_block_pair(3, m=512)
    xc, yc = x.cuda(), y.cuda()
    g1, r1 = SH.token_split_route(xc, yc, 0.05)
    g2, r2 = ql.qlinear_route(xc, yc, 0.05)
    torch.cuda.synchronize()
    assert float(_np(g1)[0]) == pytest.approx(float(_np(g2)[0]), rel=1e-12)
    assert int(_np(r1)[0]) == int(_np(r2)[0])


# ---------------------------------------------------------------- forward

def _weights(ql, kind, n, k):
    if kind == "qarvd":
        w = S.weights(n, k, 0.02, 3, n + k, outlier_frac=0.05, outlier_scale=20.0)
        return w, ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_QARVD_INT4, hadamard=False)
    w = S.weights(n, k, 0.02, 6, n + k)
    fmt = ql.QL_W_NVFP4_DECOMP if kind == "decomp" else ql.QL_W_NVFP4
    return w, ql.qlinear_prepare_weights(w.cuda(), fmt, hadamard=True)


ROUTES = {"nvfp4": 0, "decomp": 0, "int8": 1, "int6": 5, "qarvd": 2, "qarvd_int6": 7}


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("kind", list(ROUTES))
def test_token_split_forward_matches_unsplit(ql, SH, kind, world):
    m, n, k = 301, 384, 640
    x = S.activations_fixed_outliers(m, k, 8, 50.0, m + world, 1)
    xc = x.cuda()
    _, pw = _weights(ql, kind.split("_")[0], n, k)
    route = ROUTES[kind]
    y_full = ql.qlinear_forward(xc, pw, route)
    act, had, needs_amax = SH.activation_format(pw, route)
    slices = [SH.shard_rows(m, world, r) for r in range(world)]
    if needs_amax:
        amax = torch.stack([ql.qlinear_tensor_amax(xc[lo:hi], had) for lo, hi in slices]).amax(0)  # all-reduce(max)
        assert torch.equal(amax, ql.qlinear_tensor_amax(xc, had))
        wq = pw if pw.fmt == ql.QL_W_QARVD_INT4 else None
        q_full = ql.qlinear_quantize_act(xc, act, had, w=wq)
        for lo, hi in slices:
            q = ql.qlinear_quantize_act(xc[lo:hi], act, had, w=wq, amax_in=amax)
            assert torch.equal(q["codes"], q_full["codes"][lo:hi])
            assert torch.equal(q["scales"], q_full["scales"])
            if q_full["sf_rowmajor"] is not None:
                assert torch.equal(q["sf_rowmajor"], q_full["sf_rowmajor"][lo:hi])
        y = torch.cat([SH.forward_with_amax(xc[lo:hi], pw, route, amax) for lo, hi in slices])
    else:
        y = torch.cat([SH.token_split_forward(xc[lo:hi], pw, route) for lo, hi in slices])
    y_one = SH.token_split_forward(xc, pw, route)          # no process group: one rank
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    assert torch.isfinite(y.float()).all()
    assert _within_one_bf16_ulp(y, y_full)
    assert _within_one_bf16_ulp(y_one, y_full)


def test_token_split_decomposed_weights_need_the_nvfp4_route(ql, SH):
    _, pw = _weights(ql, "decomp", 64, 128)
    with pytest.raises(ValueError):
        SH.activation_format(pw, ql.QL_ROUTE_INT8)
