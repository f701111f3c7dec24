"""The forward with the route in device memory (qlinear_forward_routed):
for every route value it writes exactly what the host-routed forward
writes and what the oracle computes for that route, a value no route has
leaves the output alone, and inside one captured CUDA graph the route
written by the router is the oracle's route for that block's input/output
pair and steers the forward to the oracle's product (6Bit-Diffusion,
Methodology B.1: Gamma of the previous step routes the block)."""
import numpy as np
import pytest
import torch

from oracle import qlinear_oracle as O
from bit_quantized_linear_block_b200 import synthetic as S

pytestmark = pytest.mark.gpu


def excess_err(y, r):
    """Error beyond the bf16 rounding of the output (2^-8 of the magnitude),
    relative to max|r|.  Every product on these routes is exact and the
    accumulation is fp32, so only rounding far below 1e-5 remains."""
    ex = np.maximum(0.0, np.abs(y - r) - 2.0 ** -8 * np.maximum(np.abs(y), np.abs(r)))
    return float(ex.max() / max(np.abs(r).max(), 1e-30))


def _oracle_route_output(xb, wb, wq, route, rows):
    """The oracle's output of one route on the given rows (fp64)."""
    if route == O.ROUTE_NVFP4 or route == O.ROUTE_INT8:
        return O.forward(xb, wq, route, rows=rows)
    return O.gemm_bf16(xb, wb, rows=rows)


def _rows(m, seed):
    if m <= 512:
        return np.arange(m)
    return np.unique(np.r_[np.random.default_rng(seed).choice(m, 256, replace=False), m - 1])


@pytest.fixture(scope="module")
def ql():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from bit_quantized_linear_block_b200 import qlinear
    return qlinear


@pytest.mark.parametrize("expand", [False, True])
@pytest.mark.parametrize("m,n,k", [(300, 384, 640), (1000, 5760, 1920), (64, 640, 256)])
def test_routed_forward_matches_the_host_route(ql, m, n, k, expand):
    x = S.activations_fixed_outliers(m, k, 8, 50.0, m + k, 1).cuda()
    w = S.weights(n, k, 0.02, 6, m + n)
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4, hadamard=True, expand_f16=expand, keep_bf16=True)
    route = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(ql.lib.qlinear_forward_routed_ws_bytes(m, ql.C.byref(pw.desc)), dtype=torch.uint8, device="cuda")
    xb, wb = S.bf16_bits(x.cpu()), S.bf16_bits(w)
    wq = O.prepare_weights_nvfp4(wb)
    rows = _rows(m, m + n)
    assert (ql.QL_ROUTE_NVFP4, ql.QL_ROUTE_INT8) == (O.ROUTE_NVFP4, O.ROUTE_INT8)
    for r in (ql.QL_ROUTE_NVFP4, ql.QL_ROUTE_INT8, ql.QL_ROUTE_BF16):
        route.fill_(r)
        y = ql.qlinear_forward_routed(x, pw, route, ws=ws)
        y_host = ql.qlinear_forward(x, pw, r)
        torch.cuda.synchronize()
        assert ql.qlinear_device_status() == 0
        assert torch.equal(y, y_host), r
        # and against the oracle's product on that route, element by element
        yn = y.float().cpu().numpy()[rows].astype(np.float64)
        assert np.isfinite(yn).all()
        assert excess_err(yn, _oracle_route_output(xb, wb, wq, r, rows)) <= 1e-5, r
    route.fill_(7)                                   # no route: nothing runs
    y = torch.full((m, n), 3.0, dtype=torch.bfloat16, device="cuda")
    ql.qlinear_forward_routed(x, pw, route, Y=y, ws=ws)
    torch.cuda.synchronize()
    assert ql.qlinear_device_status() == 0
    assert bool((y == 3.0).all())


def test_router_steers_the_routed_forward_inside_one_graph(ql):
    m, k, n = 512, 1920, 768
    x = S.activations_fixed_outliers(m, k, 8, 50.0, 5, 1).cuda()
    w = S.weights(n, k, 0.02, 6, 9)
    pw = ql.qlinear_prepare_weights(w.cuda(), ql.QL_W_NVFP4, hadamard=True, expand_f16=True)
    rng = np.random.default_rng(0)
    base = rng.standard_normal((m, k)).astype(np.float32)
    bin_ = S.to_bf16(base).cuda()
    stable = S.to_bf16(base + 0.01 * rng.standard_normal((m, k)).astype(np.float32)).cuda()    # Gamma ~ 0.01
    sensitive = S.to_bf16(base + 0.3 * rng.standard_normal((m, k)).astype(np.float32)).cuda()  # Gamma ~ 0.3
    bout = torch.empty_like(bin_)
    gamma = torch.empty(1, dtype=torch.float64, device="cuda")
    route = torch.empty(1, dtype=torch.int32, device="cuda")
    rws = torch.zeros(ql.lib.qlinear_route_ws_bytes(bin_.numel()), dtype=torch.uint8, device="cuda")
    fws = torch.zeros(ql.lib.qlinear_forward_routed_ws_bytes(m, ql.C.byref(pw.desc)), dtype=torch.uint8,
                      device="cuda")
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    bout.copy_(stable)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):            # warm-up outside the capture
        ql.qlinear_route(bin_, bout, 0.05, gamma=gamma, route=route, ws=rws)
        ql.qlinear_forward_routed(x, pw, route, Y=y, ws=fws)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ql.qlinear_route(bin_, bout, 0.05, gamma=gamma, route=route, ws=rws)
        ql.qlinear_forward_routed(x, pw, route, Y=y, ws=fws)
    xb, wb = S.bf16_bits(x.cpu()), S.bf16_bits(w)
    wq = O.prepare_weights_nvfp4(wb)
    in_bits = S.bf16_bits(bin_.cpu())
    for src, want in ((stable, ql.QL_ROUTE_NVFP4), (sensitive, ql.QL_ROUTE_INT8), (stable, ql.QL_ROUTE_NVFP4)):
        g_ref = O.dmpq_gamma(in_bits, S.bf16_bits(src.cpu()))
        assert abs(g_ref - 0.05) / 0.05 > 1e-9            # away from the threshold
        assert O.dmpq_route(g_ref, 0.05) == want
        bout.copy_(src)
        y.fill_(0)
        g.replay()
        torch.cuda.synchronize()
        assert float(gamma.item()) == pytest.approx(g_ref, rel=1e-12)
        assert int(route.item()) == want
        assert torch.equal(y, ql.qlinear_forward(x, pw, want)), want
        ref = O.forward(xb, wq, O.dmpq_route(g_ref, 0.05))
        assert excess_err(y.float().cpu().numpy().astype(np.float64), ref) <= 1e-5, want
    assert ql.qlinear_device_status() == 0
    del g
