"""The forward with the route in device memory (qlinear_forward_routed):
for every route value it writes exactly what the host-routed forward
writes, a value no route has leaves the output alone, and inside one
captured CUDA graph the route written by the router steers it (6Bit-
Diffusion, Methodology B.1: Gamma of the previous step routes the block)."""
import numpy as np
import pytest
import torch

from bit_quantized_linear_block_b200 import synthetic as S

pytestmark = pytest.mark.gpu


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
    for r in (ql.QL_ROUTE_NVFP4, ql.QL_ROUTE_INT8, ql.QL_ROUTE_BF16):
        route.fill_(r)
        y = ql.qlinear_forward_routed(x, pw, route, ws=ws)
        y_host = ql.qlinear_forward(x, pw, r)
        torch.cuda.synchronize()
        assert ql.qlinear_device_status() == 0
        assert torch.equal(y, y_host), r
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
    for src, want in ((stable, ql.QL_ROUTE_NVFP4), (sensitive, ql.QL_ROUTE_INT8), (stable, ql.QL_ROUTE_NVFP4)):
        bout.copy_(src)
        y.fill_(0)
        g.replay()
        torch.cuda.synchronize()
        assert int(route.item()) == want
        assert torch.equal(y, ql.qlinear_forward(x, pw, want)), want
    assert ql.qlinear_device_status() == 0
    del g
