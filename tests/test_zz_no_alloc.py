"""The router entry point that allocates nothing, qlinear_route_noalloc, is
meant for callers that cannot allocate device memory or pass a workspace
(an engine or plugin host that owns all device memory, a loop that must not
call cudaMalloc).  It keeps its scratch in a static device array shared by
every call, so this test calls it twice in a row, on different inputs, and
checks each result against the workspace-based qlinear_route and against
the oracle's Gamma and route (6Bit-Diffusion, Methodology B.1) within the
tolerance the other router tests use.  The file is named to be collected
last."""
import ctypes as C

import numpy as np
import pytest
import torch

from oracle import qlinear_oracle as O

pytestmark = pytest.mark.gpu


def _entry():
    from bit_quantized_linear_block_b200 import qlinear as ql
    f = ql.lib.qlinear_route_noalloc
    f.restype = C.c_int
    f.argtypes = [C.c_void_p, C.c_void_p, C.c_int64, C.c_float, C.c_void_p, C.c_void_p, C.c_void_p]
    return ql, f


def test_route_noalloc_matches_route_on_two_calls():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    ql, f = _entry()
    from bit_quantized_linear_block_b200 import synthetic as S
    stream = torch.cuda.current_stream()
    cases = [(4096 * 1920 + 5, 0.2), (17776 * 1920, 0.003)]   # ragged sensitive block, stable block
    for numel, sigma in cases:
        rng = np.random.default_rng(numel)
        x = rng.standard_normal(numel).astype(np.float32)
        y = x + rng.standard_normal(numel).astype(np.float32) * np.float32(sigma)
        xd, yd = S.to_bf16(x).cuda(), S.to_bf16(y).cuda()
        g_ref, r_ref = ql.qlinear_route(xd, yd, 0.05)
        g = torch.full((1,), -1.0, dtype=torch.float64, device="cuda")
        r = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        st = f(xd.data_ptr(), yd.data_ptr(), numel, 0.05, g.data_ptr(), r.data_ptr(), stream.cuda_stream)
        assert st == 0, ql.lib.qlinear_status_string(st)
        torch.cuda.synchronize()
        assert float(g.item()) == pytest.approx(float(g_ref.item()), rel=1e-12)
        assert int(r.item()) == int(r_ref.item())
        g_or = O.dmpq_gamma(S.bf16_bits(xd.cpu()), S.bf16_bits(yd.cpu()))
        assert abs(g_or - 0.05) / 0.05 > 1e-9
        assert float(g.item()) == pytest.approx(g_or, rel=1e-12)
        assert int(r.item()) == O.dmpq_route(g_or, 0.05)
    assert int(r_ref.item()) == 0 and ql.qlinear_device_status() == 0
