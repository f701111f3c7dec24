"""GPU parity of the temporal delta cache (6Bit-Diffusion, Methodology B.2
TDC and B.3 PDR) against the oracle's state machine: the device decides
every step (skip or compute, and the route) and the oracle must agree; the
skipped outputs and the cached deltas are bit-exact, Gamma and E agree to
1e-12 (fp64 sums in another order)."""
import numpy as np
import pytest
import torch

from oracle import tdc_oracle as T
from bit_quantized_linear_block_b200 import synthetic as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ql():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from bit_quantized_linear_block_b200 import qlinear
    return qlinear


def _bits(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def _from_bits(b):
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16)


def _close(a, b):
    if np.isinf(a) or np.isinf(b):
        return a == b
    return abs(a - b) <= 1e-12 * max(abs(a), abs(b), 1e-300)


def _params(**kw):
    # the device holds the thresholds as fp32: give the oracle the same values
    p = dict(gamma_threshold=0.05, eps_threshold=0.1, acc_max=0.25, max_skips=3, kappa=8.0, rho_max=1.0)
    p.update(kw)
    f = {k: (float(np.float32(v)) if k != "max_skips" else int(v)) for k, v in p.items()}
    return f, T.TdcParams(**f)


@pytest.mark.parametrize("numel,kw", [
    (1001, dict(acc_max=0.05)),                    # ragged tail; the summed E caps the runs
    (8 * 40000 + 3, dict(acc_max=1.0)),            # several CTAs; the skip count caps the runs
    (17776 * 1920 // 8, dict(max_skips=1)),
    (4096, dict(eps_threshold=0.0)),               # never skips
    (5000 * 16 + 9, dict(rho_max=0.05)),           # outlier-heavy inputs every third step -> BF16 route
])
def test_tdc_sequence_matches_oracle(ql, numel, kw):
    f, prm = _params(**kw)
    cache = ql.TdcCache(numel, "cuda", **f)
    st = T.TdcState()
    rng = np.random.default_rng(numel)
    base = rng.standard_normal(numel).astype(np.float32) * 0.1
    pattern = ""
    seen_bf16 = False
    for step in range(14):
        dev = cache.state()
        want_skip = T.tdc_should_skip(st, prm)
        assert bool(dev.next_skip) == want_skip, step
        xin = rng.standard_normal(numel).astype(np.float32)
        if step % 3 == 1:
            xin[::61] *= 40.0          # one dominating value in about a quarter of the 16-blocks
        inp_bits = S.bf16_bits(S.to_bf16(xin))
        inp = _from_bits(inp_bits).cuda()
        if want_skip:
            out = ql.qlinear_tdc_skip(inp, cache)
            ref = T.tdc_apply(inp_bits, st.deltas[-1])
            T.tdc_after_skip(st)
            assert np.array_equal(_bits(out), ref)
            pattern += "S"
        else:
            assert dev.next_route == T.pdr_route(st, prm), step
            seen_bf16 = seen_bf16 or dev.next_route == T.ROUTE_BF16
            # block output: in + a slowly drifting delta, with a jump at step 9
            drift = 1.0 + 0.02 * step + (0.5 if step == 9 else 0.0)
            out_bits = S.bf16_bits(S.to_bf16(
                (T.bf16_bits_to_f32(inp_bits) + base * np.float32(drift)).astype(np.float32)))
            ql.qlinear_tdc_refresh(inp, _from_bits(out_bits).cuda(), cache)
            T.tdc_after_compute(st, inp_bits, out_bits)
            assert np.array_equal(_bits(cache.delta("latest")), st.deltas[-1])
            pattern += "C"
        dev = cache.state()
        assert _close(dev.gamma, st.gamma) and _close(dev.eps, st.eps), step
        assert dev.rho == st.rho, step                 # exact: a ratio of block counts
        assert dev.n_delta == len(st.deltas) and dev.skips == st.skips
        assert bool(dev.last_skipped) == st.last_skipped and dev.steps == step + 1
        assert _close(dev.acc, st.acc) or (dev.acc == 0 and st.acc == 0)
    assert ql.qlinear_device_status() == 0
    if kw.get("eps_threshold", 0.1) > 0:
        assert "S" in pattern and pattern.count("C") >= 3, pattern
    else:
        assert pattern == "C" * 14
    if kw.get("rho_max", 1.0) < 1.0:
        assert seen_bf16, pattern


def test_tdc_skip_without_delta_reports(ql):
    cache = ql.TdcCache(64, "cuda")
    inp = torch.ones(64, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(inp)
    assert ql.qlinear_device_status() == 0
    ql.qlinear_tdc_skip(inp, cache, out=out)
    assert ql.qlinear_device_status() == 1          # QL_ERR_INVALID_ARG, nothing written
    assert not out.any()
    st = cache.state()
    assert st.steps == 0 and st.next_skip == 0 and st.next_route == 1


def test_tdc_zero_input_gives_infinite_gamma(ql):
    f, prm = _params()
    cache = ql.TdcCache(256, "cuda", **f)
    z = torch.zeros(256, dtype=torch.bfloat16, device="cuda")
    ql.qlinear_tdc_refresh(z, z, cache)
    st = cache.state()
    assert np.isinf(st.gamma) and np.isinf(st.eps) and st.next_route == 1 and st.n_delta == 1
    ql.qlinear_tdc_refresh(z, z, cache)              # a zero previous delta: E = +inf, no skip
    st = cache.state()
    assert np.isinf(st.eps) and st.next_skip == 0 and st.n_delta == 2
