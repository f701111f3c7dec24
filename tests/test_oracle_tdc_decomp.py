"""Pins of the oracle's activation decomposition (SemanticDialect,
Methodology 2.2) and temporal delta cache with PDR's forced INT8
(6Bit-Diffusion, Methodology B.2 and B.3), against things other than the
oracle's own formulas: exact constructed round trips, an error bound of the
format, linearity of the product, torch's independent bf16 conversion,
closed forms and hand-traced policy sequences."""
import numpy as np
import pytest
import torch

from oracle import qlinear_oracle as O
from oracle import tdc_oracle as T


def _bf16(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _f32(bits):
    return O.bf16_bits_to_f32(bits)


# ---------------------------------------------------------------- decomposition

def _two_level_case(rng, rows, k):
    """h = v1 + v2 built from chosen codes: per 16-element block one element
    is +-6 at level one (and 0 at level two), the others are at most 4 at
    level one; level two is 2^-5 of level one's scale with one element at
    +-6.  Every value and sum is exact in fp32."""
    grid1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4], np.float32)
    grid2 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    nb = k // 16
    sb1 = rng.choice([0.5, 1.0, 2.0, 4.0], size=(rows, nb)).astype(np.float32)   # exact E4M3 values
    q1 = rng.choice(grid1, size=(rows, nb, 16)) * rng.choice([-1, 1], size=(rows, nb, 16))
    q2 = rng.choice(grid2, size=(rows, nb, 16)) * rng.choice([-1, 1], size=(rows, nb, 16))
    i1 = rng.integers(0, 16, size=(rows, nb))
    i2 = (i1 + 1 + rng.integers(0, 15, size=(rows, nb))) % 16
    r_, b_ = np.meshgrid(np.arange(rows), np.arange(nb), indexing="ij")
    q1[r_, b_, i1] = 6 * rng.choice([-1, 1], size=(rows, nb))
    q2[r_, b_, i1] = 0
    q2[r_, b_, i2] = 6 * rng.choice([-1, 1], size=(rows, nb))
    sb2 = sb1 / 32
    v1 = (q1 * sb1[:, :, None]).astype(np.float32)
    v2 = (q2 * sb2[:, :, None]).astype(np.float32)
    return (v1 + v2).reshape(rows, k), q1, sb1, q2, sb2


def test_decompose_recovers_both_levels_exactly():
    rng = np.random.default_rng(11)
    h, q1, sb1, q2, sb2 = _two_level_case(rng, 6, 256)
    packed, sb, g = O.nvfp4_decompose(h, g=np.float32(1.0))
    k = h.shape[1]
    v_first = O.e2m1_decode(O.unpack_nibbles(packed[:, :k // 2])).reshape(q1.shape)
    v_second = O.e2m1_decode(O.unpack_nibbles(packed[:, k // 2:])).reshape(q2.shape)
    assert np.array_equal(v_first, q1) and np.array_equal(v_second, q2)
    assert np.array_equal(O.e4m3_decode(sb[:, :k // 16]), sb1)
    assert np.array_equal(O.e4m3_decode(sb[:, k // 16:]), sb2)


def test_decompose_zero_residual_gives_zero_second_level():
    rng = np.random.default_rng(12)
    h, q1, sb1, q2, sb2 = _two_level_case(rng, 4, 128)
    h1 = (q1 * sb1[:, :, None]).astype(np.float32).reshape(h.shape)     # level one only
    packed, sb, _ = O.nvfp4_decompose(h1, g=np.float32(1.0))
    assert not packed[:, 64:].any() and not sb[:, 8:].any()             # +0 codes, zero scales


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_decompose_error_within_second_level_grid(seed):
    """|h - v1 - v2| is bounded by the second level's E2M1 grid: at most 2
    grid steps of s2 = E4M3(sb2) g (saturation after a subnormal E4M3 scale
    rounded down), or |r| itself when the residual's scale is zero.  A sign
    or scale mistake in the residual breaks this by orders of magnitude."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    x[:, rng.choice(512, 6, replace=False)] *= 40
    h = O.block_hadamard(_f32(_bf16(x)))
    packed, sb, g = O.nvfp4_decompose(h)
    k = h.shape[1]
    v1 = O.nvfp4_values(packed[:, :k // 2], sb[:, :k // 16], g).astype(np.float64)
    v2 = O.nvfp4_values(packed[:, k // 2:], sb[:, k // 16:], g).astype(np.float64)
    r = h.astype(np.float64) - v1
    err = np.abs(h - v1 - v2).reshape(64, k // 16, 16)
    s2 = (O.e4m3_decode(sb[:, k // 16:]) * np.float64(g))[:, :, None]
    rb = np.abs(r).reshape(64, k // 16, 16).max(axis=2, keepdims=True)
    bound = np.where(s2 > 0, 2 * s2, rb) + 1e-6 * np.abs(h).reshape(err.shape)
    assert np.all(err <= bound)
    one = np.abs(h - v1).mean()
    assert np.abs(h - v1 - v2).mean() < one / 4                      # the residual pays off


def test_decomposed_product_is_the_sum_of_both_levels():
    rng = np.random.default_rng(5)
    xb = _bf16(rng.standard_normal((24, 256)))
    wb = _bf16(rng.standard_normal((40, 256)) * 0.02)
    wq = O.prepare_weights_nvfp4(wb)
    aq = O.quantize_activations(xb, O.ROUTE_NVFP4_DECOMP)
    y = O.forward(xb, wq, O.ROUTE_NVFP4_DECOMP)
    y1 = O.gemm_w4a4(aq["packed"][:, :128], aq["sb"][:, :16], aq["g"], wq["packed"], wq["sb"], wq["g"])
    y2 = O.gemm_w4a4(aq["packed"][:, 128:], aq["sb"][:, 16:], aq["g"], wq["packed"], wq["sb"], wq["g"])
    assert np.allclose(y, y1 + y2, rtol=1e-12, atol=1e-12 * np.abs(y).max())
    exact = (_f32(xb).astype(np.float64) @ _f32(wb).astype(np.float64).T)
    e_dec = np.abs(y - exact).max() / np.abs(exact).max()
    e_one = np.abs(O.forward(xb, wq, O.ROUTE_NVFP4) - exact).max() / np.abs(exact).max()
    assert e_dec < e_one                                               # informative


# ---------------------------------------------------------------- TDC / PDR

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(4096).astype(np.float32) * 10.0 ** rng.integers(-8, 8, 4096),
                        # exact ties between two bf16 values
                        (np.arange(1, 513, dtype=np.float32) * 2 + 1) * np.float32(2.0 ** -8) + 1]).astype(np.float32)
    assert np.array_equal(T.f32_to_bf16_bits(x), _bf16(x))


def test_delta_and_apply_match_torch_arithmetic():
    rng = np.random.default_rng(4)
    a = _bf16(rng.standard_normal(5000))
    b = _bf16(rng.standard_normal(5000) * 1.3)
    ta = torch.tensor(_f32(a))
    tb = torch.tensor(_f32(b))
    want_d = (tb - ta).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(T.tdc_delta(a, b), want_d)
    want_o = (ta + tb).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(T.tdc_apply(a, b), want_o)


def test_delta_error_closed_forms():
    rng = np.random.default_rng(6)
    old = _bf16(rng.integers(-8, 9, 1000).astype(np.float32) * 0.25)   # few significant bits
    new = _bf16(_f32(old) * np.float32(1.125))                          # exact in bf16
    assert T.tdc_delta_error(new, old) == 0.125
    assert T.tdc_delta_error(old, old) == 0.0
    assert T.tdc_delta_error(old, np.zeros_like(old)) == float("inf")


def _block_with_deltas(deltas):
    """A stand-in block whose output is in + deltas[t] at its t-th computation."""
    calls = []

    def block(inp_bits, route):
        calls.append(route)
        d = deltas[len(calls) - 1]
        return _bf16(_f32(inp_bits) + np.float32(d))
    return block, calls


@pytest.mark.parametrize("acc_max,max_skips,pattern", [
    # E = 0.0625 after two computed steps (deltas 0.5 then 0.53125):
    # skips continue until max_skips, then a forced computation.
    (1.0, 3, "CCSSSC"),
    # the summed error caps the run first: 0.0625 + 0.0625 + 0.0625 > 0.15
    (0.15, 3, "CCSSCS"),
    (1.0, 0, "CCCCCC"),
])
def test_policy_traces(acc_max, max_skips, pattern):
    prm = T.TdcParams(gamma_threshold=0.05, eps_threshold=0.1, acc_max=acc_max, max_skips=max_skips)
    st = T.TdcState()
    # every computed step moves the delta by the same relative 1/16 (E = 0.0625)
    block, calls = _block_with_deltas([0.5 * (1 + 1 / 16) ** i for i in range(8)])
    inp = _bf16(np.ones(64, np.float32))
    got, routes = "", []
    for _ in range(len(pattern)):
        out, skipped, route = T.tdc_step(st, prm, inp, block)
        got += "S" if skipped else "C"
        routes.append(route)
        if skipped:
            assert np.array_equal(out, T.tdc_apply(inp, st.deltas[-1]))
    assert got == pattern
    # PDR: the first computed step after a skip runs INT8; the others follow
    # Gamma (= 0.5.. > 0.05 here, so INT8 as well) -- check the forced flag
    # with a threshold that Gamma never exceeds
    prm2 = T.TdcParams(gamma_threshold=10.0, eps_threshold=0.1, acc_max=acc_max, max_skips=max_skips)
    st2 = T.TdcState()
    block2, _ = _block_with_deltas([0.5 * (1 + 1 / 16) ** i for i in range(8)])
    seq = []
    for _ in range(len(pattern)):
        _, skipped, route = T.tdc_step(st2, prm2, inp, block2)
        seq.append("S" if skipped else ("I" if route == O.ROUTE_INT8 else "F"))
    want = []   # the very first step has no Gamma either: INT8 as well
    for i, c in enumerate(pattern):
        want.append("S" if c == "S" else ("I" if i == 0 or pattern[i - 1] == "S" else "F"))
    assert "".join(seq) == "".join(want)


@pytest.mark.parametrize("eps_threshold,pattern", [
    # deltas alternate 0.5, 0.625: E is 0.25 after the second computation and
    # 0.2 after the third (0.125 / 0.625); both are at or above 0.1
    (0.1, "CCCCCCC"),
    # E = 0.25 is not below 0.25 (strict), E = 0.2 is: three skips, then the
    # skip count forces a computation
    (0.25, "CCCSSSC"),
])
def test_error_threshold_gates_skips(eps_threshold, pattern):
    prm = T.TdcParams(gamma_threshold=0.05, eps_threshold=eps_threshold, acc_max=1.0, max_skips=3)
    st = T.TdcState()
    block, _ = _block_with_deltas([0.5, 0.625] * 4)
    inp = _bf16(np.ones(64, np.float32))
    got = ""
    for _ in range(len(pattern)):
        _, skipped, _ = T.tdc_step(st, prm, inp, block)
        got += "S" if skipped else "C"
    assert got == pattern


def test_first_two_steps_always_compute():
    st = T.TdcState()
    prm = T.TdcParams()
    assert not T.tdc_should_skip(st, prm)                 # no delta yet
    inp = _bf16(np.ones(16, np.float32))
    T.tdc_after_compute(st, inp, _bf16(np.full(16, 1.5, np.float32)))
    assert st.eps == float("inf") and not T.tdc_should_skip(st, prm)
    T.tdc_after_compute(st, inp, _bf16(np.full(16, 1.5, np.float32)))
    assert st.eps == 0.0 and T.tdc_should_skip(st, prm)


# ---------------------------------------------------------------- PDR outlier ratio

def test_outlier_ratio_hand_cases():
    blocks = np.zeros((4, 16), np.float32)
    blocks[0] = 1.0                                   # uniform: a*15 = 15, kappa*others = 8*15
    blocks[1] = 1.0
    blocks[1, 3] = 9.0                                # 9*15 = 135 > 8*15 = 120: flagged
    blocks[2] = 1.0
    blocks[2, 5] = 8.0                                # 8*15 = 120, not > 120: not flagged
    blocks[3, 0] = -0.5                               # one nonzero value: others = 0, flagged
    bits = _bf16(blocks.ravel())
    assert T.outlier_ratio(bits, 8.0) == 0.5
    assert T.outlier_ratio(bits, 7.0) == 0.75         # 8*15 = 120 > 7*15 = 105
    assert T.outlier_ratio(_bf16(np.zeros(40, np.float32)), 8.0) == 0.0   # all zero: 0 > 0 is false
    assert T.outlier_ratio(bits[:15], 8.0) == 0.0     # no whole block


def test_outlier_ratio_counts_planted_channels():
    rng = np.random.default_rng(21)
    x = rng.standard_normal((64, 1920)).astype(np.float32)
    cols = rng.choice(1920, 19, replace=False)
    x[:, cols] *= 30.0
    rho = T.outlier_ratio(_bf16(x), 8.0)
    blocks_hit = len(set(int(c) // 16 for c in cols))
    assert abs(rho - blocks_hit / 120) < 0.02          # the blocks holding a planted channel
    assert T.outlier_ratio(_bf16(rng.standard_normal((64, 1920)).astype(np.float32)), 8.0) < 0.01


def test_pdr_bf16_takes_precedence():
    prm = T.TdcParams(rho_max=0.1)
    st = T.TdcState(rho=0.2, last_skipped=True, gamma=0.0)
    assert T.pdr_route(st, prm) == T.ROUTE_BF16
    st.rho = 0.05
    assert T.pdr_route(st, prm) == O.ROUTE_INT8
    st.last_skipped = False
    assert T.pdr_route(st, prm) == O.ROUTE_NVFP4


def test_gemm_bf16_is_the_exact_product():
    rng = np.random.default_rng(22)
    xi = rng.integers(-64, 65, (5, 32)).astype(np.float32)
    wi = rng.integers(-64, 65, (7, 32)).astype(np.float32)
    r = O.gemm_bf16(_bf16(xi), _bf16(wi))
    assert np.array_equal(r, (xi.astype(np.int64) @ wi.astype(np.int64).T).astype(np.float64))
