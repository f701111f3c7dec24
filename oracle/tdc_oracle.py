"""Plain CPU oracle of the temporal delta cache (TEST INFRASTRUCTURE ONLY).

Like ``qlinear_oracle``, only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this; it shares no code with the
CUDA library.

Source: "6Bit-Diffusion" (gist.science 2603.18742), Methodology:
  * A.2 (temporal redundancy): the residual delta of a transformer block,
    Delta_t = output - input, is nearly the same at adjacent timesteps;
  * B.2 TDC: the difference E_t of the block's deltas at the two previous
    (computed) timesteps decides whether the block is skipped, in which case
    the cached delta is reused; consecutive skips are bounded by an
    accumulated-error threshold and a maximum skip count, after which the
    block is computed and the cache refreshed;
  * B.3 PDR: on the first computed step after a skip there is no routing
    information from the previous step, so the block's activations are
    forced to INT8.

Readings of what the page leaves open (every one listed in the design notes):
  * Delta is stored in the activation type: Delta = bf16(RN(out - in));
  * E_t is the relative L1 distance of the two cached deltas, in the same
    arithmetic as the router's Gamma: fp32 differences of the bf16 values,
    fp64 sums, E = sum |D_new - D_old| / sum |D_old| (+inf when the old delta
    is all zero or when fewer than two deltas are cached);
  * a skipped block's output is out = bf16(RN(in + Delta_latest));
  * skip iff two deltas are cached, E < eps_threshold, acc + E <= acc_max and
    skips < max_skips, where acc sums E over the current run of skips and
    skips counts them; a computed step resets both;
  * the route of a computed step is INT8 when the previous step skipped or
    when the block has no Gamma yet (its first step), otherwise Gamma of the
    last computed step > gamma_threshold;
  * PDR's high-precision refresh: the input outlier ratio rho is the
    fraction of 16-element blocks of the block input (in element order,
    whole blocks only) dominated by one value: with a = max |x| and s the
    fp32 sum of |x| over the block (two sequential halves of 8, then their
    sum), the block counts iff RN(a * 15) > RN(kappa * RN(s - a)), i.e. its
    largest magnitude exceeds kappa times the mean of the other 15; a
    computed step whose preceding refresh saw rho > rho_max runs in BF16
    (this takes precedence over the INT8 / NVFP4 choice).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .qlinear_oracle import ROUTE_INT8, ROUTE_NVFP4, bf16_bits_to_f32, dmpq_gamma

ROUTE_BF16 = 8   # unquantized bf16 product (PDR's high-precision refresh)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def tdc_delta(inp_bits: np.ndarray, out_bits: np.ndarray) -> np.ndarray:
    """Delta = bf16(RN(out - in)) as bf16 bit patterns."""
    d = (bf16_bits_to_f32(out_bits) - bf16_bits_to_f32(inp_bits)).astype(np.float32)
    return f32_to_bf16_bits(d)


def tdc_delta_error(new_bits: np.ndarray, old_bits: np.ndarray) -> float:
    """E = sum |RN(new - old)| / sum |old| over the bf16 deltas (fp64 sums)."""
    return dmpq_gamma(old_bits, new_bits)


def tdc_apply(inp_bits: np.ndarray, delta_bits: np.ndarray) -> np.ndarray:
    """Output of a skipped block: bf16(RN(in + Delta))."""
    y = (bf16_bits_to_f32(inp_bits) + bf16_bits_to_f32(delta_bits)).astype(np.float32)
    return f32_to_bf16_bits(y)


@dataclass
class TdcParams:
    gamma_threshold: float = 0.05   # DMPQ route threshold
    eps_threshold: float = 0.1      # skip when the delta change is below this
    acc_max: float = 0.3            # cap on the summed E over a run of skips
    max_skips: int = 3              # cap on consecutive skips
    kappa: float = 8.0              # outlier block: largest magnitude > kappa x mean of the rest
    rho_max: float = 1.0            # BF16 when the outlier-block fraction exceeds this


@dataclass
class TdcState:
    """Per-block cache state: the latest two deltas, E between them, Gamma of
    the last computed step and the skip run."""
    deltas: list = field(default_factory=list)   # oldest first, at most 2
    gamma: float = float("inf")
    eps: float = float("inf")
    acc: float = 0.0
    skips: int = 0
    last_skipped: bool = False
    rho: float = 0.0


def outlier_ratio(inp_bits: np.ndarray, kappa: float) -> float:
    """Fraction of the 16-element blocks dominated by one value (see the header)."""
    x = np.abs(bf16_bits_to_f32(inp_bits).ravel())
    nb = x.size // 16
    if nb == 0:
        return 0.0
    b = x[:nb * 16].reshape(nb, 2, 8)
    halves = np.zeros((nb, 2), np.float32)
    for j in range(8):                                           # sequential fp32 sums
        halves = (halves + b[:, :, j]).astype(np.float32)
    s = (halves[:, 0] + halves[:, 1]).astype(np.float32)
    a = b.reshape(nb, 16).max(axis=1)
    others = (s - a).astype(np.float32)
    flagged = (a * np.float32(15)).astype(np.float32) > (np.float32(kappa) * others).astype(np.float32)
    return float(np.count_nonzero(flagged)) / nb


def tdc_should_skip(st: TdcState, prm: TdcParams) -> bool:
    return (len(st.deltas) == 2 and st.eps < prm.eps_threshold and st.acc + st.eps <= prm.acc_max
            and st.skips < prm.max_skips)


def pdr_route(st: TdcState, prm: TdcParams) -> int:
    """Route of the next computed step (PDR: BF16 after a refresh that saw
    many outlier blocks, else INT8 right after a skip)."""
    if st.rho > prm.rho_max:
        return ROUTE_BF16
    if st.last_skipped:
        return ROUTE_INT8
    return ROUTE_INT8 if st.gamma > prm.gamma_threshold else ROUTE_NVFP4


def tdc_after_compute(st: TdcState, inp_bits: np.ndarray, out_bits: np.ndarray,
                      kappa: float = TdcParams.kappa) -> None:
    """Cache refresh after the block was computed: the new delta, Gamma of
    this step, E between the new and the previous delta and the input's
    outlier-block ratio."""
    d = tdc_delta(inp_bits, out_bits)
    st.rho = outlier_ratio(inp_bits, kappa)
    st.gamma = dmpq_gamma(inp_bits, out_bits)
    st.eps = tdc_delta_error(d, st.deltas[-1]) if st.deltas else float("inf")
    st.deltas = (st.deltas + [d])[-2:]
    st.acc = 0.0
    st.skips = 0
    st.last_skipped = False


def tdc_after_skip(st: TdcState) -> None:
    st.acc += st.eps
    st.skips += 1
    st.last_skipped = True


def tdc_step(st: TdcState, prm: TdcParams, inp_bits: np.ndarray, block) -> tuple[np.ndarray, bool, int]:
    """One timestep of one block under the cache.  ``block(inp_bits, route)``
    computes the block.  Returns (output bits, skipped, route used)."""
    if tdc_should_skip(st, prm):
        out = tdc_apply(inp_bits, st.deltas[-1])
        tdc_after_skip(st)
        return out, True, -1
    route = pdr_route(st, prm)
    out = block(inp_bits, route)
    tdc_after_compute(st, inp_bits, out, prm.kappa)
    return out, False, route
