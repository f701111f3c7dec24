"""Pins for the oracle's number formats (E2M1, E4M3) against the format
definitions, a library implementation and brute force."""
import struct
from fractions import Fraction

import numpy as np
import torch

from oracle import qlinear_oracle as O


def _all_bf16_values(lo, hi):
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    v = O.bf16_bits_to_f32(bits)
    v = v[np.isfinite(v)]
    return v[(v >= lo) & (v <= hi)]


def test_e2m1_table_from_definition():
    assert list(O.e2m1_magnitudes()) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e4m3_table_points(golden):
    table = O.e4m3_magnitudes()
    assert len(table) == 127 and np.all(np.diff(table) > 0)
    for line in golden("e4m3_points.txt"):
        code, val = line.split()
        assert table[int(code, 16)] == float(val)
        assert O.e4m3_encode(np.float32(float(val))) == int(code, 16)


def test_e2m1_golden_ties(golden):
    for line in golden("e2m1_ties.txt"):
        val, code = line.split()
        got = int(O.e2m1_encode(np.float32(float(val))))
        assert got == int(code, 16), (val, hex(got), code)


def _brute_e2m1(y: float) -> int:
    """Nearest of the 8 magnitudes by exact rational distance; ties to the
    even code; clamp at 6; sign bit from the float's sign."""
    mags = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2),
            Fraction(3), Fraction(4), Fraction(6)]
    a = abs(Fraction(y))
    if a >= 6:
        best = 7
    else:
        dists = [abs(a - m) for m in mags]
        dmin = min(dists)
        cands = [i for i, d in enumerate(dists) if d == dmin]
        best = [c for c in cands if c % 2 == 0][0] if len(cands) > 1 else cands[0]
    sign = 1 if struct.unpack("<I", struct.pack("<f", y))[0] >> 31 else 0
    return best | (sign << 3)


def test_e2m1_encode_matches_brute_force_on_all_bf16():
    v = _all_bf16_values(-8.0, 8.0)
    v = np.concatenate([v, np.float32([-0.0])])
    got = O.e2m1_encode(v)
    want = np.array([_brute_e2m1(float(x)) for x in v], dtype=np.uint8)
    assert np.array_equal(got, want)


def test_e2m1_decode_roundtrip():
    codes = np.arange(16, dtype=np.uint8)
    vals = O.e2m1_decode(codes).astype(np.float32)
    vals[8] = np.float32(-0.0)
    assert np.array_equal(O.e2m1_encode(vals), codes)


def test_e4m3_encode_matches_torch_float8_in_range():
    """torch's float8_e4m3fn conversion is an independent RN-even
    implementation; it agrees on every value that does not overflow."""
    v = _all_bf16_values(0.0, 448.0)
    v = v[~np.signbit(v)]              # block scales are never negative zero
    rng = np.random.default_rng(7)
    r = (rng.uniform(0, 1, 200000) ** 4 * 448).astype(np.float32)
    table = O.e4m3_magnitudes()
    mids = ((table[1:] + table[:-1]) / 2).astype(np.float32)   # exact ties
    x = np.concatenate([v, r, mids, table.astype(np.float32)])
    got = O.e4m3_encode(x)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, want)


def test_e4m3_saturates_and_subnormals():
    assert O.e4m3_encode(np.float32(448.0)) == 0x7E
    assert O.e4m3_encode(np.float32(463.9)) == 0x7E
    assert O.e4m3_encode(np.float32(1e30)) == 0x7E
    # 2^-10 is the tie between 0 and the smallest subnormal: even code 0 wins
    assert O.e4m3_encode(np.float32(2.0 ** -10)) == 0
    assert O.e4m3_encode(np.float32(2.0 ** -10 * 1.0001)) == 1
    assert O.e4m3_encode(np.float32(3 * 2.0 ** -10)) == 2   # tie 1|2 -> even


def test_nibble_pack_order():
    codes = np.array([[1, 2, 3, 4]], dtype=np.uint8)
    assert O.pack_nibbles(codes).tolist() == [[0x21, 0x43]]
    assert np.array_equal(O.unpack_nibbles(O.pack_nibbles(codes)), codes)
