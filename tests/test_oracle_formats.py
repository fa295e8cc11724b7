"""Pins for the oracle's number formats (bfloat16, OCP E4M3).

Each check ties the oracle to something outside itself: torch's own float32 ->
bfloat16 and float32 -> float8_e4m3fn conversions (library routines), closed
forms from the format definitions, and brute-force nearest-value search with
exact rational arithmetic.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore")


def _f32_bits_to_float(u):
    return float(np.array([u], dtype=np.uint32).view(np.float32)[0])


def test_bf16_decode_all_codes_match_torch():
    codes = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    ours = np.array([oracle.bf16_decode(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_bf16_encode_roundtrip_all_codes():
    for c in range(65536):
        v = oracle.bf16_decode(c)
        if math.isnan(v):
            continue
        assert oracle.bf16_encode(v) == c, hex(c)


def test_bf16_encode_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 2**32, size=20000, dtype=np.uint64).astype(np.uint32)
    # add exact ties (low 16 bits = 0x8000) and near-ties
    ties = (rng.integers(0, 2**16, size=2000, dtype=np.uint32) << 16) | 0x8000
    bits = np.concatenate([bits, ties, ties + 1, ties - 1])
    vals = bits.view(np.float32)
    vals = vals[np.isfinite(vals)]
    ref = torch.from_numpy(vals.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = np.array([oracle.bf16_encode(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(ours, ref)


def _bf16_neighbours(v: float):
    """All finite bf16 values within two codes of float32(v) (brute force)."""
    f = np.array([v], dtype=np.float32).view(np.uint32)[0]
    base = int(f >> 16)
    out = []
    for c in range(base - 2, base + 3):
        c &= 0xFFFF
        x = oracle.bf16_decode(c)
        if math.isfinite(x):
            out.append((c, x))
    return out


def test_bf16_encode_single_rounding_from_double_brute_force():
    """Doubles that are not float32 values: the result must be the nearest bf16
    (ties to even mantissa), decided with exact rationals -- no detour through
    float32, whose rounding could move a value across a bf16 tie."""
    rng = np.random.default_rng(11)
    cases = list(rng.standard_normal(3000) * 10.0 ** rng.integers(-30, 30, 3000))
    # values just above / below an exact bf16 tie, which a float32 detour rounds to the tie
    for c in rng.integers(0x3000, 0x4F00, 300):
        lo = oracle.bf16_decode(int(c))
        hi = oracle.bf16_decode(int(c) + 1)
        mid = (lo + hi) / 2
        cases += [mid + (hi - lo) * 2.0**-30, mid - (hi - lo) * 2.0**-30, mid]
    for v in cases:
        got = oracle.bf16_encode(v)
        best = None
        for c, x in _bf16_neighbours(v):
            d = abs(Fraction(x) - Fraction(v))
            key = (d, c & 1)  # ties -> even code (even mantissa LSB)
            if best is None or key < best[0]:
                best = (key, c)
        assert got == best[1], (v, hex(got), hex(best[1]))


def test_bf16_encode_special_values():
    assert oracle.bf16_encode(0.0) == 0x0000
    assert oracle.bf16_encode(-0.0) == 0x8000
    assert oracle.bf16_encode(1.0) == 0x3F80
    assert oracle.bf16_encode(-2.0) == 0xC000
    assert oracle.bf16_encode(float("inf")) == 0x7F80
    assert oracle.bf16_encode(1e39) == 0x7F80        # overflows bf16 (max ~3.39e38)
    assert oracle.bf16_encode(3.3895e38) == 0x7F7F    # largest finite
    assert oracle.bf16_encode(2.0**-133) == 0x0001    # smallest subnormal
    assert oracle.bf16_encode(2.0**-134) == 0x0000    # tie between 0 and 2^-133 -> even (0)
    assert oracle.bf16_encode(1.0 + 2.0**-8) == 0x3F80   # tie -> even
    assert oracle.bf16_encode(1.0 + 3 * 2.0**-8) == 0x3F82  # tie -> even (up)
    assert math.isnan(oracle.bf16_decode(oracle.bf16_encode(float("nan"))))


# ------------------------------------------------------------------ E4M3 ---
def _e4m3_closed_form(c: int) -> float:
    s = -1.0 if c & 0x80 else 1.0
    E, m = (c >> 3) & 15, c & 7
    if E == 15 and m == 7:
        return float("nan")
    if E == 0:
        return s * (m / 8) * 2.0**-6
    return s * (1 + m / 8) * 2.0 ** (E - 7)


def test_e4m3_decode_matches_closed_form_and_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref_t = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        ours = oracle.e4m3_decode(c)
        cf = _e4m3_closed_form(c)
        if math.isnan(cf):
            assert math.isnan(ours) and math.isnan(ref_t[c])
        else:
            assert ours == cf == ref_t[c], hex(c)
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0x08) == 2.0**-6
    assert oracle.e4m3_decode(0x01) == 2.0**-9
    assert oracle.e4m3_decode(0x38) == 1.0


def test_e4m3_encode_roundtrip_all_codes():
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if math.isnan(v):
            continue
        assert oracle.e4m3_encode(v) == c, hex(c)


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(3)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 100,
        rng.standard_normal(5000).astype(np.float32) * 0.01,
        (rng.uniform(-448, 448, 5000)).astype(np.float32),
    ])
    vals = vals[np.abs(vals) <= 448]
    ref = torch.from_numpy(vals.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.e4m3_encode(float(v)) for v in vals], dtype=np.uint8)
    assert np.array_equal(ours, ref)


def test_e4m3_encode_brute_force_nearest_even_and_saturation():
    finite = [(c, oracle.e4m3_decode(c)) for c in range(128) if not math.isnan(oracle.e4m3_decode(c))]
    rng = np.random.default_rng(5)
    vals = list(rng.uniform(0, 470, 4000)) + list(rng.uniform(0, 2.0**-5, 2000))
    # exact midpoints between neighbours
    fv = sorted(x for _, x in finite)
    vals += [(a + b) / 2 for a, b in zip(fv[:-1], fv[1:])]
    for v in vals:
        got = oracle.e4m3_encode(v)
        if v >= 448:
            assert got == 0x7E
            continue
        best = min(finite, key=lambda cx: (abs(Fraction(cx[1]) - Fraction(v)), cx[0] & 1))
        assert got == best[0], (v, got, best)
        assert oracle.e4m3_encode(-v) == (best[0] | 0x80 if best[1] != 0 else 0x80)
    for big in (449.0, 464.0, 479.9, 480.0, 1e9, float("inf")):
        assert oracle.e4m3_encode(big) == 0x7E
        assert oracle.e4m3_encode(-big) == 0xFE
