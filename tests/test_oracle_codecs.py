"""Pins for the oracle's element/scale codecs and bf16 rounding.

Each check compares the oracle with something other than itself: the public
format tables (tests/golden), PyTorch's own float8 / bfloat16 conversions, or
a brute-force nearest-value search in exact rational arithmetic.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import nvfp4_ffn as O


def _golden_table(golden, name):
    rows = golden(name)[None]
    return [(int(c, 16), float(v)) for c, v in rows]


def test_e2m1_decode_matches_spec_table(golden):
    for code, val in _golden_table(golden, "e2m1_values.txt"):
        got = float(O.e2m1_decode(code))
        assert got == val and math.copysign(1, got) == math.copysign(1, val), (code, got, val)


def test_e2m1_encode_roundtrips_every_code(golden):
    for code, val in _golden_table(golden, "e2m1_values.txt"):
        v = np.float32(val)
        assert int(O.e2m1_encode(v)) == code


def _brute_e2m1(q: float) -> int:
    """Nearest E2M1 magnitude by exhaustive search in exact rationals; ties to
    the even magnitude index; saturate at 6."""
    a = abs(Fraction(q))
    mags = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2),
            Fraction(3), Fraction(4), Fraction(6)]
    best = None
    for i, mv in enumerate(mags):
        d = abs(a - mv)
        if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
            best = (d, i)
    idx = best[1]
    return idx | (8 if math.copysign(1.0, q) < 0 else 0)


def test_e2m1_encode_ties_go_to_even_index():
    # midpoints between neighbouring magnitudes and the index they must take
    cases = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for q, idx in cases.items():
        assert int(O.e2m1_encode(np.float32(q))) == idx
        assert int(O.e2m1_encode(np.float32(-q))) == idx | 8
        assert _brute_e2m1(q) == idx


def test_e2m1_encode_saturates_and_keeps_sign():
    assert int(O.e2m1_encode(np.float32(7.0))) == 7
    assert int(O.e2m1_encode(np.float32(1e30))) == 7
    assert int(O.e2m1_encode(np.float32(-100.0))) == 15
    assert int(O.e2m1_encode(np.float32(-0.1))) == 8
    assert int(O.e2m1_encode(np.float32(-0.0))) == 8
    assert int(O.e2m1_encode(np.float32(0.0))) == 0


def test_e2m1_encode_matches_brute_force_on_random_values():
    rng = np.random.default_rng(123)
    q = (rng.standard_normal(4000) * 3).astype(np.float32)
    # include values near every midpoint
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    near = np.concatenate([np.nextafter(mids, np.float32(0)), mids, np.nextafter(mids, np.float32(9))])
    q = np.concatenate([q, near, -near])
    got = O.e2m1_encode(q)
    for v, c in zip(q.tolist(), got.tolist()):
        assert c == _brute_e2m1(v), v


def test_e4m3_decode_matches_spec_landmarks(golden):
    for code, val in _golden_table(golden, "e4m3_values.txt"):
        got = float(O.e4m3_decode(code))
        if math.isnan(val):
            assert math.isnan(got)
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val), hex(code)


def test_e4m3_decode_matches_torch_float8_for_all_bytes():
    b = torch.arange(256, dtype=torch.uint8)
    ref = b.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_decode(np.arange(256))
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.all(both_nan | (ref == got))
    assert np.all(np.signbit(ref[~both_nan]) == np.signbit(got[~both_nan]))


def test_e4m3_encode_matches_torch_round_nearest_even_in_range():
    rng = np.random.default_rng(7)
    # log-uniform over the whole non-negative range below the overflow midpoint 464
    t = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(463.0), 20000)).astype(np.float32)
    vals = O.e4m3_decode(np.arange(127))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)  # exact ties
    t = np.concatenate([t, mids, vals.astype(np.float32), np.float32([0.0, 2.0 ** -10, 463.9])])
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_encode(t)
    assert np.array_equal(ref, got)


def test_e4m3_encode_saturates_at_448():
    for t in [448.0, 463.0, 464.0, 500.0, 1e6, float("inf")]:
        assert int(O.e4m3_encode(np.float32(t))) == 0x7E


def test_round_to_bf16_matches_torch_for_fp32_inputs():
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(50000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 50000).astype(np.float32),
        # exact ties: bf16 value + half an ulp
        (np.float32(1.0) + np.float32(2.0 ** -8)) * np.float32([1, -1, 3, 1e-20, 1e20]),
    ]).astype(np.float32)
    x = x[np.isfinite(x)]
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_to_bf16(x.astype(np.float64))
    assert np.array_equal(ref, got)


def test_round_to_bf16_rounds_fp64_once():
    # 1 + 2^-8 + 2^-30 lies just above the tie between 1 and 1 + 2^-7: a single
    # rounding goes up; rounding through fp32 first would land on the tie and go
    # to even (1.0).
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert float(O.round_to_bf16(x)) == 1.0 + 2.0 ** -7
    assert float(O.round_to_bf16(-x)) == -(1.0 + 2.0 ** -7)
    assert float(O.round_to_bf16(1.0 + 2.0 ** -8)) == 1.0          # tie -> even
    assert float(O.round_to_bf16(1.0 + 3 * 2.0 ** -8)) == 1.0 + 2.0 ** -6  # tie -> even (up)
    assert math.isinf(float(O.round_to_bf16(3.4e38)))
    assert float(O.round_to_bf16(2.0 ** -133)) == 2.0 ** -133        # smallest subnormal


def test_bf16_bit_helpers_roundtrip():
    bits = np.arange(0, 65536, 7, dtype=np.uint32).astype(np.uint16)
    vals = O.bf16_bits_to_f64(bits)
    ok = np.isfinite(vals)
    assert np.array_equal(O.f64_to_bf16_bits(vals[ok]), bits[ok])
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ref), np.isnan(vals))
    assert np.array_equal(ref[ok], vals[ok])


def test_silu_identities():
    assert float(O.silu(0.0)) == 0.0
    z = np.linspace(-30, 30, 1001)
    assert np.allclose(O.silu(z) - O.silu(-z), z, rtol=0, atol=1e-12)
    # sigmoid(ln 3) = 3/4, so silu(ln 3) = 0.75 ln 3
    assert abs(float(O.silu(math.log(3.0))) - 0.75 * math.log(3.0)) < 1e-15
    # large negative arguments go to -0 without overflow warnings leaking
    assert float(O.silu(-1000.0)) == 0.0
    assert float(O.silu(1000.0)) == 1000.0
