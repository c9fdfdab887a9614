"""Pins for the oracle's NVFP4 weight and activation quantisers.

Hand-worked examples (tests/golden), brute-force nearest-code search, and
invariants every correct NVFP4 quantiser must satisfy.
"""
import numpy as np
import pytest

from oracle import nvfp4_ffn as O
from nvfp4_quantized_dense_w4a16_b200 import synth


def _floats(rows):
    return np.array([[float(v) for v in r] for r in rows], dtype=np.float32)


def _hexes(rows):
    return np.array([[int(v, 16) for v in r] for r in rows], dtype=np.uint8)


def test_weight_quant_worked_example(golden):
    g = golden("weight_quant_example.txt")
    w = _floats(g["w"])
    codes, scales, gs = O.quantize_weight(w)
    assert float(gs) == float(g["gs"][0][0])
    assert np.array_equal(scales, _hexes(g["scales"]))
    assert np.array_equal(codes, _hexes(g["codes"]))


def test_activation_quant_worked_example(golden):
    g = golden("act_quant_example.txt")
    x = _floats(g["x"])
    codes, scales = O.quantize_activation(x)
    assert np.array_equal(scales, _hexes(g["scales"]))
    assert np.array_equal(codes, _hexes(g["codes"]))


def test_pack_nibbles_low_nibble_first():
    c = np.array([[0x1, 0x2, 0xF, 0x8]], dtype=np.uint8)
    assert O.pack_nibbles(c).tolist() == [[0x21, 0x8F]]
    assert np.array_equal(O.unpack_nibbles(O.pack_nibbles(c)), c)


def _brute_codes(q: np.ndarray) -> np.ndarray:
    """Nearest of the 16 code values by exhaustive distance search (ties to the
    even magnitude index), sign from the quotient's sign bit."""
    vals = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    a = np.abs(q.astype(np.float64))[..., None]
    d = np.abs(a - vals)
    best = d.min(axis=-1, keepdims=True)
    cand = d == best
    # among equal distances prefer the even index
    pref = np.where(cand, np.where(np.arange(8) % 2 == 0, 0, 1), 9)
    idx = np.argmin(pref * 16 + np.arange(8), axis=-1)
    return (idx | (np.signbit(q).astype(np.int64) << 3)).astype(np.uint8)


@pytest.mark.parametrize("n,k,seed,outliers", [(64, 256, 0, False), (32, 512, 1, True)])
def test_weight_quant_codes_match_brute_force(n, k, seed, outliers):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((n, k)).astype(np.float32) * np.float32(0.02)
    if outliers:
        w[:, :16] *= 8
    w = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(w))
    codes, scales, gs = O.quantize_weight(w)
    assert gs == np.float32(np.abs(w).max() / np.float32(2688.0))
    sdec = (O.e4m3_decode(scales).astype(np.float32) * gs).astype(np.float32)
    q = (w.reshape(n, k // 16, 16) / sdec[..., None]).astype(np.float32)
    ref = _brute_codes(q).reshape(n, k)
    assert np.array_equal(O.unpack_nibbles(codes), ref)


def test_weight_quant_invariants():
    rng = np.random.default_rng(5)
    n, k = 48, 1024
    w = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(
        rng.standard_normal((n, k)).astype(np.float32) * np.float32(0.02)))
    w[3, 32:48] = 0.0                              # an all-zero block
    w[4, 64:80] = np.float32(0.015625)            # a constant block
    codes, scales, gs = O.quantize_weight(w)
    c = O.unpack_nibbles(codes).reshape(n, k // 16, 16)
    sdec = (O.e4m3_decode(scales).astype(np.float32) * gs).astype(np.float32)
    wb = w.reshape(n, k // 16, 16)
    # zero block: scale 0, codes 0
    assert scales[3, 2] == 0 and np.all(c[3, 2] == 0)
    # re-encoding the dequantised weight with the same scales returns the codes
    what = (O.e2m1_decode(c).astype(np.float32) * sdec[..., None]).astype(np.float32)
    again = O.e2m1_encode((what / np.where(sdec == 0, 1, sdec)[..., None]).astype(np.float32))
    nz = scales != 0
    assert np.array_equal(again[nz] & 7, c[nz] & 7)
    # error bound: within half the local code gap (scaled) when |w|/sdec <= 6
    qa = np.abs(wb / np.where(sdec == 0, 1, sdec)[..., None]).astype(np.float64)
    half_gap = np.where(qa < 2, 0.25, np.where(qa < 4, 0.5, 1.0))
    err = np.abs(wb.astype(np.float64) - what.astype(np.float64)) / np.where(sdec == 0, 1, sdec)[..., None]
    mask = nz[..., None] & (qa <= 6)
    assert np.all(err[mask] <= half_gap[mask] + 1e-12)
    # the largest element of a normal-scaled block encodes to magnitude 6
    normal = nz & (scales >= 8) & (scales < 0x7E)
    imax = np.argmax(np.abs(wb), axis=2)
    top = np.take_along_axis(c, imax[..., None], axis=2)[..., 0]
    assert np.all((top[normal] & 7) == 7)
    # constant block: every element encodes the same code
    assert len(set(c[4, 4].tolist())) == 1
    # the tensor's largest element scales to exactly 448 * gs
    i = np.unravel_index(np.argmax(np.abs(w)), w.shape)
    assert scales[i[0], i[1] // 16] == 0x7E


def test_activation_quant_codes_match_brute_force_and_row_independence():
    rng = np.random.default_rng(9)
    x = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(rng.standard_normal((16, 512)).astype(np.float32)))
    x[2] *= 1000
    x[3, :16] = 0
    codes, scales = O.quantize_activation(x)
    sdec = O.e4m3_decode(scales).astype(np.float32)
    q = (x.reshape(16, 32, 16) / np.where(sdec == 0, 1, sdec)[..., None]).astype(np.float32)
    ref = np.where((scales == 0)[..., None], 0, _brute_codes(q)).reshape(16, 512)
    assert np.array_equal(O.unpack_nibbles(codes), ref)
    assert scales[3, 0] == 0
    for r in range(16):
        c1, s1 = O.quantize_activation(x[r:r + 1])
        assert np.array_equal(c1[0], codes[r]) and np.array_equal(s1[0], scales[r])


def test_quant_scale_is_e4m3_of_block_amax_over_six():
    x = np.zeros((1, 16), np.float32)
    x[0, 5] = np.float32(-3.0)          # amax 3 -> 0.5 -> E4M3 0x30
    _, s = O.quantize_activation(x)
    assert s[0, 0] == 0x30
    x[0, 5] = np.float32(3000.0)        # 500 -> saturates to 448 (0x7E)
    c, s = O.quantize_activation(x)
    assert s[0, 0] == 0x7E and (O.unpack_nibbles(c)[0, 5] & 7) == 7
