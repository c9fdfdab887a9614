"""Pins for the oracle's projections and FFN.

* exact-rational brute force of the projection definition on tiny sizes;
* inputs whose every product and partial sum is exact (integer activations,
  power-of-two scales) give exact outputs;
* a permutation-structured FFN whose output has a closed form, which catches
  transposed operands and wrong indices;
* fused gate+up equals separate gate and up;
* every output row depends only on its own input row (both formats);
* W4A4 reduces to W4A16 when the activations are already NVFP4 values, and
  equals the integer block-sum form sum_b sa_b * sw_b * S_b.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import nvfp4_ffn as O
from nvfp4_quantized_dense_w4a16_b200 import synth

E2M1 = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4), Fraction(6)]


def _e2m1_frac(c):
    v = E2M1[c & 7]
    return -v if c & 8 else v


def _e4m3_frac(b):
    """E4M3 byte -> exact Fraction, via torch's float8 decoding (independent)."""
    import torch
    return Fraction(float(torch.tensor([b], dtype=torch.uint8).view(torch.float8_e4m3fn).float()))


def _random_weight(n, k, seed):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, (n, k // 2), dtype=np.uint8)
    scales = rng.integers(0, 0x7F, (n, k // 16), dtype=np.uint8)   # any finite non-negative E4M3
    gs = np.float32(rng.uniform(0.001, 0.01))
    return codes, scales, gs


def test_project_w4a16_matches_exact_rational_definition():
    m, n, k = 3, 5, 48
    codes, scales, gs = _random_weight(n, k, 1)
    x = synth.bf16_bits_to_f32(synth.random_bf16((m, k), 2)).astype(np.float64)
    got = O.project_w4a16(x, codes, scales, gs)
    for r in range(m):
        for j in range(n):
            acc = Fraction(0)
            for kk in range(k):
                byte = int(codes[j, kk // 2])
                nib = byte & 15 if kk % 2 == 0 else byte >> 4
                acc += Fraction(float(x[r, kk])) * _e2m1_frac(nib) * _e4m3_frac(int(scales[j, kk // 16]))
            exact = Fraction(float(gs)) * acc
            assert abs(Fraction(got[r, j]) - exact) <= abs(exact) * Fraction(1, 10 ** 12) + Fraction(1, 10 ** 300)


def test_project_exact_inputs_give_exact_outputs():
    # integer activations in [-4, 4], power-of-two block scales, gs = 1: every
    # product and partial sum is a small dyadic rational, exact in fp64.
    rng = np.random.default_rng(3)
    m, n, k = 4, 6, 64
    codes = rng.integers(0, 256, (n, k // 2), dtype=np.uint8)
    pow2 = np.array([0x20, 0x28, 0x30, 0x38, 0x40, 0x48, 0x50], dtype=np.uint8)  # 2^-3 .. 2^3
    scales = rng.choice(pow2, (n, k // 16))
    x = rng.integers(-4, 5, (m, k)).astype(np.float64)
    got = O.project_w4a16(x, codes, scales, np.float32(1.0))
    for r in range(m):
        for j in range(n):
            acc = Fraction(0)
            for kk in range(k):
                byte = int(codes[j, kk // 2])
                nib = byte & 15 if kk % 2 == 0 else byte >> 4
                acc += int(x[r, kk]) * _e2m1_frac(nib) * _e4m3_frac(int(scales[j, kk // 16]))
            assert Fraction(got[r, j]) == acc


def _perm_weight(n, k, perm, vals):
    """[n, k] weight with one nonzero per row: w[i, perm[i]] = vals[i]."""
    w = np.zeros((n, k), np.float32)
    w[np.arange(n), perm] = vals
    return w


def test_ffn_closed_form_with_permutation_weights():
    # hidden = inter = 32.  Each weight row has a single nonzero whose value
    # is amax * 2^-j with amax = 2688 * 2^-10, so gs = 2^-10, every block scale
    # is 448 * 2^-j (exact in E4M3) and every nonzero encodes to +-6 exactly:
    # the quantised weights equal the original ones.  Then
    #   g[r, i] = wg[i] * x[r, pg[i]],  u[r, i] = wu[i] * x[r, pu[i]],
    #   out[r, i] = bf16(wd[i] * h[r, pd[i]]),  h = bf16(silu(bf16 g) * bf16 u).
    H = I = 32
    rng = np.random.default_rng(4)
    amax = np.float32(2688.0 * 2.0 ** -10)
    def vals():
        v = amax * np.float32(2.0) ** -rng.integers(0, 5, I).astype(np.float32)
        v *= rng.choice(np.float32([-1, 1]), I)
        v[0] = amax
        return v.astype(np.float32)
    pg, pu, pd = rng.permutation(H), rng.permutation(H), rng.permutation(I)
    vg, vu, vd = vals(), vals(), vals()
    Wg, Wu, Wd = _perm_weight(I, H, pg, vg), _perm_weight(I, H, pu, vu), _perm_weight(H, I, pd, vd)
    qg, qu, qd = O.quantize_weight(Wg), O.quantize_weight(Wu), O.quantize_weight(Wd)
    for q, W in [(qg, Wg), (qu, Wu), (qd, Wd)]:
        assert float(q[2]) == 2.0 ** -10
        assert np.array_equal(O.dequantize(q[0], q[1]) * float(q[2]), W.astype(np.float64))
    x = synth.bf16_bits_to_f32(synth.random_bf16((3, H), 5)).astype(np.float64)
    out, h = O.ffn_w4a16(x, qg, qu, qd, return_h=True)
    g = O.round_to_bf16(vg.astype(np.float64)[None, :] * x[:, pg])
    u = O.round_to_bf16(vu.astype(np.float64)[None, :] * x[:, pu])
    hh = O.round_to_bf16(g / (1.0 + np.exp(-g)) * u)
    assert np.array_equal(h, hh)
    assert np.array_equal(out, O.round_to_bf16(vd.astype(np.float64)[None, :] * hh[:, pd]))


def _tiny_ffn_weights(H, I, seed):
    rng = np.random.default_rng(seed)
    mk = lambda n, k: synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(
        rng.standard_normal((n, k)).astype(np.float32) * np.float32(0.02)))
    return O.quantize_weight(mk(I, H)), O.quantize_weight(mk(I, H)), O.quantize_weight(mk(H, I))


def test_fused_gate_up_equals_separate():
    H, I = 64, 96
    qg, qu, qd = _tiny_ffn_weights(H, I, 6)
    fc, fs, (gsg, gsu) = O.fuse_gate_up(qg, qu)
    x = synth.bf16_bits_to_f32(synth.random_bf16((5, H), 7)).astype(np.float64)
    fused = np.concatenate([O.project_w4a16(x, fc[:I], fs[:I], gsg),
                            O.project_w4a16(x, fc[I:], fs[I:], gsu)], axis=1)
    sep = np.concatenate([O.project_w4a16(x, *qg), O.project_w4a16(x, *qu)], axis=1)
    assert np.array_equal(fused, sep)
    assert fc[:I].tobytes() == qg[0].tobytes() and fc[I:].tobytes() == qu[0].tobytes()


@pytest.mark.parametrize("ffn", [O.ffn_w4a16, O.ffn_w4a4])
def test_rows_are_independent(ffn):
    H, I = 64, 128
    qg, qu, qd = _tiny_ffn_weights(H, I, 8)
    x = synth.bf16_bits_to_f32(synth.random_bf16((7, H), 9)).astype(np.float64)
    full = ffn(x, qg, qu, qd)
    for r in range(7):
        assert np.array_equal(ffn(x[r:r + 1], qg, qu, qd)[0], full[r])


def test_w4a4_reduces_to_w4a16_on_nvfp4_activations():
    # activations that are exactly E2M1 value * E4M3 scale with the block max at
    # +-6 * scale quantise without loss, so both projections agree exactly.
    rng = np.random.default_rng(10)
    m, n, k = 3, 8, 64
    codes = rng.integers(0, 16, (m, k)).astype(np.uint8)
    codes[:, ::16] = 7                                   # block max magnitude 6
    sc = np.array([0x30, 0x38, 0x40], dtype=np.uint8)    # 0.5, 1, 2
    s = O.e4m3_decode(rng.choice(sc, (m, k // 16)))
    x = (O.e2m1_decode(codes).reshape(m, k // 16, 16) * s[..., None]).reshape(m, k)
    wc, ws, gs = _random_weight(n, k, 11)
    assert np.array_equal(O.project_w4a4(x, wc, ws, gs), O.project_w4a16(x, wc, ws, gs))


def test_w4a4_equals_integer_block_sum_form():
    m, n, k = 2, 3, 64
    wc, ws, gs = _random_weight(n, k, 12)
    x = synth.bf16_bits_to_f32(synth.random_bf16((m, k), 13))
    xc, xs = O.quantize_activation(x)
    got = O.project_w4a4(x.astype(np.float64), wc, ws, gs)
    for r in range(m):
        for j in range(n):
            tot = Fraction(0)
            for b in range(k // 16):
                S = 0   # integer block sum of (2 qa) (2 qw)
                for i in range(16):
                    kk = 16 * b + i
                    na = (int(xc[r, kk // 2]) >> (4 * (kk % 2))) & 15
                    nw = (int(wc[j, kk // 2]) >> (4 * (kk % 2))) & 15
                    S += int(2 * _e2m1_frac(na)) * int(2 * _e2m1_frac(nw))
                tot += _e4m3_frac(int(xs[r, b])) * _e4m3_frac(int(ws[j, b])) * Fraction(S, 4)
            exact = Fraction(float(gs)) * tot
            assert abs(Fraction(got[r, j]) - exact) <= abs(exact) * Fraction(1, 10 ** 12) + Fraction(1, 10 ** 300)


def test_error_stats_definition():
    ref = np.array([1.0, -2.0, 2.0, 0.0])
    out = np.array([1.0, -2.5, 2.0, 0.25])
    st = O.error_stats(out, ref)
    assert st["max_abs"] == 0.5
    assert st["rel_l1"] == 0.75 / 5.0
    assert abs(st["rms_ref"] - np.sqrt(9 / 4)) < 1e-15
