"""Pins for the oracle's LoRA adapters on the NVFP4 FFN (reading R13 of the
oracle: delta = (x A^T) B^T, rank-r product rounded to bf16, added to the
bf16 projection output and rounded again; gate/up deltas before the
activation, the down delta after the down projection).

* the delta against exact rational arithmetic on tiny sizes, with the bf16
  rounding of the rank-r product taken by torch's conversion;
* zero adapters leave the FFN unchanged;
* with every value exactly representable, the adapted FFN equals an FFN
  whose weights are merged with B A, computed by brute force in exact
  rationals (which fixes where each delta enters the layer);
* rows stay independent.
"""
from fractions import Fraction

import numpy as np
import torch

from oracle import nvfp4_ffn as O
from nvfp4_quantized_dense_w4a16_b200 import synth


def _bf16(v):
    """bf16 rounding of an exact Fraction via torch (nearest even; the value
    is first converted to fp64, exact for the small dyadic values here)."""
    return Fraction(float(torch.tensor([float(v)], dtype=torch.float64).to(torch.bfloat16).double()))


def _rand_bf16(shape, seed, std):
    return synth.bf16_bits_to_f32(synth.random_bf16(shape, seed, std=std)).astype(np.float64)


def test_lora_delta_matches_exact_rationals():
    m, k, n, r = 3, 40, 6, 4
    x, a, b = _rand_bf16((m, k), 1, 1.0), _rand_bf16((r, k), 2, 0.1), _rand_bf16((n, r), 3, 0.1)
    got = O.lora_delta(x, a, b)
    for i in range(m):
        xa = [_bf16(sum(Fraction(float(x[i, kk])) * Fraction(float(a[j, kk])) for kk in range(k)))
              for j in range(r)]
        for c in range(n):
            exact = sum(xa[j] * Fraction(float(b[c, j])) for j in range(r))
            assert abs(Fraction(got[i, c]) - exact) <= abs(exact) * Fraction(1, 10 ** 12) + Fraction(1, 10 ** 300)


def _tiny_ffn(H, I, seed):
    rng = np.random.default_rng(seed)
    mk = lambda n, k: synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(
        rng.standard_normal((n, k)).astype(np.float32) * np.float32(0.02)))
    return O.quantize_weight(mk(I, H)), O.quantize_weight(mk(I, H)), O.quantize_weight(mk(H, I))


def test_zero_adapters_leave_the_ffn_unchanged():
    H, I, r = 64, 96, 8
    qg, qu, qd = _tiny_ffn(H, I, 4)
    x = _rand_bf16((5, H), 5, 1.0)
    zero = {"gate": (np.zeros((r, H)), _rand_bf16((I, r), 6, 0.1)),
            "up": (_rand_bf16((r, H), 7, 0.1), np.zeros((I, r))),
            "down": (np.zeros((r, I)), np.zeros((H, r)))}
    assert np.array_equal(O.ffn_w4a16_lora(x, qg, qu, qd, zero), O.ffn_w4a16(x, qg, qu, qd))
    assert np.array_equal(O.ffn_w4a16_lora(x, qg, qu, qd, {}), O.ffn_w4a16(x, qg, qu, qd))


def _e2m1_frac(c):
    v = [0, Fraction(1, 2), 1, Fraction(3, 2), 2, 3, 4, 6][c & 7]
    return -Fraction(v) if c & 8 else Fraction(v)


def _dense(codes, scales):
    """Exact rational dequantised weight (tensor scale 1, power-of-two E4M3
    scale bytes 0x30/0x38 = 1/2, 1)."""
    n, half = codes.shape
    sc = {0x30: Fraction(1, 2), 0x38: Fraction(1)}
    W = [[None] * (2 * half) for _ in range(n)]
    for i in range(n):
        for kk in range(2 * half):
            nib = (int(codes[i, kk // 2]) >> (4 * (kk % 2))) & 15
            W[i][kk] = _e2m1_frac(nib) * sc[int(scales[i, kk // 16])]
    return W


def test_adapted_ffn_equals_merged_weights_by_brute_force():
    # Values chosen so that every intermediate the layer does not round is
    # exact in bf16: x in {-1, 0, 1}; gate/up weights with two non-zero E2M1
    # codes per row (scale 1/2 or 1); adapter entries in {-1, 0, 1} / 4 at
    # rank 2, so |g|, |u| < 16 on a 1/16 grid.  The down weight is zero and
    # its adapter's A has one-hot rows, so x A^T picks entries of h exactly.
    # Then the rank-r route must equal an FFN whose weights are merged with
    # B A, computed by brute force in exact rationals -- which fixes where each
    # delta enters (gate/up before the activation, down after the projection).
    rng = np.random.default_rng(8)
    m, H, I, r = 2, 32, 32, 2

    def sparse_weight(n, k, nnz):
        nib = np.zeros((n, k), np.uint8)
        for i in range(n):
            nib[i, rng.choice(k, nnz, replace=False)] = rng.integers(1, 16, nnz)
        return (O.pack_nibbles(nib), rng.choice(np.array([0x30, 0x38], np.uint8), (n, k // 16)), np.float32(1.0))
    qg, qu = sparse_weight(I, H, 2), sparse_weight(I, H, 2)
    qd = (np.zeros((H, I // 2), np.uint8), np.full((H, I // 16), 0x38, np.uint8), np.float32(1.0))
    x = rng.integers(-1, 2, (m, H)).astype(np.float64)
    ad = lambda n, k: rng.integers(-1, 2, (n, k)).astype(np.float64) * 0.25
    onehot = np.zeros((r, I))
    onehot[np.arange(r), rng.choice(I, r, replace=False)] = 1.0
    lora = {"gate": (ad(r, H), ad(I, r)), "up": (ad(r, H), ad(I, r)),
            "down": (onehot, synth.bf16_bits_to_f32(synth.random_bf16((H, r), 12, std=0.5)).astype(np.float64))}
    got = O.ffn_w4a16_lora(x, qg, qu, qd, lora)

    def merged(q, key):
        W = _dense(q[0], q[1])
        A, B = lora[key]
        return [[W[i][kk] + sum(Fraction(B[i, j]) * Fraction(A[j, kk]) for j in range(r))
                 for kk in range(len(W[0]))] for i in range(len(W))]
    Wg, Wu, Wd = merged(qg, "gate"), merged(qu, "up"), merged(qd, "down")
    for row in range(m):
        xr = [Fraction(v) for v in x[row]]
        g = [_bf16(sum(a * b for a, b in zip(xr, Wg[i]))) for i in range(I)]
        u = [_bf16(sum(a * b for a, b in zip(xr, Wu[i]))) for i in range(I)]
        # silu in fp64 (the oracle's own silu is pinned elsewhere), rounded once
        h = [_bf16(Fraction(float(O.silu(np.float64(gi)))) * ui) for gi, ui in zip(g, u)]
        out = [_bf16(sum(a * b for a, b in zip(h, Wd[i]))) for i in range(H)]
        assert [float(v) for v in out] == got[row].tolist()
    assert np.any(got != 0)


def test_rows_are_independent_with_adapters():
    H, I, r = 64, 128, 4
    qg, qu, qd = _tiny_ffn(H, I, 9)
    lora = {k: (_rand_bf16((r, n_in), 10 + i, 0.1), _rand_bf16((n_out, r), 20 + i, 0.1))
            for i, (k, n_in, n_out) in enumerate((("gate", H, I), ("up", H, I), ("down", I, H)))}
    x = _rand_bf16((6, H), 11, 1.0)
    full = O.ffn_w4a16_lora(x, qg, qu, qd, lora)
    for r_ in range(6):
        assert np.array_equal(O.ffn_w4a16_lora(x[r_:r_ + 1], qg, qu, qd, lora)[0], full[r_])
