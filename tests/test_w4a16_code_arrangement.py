"""CPU checks of the bf16-activation path's operand encoding (restated here
from the kernel's description; the GPU parity tests check the kernel itself):

* the code-bit rearrangement inside a 32-bit word is a bijection, and decoding
  output pair k by its rotations and masks yields, for every code at every
  position, the bf16 pattern s | (e1 e0 m) << 6 whose value is E2M1 * 2^-126;
* the block-scale decode (E4M3 -> f16 bits, >> 3, + 230 << 7) gives the bf16
  number s * 2^118 exactly for every non-negative finite E4M3 value, so that
  the A operand is E2M1 * s * 2^-8 and the epilogue restores it with 2^8."""
import numpy as np

from oracle import nvfp4_ffn as O

M, MA, MB = 0x81C081C0, 0x80C080C0, 0x01000100
POS = [6, 7, 8, 15]          # destination bits of code bits m, e0, e1, s


def src_bit(k, p):
    if k == 0:
        return p
    if k == 1:
        return p - 4
    if k == 2:
        return (p + 6) & 31
    return (p + 2) & 31 if (p & 15) == 8 else p - 6


def permute(nat):
    out = 0
    for e in range(8):
        for b in range(4):
            p = POS[b] + 16 * (e & 1)
            out |= ((nat >> (4 * e + b)) & 1) << src_bit(e >> 1, p)
    return out


def rotr(x, r):
    return ((x >> r) | (x << (32 - r))) & 0xFFFFFFFF if r else x


def decode(c):
    shl = lambda x, k: (x << k) & 0xFFFFFFFF
    return [c & M, shl(c, 4) & M, rotr(c, 6) & M, (shl(c, 6) & MA) | (rotr(c, 2) & MB)]


def bf16_value(bits16):
    return float(np.array([bits16 << 16], np.uint32).view(np.float32)[0])


def test_rearrangement_is_a_bijection():
    srcs = sorted(src_bit(e >> 1, POS[b] + 16 * (e & 1)) for e in range(8) for b in range(4))
    assert srcs == list(range(32))


def test_decoded_pairs_are_e2m1_times_2_pow_minus_126():
    rng = np.random.default_rng(0)
    words = [int(w) for w in rng.integers(0, 2**32, 2000, dtype=np.uint64)]
    words += [0, 0xFFFFFFFF, 0x88888888, 0x77777777] + [c * 0x11111111 for c in range(16)]
    for nat in words:
        pairs = decode(permute(nat))
        for e in range(8):
            code = (nat >> (4 * e)) & 15
            half = (pairs[e >> 1] >> (16 * (e & 1))) & 0xFFFF
            want = float(O.e2m1_decode(np.array([code], np.uint8))[0]) * 2.0 ** -126
            got = bf16_value(half)
            assert got == want and np.signbit(got) == bool(code & 8), (hex(nat), e, code, got, want)


def test_scale_rebias_is_exact():
    for s8 in range(0x7F):  # 0x7F is NaN
        f16 = np.array([O.e4m3_decode(np.array([s8], np.uint8))[0]], np.float16)
        h = int(f16.view(np.uint16)[0])
        b = ((h >> 3) + (230 << 7)) & 0xFFFF
        want = float(O.e4m3_decode(np.array([s8], np.uint8))[0]) * 2.0 ** 118
        if s8 == 0:
            assert bf16_value(b) == 2.0 ** 103  # zero-scale blocks carry zero codes
        else:
            assert bf16_value(b) == want, (s8, bf16_value(b), want)
    # largest A element stays finite, smallest stays normal
    assert 448.0 * 2.0 ** 118 < 3.3895e38 and 0.5 * 2.0 ** -9 * 2.0 ** -8 >= 2.0 ** -126
