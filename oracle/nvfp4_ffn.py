"""Plain CPU oracle of the NVFP4 SwiGLU FFN (W4A16 and fixed-format W4A4).

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and
bench.py's CPU baseline, never by the library.

What is computed, and where it comes from
-----------------------------------------
* The FFN dataflow ``out = down(silu(gate(x)) * up(x))`` with gate and up
  written to bf16 activation buffers, ``silu_mul`` overwriting the gate
  buffer in bf16, and down reading that buffer (pages
  "metrale_model_layers/layers/dense_ffn_fixed.rs", ``forward_fixed``, and
  "metrale_model_layers/layers/dense_ffn_prefill.rs", ``prefill_q2`` -- the
  projection / silu_mul / projection sequence).  The rounding points to bf16
  (g, u, h, out) follow from those buffers being bf16 activation buffers.
* The fixed activation format (W4A4): every projection quantises its input
  activation rows to NVFP4 before the block-scaled product, at every row
  count, so a row's result does not depend on the other rows of the launch
  (page "metrale_model_layers/layers/dense_ffn_fixed.rs", module comment and
  ``forward_fixed``: three ``nvfp4_proj_mx`` calls around ``silu_mul``).
* Fused gate+up: one [2*inter, hidden] weight whose rows [0, inter) are the
  gate projection and rows [inter, 2*inter) the up projection, the same bytes
  as the separate weights (page "metrale_model_layers/layers/
  dense_ffn_overlays.rs", ``set_fp8_gate_up_fused``).
* The NVFP4 encoding itself is not on the pages.  It follows the public
  format: FP4 E2M1 elements (OCP Microscaling Formats v1.0, the FP4 element
  type: magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}), one FP8 E4M3 scale per 16
  consecutive elements along K (OCP 8-bit Floating Point v1.0, E4M3: bias 7,
  no infinities, max 448), and one FP32 scale per tensor.

Readings taken where the pages are silent:
  R1 E2M1 encoding rounds to nearest, ties to the even magnitude index,
     saturating at 6; the sign bit is kept (so -0.1 encodes as 0x8).  Packing:
     element 2j in the low nibble of byte j.
  R2 fp32 -> E4M3 rounds to nearest even with saturation to 448.
  R3 weight tensor scale gs = amax / 2688 in fp32 (2688 = 6 * 448); gs = 1
     when amax == 0.
  R4 weight block scale: t = (bamax / gs) / 6 in fp32, s8 = E4M3(t),
     sdec = E4M3value(s8) * gs in fp32, code = E2M1(w / sdec) in fp32; a
     block with s8 == 0 (or sdec == 0) is all code 0.
  R5 W4A4 activation block scale: s8 = E4M3(bamax / 6) in fp32, no tensor
     scale, code = E2M1(x / E4M3value(s8)) in fp32; all-zero block when
     s8 == 0.
  R6 bf16 rounding points g, u, h, out (and, for W4A4, the quantised x and h).
  R7 fused gate+up = concatenation of the separately quantised gate and up,
     each with its own tensor scale.
  R8 relative error = sum|out - ref| / sum|ref|.
  R13 LoRA adapters (page "metrale_model_layers/layers/dense_ffn_overlays.rs",
     set_lora_weights / apply_lora_gate_up / apply_lora_down): a projection's
     adapter is a pair A [r, in], B [out, r] of bf16 values, its delta is
     (x A^T) B^T, with the rank-r product x A^T rounded to bf16 (the pages
     keep it in an activation buffer), the second product summed exactly and
     added to the projection's bf16 output, rounded once more to bf16 (the
     pages add in place into the bf16 gate/up/output buffers).  Gate and up
     deltas are added before the activation, the down delta after the down
     projection.  No separate scaling factor appears (it is folded into B).

Precision: the decisions that produce integer codes are taken in fp32 (the
precision the encoding steps are defined in, and the kernel's), so the codes
are reproducible bit for bit.  Every product and sum of the projections is
in fp64, and results are rounded once to bf16 (nearest even).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "E2M1_MAGNITUDES", "e2m1_decode", "e2m1_encode",
    "e4m3_decode", "e4m3_encode", "round_to_bf16", "bf16_bits_to_f64",
    "f64_to_bf16_bits", "silu",
    "quantize_weight", "quantize_activation", "pack_nibbles", "unpack_nibbles",
    "dequantize", "project_w4a16", "project_w4a4",
    "ffn_w4a16", "ffn_w4a4", "fuse_gate_up", "error_stats", "lora_delta", "ffn_w4a16_lora",
    "WEIGHT_SCALE_DIVISOR",
]

# ---------------------------------------------------------------------------
# Element and scale codecs
# ---------------------------------------------------------------------------

#: FP4 E2M1 magnitudes indexed by the low three bits of a code (OCP MX v1.0).
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)

#: 6 (largest E2M1 magnitude) * 448 (largest E4M3 value): reading R3.
WEIGHT_SCALE_DIVISOR = np.float32(2688.0)


def e2m1_decode(codes) -> np.ndarray:
    """Value of each 4-bit E2M1 code (bit 3 = sign, bits 0-2 = magnitude index)."""
    c = np.asarray(codes).astype(np.int64)
    mag = E2M1_MAGNITUDES[c & 7]
    return np.where((c & 8) != 0, -mag, mag)


def _nearest_index(a: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the entry of ascending ``table`` nearest to each a >= 0.

    Ties (a exactly half way between two neighbours) go to the even index;
    values above the last entry take the last index (saturation).  The
    midpoints are exact in fp64 for the tables used here.
    """
    mids = (table[:-1] + table[1:]) / 2.0
    lo = np.searchsorted(mids, a, side="left")   # number of midpoints < a
    hi = np.searchsorted(mids, a, side="right")  # number of midpoints <= a
    tie = lo != hi                               # a equals midpoint lo
    even = np.where(lo % 2 == 0, lo, hi)
    return np.where(tie, even, lo)


def e2m1_encode(v) -> np.ndarray:
    """E2M1 code of each value (reading R1): nearest magnitude, ties to the
    even magnitude index, saturating at 6, sign bit copied from the input."""
    v = np.asarray(v)
    a = np.abs(v.astype(np.float64))
    idx = _nearest_index(a, E2M1_MAGNITUDES)
    sign = np.signbit(v).astype(np.int64) << 3
    return (idx | sign).astype(np.uint8)


def _e4m3_value_of_bits(b: np.ndarray) -> np.ndarray:
    """E4M3 (OFP8 'E4M3', bias 7, no infinities) value of each byte.

    exponent field 0: subnormal  m/8 * 2^-6;  otherwise (1 + m/8) * 2^(e-7);
    exponent 15 with mantissa 7 is NaN.
    """
    b = np.asarray(b).astype(np.int64)
    s = (b >> 7) & 1
    e = (b >> 3) & 15
    m = b & 7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


_E4M3_POS = _e4m3_value_of_bits(np.arange(127))   # codes 0..126 (0 .. 448), ascending


def e4m3_decode(codes) -> np.ndarray:
    return _e4m3_value_of_bits(codes)


def e4m3_encode(t) -> np.ndarray:
    """Non-negative fp32/fp64 values -> E4M3 byte (reading R2): nearest
    value, ties to the even code (even mantissa), saturating at 448."""
    a = np.asarray(t, dtype=np.float64)
    if np.any(a < 0):
        raise ValueError("block scales are non-negative")
    return _nearest_index(a, _E4M3_POS).astype(np.uint8)


def round_to_bf16(x) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), as fp64.

    bf16 keeps 8 significant bits (exponent range as fp32); below 2^-126 the
    spacing is fixed at 2^-133 (subnormals); beyond the largest finite value
    ((2 - 2^-7) * 2^127) the result overflows to +-inf under round-to-nearest.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                       # |x| = f * 2^e, 0.5 <= f < 1
    q = np.maximum(e - 8, -133)              # exponent of one unit in the last place
    r = np.ldexp(np.rint(np.ldexp(x, -q)), q)  # rint: round half to even
    big = (2.0 - 2.0 ** -7) * 2.0 ** 127
    return np.where(np.abs(r) > big, np.copysign(np.inf, x), r)


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):   # signalling-NaN patterns widen to NaN
        return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x) -> np.ndarray:
    """bf16 bit pattern of each (already bf16-representable) fp64 value."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)  # exact for bf16 values
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def silu(z) -> np.ndarray:
    """SiLU z * sigmoid(z) = z / (1 + exp(-z)) in fp64."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


# ---------------------------------------------------------------------------
# Quantisation (readings R1-R5)
# ---------------------------------------------------------------------------

def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[..., k] nibbles -> [..., k/2] bytes, element 2j in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 15
    out[..., 1::2] = p >> 4
    return out


def _encode_blocks(v: np.ndarray, sdec: np.ndarray, s8: np.ndarray) -> np.ndarray:
    """Codes of v[..., nb, 16] under decoded block scales sdec[..., nb] (fp32)."""
    zero = (s8 == 0) | (sdec == 0)
    safe = np.where(zero, np.float32(1.0), sdec).astype(np.float32)
    q = (v / safe[..., None]).astype(np.float32)           # fp32 IEEE division
    codes = e2m1_encode(q)
    return np.where(zero[..., None], np.uint8(0), codes).astype(np.uint8)


def quantize_weight(w: np.ndarray):
    """NVFP4-quantise a weight [n, k] (bf16 values given as float32).

    Returns (codes uint8 [n, k/2], block scales uint8 [n, k/16] (E4M3),
    tensor scale gs as np.float32).  Readings R1-R4, all in fp32.
    """
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    if k % 16:
        raise ValueError("k must be a multiple of 16")
    amax = np.float32(np.max(np.abs(w))) if w.size else np.float32(0.0)
    gs = np.float32(1.0) if amax == 0 else np.float32(amax / WEIGHT_SCALE_DIVISOR)
    blocks = w.reshape(n, k // 16, 16)
    bamax = np.max(np.abs(blocks), axis=2).astype(np.float32)
    t = ((bamax / gs).astype(np.float32) / np.float32(6.0)).astype(np.float32)
    s8 = e4m3_encode(t)
    sdec = (e4m3_decode(s8).astype(np.float32) * gs).astype(np.float32)
    codes = _encode_blocks(blocks, sdec, s8).reshape(n, k)
    return pack_nibbles(codes), s8, np.float32(gs)


def quantize_activation(x: np.ndarray):
    """Per-row NVFP4 quantisation of activations [m, k] (reading R5).

    Returns (codes uint8 [m, k/2], block scales uint8 [m, k/16]).
    """
    x = np.asarray(x, dtype=np.float32)
    m, k = x.shape
    if k % 16:
        raise ValueError("k must be a multiple of 16")
    blocks = x.reshape(m, k // 16, 16)
    bamax = np.max(np.abs(blocks), axis=2).astype(np.float32)
    s8 = e4m3_encode((bamax / np.float32(6.0)).astype(np.float32))
    sdec = e4m3_decode(s8).astype(np.float32)
    codes = _encode_blocks(blocks, sdec, s8).reshape(m, k)
    return pack_nibbles(codes), s8


def dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """E2M1 value * E4M3 block scale for every element, fp64 [rows, k] (the
    tensor scale is applied by the caller, after the sum over k)."""
    vals = e2m1_decode(unpack_nibbles(codes))
    rows, k = vals.shape
    s = e4m3_decode(scales)
    return (vals.reshape(rows, k // 16, 16) * s[:, :, None]).reshape(rows, k)


# ---------------------------------------------------------------------------
# Projections and the FFN
# ---------------------------------------------------------------------------

def project_w4a16(x: np.ndarray, codes, scales, gs, chunk: int = 4096) -> np.ndarray:
    """y[r, n] = gs * sum_k x[r, k] * w_hat[n, k] in fp64 (not rounded).

    x: activations [m, k] (fp64 values).  Output columns are independent, so
    the weight is dequantised ``chunk`` rows at a time to bound memory; every
    sum over k is one full matrix product.
    """
    x = np.asarray(x, dtype=np.float64)
    n = codes.shape[0]
    y = np.empty((x.shape[0], n), dtype=np.float64)
    for c0 in range(0, n, chunk):
        wd = dequantize(codes[c0:c0 + chunk], scales[c0:c0 + chunk])
        y[:, c0:c0 + chunk] = x @ wd.T
    return float(gs) * y


def project_w4a4(x: np.ndarray, codes, scales, gs, chunk: int = 4096) -> np.ndarray:
    """Fixed-format projection: quantise each row of x (bf16 values) to NVFP4,
    then y = gs * sum_k x_hat[r, k] * w_hat[n, k] in fp64 (not rounded)."""
    xc, xs = quantize_activation(np.asarray(x, dtype=np.float32))
    return project_w4a16(dequantize(xc, xs), codes, scales, gs, chunk)


def fuse_gate_up(gate, up):
    """Fused [2*inter, hidden] weight: gate rows first, then up rows (R7).

    gate / up: (codes, scales, gs) tuples.  Returns (codes, scales, (gs_g, gs_u)).
    """
    return (np.concatenate([gate[0], up[0]], axis=0),
            np.concatenate([gate[1], up[1]], axis=0),
            (np.float32(gate[2]), np.float32(up[2])))


def _ffn(x, gate, up, down, proj):
    x = np.asarray(x, dtype=np.float64)
    g = round_to_bf16(proj(x, *gate))
    u = round_to_bf16(proj(x, *up))
    h = round_to_bf16(silu(g) * u)
    return round_to_bf16(proj(h, *down)), h


def ffn_w4a16(x, gate, up, down, return_h: bool = False):
    """The W4A16 FFN: bf16 activations times NVFP4 weights.

    x: bf16 values [m, hidden]; gate/up/down: (codes, scales, gs).
    g = bf16(x Wg^T), u = bf16(x Wu^T), h = bf16(silu(g) * u),
    out = bf16(h Wd^T)   (reading R6).
    """
    out, h = _ffn(x, gate, up, down, project_w4a16)
    return (out, h) if return_h else out


def ffn_w4a4(x, gate, up, down, return_h: bool = False):
    """Fixed-format FFN: as ``ffn_w4a16`` with x and h quantised per row to
    NVFP4 before their projections."""
    out, h = _ffn(x, gate, up, down, project_w4a4)
    return (out, h) if return_h else out


def lora_delta(x, a, b) -> np.ndarray:
    """Low-rank delta (x A^T) B^T of one projection (reading R13): the rank-r
    product rounded to bf16, the second product in fp64 (not rounded).

    x: [m, in] (bf16 values); a: [r, in]; b: [out, r] (bf16 values)."""
    xa = round_to_bf16(np.asarray(x, dtype=np.float64) @ np.asarray(a, dtype=np.float64).T)
    return xa @ np.asarray(b, dtype=np.float64).T


def ffn_w4a16_lora(x, gate, up, down, lora, return_h: bool = False):
    """The W4A16 FFN with LoRA adapters (reading R13).

    lora: dict with optional keys 'gate', 'up', 'down', each an (A, B) pair.
    g = bf16(bf16(x Wg^T) + delta_g), u likewise, h = bf16(silu(g) * u),
    out = bf16(bf16(h Wd^T) + delta_d)."""
    x = np.asarray(x, dtype=np.float64)

    def proj(inp, w, key):
        y = round_to_bf16(project_w4a16(inp, *w))
        if lora.get(key) is not None:
            y = round_to_bf16(y + lora_delta(inp, *lora[key]))
        return y
    g = proj(x, gate, "gate")
    u = proj(x, up, "up")
    h = round_to_bf16(silu(g) * u)
    out = proj(h, down, "down")
    return (out, h) if return_h else out


def error_stats(out, ref) -> dict:
    """max|out-ref| / rms(ref) and sum|out-ref| / sum|ref| (reading R8)."""
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = np.abs(out - ref)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    return {
        "max_abs": float(d.max()) if d.size else 0.0,
        "rms_ref": rms,
        "max_over_rms": float(d.max() / rms) if rms > 0 else 0.0,
        "rel_l1": float(d.sum() / np.abs(ref).sum()) if np.abs(ref).sum() > 0 else 0.0,
    }
