"""Plausible mistakes planted in the CPU oracle, to show its pins catch them.

Each entry patches the oracle module in place (on the CPU, in a test
process).  ``tests/test_oracle_mutations.py`` runs the oracle's pin tests
once per mutation in a child pytest process with ``FFN_ORACLE_MUTATION`` set
(``tests/conftest.py`` applies the patch at start-up) and requires that run
to fail.  Nothing here is used by the library or by the unmutated tests.
"""
from __future__ import annotations

import numpy as np


def _dropped_h_rounding(O):
    # h = silu(g) * u left unrounded before the down projection
    def _ffn(x, gate, up, down, proj):
        x = np.asarray(x, dtype=np.float64)
        g = O.round_to_bf16(proj(x, *gate))
        u = O.round_to_bf16(proj(x, *up))
        h = O.silu(g) * u
        return O.round_to_bf16(proj(h, *down)), h
    O._ffn = _ffn


def _swapped_silu_operands(O):
    def _ffn(x, gate, up, down, proj):
        x = np.asarray(x, dtype=np.float64)
        g = O.round_to_bf16(proj(x, *gate))
        u = O.round_to_bf16(proj(x, *up))
        h = O.round_to_bf16(O.silu(u) * g)
        return O.round_to_bf16(proj(h, *down)), h
    O._ffn = _ffn


def _ties_round_down(O):
    # nearest-code search that sends every tie to the lower neighbour
    def _nearest_index(a, table):
        mids = (table[:-1] + table[1:]) / 2.0
        return np.searchsorted(mids, a, side="left")
    O._nearest_index = _nearest_index


def _e4m3_bias_8(O):
    def _val(b):
        b = np.asarray(b).astype(np.int64)
        s, e, m = (b >> 7) & 1, (b >> 3) & 15, b & 7
        mag = np.where(e == 0, (m / 8.0) * 2.0 ** -7, (1.0 + m / 8.0) * np.exp2(e - 8.0))
        mag = np.where((e == 15) & (m == 7), np.nan, mag)
        return np.where(s == 1, -mag, mag)
    O._e4m3_value_of_bits = _val
    O._E4M3_POS = _val(np.arange(127))


def _bf16_one_bit_too_many(O):
    def round_to_bf16(x):
        x = np.asarray(x, dtype=np.float64)
        _, e = np.frexp(x)
        q = np.maximum(e - 9, -134)
        return np.ldexp(np.rint(np.ldexp(x, -q)), q)
    O.round_to_bf16 = round_to_bf16


def _scales_on_transposed_blocks(O):
    # block scale applied to element i*(k/16)+b instead of 16*b+i
    def dequantize(codes, scales):
        vals = O.e2m1_decode(O.unpack_nibbles(codes))
        rows, k = vals.shape
        s = O.e4m3_decode(scales)
        return (vals.reshape(rows, 16, k // 16) * s[:, None, :]).reshape(rows, k)
    O.dequantize = dequantize


def _high_nibble_first(O):
    def unpack_nibbles(packed):
        p = np.asarray(packed, dtype=np.uint8)
        out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
        out[..., 0::2] = p >> 4
        out[..., 1::2] = p & 15
        return out
    O.unpack_nibbles = unpack_nibbles


def _e2m1_table_entry(O):
    O.E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 2.5, 4.0, 6.0])


def _weight_scale_divisor(O):
    O.WEIGHT_SCALE_DIVISOR = np.float32(6.0 * 256.0)


def _activation_scale_amax_over_4(O):
    orig = O.quantize_activation

    def quantize_activation(x):
        return orig(np.asarray(x, dtype=np.float32) * np.float32(1.5))
    O.quantize_activation = quantize_activation


def _projection_drops_tensor_scale(O):
    orig = O.project_w4a16

    def project_w4a16(x, codes, scales, gs, chunk=4096):
        return orig(x, codes, scales, np.float32(1.0), chunk)
    O.project_w4a16 = project_w4a16


def _transposed_activation(O):
    orig = O.project_w4a16

    def project_w4a16(x, codes, scales, gs, chunk=4096):
        x = np.asarray(x, dtype=np.float64)
        return orig(x[:, ::-1].copy(), codes, scales, gs, chunk)
    O.project_w4a16 = project_w4a16


def _lora_xa_unrounded(O):
    def lora_delta(x, a, b):
        return (np.asarray(x, np.float64) @ np.asarray(a, np.float64).T) @ np.asarray(b, np.float64).T
    O.lora_delta = lora_delta


def _lora_gate_delta_after_activation(O):
    def ffn_w4a16_lora(x, gate, up, down, lora, return_h=False):
        x = np.asarray(x, dtype=np.float64)
        g = O.round_to_bf16(O.project_w4a16(x, *gate))
        u = O.round_to_bf16(O.project_w4a16(x, *up))
        if lora.get("up") is not None:
            u = O.round_to_bf16(u + O.lora_delta(x, *lora["up"]))
        h = O.round_to_bf16(O.silu(g) * u)
        if lora.get("gate") is not None:
            h = O.round_to_bf16(h + O.lora_delta(x, *lora["gate"]))
        out = O.round_to_bf16(O.project_w4a16(h, *down))
        if lora.get("down") is not None:
            out = O.round_to_bf16(out + O.lora_delta(h, *lora["down"]))
        return (out, h) if return_h else out
    O.ffn_w4a16_lora = ffn_w4a16_lora


def _lora_adapter_transposed(O):
    def lora_delta(x, a, b):
        xa = O.round_to_bf16(np.asarray(x, np.float64) @ np.asarray(a, np.float64)[:, ::-1].T)
        return xa @ np.asarray(b, np.float64).T
    O.lora_delta = lora_delta


MUTATIONS = {
    "dropped_h_rounding": _dropped_h_rounding,
    "swapped_silu_operands": _swapped_silu_operands,
    "ties_round_down": _ties_round_down,
    "e4m3_bias_8": _e4m3_bias_8,
    "bf16_one_bit_too_many": _bf16_one_bit_too_many,
    "scales_on_transposed_blocks": _scales_on_transposed_blocks,
    "high_nibble_first": _high_nibble_first,
    "e2m1_table_entry": _e2m1_table_entry,
    "weight_scale_divisor": _weight_scale_divisor,
    "activation_scale_amax_over_4": _activation_scale_amax_over_4,
    "projection_drops_tensor_scale": _projection_drops_tensor_scale,
    "transposed_activation": _transposed_activation,
    "lora_xa_unrounded": _lora_xa_unrounded,
    "lora_gate_delta_after_activation": _lora_gate_delta_after_activation,
    "lora_adapter_transposed": _lora_adapter_transposed,
}


def apply(name: str):
    from oracle import nvfp4_ffn as O
    MUTATIONS[name](O)
