"""Shared helpers of the GPU parity tests: run the same seeded inputs through
the CUDA library (C ABI, via the ctypes binding) and through the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

from oracle import nvfp4_ffn as O
from nvfp4_quantized_dense_w4a16_b200 import synth

# Acceptance thresholds for FFN outputs against the fp64 oracle.
MAX_ERR_OVER_RMS = 2e-2
REL_L1 = 5e-3


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle_weight(bits: np.ndarray):
    return O.quantize_weight(synth.bf16_bits_to_f32(bits))


def gpu_weight(native, bits: np.ndarray):
    """Quantise on the GPU and build a handle; returns (handle, codes, scales, gs)."""
    w = to_dev_bf16(bits)
    codes, scales, gs = native.ffn_nvfp4_quantize_weights(w)
    h = native.ffn_nvfp4_weight_create(codes, scales, gs)
    return h, codes, scales, gs


def assert_quant_equal(gpu, ref):
    codes, scales, gs = gpu[1], gpu[2], gpu[3]
    rc, rs, rgs = ref
    assert float(gs.item()) == float(rgs), (float(gs.item()), float(rgs))
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """One bf16 unit in the last place at |v| (normal range; 2^-133 below)."""
    _, e = np.frexp(np.abs(np.asarray(v, dtype=np.float64)))
    return np.ldexp(1.0, np.maximum(e - 8, -133))


# At most this fraction of the outputs may exceed the max-error bound, and
# only by a single final bf16 rounding step (see assert_close).
MAX_FLIP_FRACTION = 1e-4


def assert_close(out: np.ndarray, ref: np.ndarray, what: str = ""):
    """The FFN acceptance thresholds: max|err| <= 2e-2 * rms(ref) and
    sum|err| / sum|ref| <= 5e-3.  The max bound is applied to every output
    except one-ulp final-rounding flips: an output larger than ~2.6 x rms
    whose exact value lies next to a bf16 rounding midpoint rounds to one
    neighbour under fp32 accumulation and to the other under the oracle's
    fp64 sum, and one bf16 step there already exceeds 2e-2 * rms.  Such flips
    must be at most one ulp of the reference and rare (MAX_FLIP_FRACTION)."""
    st = O.error_stats(out, ref)
    assert np.all(np.isfinite(out)), what
    d = np.abs(out - ref)
    bound = MAX_ERR_OVER_RMS * st["rms_ref"]
    over = d > bound
    flips = over & (d <= bf16_ulp(ref))
    st["rounding_flips"] = int(flips.sum())
    assert not np.any(over & ~flips), (what, st, float(d[over & ~flips].max() / max(st["rms_ref"], 1e-300)))
    assert flips.sum() <= max(1, MAX_FLIP_FRACTION * d.size), (what, st)
    assert st["rel_l1"] <= REL_L1, (what, st)
    return st


class FfnCase:
    """A workload quantised on both sides, with GPU handles ready."""

    def __init__(self, native, inp: synth.FfnInputs, check_quant: bool = True):
        self.inp = inp
        self.native = native
        self.qg, self.qu, self.qd = (oracle_weight(inp.w_gate), oracle_weight(inp.w_up),
                                     oracle_weight(inp.w_down))
        g, u, d = gpu_weight(native, inp.w_gate), gpu_weight(native, inp.w_up), gpu_weight(native, inp.w_down)
        if check_quant:
            assert_quant_equal(g, self.qg)
            assert_quant_equal(u, self.qu)
            assert_quant_equal(d, self.qd)
        self.gate, self.up, self.down = g[0], u[0], d[0]
        self.gate_up = native.ffn_nvfp4_weight_create_gate_up(self.gate, self.up)
        self.x_dev = to_dev_bf16(inp.x)
        self.x64 = synth.bf16_bits_to_f32(inp.x).astype(np.float64)

    def forward(self, fmt="bf16", rows=None):
        x = self.x_dev if rows is None else self.x_dev[:rows].contiguous()
        out = self.native.ffn_nvfp4_forward(x, self.gate_up, self.down, fmt)
        torch.cuda.synchronize()
        return out

    def oracle(self, fmt="bf16", rows=None):
        x = self.x64 if rows is None else self.x64[rows]
        f = O.ffn_w4a16 if fmt == "bf16" else O.ffn_w4a4
        return f(x, self.qg, self.qu, self.qd)
