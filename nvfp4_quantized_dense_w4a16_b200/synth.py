"""Seeded synthetic inputs for the NVFP4 SwiGLU FFN.

This module only draws random numbers and stores them as bf16 bit patterns.
It holds none of the FFN's arithmetic (no quantisation, no projection, no
activation), so both the CUDA path and the CPU oracle can take their inputs
from here without sharing any of the method.

Every workload is drawn with numpy's PCG64 generator (``default_rng(seed)``)
in float32, in the fixed order x, W_gate, W_up, W_down, and each float32 draw
is rounded to the nearest bf16 (ties to even) to give the bf16 tensors the
library consumes.  Weights are returned as bf16 bit patterns (uint16) of
shape [n, k] with k contiguous (the PyTorch ``nn.Linear`` layout: gate/up are
[inter, hidden], down is [hidden, inter]).

Workloads (hidden H, inter I, rows m):

* ``tiny``      m=4,    H=256,  I=512,   seed 0: x~N(0,1), W~N(0,0.02)
* ``decode``    m=1,    H=5120, I=17408, seed 1: as tiny, and each 16-element
  block of each weight row is independently (p=0.01) scaled by 8 before
  rounding (per-row outlier blocks)
* ``smallm``    m in {8,16,32,64}, H=5120, I=17408, seed 2: as tiny
* ``prefill``   m=4096, H=5120, I=17408, seed 3: x~N(0,1) with round(0.001*H)
  channels (chosen without replacement) multiplied by 20 in every row
* ``w4a4``      m in {1,7,64,512}, H=4096, I=12288, seed 4: x~N(0,1) drawn once
  for 512 rows; smaller m take the first m rows, so the same row is compared
  across batch sizes.
"""
from __future__ import annotations

import dataclasses

import numpy as np

WEIGHT_STD = 0.02
OUTLIER_BLOCK_P = 0.01
OUTLIER_BLOCK_GAIN = 8.0
OUTLIER_CHANNEL_FRAC = 0.001
OUTLIER_CHANNEL_GAIN = 20.0


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits.

    Input preparation only: the generator draws float32 numbers and the
    library's inputs are bf16.  Inputs are finite by construction.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = (u + 0x7FFF + lsb) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class FfnInputs:
    name: str
    m: int
    hidden: int
    inter: int
    x: np.ndarray        # uint16 bf16 bits [m, hidden]
    w_gate: np.ndarray   # uint16 bf16 bits [inter, hidden]
    w_up: np.ndarray     # uint16 bf16 bits [inter, hidden]
    w_down: np.ndarray   # uint16 bf16 bits [hidden, inter]

    def with_rows(self, m: int) -> "FfnInputs":
        """The same weights with the first ``m`` rows of x."""
        assert m <= self.x.shape[0]
        return dataclasses.replace(self, m=m, x=self.x[:m].copy())


WORKLOADS = {
    # name: (m, hidden, inter, seed)
    "tiny": (4, 256, 512, 0),
    "decode": (1, 5120, 17408, 1),
    "smallm": (64, 5120, 17408, 2),
    "prefill": (4096, 5120, 17408, 3),
    "w4a4": (512, 4096, 12288, 4),
}


def _weights(rng: np.random.Generator, n: int, k: int, outlier_blocks: bool) -> np.ndarray:
    w = rng.standard_normal((n, k), dtype=np.float32) * np.float32(WEIGHT_STD)
    if outlier_blocks:
        nb = k // 16
        hit = rng.random((n, nb)) < OUTLIER_BLOCK_P
        gain = np.where(hit, np.float32(OUTLIER_BLOCK_GAIN), np.float32(1.0)).astype(np.float32)
        w = (w.reshape(n, nb, 16) * gain[:, :, None]).reshape(n, k)
    return f32_to_bf16_bits(w)


def make_inputs(name: str, m: int | None = None, hidden: int | None = None,
                inter: int | None = None, seed: int | None = None) -> FfnInputs:
    """Draw the workload ``name``; sizes and seed may be overridden (tests use
    reduced sizes of the same recipe)."""
    m0, h0, i0, s0 = WORKLOADS[name]
    m = m0 if m is None else m
    hidden = h0 if hidden is None else hidden
    inter = i0 if inter is None else inter
    seed = s0 if seed is None else seed
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((m, hidden), dtype=np.float32)
    if name == "prefill":
        nch = max(1, int(round(OUTLIER_CHANNEL_FRAC * hidden)))
        ch = rng.choice(hidden, size=nch, replace=False)
        x[:, ch] *= np.float32(OUTLIER_CHANNEL_GAIN)
    outl = name == "decode"
    wg = _weights(rng, inter, hidden, outl)
    wu = _weights(rng, inter, hidden, outl)
    wd = _weights(rng, hidden, inter, outl)
    return FfnInputs(name, m, hidden, inter, f32_to_bf16_bits(x), wg, wu, wd)


def random_bf16(shape, seed: int, std: float = 1.0) -> np.ndarray:
    """N(0, std^2) float32 draws rounded to bf16 bits (generic test tensors)."""
    rng = np.random.default_rng(seed)
    a = rng.standard_normal(shape, dtype=np.float32) * np.float32(std)
    return f32_to_bf16_bits(a)
