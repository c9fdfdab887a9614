"""Bit-exact GPU parity on exactly representable inputs, for every kernel
configuration the m-dispatch can pick.

With tensor scale 1, power-of-two E4M3 block scales and small integer (or
NVFP4-grid) activations, every product and every partial sum of a projection
is a multiple of a fixed power of two and far below 2^24 of it, so fp32
accumulation in any order is exact.  The kernel's result, rounded once to
bf16, must then equal the fp64 oracle's rounded result bit for bit -- whatever
the tile width, the split-K count, the order of the fixed-order reduction or
the block-scaled FP4 MMA.  A wrong tile row, a dropped K chunk, a misplaced
scale or a wrong unscale factor changes bits here even where it would hide
inside the FFN tolerance.

Each case asserts, through ffn_nvfp4_projection_plan, that it reaches the
configuration it is meant to cover.
"""
import numpy as np
import pytest
import torch

from oracle import nvfp4_ffn as O

pytestmark = pytest.mark.gpu

from gpu_helpers import bf16_to_f64


@pytest.fixture(scope="module")
def native():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from nvfp4_quantized_dense_w4a16_b200 import build
    build.build()
    from nvfp4_quantized_dense_w4a16_b200 import native as N
    return N


# E4M3 bytes of 2^-3, 2^-2, 2^-1, 2^0 (exponent field e, value 2^(e-7)).
POW2_SCALES = np.array([0x20, 0x28, 0x30, 0x38], np.uint8)


def exact_weight(rng, n, k, scale_bytes=POW2_SCALES, zero_block_p=0.02):
    """Random codes, power-of-two block scales (a few zero blocks), gs = 1.

    Worst case per K element: |E2M1| 6 x scale 1 x |x| 2 = 12; with K <= 4096
    every partial sum stays below 2^16 in magnitude and is a multiple of 2^-4
    (2^-12 inside the kernel, whose decoded operand carries a 2^-8 factor), so
    fp32 holds it exactly."""
    codes = rng.integers(0, 256, (n, k // 2), dtype=np.uint8)
    scales = rng.choice(scale_bytes, (n, k // 16)).astype(np.uint8)
    scales[rng.random((n, k // 16)) < zero_block_p] = 0
    return codes, scales


def make_handle(native, codes, scales):
    return native.ffn_nvfp4_weight_create(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(),
                                          torch.ones(1, dtype=torch.float32, device="cuda"))


W4A16_CASES = [
    # (m, n, k, tile rows, K splits)
    (4, 384, 512, 16, 1), (4, 128, 4096, 16, 8),
    (20, 384, 512, 32, 1), (20, 128, 4096, 32, 8),
    (50, 384, 512, 64, 1), (50, 128, 4096, 64, 8),
    (100, 384, 512, 128, 1), (100, 128, 4096, 128, 8),
    (300, 384, 512, 256, 1), (300, 128, 4096, 256, 8),
    (1, 256, 2048, 16, 4), (129, 200, 1056, 256, None), (513, 384, 2048, 256, None),
]


@pytest.mark.parametrize("m,n,k,bn,splits", W4A16_CASES)
def test_w4a16_exact_inputs_bit_exact(native, m, n, k, bn, splits):
    plan = native.ffn_nvfp4_projection_plan(m, n, k, "bf16")
    assert plan["family"] == "tc_w4a16" and plan["tile_rows"] == bn, plan
    if splits is not None:
        assert plan["k_splits"] == splits, plan
    rng = np.random.default_rng(1000 + m + n + k)
    codes, scales = exact_weight(rng, n, k)
    x = rng.integers(-2, 3, (m, k)).astype(np.float32)
    w = make_handle(native, codes, scales)
    y = native.ffn_nvfp4_linear(torch.from_numpy(x).cuda().to(torch.bfloat16), w, "bf16")
    torch.cuda.synchronize()
    ref = O.round_to_bf16(O.project_w4a16(x.astype(np.float64), codes, scales, np.float32(1.0)))
    got = bf16_to_f64(y)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} mismatches, first at {bad[:3].tolist()}: {got[tuple(bad[0])]} vs {ref[tuple(bad[0])]}"


def exact_activations(rng, m, k):
    """Activations on the NVFP4 grid: per 16-block a power-of-two scale s
    (2^-2..2^0) and E2M1 values times s, one element of each block at +-6 s,
    so the per-row quantiser reproduces them exactly (scale = amax/6 = s)."""
    nb = k // 16
    s = np.exp2(rng.integers(-2, 1, (m, nb))).astype(np.float32)
    vals = O.e2m1_decode(rng.integers(0, 16, (m, nb, 16)))
    pos = rng.integers(0, 16, (m, nb))
    sign = np.where(rng.random((m, nb)) < 0.5, -1.0, 1.0)
    np.put_along_axis(vals, pos[:, :, None], (6.0 * sign)[:, :, None], axis=2)
    return (vals * s[:, :, None]).reshape(m, k).astype(np.float32)


W4A4_CASES = [
    # (m, n, k, K splits)
    (1, 384, 256, 1), (1, 128, 4096, 8),
    (130, 384, 256, 1), (130, 128, 4096, 8),
    (7, 256, 1024, None), (64, 640, 2048, None),
]


@pytest.mark.parametrize("m,n,k,splits", W4A4_CASES)
def test_w4a4_exact_inputs_bit_exact(native, m, n, k, splits):
    plan = native.ffn_nvfp4_projection_plan(m, n, k, "nvfp4_fixed")
    assert plan["family"] == "tc_w4a4", plan
    if splits is not None:
        assert plan["k_splits"] == splits, plan
    rng = np.random.default_rng(2000 + m + n + k)
    # scales 2^-2..2^0 and |x| <= 6: products of the block-scaled values are
    # multiples of 2^-8 below 36, partial sums below 2^18 of that unit
    codes, scales = exact_weight(rng, n, k, scale_bytes=POW2_SCALES[1:])
    x = exact_activations(rng, m, k)
    xc, xs = O.quantize_activation(x)
    assert np.array_equal(O.dequantize(xc, xs), x.astype(np.float64)), "activations not on the grid"
    w = make_handle(native, codes, scales)
    y = native.ffn_nvfp4_linear(torch.from_numpy(x).cuda().to(torch.bfloat16), w, "nvfp4_fixed")
    torch.cuda.synchronize()
    ref = O.round_to_bf16(O.project_w4a4(x.astype(np.float64), codes, scales, np.float32(1.0)))
    got = bf16_to_f64(y)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} mismatches, first at {bad[:3].tolist()}"
    assert native.ffn_nvfp4_device_error(clear=False) == 0
