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


def make_handle(native, codes, scales, formats="all"):
    return native.ffn_nvfp4_weight_create(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(),
                                          torch.ones(1, dtype=torch.float32, device="cuda"), formats=formats)


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
    # three activation tiles: CTAs of two tiles and a last CTA of one
    (300, 256, 512, None), (300, 128, 4096, 8),
    # either side of the switch from 16-row to 128-row activation tiles
    (16, 256, 1024, None), (17, 256, 1024, None),
]


@pytest.mark.parametrize("m,n,k,splits", W4A4_CASES)
def test_w4a4_exact_inputs_bit_exact(native, m, n, k, splits):
    plan = native.ffn_nvfp4_projection_plan(m, n, k, "nvfp4_fixed")
    assert plan["family"] == "tc_w4a4", plan
    assert plan["tile_rows"] == (16 if m <= 16 else 128), plan
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


def exact_ffn_inputs(rng, m, H, I, down_nonzeros=4):
    """An FFN whose every intermediate is exact, so the whole layer must match
    the oracle bit for bit (all tensor scales 1):
      x in {1, 2};  gate: non-negative codes, scales 2^-3..2^0, so every
      g = x . w_g is a positive dyadic sum, here >= 32 (asserted), where
      silu(g) = g / (1 + e^-g) equals g in fp32 and rounds like g in fp64;
      up: one non-zero code (+-1 or +-2) per row in a block of scale 2^-4,
      so u = +-2^e and h = bf16(silu(g) * u) = bf16(g) * u exactly;
      down: `down_nonzeros` codes per row, scales 1, so each output is a
      short sum of exact products below 2^16 with at least 2^-7 resolution."""
    x = rng.integers(1, 3, (m, H)).astype(np.float32)
    mag = rng.integers(1, 8, (I, H)).astype(np.uint8)            # sign bit 0
    gc = (mag[:, 0::2] | (mag[:, 1::2] << 4)).astype(np.uint8)
    gsc = rng.choice(POW2_SCALES, (I, H // 16)).astype(np.uint8)
    un = np.zeros((I, H), np.uint8)
    cols = rng.integers(0, H, I)
    un[np.arange(I), cols] = rng.choice(np.array([0x2, 0xA, 0x4, 0xC], np.uint8), I)
    uc = (un[:, 0::2] | (un[:, 1::2] << 4)).astype(np.uint8)
    usc = np.full((I, H // 16), 0x18, np.uint8)                  # 2^-4
    dn = np.zeros((H, I), np.uint8)
    for r in range(H):
        dn[r, rng.choice(I, down_nonzeros, replace=False)] = rng.integers(1, 16, down_nonzeros)
    dc = (dn[:, 0::2] | (dn[:, 1::2] << 4)).astype(np.uint8)
    dsc = np.full((H, I // 16), 0x38, np.uint8)                  # 1
    one = np.float32(1.0)
    g = O.round_to_bf16(O.project_w4a16(x.astype(np.float64), gc, gsc, one))
    assert g.min() >= 32.0, g.min()
    return x, (gc, gsc, one), (uc, usc, one), (dc, dsc, one)


FFN_EXACT_CASES = [
    # (m, hidden, inter, handle formats): m <= 8 with both layouts runs the
    # block-scaled FP4 layer kernel with 8 activation planes per row,
    # bf16-only handles the per-tile kernels at the same m; tile widths
    # 16/32/64 per-tile, down K ranges that cut tiles, inter % 64 == 32, and
    # split-K with the SiLU*mul reduction for wider m
    (1, 512, 1536, "all"), (2, 512, 800, "all"), (5, 1024, 4096, "all"), (8, 512, 1536, "all"),
    (1, 512, 1536, "bf16"), (5, 1024, 4096, "bf16"), (16, 512, 800, "all"), (33, 512, 1536, "all"),
    (64, 1024, 2048, "all"), (100, 512, 1536, "all"), (300, 512, 800, "all"),
]


@pytest.mark.parametrize("m,H,I,formats", FFN_EXACT_CASES)
def test_ffn_exact_inputs_bit_exact(native, m, H, I, formats):
    rng = np.random.default_rng(3000 + m + H + I)
    x, qg, qu, qd = exact_ffn_inputs(rng, m, H, I)
    ref = O.ffn_w4a16(x.astype(np.float64), qg, qu, qd)
    hs = [make_handle(native, q[0], q[1], formats) for q in (qg, qu, qd)]
    gate_up = native.ffn_nvfp4_weight_create_gate_up(hs[0], hs[1])
    out = native.ffn_nvfp4_forward(torch.from_numpy(x).cuda().to(torch.bfloat16), gate_up, hs[2], "bf16")
    torch.cuda.synchronize()
    got = bf16_to_f64(out)
    bad = np.argwhere(got != ref)
    plan = native.ffn_nvfp4_projection_plan(m, H, I, "bf16", role="down")
    err = native.ffn_nvfp4_device_error(clear=False)
    assert bad.size == 0, (f"{plan}: {len(bad)} mismatches, first at {bad[:3].tolist()}: got "
                           f"{[got[tuple(b)] for b in bad[:3]]}, want {[ref[tuple(b)] for b in bad[:3]]}; "
                           f"device error bits {err}")
    assert err == 0


def test_persistent_path_bit_exact_in_subprocess(native):
    # the persistent few-row kernels (selectable, not the default) keep the
    # bit-exact property on the exactly representable layer
    import os
    import subprocess
    import sys
    code = (
        "import sys; sys.path.insert(0, 'tests'); sys.path.insert(0, '.');"
        "import test_gpu_exact as T; from nvfp4_quantized_dense_w4a16_b200 import native as N;"
        "assert N.ffn_nvfp4_projection_plan(5, 1024, 4096, role='down')['family'] == 'tc_w4a16_persistent';"
        "[T.test_ffn_exact_inputs_bit_exact(N, *c, 'all') for c in [(1, 512, 1536), (5, 1024, 4096),"
        " (16, 512, 800), (33, 512, 1536), (64, 1024, 2048)]]; print('persistent-ok')")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=900,
                       env=dict(os.environ, FFN_NVFP4_W4A16_PATH="persistent"))
    assert r.returncode == 0 and "persistent-ok" in r.stdout, r.stdout + r.stderr
