"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Codes and scales must match bit for bit; FFN outputs
must satisfy max|err| <= 2e-2 * rms(ref) and sum|err| / sum|ref| <= 5e-3."""
import numpy as np
import pytest
import torch

from oracle import nvfp4_ffn as O
from nvfp4_quantized_dense_w4a16_b200 import synth

pytestmark = pytest.mark.gpu

from gpu_helpers import (FfnCase, assert_close, assert_quant_equal, bf16_to_f64, gpu_weight,
                         oracle_weight, to_dev_bf16)


@pytest.fixture(scope="module")
def native():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from nvfp4_quantized_dense_w4a16_b200 import build
    build.build()
    from nvfp4_quantized_dense_w4a16_b200 import native as N
    return N


# ---------------------------------------------------------------- quantisers

@pytest.mark.parametrize("n,k,seed", [(1, 32, 0), (5, 96, 1), (64, 512, 2), (300, 1024, 3)])
def test_weight_quantizer_bit_exact_small(native, n, k, seed):
    bits = synth.random_bf16((n, k), seed, std=0.02)
    assert_quant_equal(gpu_weight(native, bits), oracle_weight(bits))


def test_weight_quantizer_worked_example(native, golden):
    g = golden("weight_quant_example.txt")
    w = np.array([[float(v) for v in r] for r in g["w"]], dtype=np.float32)
    res = gpu_weight(native, synth.f32_to_bf16_bits(w))
    assert float(res[3].item()) == float(g["gs"][0][0])
    assert res[2].cpu().numpy().tolist() == [[int(v, 16) for v in r] for r in g["scales"]]
    assert res[1].cpu().numpy().tolist() == [[int(v, 16) for v in r] for r in g["codes"]]


def test_weight_quantizer_edge_values(native):
    # zero tensor (gs = 1), constant blocks, exact ties, tiny and huge values
    z = np.zeros((4, 64), np.uint16)
    assert_quant_equal(gpu_weight(native, z), oracle_weight(z))
    rng = np.random.default_rng(0)
    w = rng.standard_normal((8, 128)).astype(np.float32)
    w[0] = 1.0
    w[1, :16] = 0.0
    w[2] *= 1e-30
    w[3] *= 1e30
    w[4, :16] = np.float32([6, 5, 3.5, 2.5, 1.75, 1.25, .75, .25, -6, -5, -3.5, -2.5, -1.75, -1.25, -.75, -.25])
    bits = synth.f32_to_bf16_bits(w)
    assert_quant_equal(gpu_weight(native, bits), oracle_weight(bits))


@pytest.mark.parametrize("name", ["decode", "w4a4"])
def test_weight_quantizer_bit_exact_full_size(native, name):
    inp = synth.make_inputs(name)
    for bits in (inp.w_gate, inp.w_down):
        assert_quant_equal(gpu_weight(native, bits), oracle_weight(bits))


@pytest.mark.parametrize("m,k,seed", [(1, 32, 0), (7, 4096, 1), (64, 12288, 2), (33, 96, 3)])
def test_activation_quantizer_bit_exact(native, m, k, seed):
    bits = synth.random_bf16((m, k), seed)
    x = to_dev_bf16(bits)
    x[0, :16] = 0
    if m > 1:
        x[1] *= 1000
    c, s = native.ffn_nvfp4_quantize_activations(x)
    rc, rs = O.quantize_activation(x.float().cpu().numpy())
    assert np.array_equal(s.cpu().numpy(), rs)
    assert np.array_equal(c.cpu().numpy(), rc)


def test_activation_quantizer_worked_example(native, golden):
    g = golden("act_quant_example.txt")
    x = np.array([[float(v) for v in r] for r in g["x"]], dtype=np.float32)
    c, s = native.ffn_nvfp4_quantize_activations(to_dev_bf16(synth.f32_to_bf16_bits(x)))
    assert s.cpu().numpy().tolist() == [[int(v, 16) for v in r] for r in g["scales"]]
    assert c.cpu().numpy().tolist() == [[int(v, 16) for v in r] for r in g["codes"]]


# --------------------------------------------------------------- projections

@pytest.mark.parametrize("m,n,k", [(1, 64, 256), (3, 96, 512), (5, 160, 1056), (17, 48, 2048),
                                   (64, 256, 5120)])
@pytest.mark.parametrize("fmt", ["bf16", "nvfp4_fixed"])
def test_linear_matches_oracle(native, m, n, k, fmt):
    wb = synth.random_bf16((n, k), 100 + m, std=0.02)
    xb = synth.random_bf16((m, k), 200 + m)
    h = gpu_weight(native, wb)
    y = native.ffn_nvfp4_linear(to_dev_bf16(xb), h[0], fmt)
    torch.cuda.synchronize()
    q = oracle_weight(wb)
    x64 = synth.bf16_bits_to_f32(xb).astype(np.float64)
    proj = O.project_w4a16 if fmt == "bf16" else O.project_w4a4
    ref = O.round_to_bf16(proj(x64, *q))
    assert_close(bf16_to_f64(y), ref, f"linear {fmt} m={m} n={n} k={k}")


def test_linear_exact_inputs_bit_exact(native):
    # gs = 1, power-of-two block scales, integer activations: every fp32
    # partial sum is exact, so the GPU must equal the oracle bit for bit.
    rng = np.random.default_rng(3)
    m, n, k = 4, 40, 256
    codes = rng.integers(0, 256, (n, k // 2), dtype=np.uint8)
    scales = rng.choice(np.array([0x20, 0x28, 0x30, 0x38, 0x40], np.uint8), (n, k // 16))
    x = rng.integers(-4, 5, (m, k)).astype(np.float32)
    w = native.ffn_nvfp4_weight_create(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(),
                                       torch.ones(1, dtype=torch.float32, device="cuda"))
    y = native.ffn_nvfp4_linear(torch.from_numpy(x).cuda().to(torch.bfloat16), w, "bf16")
    torch.cuda.synchronize()
    ref = O.round_to_bf16(O.project_w4a16(x.astype(np.float64), codes, scales, np.float32(1.0)))
    assert np.array_equal(bf16_to_f64(y), ref)


# -------------------------------------------------------------------- FFN

@pytest.fixture(scope="module")
def tiny(native):
    return FfnCase(native, synth.make_inputs("tiny"))


@pytest.mark.parametrize("fmt", ["bf16", "nvfp4_fixed"])
def test_ffn_tiny(native, tiny, fmt):
    out = bf16_to_f64(tiny.forward(fmt))
    assert_close(out, tiny.oracle(fmt), f"tiny {fmt}")


@pytest.mark.parametrize("m", [1, 2, 3, 5, 8, 13, 64, 129])
def test_ffn_ragged_rows_reduced_sizes(native, m):
    inp = synth.make_inputs("smallm", m=m, hidden=512, inter=1536, seed=20 + m)
    case = FfnCase(native, inp)
    assert_close(bf16_to_f64(case.forward("bf16")), case.oracle("bf16"), f"bf16 m={m}")
    assert_close(bf16_to_f64(case.forward("nvfp4_fixed")), case.oracle("nvfp4_fixed"), f"w4a4 m={m}")


def test_ffn_writes_only_rows_0_to_m(native, tiny):
    m, H = tiny.inp.m, tiny.inp.hidden
    big = torch.full((m + 3, H), 7.0, dtype=torch.bfloat16, device="cuda")
    native.ffn_nvfp4_forward(tiny.x_dev, tiny.gate_up, tiny.down, "bf16", out=big[:m])
    torch.cuda.synchronize()
    assert torch.all(big[m:] == 7.0)


def test_fused_gate_up_equals_separate_projections(native, tiny):
    # gate and up through ffn_nvfp4_linear with their own handles, SiLU*mul on
    # the host from the bf16 g and u, then down through the library: the same
    # result as the fused forward within the FFN tolerance.
    g = bf16_to_f64(native.ffn_nvfp4_linear(tiny.x_dev, tiny.gate, "bf16"))
    u = bf16_to_f64(native.ffn_nvfp4_linear(tiny.x_dev, tiny.up, "bf16"))
    h = O.round_to_bf16(O.silu(g) * u)
    hd = to_dev_bf16(O.f64_to_bf16_bits(h))
    out_sep = bf16_to_f64(native.ffn_nvfp4_linear(hd, tiny.down, "bf16"))
    out_fused = bf16_to_f64(tiny.forward("bf16"))
    assert_close(out_fused, out_sep, "fused vs separate")


def test_errors_are_reported_not_raised_on_device(native, tiny):
    x = tiny.x_dev
    with pytest.raises(native.FfnError) as e:
        native.ffn_nvfp4_forward(x, tiny.gate_up, tiny.down, "bf16",
                                 workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status_name == "FFN_ERR_WORKSPACE"
    with pytest.raises(native.FfnError) as e:
        native.ffn_nvfp4_forward(x, tiny.down, tiny.down, "bf16")  # not a gate+up handle
    assert e.value.status_name == "FFN_ERR_INVALID_ARG"
    with pytest.raises(native.FfnError) as e:
        native.ffn_nvfp4_weight_create_gate_up(tiny.gate, tiny.down)
    assert e.value.status_name == "FFN_ERR_SHAPE"
    xo = torch.empty(x.numel() + 8, dtype=torch.bfloat16, device="cuda")[1:1 + x.numel()].view(x.shape)
    with pytest.raises(native.FfnError) as e:
        native.ffn_nvfp4_forward(xo, tiny.gate_up, tiny.down, "bf16")
    assert e.value.status_name == "FFN_ERR_ALIGNMENT"
    # the context is still usable
    assert_close(bf16_to_f64(tiny.forward("bf16")), tiny.oracle("bf16"))


@pytest.mark.parametrize("m,H,I", [(33, 1056, 800), (300, 512, 96), (257, 256, 2048), (1, 4096, 1056)])
def test_ffn_tile_edges(native, m, H, I):
    # K % 64 == 32 (1056), inter % 64 == 32 (800, 96: partial gate+up tiles),
    # several 256-row activation tiles with a ragged last one, deep split-K.
    inp = synth.make_inputs("smallm", m=m, hidden=H, inter=I, seed=40 + m)
    case = FfnCase(native, inp)
    assert_close(bf16_to_f64(case.forward("bf16")), case.oracle("bf16"), f"m={m} H={H} I={I}")
    assert native.ffn_nvfp4_device_error() == 0


@pytest.mark.parametrize("env,fmt", [("FFN_NVFP4_W4A16_PATH", "bf16"), ("FFN_NVFP4_W4A4_PATH", "nvfp4_fixed")])
def test_cuda_core_paths_match_oracle_in_subprocess(native, env, fmt):
    # the CUDA-core projection families, selected per process by environment
    import os
    import subprocess
    import sys
    code = (
        "import sys; sys.path.insert(0, 'tests'); sys.path.insert(0, '.');"
        "from gpu_helpers import FfnCase, assert_close, bf16_to_f64;"
        "from nvfp4_quantized_dense_w4a16_b200 import native as N, synth;"
        "c = FfnCase(N, synth.make_inputs('smallm', m=5, hidden=512, inter=1536, seed=3));"
        f"assert_close(bf16_to_f64(c.forward('{fmt}')), c.oracle('{fmt}'));"
        "print('gemv-ok')")
    env_vars = dict(os.environ, **{env: "gemv"})
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=env_vars, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "gemv-ok" in r.stdout, r.stdout + r.stderr


def test_device_error_word_is_clear(native, tiny):
    tiny.forward("bf16")
    assert native.ffn_nvfp4_device_error(clear=False) == 0


def test_handles_hold_one_tiled_copy_per_format(native):
    # a bf16-only handle holds ~0.5625 B per weight (tiles pad n to 128 rows
    # and k to 64); the fused gate+up serves what both parts serve; a format
    # the handle was not built for is refused, not silently recomputed
    n, k = 512, 1024
    bits = synth.random_bf16((n, k), 7, std=0.02)
    c, s, g = native.ffn_nvfp4_quantize_weights(to_dev_bf16(bits))
    w16 = native.ffn_nvfp4_weight_create(c, s, g, formats="bf16")
    w4 = native.ffn_nvfp4_weight_create(c, s, g, formats="nvfp4_fixed")
    wall = native.ffn_nvfp4_weight_create(c, s, g)
    assert w16.formats == 1 and w4.formats == 2 and wall.formats == 3
    assert w16.device_bytes <= 0.6 * n * k and w4.device_bytes <= 0.6 * n * k
    assert wall.device_bytes <= 1.2 * n * k
    x = to_dev_bf16(synth.random_bf16((3, k), 8))
    ref = O.round_to_bf16(O.project_w4a16(synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(
        x.float().cpu().numpy())).astype(np.float64), *oracle_weight(bits)))
    assert_close(bf16_to_f64(native.ffn_nvfp4_linear(x, w16, "bf16")), ref)
    with pytest.raises(native.FfnError) as e:
        native.ffn_nvfp4_linear(x, w16, "nvfp4_fixed")
    assert e.value.status_name == "FFN_ERR_UNSUPPORTED"
    gu = native.ffn_nvfp4_weight_create_gate_up(w16, wall)
    assert gu.formats == 1 and gu.device_bytes <= 0.6 * 2 * n * k
    with pytest.raises(native.FfnError) as e:
        native.ffn_nvfp4_weight_create_gate_up(w16, w4)
    assert e.value.status_name == "FFN_ERR_UNSUPPORTED"
