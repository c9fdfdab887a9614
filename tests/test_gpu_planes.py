"""The few-row layer on the block-scaled FP4 tensor core (m <= 2, both weight
layouts): rows are independent, a row holding an Inf or NaN gives NaN outputs
for that row only (reading R9), all-zero rows give zero outputs, and rows of
very different magnitudes are each held to the FFN tolerance (each row's
planes have their own power-of-two factors).
"""
import numpy as np
import pytest
import torch

from oracle import nvfp4_ffn as O

pytestmark = pytest.mark.gpu

from gpu_helpers import assert_close, bf16_to_f64
from test_gpu_exact import make_handle


@pytest.fixture(scope="module")
def native():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from nvfp4_quantized_dense_w4a16_b200 import build
    build.build()
    from nvfp4_quantized_dense_w4a16_b200 import native as N
    return N


def layer(native, H, I, seed):
    rng = np.random.default_rng(seed)
    qs = []
    for n, k in ((I, H), (I, H), (H, I)):
        w = torch.from_numpy((rng.standard_normal((n, k)) * 0.02).astype(np.float32)).to(torch.bfloat16).cuda()
        qs.append(native.ffn_nvfp4_quantize_weights(w))
    hs = [native.ffn_nvfp4_weight_create(c, s, g, formats="all") for c, s, g in qs]
    gate_up = native.ffn_nvfp4_weight_create_gate_up(hs[0], hs[1])
    oracle_q = [(c.cpu().numpy(), s.cpu().numpy(), np.float32(g.cpu().numpy()[0])) for c, s, g in qs]
    return gate_up, hs[2], oracle_q


def run(native, x, gate_up, down):
    out = native.ffn_nvfp4_forward(x, gate_up, down, "bf16")
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("m", [1, 2])
def test_planes_path_is_taken(native, m):
    for role in ("gate_up", "down"):
        assert native.ffn_nvfp4_projection_plan(m, 2 * 1536 if role == "gate_up" else 512,
                                                512 if role == "gate_up" else 1536, "bf16",
                                                role=role)["family"] == "tc_planes"


def test_non_finite_row_gives_nan_row_only(native):
    H, I = 512, 1536
    gate_up, down, q = layer(native, H, I, 71)
    rng = np.random.default_rng(72)
    x = torch.from_numpy(rng.standard_normal((2, H)).astype(np.float32)).to(torch.bfloat16).cuda()
    ref0 = O.ffn_w4a16(bf16_to_f64(x[:1]), *q)
    for bad in (float("inf"), float("nan"), float("-inf")):
        xb = x.clone()
        xb[1, 37] = bad
        out = bf16_to_f64(run(native, xb, gate_up, down))
        assert np.all(np.isnan(out[1])), bad
        assert_close(out[:1], ref0, f"row 0 beside a row with {bad}")
    assert native.ffn_nvfp4_device_error(clear=False) == 0


def test_zero_row_and_independent_rows(native):
    H, I = 512, 1536
    gate_up, down, q = layer(native, H, I, 73)
    rng = np.random.default_rng(74)
    x = rng.standard_normal((2, H)).astype(np.float32)
    x[1] *= 1e-3  # a row a thousand times smaller: its own planes' factors
    xt = torch.from_numpy(x).to(torch.bfloat16).cuda()
    out = bf16_to_f64(run(native, xt, gate_up, down))
    ref = O.ffn_w4a16(bf16_to_f64(xt), *q)
    assert_close(out[:1], ref[:1], "row 0")
    assert_close(out[1:], ref[1:], "row 1 (x 1e-3)")
    # each row alone gives the same bits as inside the pair
    for j in range(2):
        alone = bf16_to_f64(run(native, xt[j:j + 1].contiguous(), gate_up, down))
        assert np.array_equal(alone, out[j:j + 1]), j
    zero = bf16_to_f64(run(native, torch.zeros((1, H), dtype=torch.bfloat16, device="cuda"), gate_up, down))
    assert np.all(zero == 0.0)
    assert native.ffn_nvfp4_device_error(clear=False) == 0
