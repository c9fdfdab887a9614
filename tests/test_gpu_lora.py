"""GPU parity of the LoRA adapters (the layer's NEXT-1 overlay) against the
CPU oracle: gate/up deltas before SiLU*mul, the down delta after the down
projection, through every W4A16 kernel family the m-dispatch picks (the
few-row persistent kernels, per-tile kernels with and without split-K)."""
import numpy as np
import pytest
import torch

from oracle import nvfp4_ffn as O
from nvfp4_quantized_dense_w4a16_b200 import synth

pytestmark = pytest.mark.gpu

from gpu_helpers import FfnCase, assert_close, bf16_to_f64, to_dev_bf16


@pytest.fixture(scope="module")
def native():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from nvfp4_quantized_dense_w4a16_b200 import build
    build.build()
    from nvfp4_quantized_dense_w4a16_b200 import native as N
    return N


def adapters(H, I, r, seed, which=("gate", "up", "down"), std=0.05):
    """Seeded bf16 adapters (A [r, in], B [out, r]) as bit patterns."""
    dims = {"gate": (H, I), "up": (H, I), "down": (I, H)}
    out = {}
    for i, k in enumerate(which):
        n_in, n_out = dims[k]
        out[k] = (synth.random_bf16((r, n_in), seed + 2 * i, std=std),
                  synth.random_bf16((n_out, r), seed + 2 * i + 1, std=std))
    return out


def run(native, case, lora_bits, r, rows=None):
    dev = {k: (to_dev_bf16(a), to_dev_bf16(b)) for k, (a, b) in lora_bits.items()}
    lora = native.ffn_nvfp4_lora_create(r, case.inp.hidden, case.inp.inter, **dev)
    x = case.x_dev if rows is None else case.x_dev[:rows].contiguous()
    out = native.ffn_nvfp4_forward(x, case.gate_up, case.down, "bf16", lora=lora)
    torch.cuda.synchronize()
    f64 = {k: (synth.bf16_bits_to_f32(a).astype(np.float64), synth.bf16_bits_to_f32(b).astype(np.float64))
           for k, (a, b) in lora_bits.items()}
    x64 = case.x64 if rows is None else case.x64[:rows]
    ref = O.ffn_w4a16_lora(x64, case.qg, case.qu, case.qd, f64)
    return bf16_to_f64(out), ref


@pytest.mark.parametrize("m,H,I,r", [(1, 512, 1536, 16), (5, 512, 1536, 8), (64, 1024, 2048, 32),
                                     (100, 512, 1536, 16), (300, 512, 800, 4), (3, 256, 512, 40)])
def test_lora_ffn_matches_oracle(native, m, H, I, r):
    case = FfnCase(native, synth.make_inputs("smallm", m=m, hidden=H, inter=I, seed=60 + m))
    out, ref = run(native, case, adapters(H, I, r, 70 + m), r)
    assert_close(out, ref, f"lora m={m} H={H} I={I} r={r}")
    # the deltas are not negligible here: the layer differs from the plain one
    assert O.error_stats(ref, case.oracle("bf16"))["rel_l1"] > 1e-2
    assert native.ffn_nvfp4_device_error(clear=False) == 0


@pytest.mark.parametrize("which", [("gate",), ("up",), ("down",), ("gate", "down")])
def test_lora_subsets_match_oracle(native, which):
    case = FfnCase(native, synth.make_inputs("smallm", m=7, hidden=512, inter=1536, seed=81))
    out, ref = run(native, case, adapters(512, 1536, 8, 90, which=which), 8)
    assert_close(out, ref, f"lora {which}")


def test_zero_adapters_change_no_bit(native):
    case = FfnCase(native, synth.make_inputs("smallm", m=33, hidden=512, inter=1536, seed=83))
    z = lambda shape: torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    r = 8
    lora = native.ffn_nvfp4_lora_create(r, 512, 1536, gate=(z((r, 512)), z((1536, r))),
                                        up=(z((r, 512)), z((1536, r))), down=(z((r, 1536)), z((512, r))))
    with_l = native.ffn_nvfp4_forward(case.x_dev, case.gate_up, case.down, "bf16", lora=lora)
    plain = native.ffn_nvfp4_forward(case.x_dev, case.gate_up, case.down, "bf16")
    torch.cuda.synchronize()
    assert torch.equal(with_l, plain)


def test_lora_errors(native):
    case = FfnCase(native, synth.make_inputs("tiny"))
    bits = adapters(256, 512, 4, 95)
    dev = {k: (to_dev_bf16(a), to_dev_bf16(b)) for k, (a, b) in bits.items()}
    lora = native.ffn_nvfp4_lora_create(4, 256, 512, **dev)
    with pytest.raises(native.FfnError) as e:
        native.ffn_nvfp4_forward(case.x_dev, case.gate_up, case.down, "nvfp4_fixed", lora=lora)
    assert e.value.status_name == "FFN_ERR_UNSUPPORTED"
    other = native.ffn_nvfp4_lora_create(4, 512, 512, gate=(to_dev_bf16(synth.random_bf16((4, 512), 1)),
                                                           to_dev_bf16(synth.random_bf16((512, 4), 2))))
    with pytest.raises(native.FfnError) as e:
        native.ffn_nvfp4_forward(case.x_dev, case.gate_up, case.down, "bf16", lora=other)
    assert e.value.status_name == "FFN_ERR_SHAPE"
