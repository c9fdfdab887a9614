"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times: bit-exact quantisation of every weight, FFN outputs of
sampled rows against the oracle, and bitwise row invariance of the fixed
W4A4 format across m in {1, 7, 64, 512}."""
import numpy as np
import pytest
import torch

from nvfp4_quantized_dense_w4a16_b200 import synth

pytestmark = pytest.mark.gpu

from gpu_helpers import FfnCase, assert_close, bf16_to_f64


@pytest.fixture(scope="module")
def native():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from nvfp4_quantized_dense_w4a16_b200 import build
    build.build()
    from nvfp4_quantized_dense_w4a16_b200 import native as N
    return N


def test_decode_m1_full(native):
    case = FfnCase(native, synth.make_inputs("decode"))
    out = bf16_to_f64(case.forward("bf16"))
    assert_close(out, case.oracle("bf16"), "decode m=1")


@pytest.fixture(scope="module")
def smallm(native):
    return FfnCase(native, synth.make_inputs("smallm"))


@pytest.mark.parametrize("m", [8, 16, 32, 64])
def test_small_m_sweep_full(native, smallm, m):
    out = bf16_to_f64(smallm.forward("bf16", rows=m))
    rows = sorted({0, m // 2, m - 1})
    assert_close(out[rows], smallm.oracle("bf16", rows=rows), f"small m={m}")


@pytest.fixture(scope="module")
def w4a4(native):
    return FfnCase(native, synth.make_inputs("w4a4"))


def test_w4a4_rows_bitwise_invariant_across_m(native, w4a4):
    # m <= 16 takes 16-row activation tiles (MMA N = 16), larger m 128-row
    # tiles: 16 and 17 sit on either side of that switch
    outs = {m: w4a4.forward("nvfp4_fixed", rows=m).view(torch.int16).cpu().numpy()
            for m in (1, 7, 16, 17, 64, 512)}
    for m, o in outs.items():
        assert np.array_equal(o, outs[512][:m]), f"rows of m={m} differ from m=512"
    # and the m=1 result again (same launch twice)
    again = w4a4.forward("nvfp4_fixed", rows=1).view(torch.int16).cpu().numpy()
    assert np.array_equal(again, outs[1])


@pytest.mark.parametrize("m", [1, 7, 64, 512])
def test_w4a4_full_matches_oracle(native, w4a4, m):
    out = bf16_to_f64(w4a4.forward("nvfp4_fixed", rows=m))
    rows = sorted({0, m // 2, m - 1})
    assert_close(out[rows], w4a4.oracle("nvfp4_fixed", rows=rows), f"w4a4 m={m}")


def test_prefill_m4096_full_sampled_rows(native):
    # the bench's primary workload in its launch configuration (m = 4096, 16
    # activation tiles of 256 rows): every row of the first 256-row tile, and
    # rows of the middle and last tiles at tile edges, against the oracle.
    case = FfnCase(native, synth.make_inputs("prefill"))
    out = bf16_to_f64(case.forward("bf16"))
    rows = list(range(256)) + [256, 2048, 3839, 4095]
    assert_close(out[rows], case.oracle("bf16", rows=rows), "prefill m=4096")
    assert np.all(np.isfinite(out))
    assert native.ffn_nvfp4_device_error(clear=False) == 0


def test_w4a4_fused_h_quantisation_is_bit_identical_in_subprocess(native):
    # the fixed format quantises h inside the gate+up epilogue; the layer
    # output must be bit for bit what the separate quantiser launch gives
    import os
    import subprocess
    import sys
    code = (
        "import sys, hashlib; sys.path.insert(0, 'tests'); sys.path.insert(0, '.');"
        "from gpu_helpers import FfnCase;"
        "from nvfp4_quantized_dense_w4a16_b200 import native as N, synth;"
        "c = FfnCase(N, synth.make_inputs('w4a4', m=64), check_quant=False);"
        "o = c.forward('nvfp4_fixed').view(__import__('torch').int16).cpu().numpy();"
        "print('sha', hashlib.sha1(o.tobytes()).hexdigest())")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    outs = []
    for fuse in ("1", "0"):
        r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=900,
                           env=dict(os.environ, FFN_NVFP4_W4A4_FUSE_HQ=fuse))
        assert r.returncode == 0, r.stdout + r.stderr
        outs.append([l for l in r.stdout.splitlines() if l.startswith("sha")][-1])
    assert outs[0] == outs[1]
