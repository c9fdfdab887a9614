"""The allocation-free projection entry point (ffn_nvfp4_linear_noalloc).

Some callers cannot allocate device memory while they run -- a plugin whose
host framework owns all device memory and gives it no workspace, or serving
code that must not call cudaMalloc mid-flight because it can synchronise the
device.  For them the library keeps the split-K partials in a fixed device
array.  This file checks, through the C ABI, that the variant matches the CPU
oracle (within the FFN tolerance) and returns exactly what ffn_nvfp4_linear
returns when both run the tensor-core kernels, on consecutive calls,
including calls whose partials overwrite the previous call's, and that a
shape needing more than the fixed scratch is refused.  It is collected last
and also passes when run on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import nvfp4_ffn as O
from nvfp4_quantized_dense_w4a16_b200 import synth

pytestmark = pytest.mark.gpu

from gpu_helpers import assert_close, bf16_to_f64, gpu_weight, oracle_weight, to_dev_bf16


@pytest.fixture(scope="module")
def native():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from nvfp4_quantized_dense_w4a16_b200 import build
    build.build()
    from nvfp4_quantized_dense_w4a16_b200 import native as N
    return N


def _case(native, m, n, k, seed):
    wb = synth.random_bf16((n, k), seed, std=0.02)
    xb = synth.random_bf16((m, k), seed + 1)
    w = gpu_weight(native, wb)[0]
    x = to_dev_bf16(xb)
    ref = O.round_to_bf16(O.project_w4a16(synth.bf16_bits_to_f32(xb).astype(np.float64), *oracle_weight(wb)))
    return w, x, ref


def test_noalloc_matches_oracle_and_linear_on_consecutive_calls(native):
    # shapes chosen so that the split-K partials (the scratch) are used
    a = _case(native, 4, 512, 8192, 11)     # 4 weight tiles -> many K splits
    b = _case(native, 37, 384, 6144, 12)    # different m and n: overwrites a's partials
    for w, x, ref in (a, b, a):
        m = x.shape[0]
        assert native.ffn_nvfp4_projection_plan(m, w.n, w.k, "bf16")["k_splits"] > 1
        lin = native.ffn_nvfp4_linear(x, w, "bf16")
        same_kernels = native.ffn_nvfp4_projection_plan(m, w.n, w.k, "bf16")["family"] == "tc_w4a16"
        for _ in range(2):
            y = torch.full((m, w.n), float("nan"), dtype=torch.bfloat16, device="cuda")
            st = native.lib.ffn_nvfp4_linear_noalloc(ctypes.c_void_p(x.data_ptr()), m, w.handle,
                                                      ctypes.c_void_p(y.data_ptr()),
                                                      torch.cuda.current_stream().cuda_stream)
            assert st == 0, native.status_string(st)
            torch.cuda.synchronize()
            assert_close(bf16_to_f64(y), ref, "noalloc vs oracle")
            if same_kernels:  # the same plan and kernels: identical bits
                assert torch.equal(y, lin)
    assert native.ffn_nvfp4_device_error(clear=False) == 0


def test_noalloc_refuses_shapes_beyond_the_fixed_scratch(native):
    # m=1024 rows against one 128-row weight tile with K=17408 asks for ~18 MB
    # of partials, more than the 16 MiB array: refused, nothing launched.
    w, x, _ = _case(native, 1024, 128, 17408, 13)
    y = torch.empty((1024, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(native.FfnError) as e:
        native.ffn_nvfp4_linear_noalloc(x, w, y)
    assert e.value.status_name == "FFN_ERR_WORKSPACE"
    # the library stays usable
    w, x, ref = _case(native, 2, 256, 4096, 14)
    assert_close(bf16_to_f64(native.ffn_nvfp4_linear_noalloc(x, w)), ref)
