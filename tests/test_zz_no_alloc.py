"""The allocation-free projection entry point (ffn_nvfp4_linear_noalloc).

Some callers cannot allocate device memory while they run -- a plugin whose
host framework owns all device memory and gives it no workspace, or serving
code that must not call cudaMalloc mid-flight because it can synchronise the
device.  For them the library keeps the split-K partials in a fixed device
array.  This file checks, through the C ABI, that the variant returns what
ffn_nvfp4_linear returns (within the FFN tolerance) on consecutive calls,
including calls whose partials overwrite the previous call's, and that a
shape needing more than the fixed scratch is refused.  It is collected last
and also passes when run on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from nvfp4_quantized_dense_w4a16_b200 import synth

pytestmark = pytest.mark.gpu

from gpu_helpers import assert_close, bf16_to_f64, gpu_weight, to_dev_bf16


@pytest.fixture(scope="module")
def native():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from nvfp4_quantized_dense_w4a16_b200 import build
    build.build()
    from nvfp4_quantized_dense_w4a16_b200 import native as N
    return N


def _case(native, m, n, k, seed):
    w = gpu_weight(native, synth.random_bf16((n, k), seed, std=0.02))[0]
    x = to_dev_bf16(synth.random_bf16((m, k), seed + 1))
    return w, x


def test_noalloc_matches_linear_on_consecutive_calls(native):
    # shapes chosen so that the split-K partials (the scratch) are used
    a = _case(native, 4, 512, 8192, 11)     # 4 weight tiles -> many K splits
    b = _case(native, 37, 384, 6144, 12)    # different m and n: overwrites a's partials
    for w, x in (a, b, a):
        ref = bf16_to_f64(native.ffn_nvfp4_linear(x, w, "bf16"))
        for _ in range(2):
            y = torch.full((x.shape[0], w.n), float("nan"), dtype=torch.bfloat16, device="cuda")
            st = native.lib.ffn_nvfp4_linear_noalloc(ctypes.c_void_p(x.data_ptr()), x.shape[0], w.handle,
                                                      ctypes.c_void_p(y.data_ptr()),
                                                      torch.cuda.current_stream().cuda_stream)
            assert st == 0, native.status_string(st)
            torch.cuda.synchronize()
            assert_close(bf16_to_f64(y), ref, "noalloc vs linear")
    assert native.ffn_nvfp4_device_error(clear=False) == 0


def test_noalloc_refuses_shapes_beyond_the_fixed_scratch(native):
    # m=1024 rows against one 128-row weight tile with K=17408 asks for ~18 MB
    # of partials, more than the 16 MiB array: refused, nothing launched.
    w, x = _case(native, 1024, 128, 17408, 13)
    y = torch.empty((1024, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(native.FfnError) as e:
        native.ffn_nvfp4_linear_noalloc(x, w, y)
    assert e.value.status_name == "FFN_ERR_WORKSPACE"
    # the library stays usable
    small = _case(native, 2, 256, 4096, 14)
    ref = bf16_to_f64(native.ffn_nvfp4_linear(small[1], small[0], "bf16"))
    assert_close(bf16_to_f64(native.ffn_nvfp4_linear_noalloc(small[1], small[0])), ref)
