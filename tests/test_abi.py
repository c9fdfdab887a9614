"""The C-ABI library builds, loads without a GPU, exports every symbol the
public header declares, and rejects bad arguments on the host before touching
the device."""
import ctypes

import pytest

from nvfp4_quantized_dense_w4a16_b200 import build as B


@pytest.fixture(scope="module")
def native():
    B.build()
    from nvfp4_quantized_dense_w4a16_b200 import native
    return native


def test_header_declares_the_boundary(native):
    names = native.declared_symbols()
    for required in ["ffn_nvfp4_quantize_weights", "ffn_nvfp4_quantize_activations",
                     "ffn_nvfp4_weight_create", "ffn_nvfp4_weight_create_gate_up",
                     "ffn_nvfp4_weight_destroy", "ffn_nvfp4_workspace_size",
                     "ffn_nvfp4_forward", "ffn_nvfp4_linear", "ffn_status_string"]:
        assert required in names


def test_library_exports_every_declared_symbol(native):
    lib = ctypes.CDLL(native.LIB_PATH)
    missing = [n for n in native.declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_version(native):
    assert native.status_string(0) == "FFN_OK"
    assert native.status_string(2) == "FFN_ERR_SHAPE"
    assert native.status_string(7) == "FFN_ERR_WORKSPACE"
    assert native.status_string(99) == "FFN_ERR_UNKNOWN"
    assert native.ffn_nvfp4_abi_version() == 1


def test_workspace_size_host_arithmetic(native):
    # bf16: h [m, inter] bf16 rounded to 256 bytes, plus split-K partials
    ws1 = native.ffn_nvfp4_workspace_size(1, 5120, 17408, "bf16")
    assert ws1 >= 34816 and ws1 % 256 == 0
    assert native.ffn_nvfp4_workspace_size(0, 5120, 17408, "bf16") == 0
    assert native.ffn_nvfp4_workspace_size(4096, 5120, 17408, "bf16") >= 4096 * 17408 * 2
    # fixed: at least h, the x and h codes and their scales, 256-byte granular
    m, H, I = 7, 4096, 12288
    ws = native.ffn_nvfp4_workspace_size(m, H, I, "nvfp4_fixed")
    assert ws % 256 == 0 and ws >= m * I * 2 + m * H // 2 + m * H // 16 + m * I // 2 + m * I // 16
    assert native.ffn_nvfp4_linear_workspace_size(3, 64, 128, "bf16") % 256 == 0


def test_host_side_argument_errors(native):
    L = native.lib
    out = ctypes.c_size_t()
    assert L.ffn_nvfp4_workspace_size(4, 100, 512, 0, ctypes.byref(out)) == 2   # hidden % 32
    assert L.ffn_nvfp4_workspace_size(4, 256, 512, 5, ctypes.byref(out)) == 1   # bad format
    assert L.ffn_nvfp4_workspace_size(-1, 256, 512, 0, ctypes.byref(out)) == 1
    assert L.ffn_nvfp4_workspace_size(4, 256, 512, 0, None) == 1
    fake = ctypes.c_void_p(256)
    assert L.ffn_nvfp4_quantize_weights(None, 4, 64, fake, fake, fake, None) == 1
    assert L.ffn_nvfp4_quantize_weights(fake, 4, 48, fake, fake, fake, None) == 2  # k % 32
    assert L.ffn_nvfp4_quantize_weights(fake, 0, 64, fake, fake, fake, None) == 2
    assert L.ffn_nvfp4_quantize_weights(ctypes.c_void_p(258), 4, 64, fake, fake, fake, None) == 3
    assert L.ffn_nvfp4_quantize_activations(fake, -2, 64, fake, fake, None) == 1
    assert L.ffn_nvfp4_quantize_activations(fake, 0, 64, fake, fake, None) == 0   # empty: no-op
    h = ctypes.c_void_p()
    assert L.ffn_nvfp4_weight_create(fake, fake, fake, 4, 40, None, ctypes.byref(h)) == 2
    assert L.ffn_nvfp4_weight_create(None, fake, fake, 4, 64, None, ctypes.byref(h)) == 1
    assert L.ffn_nvfp4_weight_create(fake, fake, fake, 4, 64, None, None) == 1
    assert L.ffn_nvfp4_forward(fake, 1, 256, 512, None, None, 0, fake, fake, 1 << 20, None) == 1
    assert L.ffn_nvfp4_linear(fake, 1, None, 0, fake, fake, 0, None) == 1
    assert L.ffn_nvfp4_weight_destroy(None) == 0
    assert L.ffn_nvfp4_weight_dims(None, None, None, None) == 1


def test_projection_plan_m_dispatch(native):
    # W4A16: the tile width follows m in tiers, split-K fills the GPU for
    # few output tiles; nothing is launched and no GPU is needed.
    for m, bn in ((1, 16), (16, 16), (17, 32), (32, 32), (33, 64), (64, 64), (65, 128),
                  (128, 128), (129, 256), (4096, 256)):
        p = native.ffn_nvfp4_projection_plan(m, 384, 512, "bf16")
        assert p["family"] == "tc_w4a16" and p["tile_rows"] == bn, (m, p)
    assert native.ffn_nvfp4_projection_plan(4, 384, 512)["k_splits"] == 1
    assert native.ffn_nvfp4_projection_plan(4, 128, 4096)["k_splits"] == 8
    assert native.ffn_nvfp4_projection_plan(0, 128, 4096)["family"] == "none"
    # fixed format: the K split does not depend on m (row invariance)
    splits = {native.ffn_nvfp4_projection_plan(m, 4096, 12288, "nvfp4_fixed")["k_splits"]
              for m in (1, 7, 64, 512)}
    assert len(splits) == 1
    L = native.lib
    p = native.ProjectionPlan()
    assert L.ffn_nvfp4_projection_plan(4, 128, 48, 0, 0, ctypes.byref(p)) == 2    # k % 32
    assert L.ffn_nvfp4_projection_plan(4, 129, 64, 0, 1, ctypes.byref(p)) == 2    # odd gate+up n
    assert L.ffn_nvfp4_projection_plan(-1, 128, 64, 0, 0, ctypes.byref(p)) == 1
    assert L.ffn_nvfp4_projection_plan(4, 128, 64, 0, 0, None) == 1


def test_weight_create_ex_rejects_bad_formats(native):
    L = native.lib
    fake = ctypes.c_void_p(256)
    h = ctypes.c_void_p()
    assert L.ffn_nvfp4_weight_create_ex(fake, fake, fake, 4, 64, 0, None, ctypes.byref(h)) == 1
    assert L.ffn_nvfp4_weight_create_ex(fake, fake, fake, 4, 64, 4, None, ctypes.byref(h)) == 1
    assert L.ffn_nvfp4_weight_create_ex(fake, fake, fake, 4, 40, 1, None, ctypes.byref(h)) == 2
    assert L.ffn_nvfp4_weight_info(None, None, None) == 1


def test_lora_create_host_checks(native):
    L = native.lib
    fake = ctypes.c_void_p(256)
    h = ctypes.c_void_p()
    assert L.ffn_nvfp4_lora_create(0, 256, 512, fake, fake, None, None, None, None, None, ctypes.byref(h)) == 4
    assert L.ffn_nvfp4_lora_create(257, 256, 512, fake, fake, None, None, None, None, None, ctypes.byref(h)) == 4
    assert L.ffn_nvfp4_lora_create(4, 250, 512, fake, fake, None, None, None, None, None, ctypes.byref(h)) == 2
    assert L.ffn_nvfp4_lora_create(4, 256, 512, fake, None, None, None, None, None, None, ctypes.byref(h)) == 1
    assert L.ffn_nvfp4_lora_create(4, 256, 512, None, None, None, None, None, None, None, ctypes.byref(h)) == 1
    assert L.ffn_nvfp4_lora_destroy(None) == 0
    sz = ctypes.c_size_t()
    assert L.ffn_nvfp4_workspace_size_lora(4, 256, 512, 0, None, ctypes.byref(sz)) == 0
    assert sz.value == native.ffn_nvfp4_workspace_size(4, 256, 512, "bf16")
