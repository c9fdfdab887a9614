"""CPU tests of bench.py's host-side logic: which layers rotate through weight
copies (and how many), that every timed step uses the copy it should, and the
kernel-source fingerprint that gates the reported DRAM traffic."""
import types

import numpy as np
import pytest
import torch

import bench


@pytest.fixture(scope="module")
def cpu_torch():
    # run Workload on the CPU: no device transfers, no synchronisation
    mp = pytest.MonkeyPatch()
    mp.setattr(torch.Tensor, "cuda", lambda self, *a, **k: self)
    mp.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    real_empty = torch.empty

    def empty(*a, **k):
        k.pop("device", None)
        return real_empty(*a, **k)
    mp.setattr(torch, "empty", empty)
    yield
    mp.undo()


@pytest.fixture(scope="module")
def layers(cpu_torch):
    """(Workload, list of forward calls it made) per layer, built once."""
    out = {}
    for name, m in (("decode", 1), ("w4a4", 512)):
        calls = []
        out[name] = (bench.Workload(fake_native(calls), name, m), calls)
    return out


def fake_native(calls):
    counter = iter(range(10**6))
    return types.SimpleNamespace(
        ffn_nvfp4_quantize_weights=lambda w: (w, w, w),
        ffn_nvfp4_weight_create=lambda c, s, g, formats="all": ("w", next(counter)),
        ffn_nvfp4_weight_create_gate_up=lambda g, u: ("gu", g, u),
        ffn_nvfp4_workspace_size=lambda m, H, I, f: 1024,
        ffn_nvfp4_forward=lambda x, gu, d, f, out=None, workspace=None: calls.append((gu, d)))


@pytest.mark.parametrize("name", ["decode", "w4a4"])
def test_small_layers_rotate_weight_copies(layers, name):
    wl, calls = layers[name]
    calls.clear()
    assert wl.sets >= 2
    assert wl.sets * wl.weight_bytes >= 4 * bench.L2_BYTES
    assert (wl.sets - 1) * wl.weight_bytes < 4 * bench.L2_BYTES  # no more copies than needed
    assert "rotated" in wl.l2_note
    for i in range(2 * wl.sets):
        wl.step(i)
    # step i uses copy i mod R, and the R copies are distinct handles
    used = [c[0] for c in calls]
    assert used[:wl.sets] == used[wl.sets:]
    assert len({id(h) for h in used[:wl.sets]}) == wl.sets


def test_weight_bytes_are_the_nvfp4_footprint(layers):
    wl = layers["decode"][0]
    H, I = 5120, 17408
    assert wl.weight_bytes == 3 * H * I * (0.5 + 1 / 16)


def test_fingerprint_ignores_comments_and_whitespace():
    a = "int f(int x) {\n  // note\n  return x + 1; /* block\n comment */\n}\n"
    b = "int f(int x){return x+1;}"
    c = "int f(int x){return x+2;}"
    assert bench.normalised_source(a) == bench.normalised_source(b)
    assert bench.normalised_source(a) != bench.normalised_source(c)


def test_traffic_reported_only_for_the_captured_sources():
    files = {f: "kernel body" for f in bench.KERNEL_SOURCES}
    sha = bench.kernel_sources_sha1(lambda rel: files[rel])
    files[bench.KERNEL_SOURCES[0]] = "kernel body // with a comment"
    assert bench.kernel_sources_sha1(lambda rel: files[rel]) == sha
    files[bench.KERNEL_SOURCES[0]] = "changed kernel body"
    assert bench.kernel_sources_sha1(lambda rel: files[rel]) != sha
    assert bench.measured_traffic("no_such_kernel", "prefill") is None


def test_traffic_is_keyed_by_kernel_workload_and_rows(monkeypatch):
    monkeypatch.setattr(bench, "kernel_sources_sha1", lambda read=None: "abc")
    monkeypatch.setattr(bench, "TRAFFIC", {("k", "w4a4", 512): {"bytes": 123, "sources_sha1": "abc"},
                                           ("k", "w4a4", 1): {"bytes": 7, "sources_sha1": "old"}})
    assert bench.measured_traffic("k", "w4a4", 512) == 123
    assert bench.measured_traffic("k", "w4a4", 64) is None      # another m: not captured
    assert bench.measured_traffic("k", "w4a4", 1) is None       # captured on other sources
    assert bench.measured_traffic("k", "prefill", 512) is None


def test_roofline_bound_uses_each_formats_own_peak(layers):
    peaks = {"hbm_gbs": 6557.8, "bf16_tflops": 1671.7, "bf16_tflops_sustained": 1402.4}
    assert bench.tensor_peak(peaks, "bf16")[0] == 1671.7
    assert bench.tensor_peak(peaks, "nvfp4_fixed")[0] == 1671.7 * 4   # nominal fallback
    assert bench.tensor_peak(dict(peaks, fp4_tflops=6000.0), "nvfp4_fixed")[0] == 6000.0
    assert "probe" in bench.tensor_peak(dict(peaks, fp4_tflops=6000.0), "nvfp4_fixed")[1]
    dec = layers["decode"][0]
    bound, units = dec.kernel_units("tc_w4a16_gate_up_silu", peaks)
    assert bound == "hbm" and units == bench.nvfp4_bytes(2 * 17408, 5120) + 5120 * 2 + 17408 * 2
    w4 = layers["w4a4"][0]
    bound, units = w4.kernel_units("tc_w4a4_gate_up_silu", peaks)
    assert bound == "tensor" and units == 2.0 * 512 * 2 * 12288 * 4096
    # the same intensity against the bf16 ridge (~255 flop/B) would also be
    # tensor-bound; against the FP4 ridge (~1020 flop/B) a quarter of it is not
    ridge = bench.tensor_peak(peaks, "nvfp4_fixed")[0] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    assert 1000 < ridge < 1040


def test_roofline_object_of_the_dominant_kernel(layers):
    peaks = {"hbm_gbs": 6557.8, "bf16_tflops": 1671.7, "bf16_tflops_sustained": 1402.4}
    dec = layers["decode"][0]
    prof = {"tc_w4a16_gate_up_silu": (20, 20 * 0.0430), "tc_w4a16_partial": (20, 20 * 0.0244),
            "splitk_reduce": (20, 20 * 0.0075)}
    r = bench.roofline(dec, prof, peaks, "measured", "decode")
    assert r["kernel"] == "tc_w4a16_gate_up_silu" and r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["avg_launch_us"] == 43.0 and r["launches"] == 20
    want = dec.kernel_units("tc_w4a16_gate_up_silu", peaks)[1] / 43.0e-6 / 1e9
    assert abs(r["achieved"] - want) < 0.01 and abs(r["frac"] - want / 6557.8) < 1e-4
    assert r["traffic"] is None  # no capture for this (kernel, workload)
    assert bench.roofline(dec, {}, peaks, "measured", "decode") is None
    w4 = layers["w4a4"][0]
    r = bench.roofline(w4, {"tc_w4a4_gate_up_silu": (10, 10 * 0.147)}, peaks, "measured", "w4a4")
    assert r["bound"] == "tensor" and r["peak"] == 1671.7 * 4 and "fp4" in r["peak_source"]
