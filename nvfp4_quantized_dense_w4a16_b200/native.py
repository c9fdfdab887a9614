"""ctypes binding of ``libffn_nvfp4.so`` (include/ffn_nvfp4.h).

Argument marshalling only: every function takes torch tensors, checks their
device, dtype, shape and contiguity, and passes raw pointers, sizes and the
current CUDA stream to the C ABI of the same name.  All compute happens in the
library's CUDA kernels; there is no CPU fallback, and importing this module
fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libffn_nvfp4.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "ffn_nvfp4.h")

FFN_ACT_BF16 = 0
FFN_ACT_NVFP4_FIXED = 1
# weight handle formats (FFN_FORMAT_* bits)
_WEIGHT_FORMATS = {"bf16": 1, "w4a16": 1, "nvfp4_fixed": 2, "w4a4": 2, "all": 3}
_FORMATS = {"bf16": FFN_ACT_BF16, "w4a16": FFN_ACT_BF16,
            "nvfp4_fixed": FFN_ACT_NVFP4_FIXED, "w4a4": FFN_ACT_NVFP4_FIXED}


class FfnError(RuntimeError):
    def __init__(self, fn: str, status: int, name: str):
        super().__init__(f"{fn} failed: {name} ({status})")
        self.status = status
        self.status_name = name


class ProjectionPlan(ctypes.Structure):
    _fields_ = [("family", ctypes.c_int), ("tile_rows", ctypes.c_int), ("k_splits", ctypes.c_int),
                ("grid", ctypes.c_int)]


KERNEL_FAMILIES = {0: "none", 1: "tc_w4a16", 2: "tc_w4a4", 3: "gemv_w4a16", 4: "gemv_w4a4",
                   5: "tc_w4a16_persistent", 6: "tc_planes"}
ROLES = {"linear": 0, "gate_up": 1, "down": 2}


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int), ("total_ms", ctypes.c_double)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m nvfp4_quantized_dense_w4a16_b200.build` "
            "(the NVFP4 FFN has no CPU implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
    P = ctypes.POINTER
    sig = {
        "ffn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "ffn_nvfp4_abi_version": (ctypes.c_int, []),
        "ffn_nvfp4_quantize_weights": (ctypes.c_int, [vp, i64, i64, vp, vp, vp, vp]),
        "ffn_nvfp4_quantize_activations": (ctypes.c_int, [vp, i64, i64, vp, vp, vp]),
        "ffn_nvfp4_weight_create": (ctypes.c_int, [vp, vp, vp, i64, i64, vp, P(vp)]),
        "ffn_nvfp4_weight_create_ex": (ctypes.c_int, [vp, vp, vp, i64, i64, ctypes.c_uint, vp, P(vp)]),
        "ffn_nvfp4_weight_info": (ctypes.c_int, [vp, P(ctypes.c_uint), P(sz)]),
        "ffn_nvfp4_weight_create_gate_up": (ctypes.c_int, [vp, vp, vp, P(vp)]),
        "ffn_nvfp4_weight_destroy": (ctypes.c_int, [vp]),
        "ffn_nvfp4_weight_dims": (ctypes.c_int, [vp, P(i64), P(i64), P(ctypes.c_int)]),
        "ffn_nvfp4_workspace_size": (ctypes.c_int, [i64, i64, i64, ctypes.c_int, P(sz)]),
        "ffn_nvfp4_forward": (ctypes.c_int, [vp, i64, i64, i64, vp, vp, ctypes.c_int, vp, vp, sz, vp]),
        "ffn_nvfp4_forward_lora": (ctypes.c_int, [vp, i64, i64, i64, vp, vp, vp, ctypes.c_int, vp, vp, sz, vp]),
        "ffn_nvfp4_workspace_size_lora": (ctypes.c_int, [i64, i64, i64, ctypes.c_int, vp, P(sz)]),
        "ffn_nvfp4_lora_create": (ctypes.c_int, [i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, P(vp)]),
        "ffn_nvfp4_lora_destroy": (ctypes.c_int, [vp]),
        "ffn_nvfp4_linear_workspace_size": (ctypes.c_int, [i64, i64, i64, ctypes.c_int, P(sz)]),
        "ffn_nvfp4_linear": (ctypes.c_int, [vp, i64, vp, ctypes.c_int, vp, vp, sz, vp]),
        "ffn_nvfp4_linear_noalloc": (ctypes.c_int, [vp, i64, vp, vp, vp]),
        "ffn_nvfp4_projection_plan": (ctypes.c_int, [i64, i64, i64, ctypes.c_int, ctypes.c_int,
                                                     P(ProjectionPlan)]),
        "ffn_nvfp4_tensor_peak": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                 P(ctypes.c_double)]),
        "ffn_nvfp4_profile_begin": (ctypes.c_int, []),
        "ffn_nvfp4_device_error": (ctypes.c_int, [P(ctypes.c_int), ctypes.c_int]),
        "ffn_nvfp4_profile_end": (ctypes.c_int, [P(KernelTime), ctypes.c_int, P(ctypes.c_int)]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def declared_symbols(header: str = HEADER) -> list[str]:
    """Function names declared in the public header."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ffn_[a-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    return lib.ffn_status_string(status).decode()


def _check(fn: str, status: int):
    if status != 0:
        raise FfnError(fn, status, status_string(status))


def _fmt(fmt) -> int:
    if isinstance(fmt, int):
        return fmt
    return _FORMATS[fmt]


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def ffn_nvfp4_abi_version() -> int:
    return lib.ffn_nvfp4_abi_version()


def ffn_nvfp4_quantize_weights(w: torch.Tensor, codes=None, block_scales=None, global_scale=None,
                               stream=None):
    """bf16 [n, k] -> (codes uint8 [n, k/2], block_scales uint8 [n, k/16], gs float32 [1])."""
    _need(w, "w", torch.bfloat16)
    n, k = w.shape
    dev = w.device
    codes = torch.empty((n, k // 2), dtype=torch.uint8, device=dev) if codes is None else codes
    block_scales = torch.empty((n, k // 16), dtype=torch.uint8, device=dev) if block_scales is None else block_scales
    global_scale = torch.empty((1,), dtype=torch.float32, device=dev) if global_scale is None else global_scale
    _need(codes, "codes", torch.uint8, (n, k // 2))
    _need(block_scales, "block_scales", torch.uint8, (n, k // 16))
    _need(global_scale, "global_scale", torch.float32, (1,))
    _check("ffn_nvfp4_quantize_weights", lib.ffn_nvfp4_quantize_weights(
        _ptr(w), n, k, _ptr(codes), _ptr(block_scales), _ptr(global_scale), _stream(stream)))
    return codes, block_scales, global_scale


def ffn_nvfp4_quantize_activations(x: torch.Tensor, codes=None, block_scales=None, stream=None):
    """bf16 [m, k] -> (codes uint8 [m, k/2], block_scales uint8 [m, k/16])."""
    _need(x, "x", torch.bfloat16)
    m, k = x.shape
    codes = torch.empty((m, k // 2), dtype=torch.uint8, device=x.device) if codes is None else codes
    block_scales = torch.empty((m, k // 16), dtype=torch.uint8, device=x.device) if block_scales is None else block_scales
    _need(codes, "codes", torch.uint8, (m, k // 2))
    _need(block_scales, "block_scales", torch.uint8, (m, k // 16))
    _check("ffn_nvfp4_quantize_activations", lib.ffn_nvfp4_quantize_activations(
        _ptr(x), m, k, _ptr(codes), _ptr(block_scales), _stream(stream)))
    return codes, block_scales


class Weight:
    """Owning wrapper of an ``ffn_nvfp4_weight*`` handle."""

    def __init__(self, handle: ctypes.c_void_p):
        self._h = handle
        n, k, gu = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int()
        _check("ffn_nvfp4_weight_dims", lib.ffn_nvfp4_weight_dims(
            self._h, ctypes.byref(n), ctypes.byref(k), ctypes.byref(gu)))
        self.n, self.k, self.is_gate_up = n.value, k.value, bool(gu.value)
        f, b = ctypes.c_uint(), ctypes.c_size_t()
        _check("ffn_nvfp4_weight_info", lib.ffn_nvfp4_weight_info(self._h, ctypes.byref(f), ctypes.byref(b)))
        self.formats, self.device_bytes = f.value, b.value

    @property
    def handle(self):
        return self._h

    def close(self):
        if self._h:
            _check("ffn_nvfp4_weight_destroy", lib.ffn_nvfp4_weight_destroy(self._h))
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def ffn_nvfp4_weight_create(codes: torch.Tensor, block_scales: torch.Tensor,
                            global_scale: torch.Tensor, stream=None, formats="all") -> Weight:
    """Handle for the activation formats 'bf16', 'nvfp4_fixed' or 'all'
    (one tiled copy of the weight per format)."""
    _need(codes, "codes", torch.uint8)
    n, half_k = codes.shape
    k = 2 * half_k
    _need(block_scales, "block_scales", torch.uint8, (n, k // 16))
    _need(global_scale, "global_scale", torch.float32, (1,))
    h = ctypes.c_void_p()
    f = formats if isinstance(formats, int) else _WEIGHT_FORMATS[formats]
    _check("ffn_nvfp4_weight_create_ex", lib.ffn_nvfp4_weight_create_ex(
        _ptr(codes), _ptr(block_scales), _ptr(global_scale), n, k, f, _stream(stream), ctypes.byref(h)))
    return Weight(h)


def ffn_nvfp4_weight_create_gate_up(gate: Weight, up: Weight, stream=None) -> Weight:
    h = ctypes.c_void_p()
    _check("ffn_nvfp4_weight_create_gate_up", lib.ffn_nvfp4_weight_create_gate_up(
        gate.handle, up.handle, _stream(stream), ctypes.byref(h)))
    return Weight(h)


def ffn_nvfp4_workspace_size(m: int, hidden: int, inter: int, fmt="bf16") -> int:
    out = ctypes.c_size_t()
    _check("ffn_nvfp4_workspace_size", lib.ffn_nvfp4_workspace_size(m, hidden, inter, _fmt(fmt), ctypes.byref(out)))
    return out.value


def ffn_nvfp4_linear_workspace_size(m: int, n: int, k: int, fmt="bf16") -> int:
    out = ctypes.c_size_t()
    _check("ffn_nvfp4_linear_workspace_size", lib.ffn_nvfp4_linear_workspace_size(m, n, k, _fmt(fmt), ctypes.byref(out)))
    return out.value


def _workspace(nbytes: int, device, workspace):
    """A fresh workspace of the required size, or the caller's (whose size the
    C ABI checks, returning FFN_ERR_WORKSPACE when it is too small)."""
    if workspace is None:
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=device)
    _need(workspace, "workspace", torch.uint8)
    return workspace


class Lora:
    """Owning wrapper of an ``ffn_lora*`` adapter handle."""

    def __init__(self, handle: ctypes.c_void_p, rank: int):
        self._h, self.rank = handle, rank

    @property
    def handle(self):
        return self._h

    def close(self):
        if self._h:
            _check("ffn_nvfp4_lora_destroy", lib.ffn_nvfp4_lora_destroy(self._h))
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def ffn_nvfp4_lora_create(rank: int, hidden: int, inter: int, gate=None, up=None, down=None,
                          stream=None) -> Lora:
    """Adapters for a layer: each of gate/up/down an (A, B) pair of bf16
    tensors (A [rank, in], B [out, rank]) or None."""
    ptrs = []
    for name, pair, n_in, n_out in (("gate", gate, hidden, inter), ("up", up, hidden, inter),
                                    ("down", down, inter, hidden)):
        if pair is None:
            ptrs += [None, None]
            continue
        a, b = pair
        _need(a, name + "_a", torch.bfloat16, (rank, n_in))
        _need(b, name + "_b", torch.bfloat16, (n_out, rank))
        ptrs += [_ptr(a), _ptr(b)]
    h = ctypes.c_void_p()
    _check("ffn_nvfp4_lora_create", lib.ffn_nvfp4_lora_create(rank, hidden, inter, *ptrs, _stream(stream),
                                                              ctypes.byref(h)))
    return Lora(h, rank)


def ffn_nvfp4_forward(x: torch.Tensor, gate_up: Weight, down: Weight, fmt="bf16", out=None,
                      workspace=None, stream=None, lora: Lora | None = None) -> torch.Tensor:
    """out[m, hidden] = down(silu(gate(x)) * up(x)) through the C ABI (with
    the adapters' deltas when `lora` is given)."""
    _need(x, "x", torch.bfloat16)
    m, hidden = x.shape
    inter = down.k
    out = torch.empty((m, hidden), dtype=torch.bfloat16, device=x.device) if out is None else out
    _need(out, "out", torch.bfloat16, (m, hidden))
    if lora is None:
        nbytes = ffn_nvfp4_workspace_size(m, hidden, inter, fmt)
        workspace = _workspace(nbytes, x.device, workspace)
        _check("ffn_nvfp4_forward", lib.ffn_nvfp4_forward(
            _ptr(x), m, hidden, inter, gate_up.handle, down.handle, _fmt(fmt), _ptr(out),
            _ptr(workspace), workspace.numel(), _stream(stream)))
        return out
    nb = ctypes.c_size_t()
    _check("ffn_nvfp4_workspace_size_lora", lib.ffn_nvfp4_workspace_size_lora(
        m, hidden, inter, _fmt(fmt), lora.handle, ctypes.byref(nb)))
    workspace = _workspace(nb.value, x.device, workspace)
    _check("ffn_nvfp4_forward_lora", lib.ffn_nvfp4_forward_lora(
        _ptr(x), m, hidden, inter, gate_up.handle, down.handle, lora.handle, _fmt(fmt), _ptr(out),
        _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def ffn_nvfp4_linear(x: torch.Tensor, w: Weight, fmt="bf16", y=None, workspace=None,
                     stream=None) -> torch.Tensor:
    """y[m, n] = bf16(gs * x @ w^T) (x quantised per row first in the fixed format)."""
    _need(x, "x", torch.bfloat16)
    m, k = x.shape
    if k != w.k:
        raise ValueError(f"x has {k} columns, the weight expects {w.k}")
    y = torch.empty((m, w.n), dtype=torch.bfloat16, device=x.device) if y is None else y
    _need(y, "y", torch.bfloat16, (m, w.n))
    nbytes = ffn_nvfp4_linear_workspace_size(m, w.n, k, fmt)
    workspace = _workspace(nbytes, x.device, workspace)
    _check("ffn_nvfp4_linear", lib.ffn_nvfp4_linear(
        _ptr(x), m, w.handle, _fmt(fmt), _ptr(y), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return y


def ffn_nvfp4_profile_begin():
    """Start timing every kernel the library launches from this thread."""
    _check("ffn_nvfp4_profile_begin", lib.ffn_nvfp4_profile_begin())


def ffn_nvfp4_profile_end() -> dict:
    """Stop timing; {kernel name: (launches, total ms)} (synchronises the device)."""
    cap = 64
    arr = (KernelTime * cap)()
    n = ctypes.c_int()
    _check("ffn_nvfp4_profile_end", lib.ffn_nvfp4_profile_end(arr, cap, ctypes.byref(n)))
    return {arr[i].name.decode(): (arr[i].launches, arr[i].total_ms) for i in range(n.value)}


def ffn_nvfp4_device_error(clear: bool = True) -> int:
    """Device-side error bits of kernels whose bounded waits gave up (0 = none)."""
    v = ctypes.c_int()
    _check("ffn_nvfp4_device_error", lib.ffn_nvfp4_device_error(ctypes.byref(v), int(clear)))
    return v.value


def ffn_nvfp4_linear_noalloc(x: torch.Tensor, w: Weight, y=None, stream=None) -> torch.Tensor:
    """bf16 projection through the allocation-free entry point (fixed device
    scratch inside the library; concurrent calls must be serialised)."""
    _need(x, "x", torch.bfloat16)
    m, k = x.shape
    if k != w.k:
        raise ValueError(f"x has {k} columns, the weight expects {w.k}")
    y = torch.empty((m, w.n), dtype=torch.bfloat16, device=x.device) if y is None else y
    _need(y, "y", torch.bfloat16, (m, w.n))
    _check("ffn_nvfp4_linear_noalloc", lib.ffn_nvfp4_linear_noalloc(
        _ptr(x), m, w.handle, _ptr(y), _stream(stream)))
    return y


def ffn_nvfp4_projection_plan(m: int, n: int, k: int, fmt="bf16", role: str = "linear") -> dict:
    """The kernel configuration a projection of m rows selects (nothing
    launched); role: 'linear', or the forward's 'gate_up' / 'down'."""
    p = ProjectionPlan()
    _check("ffn_nvfp4_projection_plan", lib.ffn_nvfp4_projection_plan(m, n, k, _fmt(fmt), ROLES[role],
                                                                      ctypes.byref(p)))
    return {"family": KERNEL_FAMILIES.get(p.family, str(p.family)), "tile_rows": p.tile_rows,
            "k_splits": p.k_splits, "grid": p.grid}


def ffn_nvfp4_tensor_peak(kind: str = "bf16", issuers: int = 1, iters: int = 20000) -> float:
    """Measured dense tensor-core TFLOP/s of the current GPU for the MMA kind
    the library issues ('bf16': kind::f16; 'nvfp4': kind::mxf4nvf4)."""
    out = ctypes.c_double()
    _check("ffn_nvfp4_tensor_peak", lib.ffn_nvfp4_tensor_peak({"bf16": 0, "nvfp4": 1}[kind], issuers, iters,
                                                              ctypes.byref(out)))
    return out.value
