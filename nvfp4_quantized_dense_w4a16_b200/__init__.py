"""NVFP4 dense SwiGLU FFN for NVIDIA B200 (sm_100a).

The compute lives in ``libffn_nvfp4.so`` (hand-written CUDA behind the C ABI
in ``include/ffn_nvfp4.h``); :mod:`.native` binds it with ctypes and raises
ImportError when the library is missing -- there is no CPU implementation.
:mod:`.synth` draws the seeded synthetic workloads.
"""
__all__ = ["native", "synth", "build"]
