"""NVFP4 W4A4 linear layer for NVIDIA B200 (sm_100a).

The compute path is ``libnvfp4.so`` (hand-written CUDA, C ABI declared in
``include/nvfp4.h``); :mod:`.nvfp4` is its thin ctypes binding and
:mod:`.workloads` draws the seeded synthetic inputs.
"""
__all__ = ["nvfp4", "workloads"]
