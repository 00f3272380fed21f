"""Fill CUDA tensors with the seeded inputs (ctypes binding of libkvsynth.so).

Same bits as ``synth.philox`` / ``Config.make`` for the same recipe; used for
inputs too large to draw on the host. Holds no method arithmetic.
"""
from __future__ import annotations

import ctypes
import os

from . import philox  # noqa: F401  (documentation: the numpy twin)

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkvsynth.so")
_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m synth.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        lib.kvsynth_normal.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64,
                                       ctypes.c_uint32, ctypes.c_uint32, ctypes.c_double, ctypes.c_void_p]
        lib.kvsynth_normal.restype = ctypes.c_int
        lib.kvsynth_uniform_f32.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32,
                                            ctypes.c_uint32, ctypes.c_void_p]
        lib.kvsynth_uniform_f32.restype = ctypes.c_int
        _lib = lib
    return _lib


def _stream():
    import torch
    return int(torch.cuda.current_stream().cuda_stream)


def fill_normal(t, seed: int, tensor_id: int, scale: float, offset: int = 0):
    """t: contiguous CUDA tensor, float32 (values) or int16/uint16/bfloat16 (bf16 patterns)."""
    import torch
    dt = 0 if t.dtype == torch.float32 else 1
    rc = _load().kvsynth_normal(t.data_ptr(), dt, t.numel(), offset, seed, tensor_id, float(scale), _stream())
    if rc != 0:
        raise RuntimeError(f"kvsynth_normal failed: cuda error {rc}")
    return t


def fill_uniform(t, seed: int, tensor_id: int, offset: int = 0):
    rc = _load().kvsynth_uniform_f32(t.data_ptr(), t.numel(), offset, seed, tensor_id, _stream())
    if rc != 0:
        raise RuntimeError(f"kvsynth_uniform_f32 failed: cuda error {rc}")
    return t


def make_device(cfg, name: str, device="cuda"):
    """Draw input ``name`` of config ``cfg`` directly on the device (same bits as cfg.make(name))."""
    import torch
    shape, tid, scale, dt, dist = cfg.recipe()[name]
    if dist == "uniform":
        return fill_uniform(torch.empty(shape, dtype=torch.float32, device=device), cfg.seed, tid)
    dtype = torch.float32 if dt == "f32" else torch.bfloat16
    return fill_normal(torch.empty(shape, dtype=dtype, device=device), cfg.seed, tid, scale)
