"""Seeded synthetic inputs (weights, prompts, pre-filled KV) for the decoder.

Shared by the CUDA path's tests and bench and by the CPU oracle.  It holds no
decoder arithmetic: the C generator in ``synth.c`` maps (seed, stream, index)
to numbers (counter-based SplitMix64; approximately normal draws from an
Irwin-Hall sum of eight 16-bit uniforms).  Stream ids come from the tensor's
name (FNV-1a 64), so every tensor is reproducible on its own.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", _SO, src, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        i64, u64, vp = ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p
        lib.synth_normal_bf16.argtypes = [vp, i64, u64, u64, ctypes.c_double]
        lib.synth_normal_f64.argtypes = [vp, i64, u64, u64, ctypes.c_double]
        lib.synth_uniform_int64.argtypes = [vp, i64, u64, u64, i64, i64]
        lib.synth_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def stream_id(name: str) -> int:
    """FNV-1a 64-bit hash of a tensor name: the generator stream of that tensor."""
    h = 0xCBF29CE484222325
    for b in name.encode():
        h ^= b
        h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def normal_bf16(shape, seed: int, name: str, std: float, pin: bool = False) -> torch.Tensor:
    """bf16 CPU tensor of approximately N(0, std^2) draws for tensor ``name``."""
    n = int(np.prod(shape)) if len(shape) else 1
    t = torch.empty(tuple(shape), dtype=torch.int16, pin_memory=pin)
    if n:
        _load().synth_normal_bf16(t.data_ptr(), n, seed, stream_id(name), float(std))
    return t.view(torch.bfloat16)


def normal_f64(n: int, seed: int, name: str, std: float = 1.0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    if n:
        _load().synth_normal_f64(out.ctypes.data, n, seed, stream_id(name), float(std))
    return out


def uniform_ids(n: int, seed: int, name: str, lo: int, hi: int) -> torch.Tensor:
    """int64 CPU tensor of uniform integers in [lo, hi] (inclusive)."""
    t = torch.empty(n, dtype=torch.int64)
    if n:
        _load().synth_uniform_int64(t.data_ptr(), n, seed, stream_id(name), lo, hi)
    return t


def num_threads() -> int:
    return int(_load().synth_num_threads())
