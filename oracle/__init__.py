"""CPU oracle of the decode path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package.  It loads ``liboracle.so`` built from ``oracle.c``
(plain C, double arithmetic, OpenMP over output rows) and never touches the
CUDA library.

Parity unpinned: none of the functions here; each building block is pinned by
``tests/test_oracle_pins.py`` (closed forms, invariants, brute force, special
cases) and the whole decoder by special-case models and an independent
restatement through PyTorch's own library routines.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None

ROUND_NONE = 0
ROUND_BF16 = 1

_P = ctypes.POINTER(ctypes.c_uint16)
_PP = ctypes.POINTER(_P)


class _Model(ctypes.Structure):
    _fields_ = [
        ("L", ctypes.c_int), ("H", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
        ("d", ctypes.c_int), ("I", ctypes.c_int), ("V", ctypes.c_int),
        ("eps", ctypes.c_double), ("theta", ctypes.c_double),
        ("embed", _P), ("final_norm", _P), ("lm_head", _P),
        ("in_norm", _PP), ("wq", _PP), ("wk", _PP), ("wv", _PP), ("q_norm", _PP),
        ("k_norm", _PP), ("wo", _PP), ("post_norm", _PP), ("wg", _PP), ("wu", _PP), ("wd", _PP),
    ]


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "oracle.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", _SO, src, "-lm"])
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        d, vp, i64 = ctypes.c_double, ctypes.c_void_p, ctypes.c_int64
        L.orc_bf16_to_f64.restype = d
        L.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_round_bf16.restype = d
        L.orc_round_bf16.argtypes = [d]
        L.orc_f64_to_bf16_bits.restype = ctypes.c_uint16
        L.orc_f64_to_bf16_bits.argtypes = [d]
        L.orc_rmsnorm.argtypes = [vp, vp, i64, d, vp]
        L.orc_gemv.argtypes = [vp, i64, i64, vp, vp]
        L.orc_rope.argtypes = [vp, ctypes.c_int, i64, d]
        L.orc_silu.restype = d
        L.orc_silu.argtypes = [d]
        L.orc_attend.argtypes = [vp, vp, vp, i64, ctypes.c_int, vp]
        L.orc_argmax_f32.restype = i64
        L.orc_argmax_f32.argtypes = [vp, i64]
        L.orc_decode_iteration.restype = ctypes.c_int
        L.orc_decode_iteration.argtypes = [ctypes.POINTER(_Model), ctypes.c_int, i64, vp, vp, vp,
                                           vp, vp, ctypes.c_int, vp, vp, vp]
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_set_num_threads.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def _u16(t: torch.Tensor) -> np.ndarray:
    """bf16 CPU tensor -> uint16 numpy view (no copy)."""
    assert t.dtype == torch.bfloat16 and not t.is_cuda
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_P)


# ---------------------------------------------------------------- building blocks

def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_bf16(x: float) -> float:
    return lib().orc_round_bf16(float(x))


def rmsnorm(x: np.ndarray, w_bf16: torch.Tensor, eps: float) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    w = _u16(w_bf16)
    y = np.empty_like(x)
    lib().orc_rmsnorm(x.ctypes.data, w.ctypes.data, x.size, eps, y.ctypes.data)
    return y


def gemv(W_bf16: torch.Tensor, x: np.ndarray) -> np.ndarray:
    W = _u16(W_bf16)
    N, K = W.shape
    x = np.ascontiguousarray(x, dtype=np.float64)
    assert x.size == K
    y = np.empty(N, dtype=np.float64)
    lib().orc_gemv(W.ctypes.data, N, K, x.ctypes.data, y.ctypes.data)
    return y


def rope(v: np.ndarray, pos: int, theta: float) -> np.ndarray:
    v = np.array(v, dtype=np.float64, copy=True)
    lib().orc_rope(v.ctypes.data, v.size, int(pos), float(theta))
    return v


def silu(z: float) -> float:
    return lib().orc_silu(float(z))


def attend(q: np.ndarray, K_bf16: torch.Tensor, V_bf16: torch.Tensor) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.float64)
    K, V = _u16(K_bf16), _u16(V_bf16)
    npos, d = K.shape
    o = np.empty(d, dtype=np.float64)
    lib().orc_attend(q.ctypes.data, K.ctypes.data, V.ctypes.data, npos, d, o.ctypes.data)
    return o


def argmax_f32(z: np.ndarray) -> int:
    z = np.ascontiguousarray(z, dtype=np.float64)
    return int(lib().orc_argmax_f32(z.ctypes.data, z.size))


def num_threads() -> int:
    return int(lib().orc_num_threads())


def set_num_threads(n: int) -> None:
    lib().orc_set_num_threads(int(n))


# ---------------------------------------------------------------- the decoder

class Decoder:
    """The oracle decoder over a dict of bf16 CPU weights (names as in ``synth.qwen3``)."""

    def __init__(self, shape, weights: Dict[str, torch.Tensor]):
        self.shape = shape
        s = shape
        assert s.head_dim <= 512 and s.head_dim % 2 == 0
        self._keep = []

        def arr(name):
            a = _u16(weights[name])
            self._keep.append(a)
            return a

        def layer_ptrs(suffix):
            ps = [_ptr(arr(f"layers.{l}.{suffix}")) for l in range(s.layers)]
            a = (_P * s.layers)(*ps)
            self._keep.append(a)
            return ctypes.cast(a, _PP)

        m = _Model()
        m.L, m.H, m.Hq, m.Hkv = s.layers, s.hidden, s.q_heads, s.kv_heads
        m.d, m.I, m.V = s.head_dim, s.intermediate, s.vocab
        m.eps, m.theta = s.eps, s.rope_theta
        m.embed = _ptr(arr("embed_tokens"))
        m.final_norm = _ptr(arr("norm"))
        m.lm_head = m.embed if s.tied else _ptr(arr("lm_head"))
        m.in_norm = layer_ptrs("input_layernorm")
        m.wq, m.wk, m.wv = layer_ptrs("q_proj"), layer_ptrs("k_proj"), layer_ptrs("v_proj")
        m.q_norm, m.k_norm = layer_ptrs("q_norm"), layer_ptrs("k_norm")
        m.wo = layer_ptrs("o_proj")
        m.post_norm = layer_ptrs("post_attention_layernorm")
        m.wg, m.wu, m.wd = layer_ptrs("gate_proj"), layer_ptrs("up_proj"), layer_ptrs("down_proj")
        self._m = m

    def new_cache(self, requests: int, max_seq: int):
        s = self.shape
        shp = (s.layers, requests, s.kv_heads, max_seq, s.head_dim)
        return np.zeros(shp, dtype=np.uint16), np.zeros(shp, dtype=np.uint16)

    def iteration(self, kc: np.ndarray, vc: np.ndarray, step: np.ndarray, tokens: np.ndarray,
                  step_end: Optional[np.ndarray] = None, round_mode: int = ROUND_NONE,
                  logits: Optional[np.ndarray] = None, hidden: Optional[np.ndarray] = None,
                  pred: Optional[np.ndarray] = None) -> int:
        """One decoding iteration in place (see ``orc_decode_iteration``)."""
        R, S = tokens.shape
        assert tokens.dtype == np.int64 and tokens.flags.c_contiguous
        assert step.dtype == np.int32 and step.size == R
        assert kc.dtype == np.uint16 and kc.shape[1] == R and kc.shape[3] == S
        se = None if step_end is None else np.ascontiguousarray(step_end, dtype=np.int32)
        for a, shp in ((logits, (R, self.shape.vocab)),
                       (hidden, (self.shape.layers + 1, R, self.shape.hidden)),
                       (pred, (R, S))):
            if a is not None:
                assert a.shape == shp and a.flags.c_contiguous
        return lib().orc_decode_iteration(
            ctypes.byref(self._m), R, S, kc.ctypes.data, vc.ctypes.data, step.ctypes.data,
            tokens.ctypes.data, None if se is None else se.ctypes.data, round_mode,
            None if logits is None else logits.ctypes.data,
            None if hidden is None else hidden.ctypes.data,
            None if pred is None else pred.ctypes.data)

    def generate(self, tokens: np.ndarray, step: np.ndarray, step_end: np.ndarray,
                 kc=None, vc=None, round_mode: int = ROUND_NONE, capture: bool = False):
        """Iterate until no request is active.  Returns (tokens, step, kc, vc, captures)
        where captures is a list of (logits, hidden) per iteration when ``capture``."""
        tokens = np.array(tokens, dtype=np.int64, copy=True)
        step = np.array(step, dtype=np.int32, copy=True)
        R, S = tokens.shape
        if kc is None:
            kc, vc = self.new_cache(R, S)
        caps = []
        while True:
            lg = hd = None
            if capture:
                lg = np.full((R, self.shape.vocab), np.nan)
                hd = np.full((self.shape.layers + 1, R, self.shape.hidden), np.nan)
            n = self.iteration(kc, vc, step, tokens, step_end, round_mode, lg, hd)
            if n == 0:
                break
            if capture:
                caps.append((lg, hd))
        return tokens, step, kc, vc, caps
