"""Qwen3-style decoder shapes and their seeded synthetic inputs.

Only shapes, names and random draws live here (no decoder arithmetic), so the
CUDA path and the CPU oracle can both take their inputs from this module.

Weights: every linear / embedding tensor is drawn as bf16 N(0, 0.02^2) from its
own generator stream (the stream is the tensor's name); every norm weight is
1.0.  Prompts: uniform ids in [0, vocab).  Pre-filled KV: bf16 N(0, 1).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List

import torch

from . import normal_bf16, uniform_ids


@dataclass(frozen=True)
class Qwen3Shape:
    name: str
    layers: int
    hidden: int
    q_heads: int
    kv_heads: int
    head_dim: int
    intermediate: int
    vocab: int
    tied: bool
    rope_theta: float = 1.0e6
    eps: float = 1.0e-6
    weight_std: float = 0.02

    @property
    def q_dim(self) -> int:
        return self.q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.kv_heads * self.head_dim

    def weight_shapes(self) -> Dict[str, tuple]:
        H, I, V, d = self.hidden, self.intermediate, self.vocab, self.head_dim
        s: Dict[str, tuple] = {"embed_tokens": (V, H)}
        for l in range(self.layers):
            p = f"layers.{l}."
            s[p + "input_layernorm"] = (H,)
            s[p + "q_proj"] = (self.q_dim, H)
            s[p + "k_proj"] = (self.kv_dim, H)
            s[p + "v_proj"] = (self.kv_dim, H)
            s[p + "q_norm"] = (d,)
            s[p + "k_norm"] = (d,)
            s[p + "o_proj"] = (H, self.q_dim)
            s[p + "post_attention_layernorm"] = (H,)
            s[p + "gate_proj"] = (I, H)
            s[p + "up_proj"] = (I, H)
            s[p + "down_proj"] = (H, I)
        s["norm"] = (H,)
        if not self.tied:
            s["lm_head"] = (V, H)
        return s

    def weight_bytes(self) -> int:
        """bf16 bytes of all weights (each tensor once; a tied LM head is the embedding)."""
        n = 0
        for shp in self.weight_shapes().values():
            m = 1
            for x in shp:
                m *= x
            n += m
        return 2 * n

    def streamed_weight_bytes(self) -> int:
        """Weight bytes one decode step must read: everything but the embedding table,
        plus one embedding row; a tied LM head reads the whole table once."""
        total = self.weight_bytes()
        V, H = self.vocab, self.hidden
        emb = 2 * V * H
        if self.tied:
            return total + 2 * H  # table read once as LM head, one row as embedding
        return total - emb + 2 * H

    def kv_bytes_per_position(self) -> int:
        """bf16 K and V bytes of one cached position across all layers (one request)."""
        return 2 * 2 * self.layers * self.kv_heads * self.head_dim


TINY = Qwen3Shape("tiny", 2, 256, 4, 2, 64, 768, 1024, tied=False)
QWEN3_0_6B = Qwen3Shape("qwen3-0.6b", 28, 1024, 16, 8, 128, 3072, 151936, tied=True)
QWEN3_8B = Qwen3Shape("qwen3-8b", 36, 4096, 32, 8, 128, 12288, 151936, tied=False)
SHAPES = {s.name: s for s in (TINY, QWEN3_0_6B, QWEN3_8B)}


def is_norm(name: str) -> bool:
    return name.endswith("layernorm") or name.endswith("_norm") or name == "norm"


def make_weights(shape: Qwen3Shape, seed: int = 0, pin: bool = False,
                 names: List[str] | None = None) -> Dict[str, torch.Tensor]:
    """bf16 CPU tensors keyed by name (norm weights are ones)."""
    out: Dict[str, torch.Tensor] = {}
    for n, shp in shape.weight_shapes().items():
        if names is not None and n not in names:
            continue
        if is_norm(n):
            t = torch.ones(shp, dtype=torch.bfloat16)
            out[n] = t.pin_memory() if pin else t
        else:
            out[n] = normal_bf16(shp, seed, n, shape.weight_std, pin=pin)
    return out


def make_prompts(shape: Qwen3Shape, requests: int, length: int, seed: int = 0,
                 tag: str = "prompt") -> torch.Tensor:
    """int64 [requests, length] uniform ids in [0, vocab)."""
    ids = uniform_ids(requests * length, seed, f"{tag}.ids", 0, shape.vocab - 1)
    return ids.view(requests, length)


def make_prompt_lengths(requests: int, lo: int, hi: int, seed: int = 0) -> torch.Tensor:
    return uniform_ids(requests, seed, "prompt.lengths", lo, hi)


def make_tokens(shape: Qwen3Shape, requests: int, seq_len: int, prompt_lens, seed: int = 0,
                teacher_forced: bool = False) -> torch.Tensor:
    """tokens[requests, seq_len] int64: prompt ids, then -1 (slots to generate).
    With ``teacher_forced`` every slot holds a random id (nothing is generated)."""
    ids = make_prompts(shape, requests, seq_len, seed)
    tok = ids.clone()
    if not teacher_forced:
        for r in range(requests):
            tok[r, int(prompt_lens[r]):] = -1
    return tok


def make_kv_prefill(shape: Qwen3Shape, requests: int, max_seq: int, positions: int,
                    seed: int = 0, pin: bool = False):
    """(K, V) bf16 caches [L, R, Hkv, max_seq, d]; positions [0, positions) hold
    N(0,1) draws, the rest zeros."""
    L, Hkv, d = shape.layers, shape.kv_heads, shape.head_dim
    caches = []
    for which in ("k", "v"):
        c = torch.zeros((L, requests, Hkv, max_seq, d), dtype=torch.bfloat16, pin_memory=pin)
        if positions:
            for l in range(L):
                for r in range(requests):
                    blk = normal_bf16((Hkv, positions, d), seed, f"kv.{which}.{l}.{r}", 1.0)
                    c[l, r, :, :positions, :] = blk
        caches.append(c)
    return caches[0], caches[1]
