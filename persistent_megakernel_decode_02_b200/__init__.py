"""Persistent-megakernel decoding for NVIDIA B200 (sm_100a).

The whole decode iteration of a Qwen3-style decoder runs in ONE persistent
kernel launch (libmpk.so, C ABI in include/mpk.h); this package is the thin
Python binding over it.  There is no CPU or PyTorch fallback: without the
compiled library every entry point raises.
"""
from ._lib import MpkError, load  # noqa: F401
from .kernel import PersistentKernel  # noqa: F401
from .qwen3 import Decoder, build_decoder, default_attn_chunks, layer_plan  # noqa: F401

__all__ = ["MpkError", "PersistentKernel", "Decoder", "build_decoder", "layer_plan", "default_attn_chunks", "load"]
