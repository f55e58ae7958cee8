"""Python face of the C ABI, shaped like the pages' API.

"Mirage Persistent Kernel: Fusing Multi-GPU LLM Inference into One Kernel
Launch", sections "How MPK Works" and "The API": a PersistentKernel is created
with num_workers / num_local_schedulers / num_remote_schedulers (plus
world_size and mpi_rank), existing PyTorch tensors are attached by name,
intermediate tensors are allocated with new_tensor(dims, dtype, name,
io_category), fused layers such as rmsnorm_linear_layer are chained with a
grid_dim and block_dim each, compile() builds the kernel and calling the object
runs it over the `step` / `tokens` meta tensors.

This module only marshals arguments; all computation runs in libmpk.so.
PyTorch provides device memory and streams.
"""
from __future__ import annotations

import ctypes
from typing import Dict, Iterable, List, Optional, Sequence, Union

import torch

from . import _lib
from ._lib import MpkError, check

_DTYPES = {torch.bfloat16: _lib.BF16, torch.float32: _lib.FP32, torch.int32: _lib.INT32,
           torch.int64: _lib.INT64}
_TORCH = {v: k for k, v in _DTYPES.items()}
# Activations passed between operations (MPK_FP32T): 8 bytes per element, the
# fp32 value in the low half, a version tag in the high half.  Seen from torch
# as int64; `untag` gives the values.
FP32_TAGGED = "fp32_tagged"
_IO = {"cuda_tensor": _lib.IO_CUDA, "nvshmem_tensor": _lib.IO_NVSHMEM}

Name = Union[str, torch.Tensor]


def untag(t: torch.Tensor) -> torch.Tensor:
    """fp32 values of a tagged activation tensor (int64 view of MPK_FP32T)."""
    return t.contiguous().view(torch.float32)[..., 0::2]


class _DeviceArray:
    """__cuda_array_interface__ view of library-owned memory (for torch.as_tensor)."""

    _TYPESTR = {_lib.BF16: "<f2", _lib.FP32: "<f4", _lib.INT32: "<i4", _lib.INT64: "<i8", _lib.FP32T: "<i8"}

    def __init__(self, ptr: int, dims: Sequence[int], dtype: int):
        self.__cuda_array_interface__ = {
            "shape": tuple(int(d) for d in dims), "typestr": self._TYPESTR[dtype],
            "data": (int(ptr), False), "version": 3, "strides": None,
        }


def _dim3(v) -> _lib.Dim3:
    if isinstance(v, int):
        return _lib.Dim3(v, 1, 1)
    v = tuple(v) + (1, 1, 1)
    return _lib.Dim3(int(v[0]), int(v[1]), int(v[2]))


class PersistentKernel:
    """block_dim 0 (the default of every layer method) means all worker threads
    (mpk_worker_threads())."""

    def __init__(self, num_workers: int, num_local_schedulers: int, num_remote_schedulers: int = 0,
                 world_size: int = 1, mpi_rank: int = 0):
        self._lib = _lib.load()
        if world_size != 1 or mpi_rank != 0:
            raise MpkError(_lib.ERR_CODE["UNSUPPORTED"],
                           "world_size > 1 needs remote schedulers and NVSHMEM tensors; this build runs on one GPU")
        ctx = ctypes.c_void_p()
        check(self._lib.mpk_create(num_workers, num_local_schedulers, num_remote_schedulers, ctypes.byref(ctx)))
        self._ctx = ctx
        self.num_workers = num_workers
        self.num_local_schedulers = num_local_schedulers
        self._names: Dict[int, str] = {}
        self._keep: List[object] = []
        self._layers: List[_lib.Layer] = []
        self.tensors: Dict[str, torch.Tensor] = {}
        self.compiled = False

    # ------------------------------------------------------------------ tensors
    def attach_input(self, torch_tensor: torch.Tensor, name: str) -> torch.Tensor:
        t = torch_tensor
        if not t.is_cuda or not t.is_contiguous():
            raise MpkError(_lib.ERR_CODE["INVALID_ARG"], f"'{name}': needs a contiguous CUDA tensor")
        if t.dtype not in _DTYPES:
            raise MpkError(_lib.ERR_CODE["DTYPE"], f"'{name}': dtype {t.dtype} not supported")
        dims = (ctypes.c_int64 * t.dim())(*t.shape)
        check(self._lib.mpk_attach_input(self._ctx, name.encode(), ctypes.c_void_p(t.data_ptr()), _DTYPES[t.dtype],
                                         t.dim(), dims), self._ctx)
        self._names[id(t)] = name
        self.tensors[name] = t
        return t

    def new_tensor(self, dims: Sequence[int], dtype: torch.dtype, name: str,
                   io_category: str = "cuda_tensor") -> torch.Tensor:
        if io_category not in _IO:
            raise MpkError(_lib.ERR_CODE["INVALID_ARG"], f"io_category {io_category!r}")
        if dtype != FP32_TAGGED and dtype not in _DTYPES:
            raise MpkError(_lib.ERR_CODE["DTYPE"], f"dtype {dtype} not supported")
        code = _lib.FP32T if dtype == FP32_TAGGED else _DTYPES[dtype]
        cd = (ctypes.c_int64 * len(dims))(*dims)
        ptr = ctypes.c_void_p()
        check(self._lib.mpk_new_tensor(self._ctx, name.encode(), code, len(dims), cd, _IO[io_category],
                                       ctypes.byref(ptr)), self._ctx)
        if dtype == torch.bfloat16:
            view = torch.as_tensor(_DeviceArray(ptr.value, dims, code), device="cuda").view(torch.bfloat16)
        else:
            view = torch.as_tensor(_DeviceArray(ptr.value, dims, code), device="cuda")
        self._names[id(view)] = name
        self.tensors[name] = view
        return view

    def _name(self, x: Optional[Name]) -> Optional[bytes]:
        if x is None:
            return None
        if isinstance(x, str):
            return x.encode()
        n = self._names.get(id(x))
        if n is None:
            raise MpkError(_lib.ERR_CODE["NOT_FOUND"], "tensor was not attached or allocated by this kernel")
        return n.encode()

    # ------------------------------------------------------------------ layers
    def _add(self, op: int, inputs: Iterable[Optional[Name]] = (), weights: Iterable[Optional[Name]] = (),
             outputs: Iterable[Optional[Name]] = (), grid_dim=1, block_dim=0, layer: int = 0,
             capture_slot: int = -1, eps: float = 1e-6, rope_theta: float = 1e6) -> None:
        L = _lib.Layer()
        L.op = op
        for arr, vals in ((L.inputs, inputs), (L.weights, weights), (L.outputs, outputs)):
            vals = list(vals)
            if len(vals) > _lib.MAX_IO:
                raise MpkError(_lib.ERR_CODE["INVALID_ARG"], "too many tensors for one operation")
            for i, v in enumerate(vals):
                n = self._name(v)
                if n is not None:
                    self._keep.append(n)
                    arr[i] = n
        L.grid_dim = _dim3(grid_dim)
        L.block_dim = _dim3(block_dim)
        L.layer = layer
        L.capture_slot = capture_slot
        L.eps = eps
        L.rope_theta = rope_theta
        self._layers.append(L)

    def embed_layer(self, embedding: Name, output: Name, grid_dim, block_dim=0, capture_slot: int = -1):
        self._add(_lib.OP_EMBED, (), (embedding,), (output,), grid_dim, block_dim, capture_slot=capture_slot)

    def rmsnorm_linear_layer(self, input: Name, weight_norm: Name, weight_linear, output, grid_dim,
                             block_dim=0, eps: float = 1e-6):
        wl = weight_linear if isinstance(weight_linear, (list, tuple)) else [weight_linear]
        out = output if isinstance(output, (list, tuple)) else [output]
        self._add(_lib.OP_RMSNORM_LINEAR, (input,), [weight_norm, *wl], out, grid_dim, block_dim, eps=eps)

    def attention_layer(self, q: Name, k: Name, v: Name, q_norm: Name, k_norm: Name, k_cache: Name,
                        v_cache: Name, output: Name, layer: int, grid_dim, block_dim=0, eps: float = 1e-6,
                        rope_theta: float = 1e6):
        self._add(_lib.OP_ATTENTION, (q, k, v), (q_norm, k_norm, k_cache, v_cache), (output,), grid_dim,
                  block_dim, layer=layer, eps=eps, rope_theta=rope_theta)

    def rmsnorm_qkv_attention_layer(self, input: Name, weight_norm: Name, wq: Name, wk: Name, wv: Name,
                                    q_norm: Name, k_norm: Name, k_cache: Name, v_cache: Name, q: Name, k: Name,
                                    v: Name, output: Name, layer: int, grid_dim, block_dim=0, eps: float = 1e-6,
                                    rope_theta: float = 1e6):
        self._add(_lib.OP_RMSNORM_QKV_ATTENTION, (input,),
                  (weight_norm, wq, wk, wv, q_norm, k_norm, k_cache, v_cache), (q, k, v, output), grid_dim,
                  block_dim, layer=layer, eps=eps, rope_theta=rope_theta)

    def linear_residual_layer(self, input: Name, weight: Name, residual: Name, grid_dim, block_dim=0,
                              capture_slot: int = -1):
        self._add(_lib.OP_LINEAR_RESIDUAL, (input,), (weight,), (residual,), grid_dim, block_dim,
                  capture_slot=capture_slot)

    def rmsnorm_linear_silu_mul_layer(self, input: Name, weight_norm: Name, weight_gate: Name, weight_up: Name,
                                      output: Name, grid_dim, block_dim=0, eps: float = 1e-6):
        self._add(_lib.OP_RMSNORM_LINEAR_SILU_MUL, (input,), (weight_norm, weight_gate, weight_up), (output,),
                  grid_dim, block_dim, eps=eps)

    def rmsnorm_lmhead_argmax_layer(self, input: Name, weight_norm: Name, weight_lm: Name,
                                    pred: Optional[Name] = None, grid_dim=1, block_dim=0, eps: float = 1e-6):
        self._add(_lib.OP_RMSNORM_LMHEAD_ARGMAX, (input,), (weight_norm, weight_lm), (pred,), grid_dim, block_dim,
                  eps=eps)

    # ------------------------------------------------------------------ compile / run
    def compile(self, profiling: bool = False, sched_lookahead: int = 0, timeout_s: float = 0.0,
                max_timeline: int = 0, prefetch_kb: int = 0, debug_stall_op: int = 0,
                dynamic_tasks: bool = False, poll_inputs: bool = False, prefill_tokens: int = 0,
                kv_page_size: int = 0) -> str:
        arr = (_lib.Layer * len(self._layers))(*self._layers)
        opts = _lib.Options(int(profiling), int(sched_lookahead), float(timeout_s), int(max_timeline),
                            int(prefetch_kb), 1 if dynamic_tasks else 0, int(debug_stall_op),
                            1 if poll_inputs else 0, int(prefill_tokens), int(kv_page_size))
        check(self._lib.mpk_compile(self._ctx, arr, len(self._layers), ctypes.byref(opts)), self._ctx)
        self._keep.append(arr)
        self.compiled = True
        return self.warnings()

    def num_ops(self) -> int:
        return len(self._layers)

    def warnings(self) -> str:
        w = self._lib.mpk_warnings(self._ctx)
        return w.decode() if w else ""

    @staticmethod
    def _stream_ptr(stream) -> ctypes.c_void_p:
        if stream is None:
            stream = torch.cuda.current_stream()
        return ctypes.c_void_p(stream.cuda_stream)

    def _meta(self, step: torch.Tensor, tokens: torch.Tensor, step_end: Optional[torch.Tensor]):
        if step.dtype != torch.int32 or tokens.dtype != torch.int64:
            raise MpkError(_lib.ERR_CODE["DTYPE"], "step must be int32 and tokens int64")
        if not (step.is_cuda and tokens.is_cuda and step.is_contiguous() and tokens.is_contiguous()):
            raise MpkError(_lib.ERR_CODE["INVALID_ARG"], "step / tokens must be contiguous CUDA tensors")
        if tokens.dim() != 2 or step.numel() != tokens.shape[0]:
            raise MpkError(_lib.ERR_CODE["SHAPE"], "tokens must be [num_requests, seq_length], step [num_requests]")
        se = None
        if step_end is not None:
            if step_end.dtype != torch.int32 or not step_end.is_cuda or step_end.numel() != step.numel():
                raise MpkError(_lib.ERR_CODE["INVALID_ARG"], "step_end must be a CUDA int32 [num_requests]")
            se = ctypes.c_void_p(step_end.data_ptr())
        return (ctypes.c_void_p(step.data_ptr()), ctypes.c_void_p(tokens.data_ptr()), int(tokens.shape[0]),
                int(tokens.shape[1]), se)

    def __call__(self, step: torch.Tensor, tokens: torch.Tensor, step_end: Optional[torch.Tensor] = None,
                 stream=None) -> None:
        """Run iterations in one persistent launch (asynchronous on `stream`)."""
        s, t, R, S, se = self._meta(step, tokens, step_end)
        check(self._lib.mpk_run(self._ctx, s, t, R, S, se, self._stream_ptr(stream)), self._ctx)

    run = __call__

    def run_op_by_op(self, step: torch.Tensor, tokens: torch.Tensor, step_end: Optional[torch.Tensor] = None,
                     stream=None) -> None:
        s, t, R, S, se = self._meta(step, tokens, step_end)
        check(self._lib.mpk_run_op_by_op(self._ctx, s, t, R, S, se, self._stream_ptr(stream)), self._ctx)

    def set_capture(self, iteration: int, logits: Optional[torch.Tensor] = None,
                    hidden: Optional[torch.Tensor] = None) -> None:
        for t in (logits, hidden):
            if t is not None and (t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous()):
                raise MpkError(_lib.ERR_CODE["INVALID_ARG"], "capture buffers must be contiguous CUDA fp32")
        self._keep.extend([logits, hidden])
        check(self._lib.mpk_set_capture(self._ctx, int(iteration),
                                        ctypes.c_void_p(logits.data_ptr() if logits is not None else 0),
                                        ctypes.c_void_p(hidden.data_ptr() if hidden is not None else 0)), self._ctx)

    def status(self) -> int:
        """Device status of the last run (call after synchronising its stream)."""
        return int(self._lib.mpk_status(self._ctx))

    def check_status(self) -> None:
        check(self._lib.mpk_status(self._ctx), self._ctx)

    def last_error(self) -> str:
        m = self._lib.mpk_last_error(self._ctx)
        return m.decode() if m else ""

    def request_abort(self) -> None:
        check(self._lib.mpk_request_abort(self._ctx), self._ctx)

    TIMELINE_FIELDS = ("entry", "worker", "popped", "ready", "end", "prologue", "first_data", "first_issue",
                       "stage_wait", "last_data", "rows_done")

    def timeline(self) -> torch.Tensor:
        """[n, 11] records (see TIMELINE_FIELDS; times in %globaltimer ns, stage_wait a duration in ns)."""
        n = int(self._lib.mpk_timeline(self._ctx, None, 0))
        out = torch.zeros((max(n, 0), len(self.TIMELINE_FIELDS)), dtype=torch.int64)
        if n > 0:
            self._lib.mpk_timeline(self._ctx, ctypes.c_void_p(out.data_ptr()), n)
        return out

    def close(self) -> None:
        if getattr(self, "_ctx", None) is not None and self._ctx.value:
            self._lib.mpk_destroy(self._ctx)
            self._ctx = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
