"""ctypes binding of libmpk.so (the C ABI in include/mpk.h).

Argument marshalling only: every step of the decode path runs in the CUDA
library.  Importing this module never builds anything; a missing library is a
hard error (there is no fallback path).
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
SO_PATH = os.path.join(HERE, "libmpk.so")

MPK_OK = 0
ERRORS = {
    -1: "INVALID_ARG", -2: "SM_FORMULA", -3: "UNSUPPORTED", -4: "NOT_FOUND", -5: "SHAPE",
    -6: "DTYPE", -7: "STATE", -8: "CUDA", -9: "TIMEOUT", -10: "ABORTED", -11: "DEVICE",
}
ERR_CODE = {v: k for k, v in ERRORS.items()}

BF16, FP32, INT32, INT64, FP32T = 0, 1, 2, 3, 4
IO_CUDA, IO_NVSHMEM = 0, 1
OP_EMBED, OP_RMSNORM_LINEAR, OP_ATTENTION, OP_LINEAR_RESIDUAL = 1, 2, 3, 4
OP_RMSNORM_LINEAR_SILU_MUL, OP_RMSNORM_LMHEAD_ARGMAX, OP_RMSNORM_QKV_ATTENTION = 5, 6, 7
MAX_IO = 8
MAX_GEMV_K = 4096  # MPK_MAX_GEMV_K


class Dim3(ctypes.Structure):
    _fields_ = [("x", ctypes.c_int32), ("y", ctypes.c_int32), ("z", ctypes.c_int32)]


class Layer(ctypes.Structure):
    _fields_ = [
        ("op", ctypes.c_int32),
        ("inputs", ctypes.c_char_p * MAX_IO),
        ("weights", ctypes.c_char_p * MAX_IO),
        ("outputs", ctypes.c_char_p * MAX_IO),
        ("grid_dim", Dim3),
        ("block_dim", Dim3),
        ("layer", ctypes.c_int32),
        ("capture_slot", ctypes.c_int32),
        ("eps", ctypes.c_float),
        ("rope_theta", ctypes.c_float),
    ]


class Options(ctypes.Structure):
    _fields_ = [
        ("profiling", ctypes.c_int32),
        ("sched_lookahead", ctypes.c_int32),
        ("timeout_s", ctypes.c_double),
        ("max_timeline", ctypes.c_int32),
        ("prefetch_kb", ctypes.c_int32),
        ("dynamic_tasks", ctypes.c_int32),
        ("debug_stall_op", ctypes.c_int32),
        ("poll_inputs", ctypes.c_int32),
        ("prefill_tokens", ctypes.c_int32),
        ("kv_page_size", ctypes.c_int32),
    ]


class MpkError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code
        self.name = ERRORS.get(code, str(code))


# name -> (restype, argtypes); mirrors include/mpk.h
_VP, _I, _I64, _CP = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_char_p
SIGNATURES = {
    "mpk_abi_version": (_I, []),
    "mpk_worker_threads": (_I, []),
    "mpk_device_sm_count": (_I, []),
    "mpk_validate_split": (_I, [_I, _I, _I, _I]),
    "mpk_create": (_I, [_I, _I, _I, ctypes.POINTER(_VP)]),
    "mpk_attach_input": (_I, [_VP, _CP, _VP, _I, _I, ctypes.POINTER(_I64)]),
    "mpk_new_tensor": (_I, [_VP, _CP, _I, _I, ctypes.POINTER(_I64), _I, ctypes.POINTER(_VP)]),
    "mpk_tensor_ptr": (_VP, [_VP, _CP]),
    "mpk_compile": (_I, [_VP, ctypes.POINTER(Layer), _I, ctypes.POINTER(Options)]),
    "mpk_warnings": (_CP, [_VP]),
    "mpk_run": (_I, [_VP, _VP, _VP, _I, _I64, _VP, _VP]),
    "mpk_run_op_by_op": (_I, [_VP, _VP, _VP, _I, _I64, _VP, _VP]),
    "mpk_set_capture": (_I, [_VP, _I, _VP, _VP]),
    "mpk_status": (_I, [_VP]),
    "mpk_request_abort": (_I, [_VP]),
    "mpk_timeline": (_I, [_VP, _VP, _I]),
    "mpk_destroy": (_I, [_VP]),
    "mpk_last_error": (_CP, [_VP]),
    "mpk_lmhead_argmax_noalloc": (_I, [_VP, _VP, _VP, _I, _I, _I, ctypes.c_float, _VP, _VP, _VP]),
    "mpk_noalloc_last_error": (_CP, []),
}

_lib = None


def load():
    """Load libmpk.so (built by build.py / __graft_entry__.build()).  MPK_LIBRARY
    may name another build of the same library (e.g. a ring-depth variant)."""
    global _lib
    if _lib is None:
        path = os.environ.get("MPK_LIBRARY", SO_PATH)
        if not os.path.exists(path):
            raise ImportError(f"libmpk.so not found at {path}: run persistent_megakernel_decode_02_b200/build.py")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def check(rc: int, ctx=None):
    if rc != MPK_OK:
        msg = load().mpk_last_error(ctx)
        raise MpkError(rc, msg.decode() if msg else "")
    return rc
