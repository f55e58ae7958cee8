"""Error paths of the C ABI on a device (they need a context).

The contracts come from the pages' API ("Mirage Persistent Kernel: Fusing
Multi-GPU LLM Inference into One Kernel Launch", sections "How MPK Works" and
"The API"; the Chinese page's "关键 API 与张量管理"): the worker / scheduler
split must satisfy num_workers + schedulers / 4 = #SMs, remote schedulers and
nvshmem tensors serve other GPUs (this build runs on one GPU), fused layers
name tensors that were attached or allocated first, and the kernel runs only
once compiled.  Each case calls the C entry point directly and checks the
returned code (and that mpk_last_error explains it); a context that rejected a
call stays usable.
"""
import ctypes

import pytest
import torch

from synth import qwen3 as sq
from tests.gpu_util import to_cuda

pytestmark = pytest.mark.gpu

SHAPE = sq.TINY
S = 16


def _lib():
    from persistent_megakernel_decode_02_b200 import _lib as L
    return L


def _err(rc):
    return _lib().ERRORS.get(rc, "OK")


def _last(mk):
    return mk.last_error()


@pytest.fixture(scope="module")
def weights():
    return to_cuda(sq.make_weights(SHAPE, seed=0))


def _kernel():
    from persistent_megakernel_decode_02_b200 import PersistentKernel
    L = _lib().load()
    return PersistentKernel(L.mpk_device_sm_count() - 4, 16, 0)


def _graph(mk, w, drop=(), replace=None):
    """Attach the tiny decoder's tensors to mk and add its layers (not compiled).
    drop: weight names left unattached; replace: name -> tensor attached instead."""
    from persistent_megakernel_decode_02_b200 import layer_plan
    from persistent_megakernel_decode_02_b200.kernel import FP32_TAGGED
    replace = replace or {}
    for name, t in w.items():
        if name not in drop:
            mk.attach_input(replace.get(name, t), name)
    s = SHAPE
    kv = (s.layers, 1, s.kv_heads, S, s.head_dim)
    for n in ("k_cache", "v_cache"):
        mk.attach_input(torch.zeros(kv, dtype=torch.bfloat16, device="cuda"), n)
    for n, dim in (("x", s.hidden), ("q", s.q_dim), ("k", s.kv_dim), ("v", s.kv_dim), ("o", s.q_dim),
                   ("a", s.intermediate)):
        mk.new_tensor((1, dim), FP32_TAGGED, n)
    mk.attach_input(torch.full((1, S), -1, dtype=torch.int64, device="cuda"), "pred")
    for op in layer_plan(s, 1, mk.num_workers, 2, fused_attention=True):
        op = dict(op)
        getattr(mk, op.pop("method"))(**op)


def _compile_rc(mk):
    L = _lib()
    arr = (L.Layer * len(mk._layers))(*mk._layers)
    opts = L.Options()
    return mk._lib.mpk_compile(mk._ctx, arr, len(mk._layers), ctypes.byref(opts))


def test_create_rejects_remote_schedulers_and_broken_split():
    L = _lib()
    lib = L.load()
    sms = lib.mpk_device_sm_count()
    ctx = ctypes.c_void_p()
    assert _err(lib.mpk_create(sms - 5, 16, 4, ctypes.byref(ctx))) == "UNSUPPORTED" and not ctx.value
    assert b"remote" in lib.mpk_last_error(None)
    assert _err(lib.mpk_create(sms - 3, 16, 0, ctypes.byref(ctx))) == "SM_FORMULA" and not ctx.value
    assert _err(lib.mpk_create(sms - 4, 14, 0, ctypes.byref(ctx))) == "SM_FORMULA" and not ctx.value
    assert _err(lib.mpk_create(sms, 0, 0, ctypes.byref(ctx))) == "INVALID_ARG" and not ctx.value
    assert _err(lib.mpk_create(sms - 4, 16, 0, None)) == "INVALID_ARG"


def test_python_world_size_is_unsupported():
    from persistent_megakernel_decode_02_b200 import PersistentKernel, MpkError
    L = _lib().load()
    with pytest.raises(MpkError) as e:
        PersistentKernel(L.mpk_device_sm_count() - 4, 16, 0, world_size=2)
    assert e.value.name == "UNSUPPORTED"


def test_nvshmem_tensor_is_unsupported():
    L = _lib()
    mk = _kernel()
    dims = (ctypes.c_int64 * 2)(1, 256)
    ptr = ctypes.c_void_p()
    rc = mk._lib.mpk_new_tensor(mk._ctx, b"remote_x", L.FP32, 2, dims, L.IO_NVSHMEM, ctypes.byref(ptr))
    assert _err(rc) == "UNSUPPORTED" and "nvshmem" in _last(mk) and not ptr.value
    rc = mk._lib.mpk_new_tensor(mk._ctx, b"x2", L.FP32, 2, dims, 7, ctypes.byref(ptr))
    assert _err(rc) == "INVALID_ARG"
    # the context is still usable
    assert _err(mk._lib.mpk_new_tensor(mk._ctx, b"x3", L.FP32, 2, dims, L.IO_CUDA, ctypes.byref(ptr))) == "OK"
    mk.close()


def test_attach_input_rejects_duplicates_null_and_misaligned():
    L = _lib()
    mk = _kernel()
    t = torch.zeros(64, dtype=torch.float32, device="cuda")
    dims = (ctypes.c_int64 * 1)(64)
    ok = mk._lib.mpk_attach_input(mk._ctx, b"t", ctypes.c_void_p(t.data_ptr()), L.FP32, 1, dims)
    assert _err(ok) == "OK"
    assert _err(mk._lib.mpk_attach_input(mk._ctx, b"t", ctypes.c_void_p(t.data_ptr()), L.FP32, 1, dims)) == \
        "INVALID_ARG" and "already" in _last(mk)
    assert _err(mk._lib.mpk_attach_input(mk._ctx, b"n", None, L.FP32, 1, dims)) == "INVALID_ARG"
    assert _err(mk._lib.mpk_attach_input(mk._ctx, b"m", ctypes.c_void_p(t.data_ptr() + 4), L.FP32, 1, dims)) == \
        "INVALID_ARG" and "aligned" in _last(mk)
    assert _err(mk._lib.mpk_attach_input(mk._ctx, b"", ctypes.c_void_p(t.data_ptr()), L.FP32, 1, dims)) == \
        "INVALID_ARG"
    mk.close()


def test_compile_unknown_tensor_is_not_found(weights):
    mk = _kernel()
    _graph(mk, weights, drop=("layers.1.o_proj",))
    assert _err(_compile_rc(mk)) == "NOT_FOUND" and "layers.1.o_proj" in _last(mk)
    mk.close()


def test_compile_weight_dtype_mismatch(weights):
    mk = _kernel()
    bad = weights["layers.0.gate_proj"].float()
    _graph(mk, weights, replace={"layers.0.gate_proj": bad})
    assert _err(_compile_rc(mk)) == "DTYPE" and "layers.0.gate_proj" in _last(mk)
    mk.close()


def test_compile_weight_shape_mismatch(weights):
    mk = _kernel()
    w = weights["layers.0.down_proj"]
    bad = torch.zeros((w.shape[0], w.shape[1] + 256), dtype=torch.bfloat16, device="cuda")
    _graph(mk, weights, replace={"layers.0.down_proj": bad})
    assert _err(_compile_rc(mk)) == "SHAPE" and f"[{w.shape[0]},{w.shape[1] + 256}]" in _last(mk)
    mk.close()


def test_run_before_compile_and_double_compile(weights):
    L = _lib()
    mk = _kernel()
    _graph(mk, weights)
    step = torch.zeros(1, dtype=torch.int32, device="cuda")
    tok = torch.full((1, S), -1, dtype=torch.int64, device="cuda")
    tok[0, 0] = 3
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = mk._lib.mpk_run(mk._ctx, ctypes.c_void_p(step.data_ptr()), ctypes.c_void_p(tok.data_ptr()), 1, S, None,
                         stream)
    assert _err(rc) == "STATE" and "before" in _last(mk)
    assert _err(_compile_rc(mk)) == "OK"
    assert _err(_compile_rc(mk)) == "STATE" and "already compiled" in _last(mk)
    dims = (ctypes.c_int64 * 1)(8)
    ptr = ctypes.c_void_p()
    rc = mk._lib.mpk_new_tensor(mk._ctx, b"late", L.FP32, 1, dims, L.IO_CUDA, ctypes.byref(ptr))
    assert _err(rc) == "STATE"
    # a request count the graph was not built for, then a valid run
    tok2 = torch.full((2, S), -1, dtype=torch.int64, device="cuda")
    step2 = torch.zeros(2, dtype=torch.int32, device="cuda")
    rc = mk._lib.mpk_run(mk._ctx, ctypes.c_void_p(step2.data_ptr()), ctypes.c_void_p(tok2.data_ptr()), 2, S, None,
                         stream)
    assert _err(rc) == "SHAPE"
    end = torch.full((1,), 4, dtype=torch.int32, device="cuda")
    rc = mk._lib.mpk_run(mk._ctx, ctypes.c_void_p(step.data_ptr()), ctypes.c_void_p(tok.data_ptr()), 1, S,
                         ctypes.c_void_p(end.data_ptr()), stream)
    assert _err(rc) == "OK"
    torch.cuda.synchronize()
    mk.check_status()
    assert int(step.item()) == 4 and bool((tok[0, 1:5] >= 0).all())
    mk.close()
