"""The allocation-free LM-head + argmax entry point (mpk_lmhead_argmax_noalloc).

Some callers cannot allocate device memory on their decode path (a serving
framework whose memory pool owns the GPU, for example), so this entry point
keeps its scratch in a fixed array inside the library.  The test feeds it the
residual stream that the persistent kernel captured right before its own final
norm + LM head and checks, on two calls in a row (the scratch is shared and
must be cleared by each call), that the logits agree within the tests' logits
tolerance and the greedy token is the persistent kernel's.  It also checks the
call against the CPU oracle's final RMSNorm + LM head + argmax on the same
input: several requests with different rows, without a logits buffer, the
8B width (K = 4096) and the longest reduction (K = 16384, whose input vector
needs more than 48 KB of shared memory).  This file is collected last on
purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import qwen3 as sq
from tests.gpu_util import LOGITS_TOL, rel_l2, to_cuda

pytestmark = pytest.mark.gpu


def _vp(t):
    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


def test_lmhead_argmax_noalloc_matches_persistent_kernel():
    from persistent_megakernel_decode_02_b200 import _lib, build_decoder

    lib = _lib.load()
    shape = sq.TINY
    S = 12
    w = to_cuda(sq.make_weights(shape, seed=0))
    tokens = sq.make_tokens(shape, 1, S, [S], seed=9, teacher_forced=True).cuda()
    dec = build_decoder(shape, w, requests=1, max_seq=S)
    step = torch.zeros(1, dtype=torch.int32, device="cuda")
    for it in range(3):
        logits = torch.zeros((1, shape.vocab), device="cuda")
        hidden = torch.zeros((shape.layers + 1, 1, shape.hidden), device="cuda")
        dec.kernel.set_capture(0, logits, hidden)
        s0 = int(step.item())
        dec.run(step, tokens, (step + 1).to(torch.int32))
        torch.cuda.synchronize()
        dec.kernel.check_status()
        pred = int(dec.pred[0, s0 + 1].item())
        x = hidden[shape.layers].contiguous()  # residual entering the final norm
        lm = w["embed_tokens"] if shape.tied else w["lm_head"]
        for _ in range(2):
            tok = torch.full((1,), -7, dtype=torch.int64, device="cuda")
            lg = torch.zeros((1, shape.vocab), device="cuda")
            rc = lib.mpk_lmhead_argmax_noalloc(_vp(x), _vp(w["norm"]), _vp(lm), 1, shape.hidden, shape.vocab,
                                               ctypes.c_float(shape.eps), _vp(tok), _vp(lg),
                                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
            assert rc == 0, lib.mpk_noalloc_last_error()
            torch.cuda.synchronize()
            err = rel_l2(lg.cpu().numpy(), logits.cpu().numpy())
            assert err <= LOGITS_TOL, (it, err)
            assert int(tok.item()) == pred, (it, int(tok.item()), pred)
    dec.kernel.close()


def test_lmhead_argmax_noalloc_rejects_oversize():
    from persistent_megakernel_decode_02_b200 import _lib

    lib = _lib.load()
    x = torch.zeros((1, 64), device="cuda")
    nw = torch.ones(64, dtype=torch.bfloat16, device="cuda")
    wl = torch.zeros((10, 64), dtype=torch.bfloat16, device="cuda")
    tok = torch.zeros(1, dtype=torch.int64, device="cuda")
    big = 10 ** 6
    rc = lib.mpk_lmhead_argmax_noalloc(_vp(x), _vp(nw), _vp(wl), 1, big, 10, ctypes.c_float(1e-6), _vp(tok), None,
                                       None)
    assert _lib.ERRORS[rc] == "SHAPE" and b"MAX_K" in lib.mpk_noalloc_last_error()
    rc = lib.mpk_lmhead_argmax_noalloc(_vp(x), _vp(nw), _vp(wl), 100000, 64, 10, ctypes.c_float(1e-6), _vp(tok),
                                       None, None)
    assert _lib.ERRORS[rc] == "INVALID_ARG"


def _oracle_lm(x: np.ndarray, nw: torch.Tensor, wl: torch.Tensor, eps: float):
    """Final RMSNorm + LM head + argmax of the oracle, one request row at a time."""
    z = [oracle.gemv(wl, oracle.rmsnorm(x[r], nw, eps)) for r in range(x.shape[0])]
    return np.stack(z), [oracle.argmax_f32(zr) for zr in z]


@pytest.mark.parametrize("R,K,V,with_logits", [(4, 256, 1000, True), (4, 256, 1000, False), (2, 4096, 3000, True),
                                               (1, 16384, 1000, True)])
def test_lmhead_argmax_noalloc_matches_oracle(R, K, V, with_logits):
    from persistent_megakernel_decode_02_b200 import _lib

    lib = _lib.load()
    tag = f"noalloc.{R}.{K}.{V}"
    x_cpu = np.stack([synth.normal_f64(K, 3, f"{tag}.x{r}", 1.0 + r) for r in range(R)]).astype(np.float32)
    nw_cpu = synth.normal_bf16((K,), 3, tag + ".norm", 0.5)
    wl_cpu = synth.normal_bf16((V, K), 3, tag + ".lm", 0.02)
    ref_z, ref_t = _oracle_lm(x_cpu.astype(np.float64), nw_cpu, wl_cpu, 1e-6)
    x, nw, wl = torch.from_numpy(x_cpu).cuda(), nw_cpu.cuda(), wl_cpu.cuda()
    for _ in range(2):  # two calls in a row: the shared scratch is cleared by each
        tok = torch.full((R,), -7, dtype=torch.int64, device="cuda")
        lg = torch.full((R, V), float("nan"), device="cuda") if with_logits else None
        rc = lib.mpk_lmhead_argmax_noalloc(_vp(x), _vp(nw), _vp(wl), R, K, V, ctypes.c_float(1e-6), _vp(tok),
                                           _vp(lg), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == 0, lib.mpk_noalloc_last_error()
        torch.cuda.synchronize()
        if with_logits:
            for r in range(R):
                assert rel_l2(lg[r].cpu().numpy(), ref_z[r]) <= LOGITS_TOL
        for r in range(R):
            # the token is the oracle's unless the top two logits are closer than
            # the fp32 error of a K-long dot product (then either is a valid argmax)
            top2 = np.sort(ref_z[r])[-2:]
            got = int(tok[r].item())
            assert got == ref_t[r] or (top2[1] - top2[0] < 1e-4 * max(1.0, abs(top2[1])) and
                                       abs(ref_z[r][got] - top2[1]) < 1e-4 * max(1.0, abs(top2[1]))), (r, got, ref_t[r])


def test_lmhead_argmax_noalloc_rejects_bad_eps():
    from persistent_megakernel_decode_02_b200 import _lib

    lib = _lib.load()
    x = torch.zeros((1, 64), device="cuda")
    nw = torch.ones(64, dtype=torch.bfloat16, device="cuda")
    wl = torch.zeros((10, 64), dtype=torch.bfloat16, device="cuda")
    tok = torch.zeros(1, dtype=torch.int64, device="cuda")
    for eps in (0.0, -1e-6, float("nan"), float("inf")):
        rc = lib.mpk_lmhead_argmax_noalloc(_vp(x), _vp(nw), _vp(wl), 1, 64, 10, ctypes.c_float(eps), _vp(tok), None,
                                           None)
        assert _lib.ERRORS[rc] == "INVALID_ARG" and b"eps" in lib.mpk_noalloc_last_error(), eps
