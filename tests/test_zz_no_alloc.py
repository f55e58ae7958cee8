"""The allocation-free LM-head + argmax entry point (mpk_lmhead_argmax_noalloc).

Some callers cannot allocate device memory on their decode path (a serving
framework whose memory pool owns the GPU, for example), so this entry point
keeps its scratch in a fixed array inside the library.  The test feeds it the
residual stream that the persistent kernel captured right before its own final
norm + LM head and checks, on two calls in a row (the scratch is shared and
must be cleared by each call), that the logits agree within the tests' logits
tolerance and the greedy token is the persistent kernel's.  This file is
collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

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
