"""Failure detection without a GPU fault: every device wait is bounded and ends
in a status the host reads.

A dependency made unsatisfiable on the host (one more completion per iteration
than its producer delivers) must end the run with MPK_ERR_TIMEOUT within the
wait limit; a host abort request must end a long run with MPK_ERR_ABORTED.  In
both cases the context and the GPU stay usable, and after an abort a later run
resumes from `step` and ends where an uninterrupted run ends."""
import time

import pytest
import torch

from synth import qwen3 as sq
from tests.gpu_util import to_cuda

pytestmark = pytest.mark.gpu

SHAPE = sq.TINY


@pytest.fixture(scope="module")
def weights():
    return to_cuda(sq.make_weights(SHAPE, seed=0))


def _inputs(S, prompt=8):
    tok = sq.make_tokens(SHAPE, 1, S, [prompt], seed=0).cuda()
    step = torch.zeros(1, dtype=torch.int32, device="cuda")
    return tok, step


@pytest.mark.parametrize("stall_op", [1, 2, 4, 6])
def test_unsatisfiable_dependency_times_out(weights, stall_op):
    from persistent_megakernel_decode_02_b200 import build_decoder
    from persistent_megakernel_decode_02_b200._lib import ERR_CODE

    S = 24
    dec = build_decoder(SHAPE, weights, requests=1, max_seq=S, timeout_s=0.2, debug_stall_op=stall_op)
    tok, step = _inputs(S)
    before = tok.cpu()
    torch.cuda.synchronize()
    t0 = time.time()
    dec.run(step, tok)
    torch.cuda.synchronize()
    took = time.time() - t0
    assert dec.kernel.status() == ERR_CODE["TIMEOUT"], dec.kernel.last_error()
    assert "device status -9" in dec.kernel.last_error()
    assert took < 5.0, took
    # the first iteration never completed: nothing advanced
    assert int(step.item()) == 0
    assert torch.equal(tok.cpu(), before)
    dec.kernel.close()
    # the device is still healthy: a normal decoder runs to completion
    ok = build_decoder(SHAPE, weights, requests=1, max_seq=S)
    tok, step = _inputs(S)
    ok.run(step, tok)
    torch.cuda.synchronize()
    ok.kernel.check_status()
    assert int(step.item()) == S - 1
    ok.kernel.close()


def test_stall_op_out_of_range_is_rejected(weights):
    from persistent_megakernel_decode_02_b200 import build_decoder
    from persistent_megakernel_decode_02_b200._lib import MpkError

    with pytest.raises(MpkError, match="debug_stall_op"):
        build_decoder(SHAPE, weights, requests=1, max_seq=24, debug_stall_op=1000)


def test_host_abort_then_resume(weights):
    from persistent_megakernel_decode_02_b200 import build_decoder
    from persistent_megakernel_decode_02_b200._lib import ERR_CODE

    S = 8192
    dec = build_decoder(SHAPE, weights, requests=1, max_seq=S)
    tok, step = _inputs(S)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    dec.run(step, tok, stream=stream)
    time.sleep(0.05)
    dec.kernel.request_abort()
    stream.synchronize()
    assert dec.kernel.status() == ERR_CODE["ABORTED"], dec.kernel.last_error()
    s_abort = int(step.item())
    assert 0 <= s_abort < S - 1
    # resume on the same context: the abort flag is cleared by the next run
    dec.run(step, tok)
    torch.cuda.synchronize()
    dec.kernel.check_status()
    assert int(step.item()) == S - 1
    ref = build_decoder(SHAPE, weights, requests=1, max_seq=S)
    tok2, step2 = _inputs(S)
    ref.run(step2, tok2)
    torch.cuda.synchronize()
    ref.kernel.check_status()
    assert torch.equal(tok.cpu(), tok2.cpu())
    assert torch.equal(dec.k_cache.view(torch.int16), ref.k_cache.view(torch.int16))
    print(f"aborted at step {s_abort} of {S - 1}")
    dec.kernel.close()
    ref.kernel.close()


@pytest.mark.parametrize("stall_op", [2, 3, 4, 6, 12])
def test_batched_unsatisfiable_dependency_times_out(weights, stall_op):
    """The batched kernel (tensor-core projections, streamed split-K attention)
    under a stalled operation: RMSNorm + QKV (op 2), attention (3), o projection
    (4), down projection (6), LM head (12).  The run ends with MPK_ERR_TIMEOUT
    within the wait limit, after the accumulators' tensor memory is drained and
    released, and a fresh batched decoder then runs normally."""
    from persistent_megakernel_decode_02_b200 import build_decoder
    from persistent_megakernel_decode_02_b200._lib import ERR_CODE

    S, R = 24, 4
    tok = sq.make_tokens(SHAPE, R, S, [8, 5, 7, 3], seed=1).cuda()
    step = torch.zeros(R, dtype=torch.int32, device="cuda")
    dec = build_decoder(SHAPE, weights, requests=R, max_seq=S, timeout_s=0.2, debug_stall_op=stall_op)
    before = tok.cpu()
    torch.cuda.synchronize()
    t0 = time.time()
    dec.run(step, tok)
    torch.cuda.synchronize()
    took = time.time() - t0
    assert dec.kernel.status() == ERR_CODE["TIMEOUT"], dec.kernel.last_error()
    assert took < 5.0, took
    assert not step.any()
    assert torch.equal(tok.cpu(), before)
    dec.kernel.close()
    ok = build_decoder(SHAPE, weights, requests=R, max_seq=S)
    tok = sq.make_tokens(SHAPE, R, S, [8, 5, 7, 3], seed=1).cuda()
    step = torch.zeros(R, dtype=torch.int32, device="cuda")
    ok.run(step, tok)
    torch.cuda.synchronize()
    ok.kernel.check_status()
    assert (step == S - 1).all()
    ok.kernel.close()
