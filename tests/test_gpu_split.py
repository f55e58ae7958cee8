"""Residual projections longer than the shared-memory input buffer (4096) are
split into reduction segments computed by separate tasks; the last segment
task of each row block adds the partial sums in segment order.  A tiny model
with a 12288-wide MLP exercises the split (3 segments) against the oracle."""
import numpy as np
import pytest
import torch

from synth import qwen3 as sq
from tests.gpu_util import compare_captures, gpu_teacher_forced, oracle_teacher_forced, to_cuda

pytestmark = pytest.mark.gpu

WIDE = sq.Qwen3Shape("tiny-wide", 2, 256, 4, 2, 64, 12288, 1024, tied=False)
PROMPT, S = 6, 14


@pytest.fixture(scope="module")
def weights():
    w_cpu = sq.make_weights(WIDE, seed=3)
    return w_cpu, to_cuda(w_cpu)


@pytest.mark.parametrize("tasks", [3, 9, 144, 288])
def test_split_down_projection_matches_oracle(weights, tasks):
    from persistent_megakernel_decode_02_b200 import build_decoder

    w_cpu, w = weights
    tokens = sq.make_tokens(WIDE, 1, S, [PROMPT], seed=21, teacher_forced=True)
    dec = build_decoder(WIDE, w, requests=1, max_seq=S, gemv_tasks=tasks)
    gpu, _, _ = gpu_teacher_forced(dec, tokens, 6)
    ref, _, _, _ = oracle_teacher_forced(WIDE, w_cpu, tokens, 6)
    compare_captures(gpu, ref)
    dec.kernel.close()


def test_split_op_by_op_bit_identical(weights):
    from persistent_megakernel_decode_02_b200 import build_decoder

    _, w = weights
    tokens = sq.make_tokens(WIDE, 1, S, [PROMPT], seed=22)
    outs = []
    for mode in ("run", "run_op_by_op"):
        dec = build_decoder(WIDE, w, requests=1, max_seq=S)
        hd = torch.zeros((WIDE.layers + 1, 1, WIDE.hidden), device="cuda")
        dec.kernel.set_capture(S - 3, None, hd)
        tok = tokens.cuda()
        step = torch.zeros(1, dtype=torch.int32, device="cuda")
        getattr(dec, mode)(step, tok)
        torch.cuda.synchronize()
        dec.kernel.check_status()
        outs.append((tok.cpu(), dec.pred.cpu(), hd.cpu(), dec.k_cache.cpu().view(torch.int16)))
        dec.kernel.close()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_split_needs_task_multiple(weights):
    from persistent_megakernel_decode_02_b200 import build_decoder
    from persistent_megakernel_decode_02_b200._lib import MpkError

    _, w = weights
    with pytest.raises(MpkError, match="multiple of 3 tasks"):
        build_decoder(WIDE, w, requests=1, max_seq=S, gemv_tasks=100)


def test_split_claimed_tasks_bit_identical_to_fixed_mapping(weights):
    from persistent_megakernel_decode_02_b200 import build_decoder

    _, w = weights
    tokens = sq.make_tokens(WIDE, 1, S, [PROMPT], seed=23)
    outs = []
    for dynamic in (False, True):
        dec = build_decoder(WIDE, w, requests=1, max_seq=S, gemv_tasks=96, dynamic_tasks=dynamic)
        hd = torch.zeros((WIDE.layers + 1, 1, WIDE.hidden), device="cuda")
        dec.kernel.set_capture(S - 3, None, hd)
        tok = tokens.cuda()
        step = torch.zeros(1, dtype=torch.int32, device="cuda")
        dec.run(step, tok)
        torch.cuda.synchronize()
        dec.kernel.check_status()
        outs.append((tok.cpu(), dec.pred.cpu(), hd.cpu()))
        dec.kernel.close()
    for a, b in zip(*outs):
        assert torch.equal(a, b)
