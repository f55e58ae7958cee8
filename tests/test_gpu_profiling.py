"""The task-timeline profiler on the GPU ("Mirage Persistent Kernel: Fusing
Multi-GPU LLM Inference into One Kernel Launch", "Getting Started": with
profiling on, the task timeline is recorded for visualisation).  Recording must
not change what is computed, and every task of every iteration leaves one
well-ordered record."""
import numpy as np
import pytest
import torch

from synth import qwen3 as sq
from tests.gpu_util import to_cuda

pytestmark = pytest.mark.gpu

SHAPE = sq.TINY
PROMPT, GEN = 8, 12
S = PROMPT + GEN


@pytest.fixture(scope="module")
def weights():
    return to_cuda(sq.make_weights(SHAPE, seed=0))


def _decode(w, profiling, fused, requests=1):
    from persistent_megakernel_decode_02_b200 import build_decoder
    lens = [PROMPT, 5, 7, 3][:requests]
    tokens = sq.make_tokens(SHAPE, requests, S, lens, seed=4)
    dec = build_decoder(SHAPE, w, requests=requests, max_seq=S, profiling=profiling,
                        fused_attention=fused if requests == 1 else None)
    step = torch.zeros(requests, dtype=torch.int32, device="cuda")
    tok = tokens.cuda()
    dec.run(step, tok)
    torch.cuda.synchronize()
    dec.kernel.check_status()
    out = (tok.cpu(), step.cpu(), dec.pred.cpu(), dec.k_cache.cpu(), dec.v_cache.cpu())
    tl = dec.kernel.timeline() if profiling else None
    ntasks = [L.grid_dim.x * L.grid_dim.y * L.grid_dim.z for L in dec.kernel._layers]
    dec.kernel.close()
    return out, tl, ntasks


@pytest.mark.parametrize("fused,requests", [(True, 1), (False, 1), (None, 4)],
                         ids=["fused-attention", "split-attention", "batched-4"])
def test_profiling_leaves_results_bit_identical(weights, fused, requests):
    a, _, _ = _decode(weights, False, fused, requests)
    b, tl, _ = _decode(weights, True, fused, requests)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert tl.shape[0] > 0


@pytest.mark.parametrize("fused,requests", [(True, 1), (False, 1), (None, 4)],
                         ids=["fused-attention", "split-attention", "batched-4"])
def test_timeline_one_ordered_record_per_task_and_iteration(weights, fused, requests):
    (_, step, _, _, _), tl, ntasks = _decode(weights, True, fused, requests)
    iters = int(step.max().item())  # every run starts at step 0 and ends when the longest request is done
    rec = tl.numpy()
    entry = rec[:, 0].astype(np.uint64)
    it = (entry >> np.uint64(32)).astype(np.int64)
    op = ((entry >> np.uint64(16)) & np.uint64(0xFFFF)).astype(np.int64)
    task = (entry & np.uint64(0xFFFF)).astype(np.int64)
    assert rec.shape[0] == iters * sum(ntasks)
    seen = set(zip(it.tolist(), op.tolist(), task.tolist()))
    assert len(seen) == rec.shape[0]  # no duplicate record
    for n in range(iters):
        for p, nt in enumerate(ntasks):
            for t in range(nt):
                assert (n, p, t) in seen
    popped, ready, end = rec[:, 2], rec[:, 3], rec[:, 4]
    assert (popped > 0).all() and (popped <= ready).all() and (ready <= end).all()
    for col in (5, 6, 9, 10):  # prologue, first data, last data, rows done: 0 when the task has none
        v = rec[:, col]
        has = v != 0
        assert ((v[has] >= ready[has]) & (v[has] <= end[has])).all(), col
    assert (rec[:, 8] >= 0).all()  # time waited for weight stages
    workers = rec[:, 1]
    assert (workers >= 0).all() and (workers < 148).all()
