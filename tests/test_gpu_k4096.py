"""GEMV tasks with reduction length 4096 (the Qwen3-8B hidden size, the longest
input the GEMV path keeps in shared memory): every consumer warp takes whole
weight rows (two at a time, sharing each load of the fp32 input vector) from
the weight stages.  A one-layer model with hidden size 4096 runs every GEMV
kind through that path: against the oracle, with task splits that leave
ragged last stages, against op-by-op execution, and with fewer consumer warps
per task (block_dim 128)."""
import pytest
import torch

from synth import qwen3 as sq
from tests.gpu_util import compare_captures, gpu_teacher_forced, oracle_teacher_forced, to_cuda

pytestmark = pytest.mark.gpu

H4096 = sq.Qwen3Shape("h4096", 1, 4096, 32, 8, 128, 4096, 2048, tied=False)
S = 10


@pytest.fixture(scope="module")
def weights():
    w_cpu = sq.make_weights(H4096, seed=5)
    return w_cpu, to_cuda(w_cpu)


@pytest.mark.parametrize("tasks,block_dim", [(144, 0), (7, 0), (37, 0), (144, 128)])
def test_k4096_matches_oracle(weights, tasks, block_dim):
    from persistent_megakernel_decode_02_b200 import build_decoder

    w_cpu, w = weights
    tokens = sq.make_tokens(H4096, 1, S, [S], seed=31, teacher_forced=True)
    dec = build_decoder(H4096, w, requests=1, max_seq=S, gemv_tasks=tasks, block_dim=block_dim)
    gpu, _, _ = gpu_teacher_forced(dec, tokens, 4)
    ref, _, _, _ = oracle_teacher_forced(H4096, w_cpu, tokens, 4)
    wl, wh = compare_captures(gpu, ref)
    print(f"tasks {tasks} block_dim {block_dim}: logits {wl:.2e} hidden {wh:.2e}")
    dec.kernel.close()


@pytest.mark.parametrize("fused", [True, False], ids=["fused-attention", "split-attention"])
def test_k4096_op_by_op_bit_identical(weights, fused):
    from persistent_megakernel_decode_02_b200 import build_decoder

    _, w = weights
    tokens = sq.make_tokens(H4096, 1, S, [4], seed=32)
    outs = []
    for mode in ("run", "run_op_by_op"):
        dec = build_decoder(H4096, w, requests=1, max_seq=S, fused_attention=fused)
        lg = torch.zeros((1, H4096.vocab), device="cuda")
        hd = torch.zeros((H4096.layers + 1, 1, H4096.hidden), device="cuda")
        dec.kernel.set_capture(S - 3, lg, hd)
        tok = tokens.cuda()
        step = torch.zeros(1, dtype=torch.int32, device="cuda")
        getattr(dec, mode)(step, tok)
        torch.cuda.synchronize()
        dec.kernel.check_status()
        outs.append((tok.cpu(), dec.pred.cpu(), lg.cpu(), hd.cpu(), dec.k_cache.cpu().view(torch.int16)))
        dec.kernel.close()
    for a, b in zip(*outs):
        assert torch.equal(a, b)
