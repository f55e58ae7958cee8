"""GPU parity of the whole decode path on the tiny Qwen3-style config.

Every call goes through the C ABI (libmpk.so via the thin ctypes binding);
expected values come from the CPU oracle only.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import qwen3 as sq
from tests.gpu_util import (HIDDEN_TOL, LOGITS_TOL, bf16_u16, compare_captures, gpu_teacher_forced,
                            oracle_teacher_forced, rel_l2, to_cuda, u16_to_f64)

pytestmark = pytest.mark.gpu

SHAPE = sq.TINY
PROMPT, GEN = 8, 16
S = PROMPT + GEN


@pytest.fixture(scope="module")
def weights():
    w_cpu = sq.make_weights(SHAPE, seed=0)
    return w_cpu, to_cuda(w_cpu)


def _build(w, **kw):
    from persistent_megakernel_decode_02_b200 import build_decoder
    return build_decoder(SHAPE, w, requests=kw.pop("requests", 1), max_seq=kw.pop("max_seq", S), **kw)


def _greedy(dec, tokens_cpu, step0=0):
    tok = tokens_cpu.cuda()
    step = torch.full((tokens_cpu.shape[0],), step0, dtype=torch.int32, device="cuda")
    dec.run(step, tok)
    torch.cuda.synchronize()
    dec.kernel.check_status()
    return tok.cpu(), step.cpu()


@pytest.mark.parametrize("fused", [True, False], ids=["fused-attention", "split-attention"])
def test_greedy_tokens_bit_identical_to_oracle(weights, fused):
    """The tiny config's greedy tokens must match the oracle exactly; the oracle's
    top-2 margins show how far each choice is from a tie."""
    w_cpu, w = weights
    tokens = sq.make_tokens(SHAPE, 1, S, [PROMPT], seed=0)
    dec = _build(w, fused_attention=fused)
    got, step = _greedy(dec, tokens)
    ref = oracle.Decoder(SHAPE, w_cpu)
    toks = tokens.numpy().copy()
    kc, vc = ref.new_cache(1, S)
    st = np.zeros(1, np.int32)
    margins = []
    while True:
        lg = np.zeros((1, SHAPE.vocab))
        if ref.iteration(kc, vc, st, toks, None, oracle.ROUND_NONE, lg, None) == 0:
            break
        z = np.sort(lg[0].astype(np.float32))
        margins.append(float(z[-1] - z[-2]))
    assert int(step[0]) == S - 1
    assert np.array_equal(got.numpy(), toks), (got.tolist(), toks.tolist(), margins)
    # pred holds every prediction, prompt positions included
    pred = dec.pred.cpu().numpy()
    assert np.array_equal(pred[0, PROMPT:], toks[0, PROMPT:])
    # KV cache: bf16 values within bf16 rounding of the oracle's
    gk = u16_to_f64(bf16_u16(dec.k_cache))[:, :, :, : S - 1]
    rk = u16_to_f64(kc)[:, :, :, : S - 1]
    assert rel_l2(gk, rk) < 1e-2
    gv = u16_to_f64(bf16_u16(dec.v_cache))[:, :, :, : S - 1]
    rv = u16_to_f64(vc)[:, :, :, : S - 1]
    assert rel_l2(gv, rv) < 1e-2
    assert np.all(bf16_u16(dec.k_cache)[:, :, :, S - 1:] == 0)
    dec.kernel.close()


@pytest.mark.parametrize("fused", [True, False], ids=["fused-attention", "split-attention"])
def test_teacher_forced_logits_and_hidden_states(weights, fused):
    w_cpu, w = weights
    tokens = sq.make_tokens(SHAPE, 1, S, [PROMPT], seed=1, teacher_forced=True)
    dec = _build(w, fused_attention=fused)
    gpu, gtok, _ = gpu_teacher_forced(dec, tokens, S - 1)
    ref, rtok, _, _ = oracle_teacher_forced(SHAPE, w_cpu, tokens, S - 1)
    wl, wh = compare_captures(gpu, ref)
    print(f"worst logits rel-L2 {wl:.2e} (tol {LOGITS_TOL}), hidden {wh:.2e} (tol {HIDDEN_TOL})")
    # teacher-forced slots are never overwritten
    assert torch.equal(gtok, tokens)
    dec.kernel.close()


@pytest.mark.parametrize("fused", [True, False], ids=["fused-attention", "split-attention"])
def test_op_by_op_is_bit_identical_to_persistent(weights, fused):
    _, w = weights
    tokens = sq.make_tokens(SHAPE, 1, S, [PROMPT], seed=2)
    outs = []
    for mode in ("persistent", "op_by_op"):
        dec = _build(w, fused_attention=fused)
        lg = torch.zeros((1, SHAPE.vocab), device="cuda")
        hd = torch.zeros((SHAPE.layers + 1, 1, SHAPE.hidden), device="cuda")
        dec.kernel.set_capture(S - 3, lg, hd)
        tok = tokens.cuda()
        step = torch.zeros(1, dtype=torch.int32, device="cuda")
        (dec.run if mode == "persistent" else dec.run_op_by_op)(step, tok)
        torch.cuda.synchronize()
        dec.kernel.check_status()
        outs.append((tok.cpu(), dec.pred.cpu(), lg.cpu(), hd.cpu(), dec.k_cache.cpu(), dec.v_cache.cpu()))
        dec.kernel.close()
    for a, b in zip(*outs):
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                           b.view(torch.int16) if b.dtype == torch.bfloat16 else b)


@pytest.mark.parametrize("split", [(140, 32), (128, 80), (146, 8)])
def test_worker_scheduler_split_invariance(weights, split):
    """Results do not depend on how SMs are split between workers and schedulers."""
    _, w = weights
    import persistent_megakernel_decode_02_b200 as pkg
    sms = pkg.load().mpk_device_sm_count()
    tokens = sq.make_tokens(SHAPE, 1, S, [PROMPT], seed=3)
    res = []
    for W, Ls in ((sms - 4, 16), (sms - split[1] // 4, split[1])):
        dec = _build(w, num_workers=W, num_local_schedulers=Ls, gemv_tasks=144, attn_chunks=5,
                     fused_attention=split[0] % 2 == 0)
        lg = torch.zeros((1, SHAPE.vocab), device="cuda")
        dec.kernel.set_capture(S - 2, lg, None)
        got, _ = _greedy(dec, tokens)
        res.append((got, lg.cpu(), dec.k_cache.cpu()))
        dec.kernel.close()
    assert torch.equal(res[0][0], res[1][0])
    assert torch.equal(res[0][1], res[1][1])
    assert torch.equal(res[0][2].view(torch.int16), res[1][2].view(torch.int16))


def test_resume_one_step_runs_equal_one_long_run(weights):
    _, w = weights
    tokens = sq.make_tokens(SHAPE, 1, S, [PROMPT], seed=4)
    dec = _build(w)
    a, _ = _greedy(dec, tokens)
    kc_a = dec.k_cache.clone()
    dec.kernel.close()
    dec = _build(w)
    tok = tokens.cuda()
    step = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(S - 1):
        dec.run(step, tok, (step + 1).to(torch.int32))
    torch.cuda.synchronize()
    dec.kernel.check_status()
    assert int(step.item()) == S - 1
    assert torch.equal(tok.cpu(), a)
    assert torch.equal(dec.k_cache.view(torch.int16), kc_a.view(torch.int16))
    dec.kernel.close()


@pytest.mark.parametrize("chunks", [1, 3, 16, 40])
def test_attention_chunking_ragged(weights, chunks):
    """Split-K chunk counts larger than the context (empty chunks), ragged chunk
    sizes and a single chunk all agree with the oracle."""
    w_cpu, w = weights
    tokens = sq.make_tokens(SHAPE, 1, S, [PROMPT], seed=5, teacher_forced=True)
    dec = _build(w, attn_chunks=chunks, fused_attention=False)
    gpu, _, _ = gpu_teacher_forced(dec, tokens, 12)
    ref, _, _, _ = oracle_teacher_forced(SHAPE, w_cpu, tokens, 12)
    compare_captures(gpu, ref)
    dec.kernel.close()


@pytest.mark.parametrize("tasks", [1, 7, 100, 288])
@pytest.mark.parametrize("fused", [True, False], ids=["fused-attention", "split-attention"])
def test_ragged_task_splits(weights, tasks, fused):
    """Row splits that are not multiples of the worker count (warning only), one
    task for a whole matrix (or kv-head group), and more tasks than workers."""
    w_cpu, w = weights
    tokens = sq.make_tokens(SHAPE, 1, S, [PROMPT], seed=6, teacher_forced=True)
    dec = _build(w, gemv_tasks=tasks, fused_attention=fused)
    gpu, _, _ = gpu_teacher_forced(dec, tokens, 6)
    ref, _, _, _ = oracle_teacher_forced(SHAPE, w_cpu, tokens, 6)
    compare_captures(gpu, ref)
    if tasks % dec.kernel.num_workers:
        assert "not a multiple of num_workers" in dec.kernel.warnings()
    dec.kernel.close()


def test_block_dim_variants(weights):
    w_cpu, w = weights
    tokens = sq.make_tokens(SHAPE, 1, S, [PROMPT], seed=7, teacher_forced=True)
    ref, _, _, _ = oracle_teacher_forced(SHAPE, w_cpu, tokens, 5)
    for bd in (128, 256):
        dec = _build(w, block_dim=bd)
        gpu, _, _ = gpu_teacher_forced(dec, tokens, 5)
        compare_captures(gpu, ref)
        dec.kernel.close()


def test_no_active_request_is_a_no_op(weights):
    _, w = weights
    tokens = sq.make_tokens(SHAPE, 1, S, [PROMPT], seed=8)
    dec = _build(w)
    tok = tokens.cuda()
    step = torch.full((1,), S - 1, dtype=torch.int32, device="cuda")
    dec.run(step, tok)
    torch.cuda.synchronize()
    dec.kernel.check_status()
    assert int(step.item()) == S - 1 and torch.equal(tok.cpu(), tokens)
    step = torch.full((1,), 3, dtype=torch.int32, device="cuda")
    dec.run(step, tok, torch.full((1,), 3, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    dec.kernel.check_status()
    assert int(step.item()) == 3
    dec.kernel.close()


@pytest.mark.parametrize("fused", [True, False], ids=["fused-attention", "split-attention"])
def test_claimed_tasks_bit_identical_to_fixed_mapping(weights, fused):
    """Claiming GEMV tasks from a shared counter (whichever worker is free takes
    the next) gives exactly the results of the fixed task-to-worker mapping with
    the same task split."""
    _, w = weights
    tokens = sq.make_tokens(SHAPE, 1, S, [PROMPT], seed=10)
    outs = []
    for dynamic in (False, True):
        dec = _build(w, gemv_tasks=40, fused_attention=fused, dynamic_tasks=dynamic)
        lg = torch.zeros((1, SHAPE.vocab), device="cuda")
        hd = torch.zeros((SHAPE.layers + 1, 1, SHAPE.hidden), device="cuda")
        dec.kernel.set_capture(S - 3, lg, hd)
        got, _ = _greedy(dec, tokens)
        outs.append((got, dec.pred.cpu(), lg.cpu(), hd.cpu(), dec.k_cache.cpu().view(torch.int16)))
        dec.kernel.close()
    for a, b in zip(*outs):
        assert torch.equal(a, b)
