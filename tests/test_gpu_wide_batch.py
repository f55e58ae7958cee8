"""GPU parity of the batched decode path over 9..16 requests, where every
projection runs as one tensor-core contraction 16 requests wide (MMA N = 32:
the hi and lo parts of 16 input rows) while the weights are still read once
per iteration.

Expected values come from the CPU oracle only (its plain ROUND_NONE reading);
the tolerances are those of the 8-wide path (inputs to ~16 bits, fp32
accumulation: 1e-3 rel-L2 in logits and every layer's residual stream, far
inside the decode bars of 2e-2 and 1e-2), and greedy tokens match exactly.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import qwen3 as sq
from tests.gpu_util import compare_captures, gpu_teacher_forced, oracle_teacher_forced, to_cuda

pytestmark = pytest.mark.gpu

SHAPE = sq.TINY
S = 48


@pytest.fixture(scope="module")
def weights():
    w_cpu = sq.make_weights(SHAPE, seed=0)
    return w_cpu, to_cuda(w_cpu)


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def _build(shape, w, R, **kw):
    from persistent_megakernel_decode_02_b200 import build_decoder
    return build_decoder(shape, w, requests=R, max_seq=kw.pop("max_seq", S), **kw)


def _positions(R, seed):
    return np.array(sq.make_prompt_lengths(R, 0, 20, seed=seed).tolist(), np.int32)


@pytest.mark.parametrize("R", [9, 16])
@pytest.mark.parametrize("poll", [False, True])
def test_teacher_forced_wide_batch(weights, R, poll):
    """R requests at different positions over a pre-filled cache, inputs taken
    from the writers' published rows or polled element by element: logits and
    every layer's residual stream within 1e-3 of the oracle, every request's
    appended cache rows, rows below each request's position untouched."""
    w_cpu, w = weights
    p0 = _positions(R, seed=R + 40)
    kc, vc = sq.make_kv_prefill(SHAPE, R, S, int(p0.max()), seed=41)
    tokens = sq.make_tokens(SHAPE, R, S, [S] * R, seed=42, teacher_forced=True)
    dec = _build(SHAPE, w, R, k_cache=kc.cuda(), v_cache=vc.cuda(), poll_inputs=poll)
    iters = 3
    gpu, gtok, gstep = gpu_teacher_forced(dec, tokens, iters, step0=p0)
    ref, _, rkc, _ = oracle_teacher_forced(SHAPE, w_cpu, tokens, iters, _u16(kc), _u16(vc), step0=p0)
    wl, wh = compare_captures(gpu, ref, logits_tol=1e-3, hidden_tol=1e-3)
    print(f"R={R} poll_inputs={poll}: worst logits rel-L2 {wl:.2e}, hidden {wh:.2e}")
    assert np.array_equal(gstep.numpy(), p0 + iters)
    assert torch.equal(gtok, tokens)
    for r in range(R):
        a, b = int(p0[r]), int(p0[r]) + iters
        gk = dec.k_cache[:, r, :, a:b].float().cpu().numpy()
        rk = (rkc[:, r, :, a:b].astype(np.uint32) << 16).view(np.float32)
        assert np.linalg.norm(gk - rk) <= 1e-2 * np.linalg.norm(rk)
        assert torch.equal(dec.k_cache[:, r, :, :a].cpu().view(torch.int16), kc[:, r, :, :a].view(torch.int16))
    dec.kernel.close()


def test_wide_greedy_tokens_match_oracle(weights):
    """Free-running greedy decode of 16 requests with prompts of different
    lengths and different ends (requests go inactive while the others run on):
    every generated token equals the oracle's, nothing is written past a
    request's end."""
    w_cpu, w = weights
    R = 16
    lens = sq.make_prompt_lengths(R, 2, 12, seed=43)
    tokens = sq.make_tokens(SHAPE, R, S, lens, seed=44)
    se = (lens + torch.tensor([16, 5, 12, 16, 9, 16, 3, 14, 16, 7, 11, 16, 6, 16, 10, 13])).numpy().astype(np.int32)
    dec = _build(SHAPE, w, R)
    tok = tokens.cuda()
    step = torch.zeros(R, dtype=torch.int32, device="cuda")
    dec.run(step, tok, torch.from_numpy(se).cuda())
    torch.cuda.synchronize()
    dec.kernel.check_status()
    got = tok.cpu().numpy()

    ref = oracle.Decoder(SHAPE, w_cpu)
    toks = tokens.numpy().copy()
    kc, vc = ref.new_cache(R, S)
    st = np.zeros(R, np.int32)
    while ref.iteration(kc, vc, st, toks, se, oracle.ROUND_NONE, None, None):
        pass
    assert np.array_equal(step.cpu().numpy(), se)
    assert np.array_equal(got, toks)
    for r in range(R):
        e = int(se[r])
        assert not dec.k_cache[:, r, :, e:].any()
        assert (got[r, e + 1:] == -1).all()
    dec.kernel.close()


def test_wide_op_by_op_is_bit_identical_to_persistent(weights):
    """The 16-wide contractions as one launch per operation give the persistent
    kernel's tokens, predictions and cache bit for bit."""
    _, w = weights
    R = 12
    tokens = sq.make_tokens(SHAPE, R, S, sq.make_prompt_lengths(R, 2, 10, seed=45), seed=46)
    outs = []
    for mode in ("run", "run_op_by_op"):
        dec = _build(SHAPE, w, R)
        tok = tokens.cuda()
        step = torch.zeros(R, dtype=torch.int32, device="cuda")
        getattr(dec, mode)(step, tok, torch.full((R,), 22, dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        dec.kernel.check_status()
        outs.append((tok.cpu(), dec.pred.cpu(), dec.k_cache.cpu().view(torch.int16)))
        dec.kernel.close()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_wide_and_narrow_batches_agree(weights):
    """The first four requests of a 12-request graph (16 wide) decode to the
    same tokens and predictions as the same four requests alone (8 wide), and
    their cache rows agree to rounding: each request is its own column of
    every contraction."""
    _, w = weights
    lens = sq.make_prompt_lengths(12, 2, 10, seed=47)
    tokens = sq.make_tokens(SHAPE, 12, S, lens, seed=48)
    outs = []
    for R in (4, 12):
        dec = _build(SHAPE, w, R, attn_chunks=2)
        tok = tokens[:R].cuda()
        step = torch.zeros(R, dtype=torch.int32, device="cuda")
        dec.run(step, tok, torch.full((R,), 28, dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        dec.kernel.check_status()
        outs.append((tok[:4].cpu(), dec.pred[:4].cpu(), dec.k_cache[:, :4].float().cpu()))
        dec.kernel.close()
    (t0, p0, k0), (t1, p1, k1) = outs
    assert torch.equal(t0, t1)
    assert torch.equal(p0, p1)
    assert float(torch.linalg.vector_norm(k0 - k1)) <= 1e-5 * float(torch.linalg.vector_norm(k0))


WIDE = sq.Qwen3Shape("tiny-wide", 2, 256, 4, 2, 64, 4096, 1024, tied=False)


@pytest.mark.parametrize("down_grid,gu_grid,lm_grid", [
    ((1, 1), (1, 1), (1, 1)),    # one task per op: the 4096-long down reduction in 6 passes of 768
    ((2, 2), (4, 1), (8, 1)),    # down split in two segments of 2048, each in 3 passes
])
def test_wide_reduction_passes(monkeypatch, down_grid, gu_grid, lm_grid):
    """16-wide contractions hold 768 reduction elements per pass (the 16 hi and
    16 lo input rows of a K block take 4 KB): longer reductions run in passes,
    each row block in its own accumulator slot, alone or with a split."""
    import persistent_megakernel_decode_02_b200.qwen3 as q3

    w_cpu = sq.make_weights(WIDE, seed=4)
    w = to_cuda(w_cpu)
    grids = {(WIDE.hidden, WIDE.intermediate, False): down_grid, (WIDE.intermediate, WIDE.hidden, True): gu_grid,
             (WIDE.vocab, WIDE.hidden, False): lm_grid}
    orig = q3.batched_grid
    monkeypatch.setattr(q3, "batched_grid", lambda rows, K, wk, pair=False, **kw: grids.get((rows, K, pair)) or
                        orig(rows, K, wk, pair, **kw))
    R = 10
    p0 = _positions(R, seed=49)
    kc, vc = sq.make_kv_prefill(WIDE, R, S, int(p0.max()), seed=50)
    tokens = sq.make_tokens(WIDE, R, S, [S] * R, seed=51, teacher_forced=True)
    dec = _build(WIDE, w, R, k_cache=kc.cuda(), v_cache=vc.cuda())
    gpu, _, gstep = gpu_teacher_forced(dec, tokens, 2, step0=p0)
    ref, _, _, _ = oracle_teacher_forced(WIDE, w_cpu, tokens, 2, _u16(kc), _u16(vc), step0=p0)
    wl, wh = compare_captures(gpu, ref, logits_tol=1e-3, hidden_tol=1e-3)
    print(f"R={R} down {down_grid} gate/up {gu_grid} lm {lm_grid}: worst logits rel-L2 {wl:.2e}, hidden {wh:.2e}")
    assert np.array_equal(gstep.numpy(), p0 + 2)
    dec.kernel.close()


def test_more_than_sixteen_requests_rejected(weights):
    """17 requests exceed the widest contraction: refused at compile time."""
    from persistent_megakernel_decode_02_b200._lib import MpkError

    _, w = weights
    with pytest.raises(MpkError, match="at most 16"):
        _build(SHAPE, w, 17)
