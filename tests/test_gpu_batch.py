"""GPU parity of the batched decode path: several requests per iteration, every
projection a tensor-core (tcgen05) contraction over the batch.

Expected values come from the CPU oracle only (its plain ROUND_NONE reading).
The batched projections feed each fp32 input to the MMA as a bf16 hi/lo pair,
so they see it to about 16 significant bits; the results stay within the
decode tolerances (logits 2e-2, hidden 1e-2 rel-L2) with a wide margin, and
greedy tokens match exactly.
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


def _build(w, R, **kw):
    from persistent_megakernel_decode_02_b200 import build_decoder
    return build_decoder(SHAPE, w, requests=R, max_seq=kw.pop("max_seq", S), **kw)


def _positions(R, seed):
    """Distinct starting positions per request (the requests of a batch sit at
    different points of their sequences)."""
    return np.array(sq.make_prompt_lengths(R, 0, 20, seed=seed).tolist(), np.int32)


@pytest.mark.parametrize("R", [3, 8])
def test_polled_inputs_and_published_rows_agree(weights, R):
    """The projections' two ways of taking their inputs: rows their writers
    publish in the shared-memory layout (default), or every tagged element
    polled, normalised and split in the prologue (poll_inputs).  Both stay
    within 1e-3 rel-L2 of the oracle in logits and every layer's residual
    stream, and within 1e-3 of each other (the RMS factor scales the products
    instead of the inputs, so they agree to rounding, not bit for bit)."""
    w_cpu, w = weights
    p0 = _positions(R, seed=R + 11)
    P = int(p0.max())
    kc, vc = sq.make_kv_prefill(SHAPE, R, S, P, seed=7)
    tokens = sq.make_tokens(SHAPE, R, S, [S] * R, seed=8, teacher_forced=True)
    iters = 3
    ref, _, _, _ = oracle_teacher_forced(SHAPE, w_cpu, tokens, iters, _u16(kc), _u16(vc), step0=p0)
    caps = []
    for poll in (False, True):
        dec = _build(w, R, k_cache=kc.cuda(), v_cache=vc.cuda(), poll_inputs=poll)
        gpu, gtok, gstep = gpu_teacher_forced(dec, tokens, iters, step0=p0)
        wl, wh = compare_captures(gpu, ref, logits_tol=1e-3, hidden_tol=1e-3)
        print(f"R={R} poll_inputs={poll}: worst logits rel-L2 {wl:.2e}, hidden {wh:.2e}")
        assert np.array_equal(gstep.numpy(), p0 + iters)
        caps.append(gpu)
        del dec
    compare_captures(caps[0], caps[1], logits_tol=1e-3, hidden_tol=1e-3)


@pytest.mark.parametrize("R", [2, 3, 8])
def test_teacher_forced_batch(weights, R):
    """R requests at different positions (KV pre-filled below the largest):
    logits (rel-L2 2e-2) and every layer's residual stream (1e-2) within tolerance,
    and the cache rows each request appends."""
    w_cpu, w = weights
    p0 = _positions(R, seed=R)
    P = int(p0.max())
    kc, vc = sq.make_kv_prefill(SHAPE, R, S, P, seed=5)
    tokens = sq.make_tokens(SHAPE, R, S, [S] * R, seed=6, teacher_forced=True)
    dec = _build(w, R, k_cache=kc.cuda(), v_cache=vc.cuda())
    iters = 3
    gpu, gtok, gstep = gpu_teacher_forced(dec, tokens, iters, step0=p0)
    ref, _, rkc, _ = oracle_teacher_forced(SHAPE, w_cpu, tokens, iters, _u16(kc), _u16(vc), step0=p0)
    wl, wh = compare_captures(gpu, ref)
    print(f"R={R}: worst logits rel-L2 {wl:.2e}, hidden {wh:.2e}")
    # inputs to ~16 bits, fp32 accumulation: far inside the tolerances
    assert wl <= 1e-3 and wh <= 1e-3
    assert np.array_equal(gstep.numpy(), p0 + iters)
    assert torch.equal(gtok, tokens)
    for r in range(R):
        a, b = int(p0[r]), int(p0[r]) + iters
        gk = dec.k_cache[:, r, :, a:b].float().cpu().numpy()
        rk = (rkc[:, r, :, a:b].astype(np.uint32) << 16).view(np.float32)
        assert np.linalg.norm(gk - rk) <= 1e-2 * np.linalg.norm(rk)
        # rows below the request's position are untouched
        assert torch.equal(dec.k_cache[:, r, :, :a].cpu().view(torch.int16), kc[:, r, :, :a].view(torch.int16))
    dec.kernel.close()


def test_greedy_tokens_match_oracle(weights):
    """Free-running greedy decode of 8 requests with prompts of different
    lengths (one launch, prompts ingested as decode iterations): the generated
    tokens equal the oracle's."""
    w_cpu, w = weights
    R = 8
    lens = sq.make_prompt_lengths(R, 2, 12, seed=3)
    tokens = sq.make_tokens(SHAPE, R, S, lens, seed=4)
    dec = _build(w, R)
    tok = tokens.cuda()
    step = torch.zeros(R, dtype=torch.int32, device="cuda")
    end = (lens + 16).to(torch.int32).cuda()
    dec.run(step, tok, end)
    torch.cuda.synchronize()
    dec.kernel.check_status()
    got = tok.cpu()

    ref = oracle.Decoder(SHAPE, w_cpu)
    toks = tokens.numpy().copy()
    kc, vc = ref.new_cache(R, S)
    st = np.zeros(R, np.int32)
    se = (lens + 16).numpy().astype(np.int32)
    while ref.iteration(kc, vc, st, toks, se, oracle.ROUND_NONE, None, None):
        pass
    assert np.array_equal(step.cpu().numpy(), se)
    assert np.array_equal(got.numpy(), toks)
    for r in range(R):
        # generated slots filled, nothing past the request's end
        L = int(lens[r])
        assert (got[r, L:L + 17] >= 0).all() and (got[r, L + 17:] == -1).all()
    dec.kernel.close()


def test_requests_finishing_at_different_steps(weights):
    """Requests whose step_end comes earlier go inactive while the others run
    on: the active ones match the oracle, the finished ones keep their cache
    and tokens untouched past their end."""
    w_cpu, w = weights
    R = 4
    tokens = sq.make_tokens(SHAPE, R, S, [4, 6, 3, 5], seed=8)
    se = np.array([7, 20, 4, 12], np.int32)
    dec = _build(w, R)
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
        assert not dec.k_cache[:, r, :, e:].any()   # never written past the last position it ran
        assert dec.k_cache[:, r, :, :e].abs().sum() > 0
    dec.kernel.close()


def test_op_by_op_is_bit_identical_to_persistent(weights):
    _, w = weights
    R = 8
    tokens = sq.make_tokens(SHAPE, R, S, sq.make_prompt_lengths(R, 2, 10, seed=9), seed=10)
    outs = []
    for mode in ("run", "run_op_by_op"):
        dec = _build(w, R)
        tok = tokens.cuda()
        step = torch.zeros(R, dtype=torch.int32, device="cuda")
        getattr(dec, mode)(step, tok, torch.full((R,), 24, dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        dec.kernel.check_status()
        outs.append((tok.cpu(), dec.pred.cpu(), dec.k_cache.cpu().view(torch.int16)))
        dec.kernel.close()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


@pytest.mark.parametrize("split", [(144, 16), (140, 32), (128, 80)])
def test_worker_scheduler_split_invariance(weights, split):
    """Same task plan (planned for 144 workers), different worker/scheduler
    splits: bit-identical tokens, predictions and caches."""
    _, w = weights
    R = 8
    tokens = sq.make_tokens(SHAPE, R, S, sq.make_prompt_lengths(R, 2, 10, seed=11), seed=12)
    ref = None
    for W, Ls in [(144, 16), split]:
        dec = _build(w, R, num_workers=W, num_local_schedulers=Ls, gemv_tasks=144, attn_chunks=3)
        tok = tokens.cuda()
        step = torch.zeros(R, dtype=torch.int32, device="cuda")
        dec.run(step, tok, torch.full((R,), 30, dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        dec.kernel.check_status()
        out = (tok.cpu(), dec.pred.cpu(), dec.k_cache.cpu().view(torch.int16))
        dec.kernel.close()
        if ref is None:
            ref = out
        else:
            for a, b in zip(ref, out):
                assert torch.equal(a, b)


@pytest.mark.parametrize("plan_workers", [1, 7, 37, 144, 300])
def test_task_plans_agree(weights, plan_workers):
    """Very different task plans (whole row blocks per task, reductions split
    into up to every K block): all within tolerance of the oracle."""
    w_cpu, w = weights
    R = 5
    p0 = _positions(R, seed=13)
    kc, vc = sq.make_kv_prefill(SHAPE, R, S, int(p0.max()), seed=14)
    tokens = sq.make_tokens(SHAPE, R, S, [S] * R, seed=15, teacher_forced=True)
    dec = _build(w, R, k_cache=kc.cuda(), v_cache=vc.cuda(), gemv_tasks=plan_workers)
    gpu, _, _ = gpu_teacher_forced(dec, tokens, 2, step0=p0)
    ref, _, _, _ = oracle_teacher_forced(SHAPE, w_cpu, tokens, 2, _u16(kc), _u16(vc), step0=p0)
    wl, wh = compare_captures(gpu, ref)
    print(f"plan for {plan_workers} workers: worst logits rel-L2 {wl:.2e}, hidden {wh:.2e}")
    assert wl <= 1e-3 and wh <= 1e-3
    dec.kernel.close()


def test_request_permutation_is_exact(weights):
    """Every request is its own column of each contraction and its own
    attention: permuting the requests of a batch permutes every result bit for
    bit (a cross-request indexing slip would not)."""
    _, w = weights
    R = 8
    p0 = _positions(R, seed=16)
    kc, vc = sq.make_kv_prefill(SHAPE, R, S, int(p0.max()), seed=17)
    tokens = sq.make_tokens(SHAPE, R, S, [S] * R, seed=18, teacher_forced=True)
    perm = np.array([5, 2, 7, 0, 3, 6, 1, 4])
    outs = []
    for order in (np.arange(R), perm):
        dec = _build(w, R, k_cache=kc[:, order].contiguous().cuda(), v_cache=vc[:, order].contiguous().cuda())
        gpu, _, _ = gpu_teacher_forced(dec, tokens[order], 2, step0=p0[order])
        outs.append((gpu, dec.k_cache.cpu().view(torch.int16)))
        dec.kernel.close()
    (g0, k0), (g1, k1) = outs
    for (l0, h0), (l1, h1) in zip(g0, g1):
        assert np.array_equal(l0[perm], l1)
        assert np.array_equal(h0[:, perm], h1)
    assert torch.equal(k0[:, perm], k1)


WIDE = sq.Qwen3Shape("tiny-wide", 2, 256, 4, 2, 64, 4096, 1024, tied=False)


@pytest.fixture(scope="module")
def wide_weights():
    w_cpu = sq.make_weights(WIDE, seed=4)
    return w_cpu, to_cuda(w_cpu)


@pytest.mark.parametrize("down_grid,gu_grid,lm_grid", [
    ((1, 1), (1, 1), (1, 1)),    # one task per op: the 4096-long down reduction in 3 passes, 16 gate/up blocks
    ((2, 2), (4, 1), (8, 1)),    # split in two segments of 2048, each in 2 passes
    ((2, 3), (32, 1), (8, 4)),   # three segments of 1365 (single pass), one block per gate/up task
    ((1, 64), (2, 4), (4, 2)),   # every K block its own task (64-way split)
])
def test_reduction_passes_and_splits(wide_weights, monkeypatch, down_grid, gu_grid, lm_grid):
    """Reductions longer than the shared-memory input rows run in passes that
    keep each row block in its own tensor-memory accumulator, alone or combined
    with cross-task splits: all within tight tolerance of the oracle."""
    import persistent_megakernel_decode_02_b200.qwen3 as q3
    from persistent_megakernel_decode_02_b200 import build_decoder

    grids = {(WIDE.hidden, WIDE.intermediate, False): down_grid, (WIDE.intermediate, WIDE.hidden, True): gu_grid,
             (WIDE.vocab, WIDE.hidden, False): lm_grid}
    orig = q3.batched_grid
    monkeypatch.setattr(q3, "batched_grid", lambda rows, K, w, pair=False, **kw: grids.get((rows, K, pair)) or
                        orig(rows, K, w, pair))
    w_cpu, w = wide_weights
    R = 4
    p0 = _positions(R, seed=19)
    kc, vc = sq.make_kv_prefill(WIDE, R, S, int(p0.max()), seed=20)
    tokens = sq.make_tokens(WIDE, R, S, [S] * R, seed=21, teacher_forced=True)
    dec = build_decoder(WIDE, w, requests=R, max_seq=S, k_cache=kc.cuda(), v_cache=vc.cuda())
    gpu, _, gstep = gpu_teacher_forced(dec, tokens, 2, step0=p0)
    ref, _, _, _ = oracle_teacher_forced(WIDE, w_cpu, tokens, 2, _u16(kc), _u16(vc), step0=p0)
    wl, wh = compare_captures(gpu, ref)
    print(f"down {down_grid} gate/up {gu_grid} lm {lm_grid}: worst logits rel-L2 {wl:.2e}, hidden {wh:.2e}")
    assert wl <= 1e-3 and wh <= 1e-3
    assert np.array_equal(gstep.numpy(), p0 + 2)
    dec.kernel.close()


def test_too_many_blocks_for_passes_is_rejected(wide_weights, monkeypatch):
    """A task that needs passes must fit its row blocks in the accumulator
    slots: 32 gate/up blocks of one task over a reduction longer than the
    input rows are refused at compile time."""
    import persistent_megakernel_decode_02_b200.qwen3 as q3
    from persistent_megakernel_decode_02_b200 import build_decoder
    from persistent_megakernel_decode_02_b200._lib import MpkError

    shape = sq.Qwen3Shape("tiny-long", 1, 2048, 4, 2, 64, 4096, 1024, tied=False)
    w = to_cuda(sq.make_weights(shape, seed=5))
    orig = q3.batched_grid
    monkeypatch.setattr(q3, "batched_grid", lambda rows, K, wk, pair=False, **kw: (1, 1) if pair else orig(rows, K, wk, pair))
    with pytest.raises(MpkError, match="at most 16 row blocks"):
        build_decoder(shape, w, requests=2, max_seq=16)


def test_results_do_not_depend_on_the_batch(weights):
    """A request decodes to the same tokens, predictions and cache whether it
    shares its iterations with one other request or with seven of different
    lengths (every step of the path treats a request on its own)."""
    _, w = weights
    lens = [9, 3, 11, 5, 2, 7, 10, 4]
    tokens = sq.make_tokens(SHAPE, 8, S, lens, seed=23)
    outs = []
    for R in (2, 8):
        dec = _build(w, R)
        tok = tokens[:R].cuda()
        step = torch.zeros(R, dtype=torch.int32, device="cuda")
        dec.run(step, tok, torch.full((R,), 30, dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        dec.kernel.check_status()
        outs.append((tok[0].cpu(), dec.pred[0].cpu(), dec.k_cache[:, 0].cpu().view(torch.int16)))
        dec.kernel.close()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


RAGGED = sq.Qwen3Shape("tiny-ragged", 2, 320, 4, 2, 64, 832, 1000, tied=False)


@pytest.mark.parametrize("plan_workers", [3, 144])
def test_ragged_row_blocks(plan_workers):
    """Row counts that are not multiples of 128 (hidden 320, intermediate 832,
    vocabulary 1000): the last row block of a projection reads past the matrix
    (the TMA fills zeros) and its epilogue stops at the last row.  Teacher-forced
    against the oracle and greedy tokens."""
    from persistent_megakernel_decode_02_b200 import build_decoder

    w_cpu = sq.make_weights(RAGGED, seed=6)
    w = to_cuda(w_cpu)
    R = 3
    p0 = _positions(R, seed=24)
    kc, vc = sq.make_kv_prefill(RAGGED, R, S, int(p0.max()), seed=25)
    tokens = sq.make_tokens(RAGGED, R, S, [S] * R, seed=26, teacher_forced=True)
    dec = build_decoder(RAGGED, w, requests=R, max_seq=S, k_cache=kc.cuda(), v_cache=vc.cuda(),
                        gemv_tasks=plan_workers)
    gpu, _, _ = gpu_teacher_forced(dec, tokens, 2, step0=p0)
    ref, _, _, _ = oracle_teacher_forced(RAGGED, w_cpu, tokens, 2, _u16(kc), _u16(vc), step0=p0)
    wl, wh = compare_captures(gpu, ref)
    print(f"ragged, plan for {plan_workers}: worst logits rel-L2 {wl:.2e}, hidden {wh:.2e}")
    assert wl <= 1e-3 and wh <= 1e-3
    dec.kernel.close()

    lens = [5, 9, 3]
    tokens = sq.make_tokens(RAGGED, R, S, lens, seed=27)
    dec = build_decoder(RAGGED, w, requests=R, max_seq=S, gemv_tasks=plan_workers)
    tok = tokens.cuda()
    step = torch.zeros(R, dtype=torch.int32, device="cuda")
    end = torch.tensor([l + 10 for l in lens], dtype=torch.int32, device="cuda")
    dec.run(step, tok, end)
    torch.cuda.synchronize()
    dec.kernel.check_status()
    ref = oracle.Decoder(RAGGED, w_cpu)
    out, _, _, _, _ = ref.generate(tokens.numpy(), np.zeros(R, np.int32), np.array([l + 10 for l in lens], np.int32))
    assert np.array_equal(tok.cpu().numpy(), out)
    dec.kernel.close()
