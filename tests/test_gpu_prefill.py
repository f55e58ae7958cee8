"""Prompt ingestion by prefill graphs (mpk_options.prefill_tokens): T
consecutive prompt positions of one request per iteration, as the T columns
of the tensor-core projections, the requests of the cache one after another,
inside the same persistent kernel ("Mirage Persistent Kernel: Fusing
Multi-GPU LLM Inference into One Kernel Launch", "How MPK Works": the
`tokens` meta tensor holds the prompt; the runtime advances `step`).

Each column at position p of request q consumes tokens[q, p], appends its K/V
at p and attends to positions 0..p: the chunk's earlier positions from this
iteration's k and v, the rest from the cache.  Checked against the CPU
oracle, which ingests the prompt one position at a time: greedy tokens after
a prefilled prompt are the oracle's, the per-column logits and residual
streams of a prefill iteration are within the tests' tolerances of the
oracle's per-position ones, the prefilled cache rows agree, and op-by-op
execution is bit-identical to the persistent kernel.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import qwen3 as sq
from tests.gpu_util import HIDDEN_TOL, LOGITS_TOL, rel_l2, to_cuda, u16_to_f64, bf16_u16

pytestmark = pytest.mark.gpu

SHAPE = sq.TINY
PROMPT, GEN = 19, 10
S = PROMPT + GEN + 1


@pytest.fixture(scope="module")
def weights():
    w_cpu = sq.make_weights(SHAPE, seed=0)
    return w_cpu, to_cuda(w_cpu)


def _decoders(w, T, **kw):
    from persistent_megakernel_decode_02_b200 import build_decoder
    dec = build_decoder(SHAPE, w, requests=1, max_seq=S, **kw)
    pre = build_decoder(SHAPE, w, requests=1, max_seq=S, prefill_tokens=T, k_cache=dec.k_cache,
                        v_cache=dec.v_cache, **kw)
    return pre, dec


@pytest.mark.parametrize("T", [2, 5, 8])
def test_prefill_then_greedy_decode_matches_oracle(weights, T):
    """Prompt positions 0..PROMPT-2 by prefill (the last chunk partial), then
    greedy decoding from the last prompt token with the ordinary graph: every
    generated token is the oracle's, and the prefilled cache rows agree with
    the oracle's up to bf16 rounding."""
    w_cpu, w = weights
    tokens = sq.make_tokens(SHAPE, 1, S, [PROMPT], seed=31)
    pre, dec = _decoders(w, T)
    tok = tokens.cuda()
    step = torch.zeros(1, dtype=torch.int32, device="cuda")
    pre.run(step, tok, torch.full((1,), PROMPT - 1, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    pre.kernel.check_status()
    assert int(step.item()) == PROMPT - 1
    assert torch.equal(tok.cpu()[0, :PROMPT], tokens[0, :PROMPT])  # prompt slots kept
    kc_pre = bf16_u16(dec.k_cache).copy()
    end = torch.full((1,), S - 1, dtype=torch.int32, device="cuda")
    dec.run(step, tok, end)
    torch.cuda.synchronize()
    dec.kernel.check_status()
    got = tok.cpu().numpy()

    ref = oracle.Decoder(SHAPE, w_cpu)
    out, st, rkc, _, _ = ref.generate(tokens.numpy(), np.zeros(1, np.int32), np.array([S - 1], np.int32))
    assert int(st[0]) == S - 1 and int(step.item()) == S - 1
    assert np.array_equal(got, out), f"\n gpu    {got.tolist()}\n oracle {out.tolist()}"
    gk = u16_to_f64(kc_pre[:, :, :, :PROMPT - 1])
    rk = u16_to_f64(rkc[:, :, :, :PROMPT - 1])
    assert np.linalg.norm(gk - rk) <= 1e-2 * np.linalg.norm(rk)
    # the prefill's predictions of the prompt positions are the oracle's argmax there
    gp = pre.pred.cpu().numpy()[0]
    ref2 = oracle.Decoder(SHAPE, w_cpu)
    toks2 = tokens.numpy().copy()
    kc2, vc2 = ref2.new_cache(1, S)
    st2 = np.zeros(1, np.int32)
    pred2 = np.full((1, S), -1, np.int64)
    for _ in range(PROMPT - 1):
        ref2.iteration(kc2, vc2, st2, toks2, None, oracle.ROUND_NONE, None, None, pred2)
    assert np.array_equal(gp[1:PROMPT], pred2[0, 1:PROMPT])
    pre.kernel.close()
    dec.kernel.close()


@pytest.mark.parametrize("T", [3, 8])
def test_prefill_teacher_forced_logits_and_hidden(weights, T):
    """Every prefill iteration's per-column logits and residual streams against
    the oracle's per-position values (rel-L2 2e-2 / 1e-2)."""
    w_cpu, w = weights
    tokens = sq.make_tokens(SHAPE, 1, S, [S], seed=32, teacher_forced=True)
    pre, dec = _decoders(w, T)
    tok = tokens.cuda()
    step = torch.zeros(1, dtype=torch.int32, device="cuda")
    n_iter = -(-(S - 1) // T)
    gl, gh = [], []
    for it in range(n_iter):
        lg = torch.full((T, SHAPE.vocab), float("nan"), device="cuda")
        hd = torch.full((SHAPE.layers + 1, T, SHAPE.hidden), float("nan"), device="cuda")
        pre.kernel.set_capture(0, lg, hd)
        pre.run(step, tok, torch.full((1,), min(S - 1, (it + 1) * T), dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        pre.kernel.check_status()
        gl.append(lg.double().cpu().numpy())
        gh.append(hd.double().cpu().numpy())
    assert int(step.item()) == S - 1
    ref = oracle.Decoder(SHAPE, w_cpu)
    toks = tokens.numpy().copy()
    kc, vc = ref.new_cache(1, S)
    st = np.zeros(1, np.int32)
    worst_l = worst_h = 0.0
    for p in range(S - 1):
        lg = np.full((1, SHAPE.vocab), np.nan)
        hd = np.full((SHAPE.layers + 1, 1, SHAPE.hidden), np.nan)
        ref.iteration(kc, vc, st, toks, None, oracle.ROUND_NONE, lg, hd)
        it, col = divmod(p, T)
        e = rel_l2(gl[it][col], lg[0])
        worst_l = max(worst_l, e)
        assert e <= LOGITS_TOL, (p, e)
        for layer in range(SHAPE.layers + 1):
            e = rel_l2(gh[it][layer, col], hd[layer, 0])
            worst_h = max(worst_h, e)
            assert e <= HIDDEN_TOL, (p, layer, e)
    print(f"prefill T={T}: worst logits rel-L2 {worst_l:.2e}, hidden {worst_h:.2e}")
    pre.kernel.close()
    dec.kernel.close()


def test_prefill_op_by_op_bit_identical(weights):
    _, w = weights
    tokens = sq.make_tokens(SHAPE, 1, S, [PROMPT], seed=33)
    outs = []
    for mode in ("run", "run_op_by_op"):
        pre, dec = _decoders(w, 8)
        tok = tokens.cuda()
        step = torch.zeros(1, dtype=torch.int32, device="cuda")
        getattr(pre, mode)(step, tok, torch.full((1,), PROMPT - 1, dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        pre.kernel.check_status()
        outs.append((step.cpu(), tok.cpu(), pre.pred.cpu(), dec.k_cache.cpu().view(torch.int16),
                     dec.v_cache.cpu().view(torch.int16)))
        pre.kernel.close()
        dec.kernel.close()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_prefill_several_requests_then_batched_decode(weights):
    """A prefill graph over a KV cache of four requests ingests their prompts one
    request after another (a one-token prompt has nothing to ingest, an
    inactive request stays untouched), then the batched decode graph on the
    same cache continues all of them: every generated token is the oracle's."""
    w_cpu, w = weights
    from persistent_megakernel_decode_02_b200 import build_decoder
    prompts = [19, 1, 7, 12]
    R, T = len(prompts), 5
    tokens = sq.make_tokens(SHAPE, R, S, prompts, seed=34)
    dec = build_decoder(SHAPE, w, requests=R, max_seq=S)
    pre = build_decoder(SHAPE, w, requests=R, max_seq=S, prefill_tokens=T, k_cache=dec.k_cache,
                        v_cache=dec.v_cache)
    tok = tokens.cuda()
    step = torch.zeros(R, dtype=torch.int32, device="cuda")
    p_end = torch.tensor([p - 1 for p in prompts], dtype=torch.int32, device="cuda")
    pre.run(step, tok, p_end)
    torch.cuda.synchronize()
    pre.kernel.check_status()
    assert step.cpu().tolist() == [p - 1 for p in prompts]
    assert torch.equal(tok.cpu(), tokens)  # every slot the prefill reached holds a prompt token
    dec.run(step, tok, torch.full((R,), S - 1, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    dec.kernel.check_status()
    ref = oracle.Decoder(SHAPE, w_cpu)
    out, st, rkc, _, _ = ref.generate(tokens.numpy(), np.zeros(R, np.int32), np.full(R, S - 1, np.int32))
    assert step.cpu().tolist() == [S - 1] * R and st.tolist() == [S - 1] * R
    got = tok.cpu().numpy()
    assert np.array_equal(got, out), f"\n gpu    {got.tolist()}\n oracle {out.tolist()}"
    gk = u16_to_f64(bf16_u16(dec.k_cache))
    rk = u16_to_f64(rkc)
    assert np.linalg.norm(gk - rk) <= 1e-2 * np.linalg.norm(rk)
    pre.kernel.close()
    dec.kernel.close()


def test_prefill_skips_an_inactive_request(weights):
    """step = -1 marks a request the run leaves alone: its step, tokens and
    cache rows stay as they were while the others are prefilled."""
    _, w = weights
    from persistent_megakernel_decode_02_b200 import build_decoder
    R, T = 3, 4
    tokens = sq.make_tokens(SHAPE, R, S, [PROMPT] * R, seed=35)
    pre = build_decoder(SHAPE, w, requests=R, max_seq=S, prefill_tokens=T)
    tok = tokens.cuda()
    step = torch.tensor([0, -1, 0], dtype=torch.int32, device="cuda")
    pre.run(step, tok, torch.full((R,), PROMPT - 1, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    pre.kernel.check_status()
    assert step.cpu().tolist() == [PROMPT - 1, -1, PROMPT - 1]
    assert torch.equal(tok.cpu(), tokens)
    kc = pre.k_cache.cpu().float()
    assert not bool(kc[:, 1].any()) and bool(kc[:, 0, :, :PROMPT - 1].any()) and bool(kc[:, 2, :, :PROMPT - 1].any())
    assert not bool(kc[:, :, :, PROMPT - 1:].any())  # nothing past the ingested positions
    assert bool((pre.pred.cpu()[1] == -1).all())
    pre.kernel.close()


def test_prefill_several_requests_op_by_op_bit_identical(weights):
    _, w = weights
    from persistent_megakernel_decode_02_b200 import build_decoder
    prompts = [9, 17, 4]
    R = len(prompts)
    tokens = sq.make_tokens(SHAPE, R, S, prompts, seed=36)
    outs = []
    for mode in ("run", "run_op_by_op"):
        pre = build_decoder(SHAPE, w, requests=R, max_seq=S, prefill_tokens=6)
        tok = tokens.cuda()
        step = torch.zeros(R, dtype=torch.int32, device="cuda")
        getattr(pre, mode)(step, tok, torch.tensor([p - 1 for p in prompts], dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        pre.kernel.check_status()
        outs.append((step.cpu(), tok.cpu(), pre.pred.cpu(), pre.k_cache.cpu().view(torch.int16),
                     pre.v_cache.cpu().view(torch.int16)))
        pre.kernel.close()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_prefill_run_needs_every_cached_request(weights):
    """A prefill graph over a cache of three requests takes tokens and step of
    three rows: a run with one is a SHAPE error and the context stays usable."""
    from persistent_megakernel_decode_02_b200 import MpkError, build_decoder
    _, w = weights
    pre = build_decoder(SHAPE, w, requests=3, max_seq=S, prefill_tokens=4)
    tok = sq.make_tokens(SHAPE, 1, S, [PROMPT], seed=37).cuda()
    with pytest.raises(MpkError) as e:
        pre.run(torch.zeros(1, dtype=torch.int32, device="cuda"), tok)
    assert e.value.name == "SHAPE"
    tok3 = sq.make_tokens(SHAPE, 3, S, [PROMPT] * 3, seed=37).cuda()
    step = torch.zeros(3, dtype=torch.int32, device="cuda")
    pre.run(step, tok3, torch.full((3,), 4, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    pre.kernel.check_status()
    assert step.cpu().tolist() == [4, 4, 4]
    pre.kernel.close()
