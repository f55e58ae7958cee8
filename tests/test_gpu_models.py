"""GPU parity at the model sizes of the measured workloads (Qwen3-0.6B and
Qwen3-8B shapes), in the launch configuration the benchmark uses (all SMs but
four worker SMs' worth of scheduler warps, default task splits and attention
mode for the sequence length).

The oracle cannot afford hundreds of full-size iterations, so these tests
sample: the KV cache is pre-filled with seeded N(0,1) bf16 keys/values for
positions [0, P) (the same input on both sides), and a few teacher-forced
iterations from step P are compared — logits within rel-L2 2e-2 and every
layer's residual stream within 1e-2.  P sits at the end of the 39 + 512 token
workload, and at 32768 for the long-context workload (split-K attention).
"""
import numpy as np
import pytest
import torch

from synth import qwen3 as sq
from tests.gpu_util import compare_captures, gpu_teacher_forced, oracle_teacher_forced, to_cuda

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

PROMPT, GENERATED = 39, 512


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def _check(shape, w_cpu, w, P, S, iters, **build_kw):
    from persistent_megakernel_decode_02_b200 import build_decoder

    kc, vc = sq.make_kv_prefill(shape, 1, S, P, seed=11)
    tokens = sq.make_tokens(shape, 1, S, [S], seed=12, teacher_forced=True)
    dec = build_decoder(shape, w, requests=1, max_seq=S, k_cache=kc.cuda(), v_cache=vc.cuda(), **build_kw)
    gpu, gtok, gstep = gpu_teacher_forced(dec, tokens, iters, step0=P)
    ref, _, rkc, _ = oracle_teacher_forced(shape, w_cpu, tokens, iters, _u16(kc), _u16(vc), step0=P)
    wl, wh = compare_captures(gpu, ref)
    print(f"{shape.name} P={P}: worst logits rel-L2 {wl:.2e}, hidden {wh:.2e}")
    assert int(gstep[0]) == P + iters
    assert torch.equal(gtok, tokens)
    # the K cache rows this run wrote are the oracle's up to bf16 rounding flips
    gk = dec.k_cache[:, :, :, P:P + iters].float().cpu().numpy()
    rk = (rkc[:, :, :, P:P + iters].astype(np.uint32) << 16).view(np.float32)
    assert np.linalg.norm(gk - rk) <= 1e-2 * np.linalg.norm(rk)
    # the pre-filled rows are untouched
    assert torch.equal(dec.k_cache[:, :, :, :P].cpu().view(torch.int16), kc[:, :, :, :P].view(torch.int16))
    dec.kernel.close()


@pytest.fixture(scope="module")
def qwen3_0_6b():
    w_cpu = sq.make_weights(sq.QWEN3_0_6B, seed=0)
    return w_cpu, to_cuda(w_cpu)


@pytest.fixture(scope="module")
def qwen3_8b():
    w_cpu = sq.make_weights(sq.QWEN3_8B, seed=0)
    yield w_cpu, to_cuda(w_cpu)
    torch.cuda.empty_cache()


def test_qwen3_0_6b_from_scratch(qwen3_0_6b):
    """0.6B shape (tied embeddings): iterations from an empty cache."""
    w_cpu, w = qwen3_0_6b
    _check(sq.QWEN3_0_6B, w_cpu, w, 0, PROMPT + GENERATED, 4)


def test_qwen3_0_6b_end_of_workload(qwen3_0_6b):
    w_cpu, w = qwen3_0_6b
    S = PROMPT + GENERATED
    _check(sq.QWEN3_0_6B, w_cpu, w, S - 4, S, 3)


def test_qwen3_0_6b_op_by_op_bit_identical(qwen3_0_6b):
    from persistent_megakernel_decode_02_b200 import build_decoder

    _, w = qwen3_0_6b
    shape, S = sq.QWEN3_0_6B, 16
    tokens = sq.make_tokens(shape, 1, S, [8], seed=13)
    outs = []
    for mode in ("run", "run_op_by_op"):
        dec = build_decoder(shape, w, requests=1, max_seq=S)
        tok = tokens.cuda()
        step = torch.zeros(1, dtype=torch.int32, device="cuda")
        getattr(dec, mode)(step, tok)
        torch.cuda.synchronize()
        dec.kernel.check_status()
        outs.append((tok.cpu(), dec.pred.cpu(), dec.k_cache.cpu().view(torch.int16)))
        dec.kernel.close()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_qwen3_8b_end_of_workload(qwen3_8b):
    """The benchmarked workload: 8B shape, 551 positions, fused attention."""
    w_cpu, w = qwen3_8b
    S = PROMPT + GENERATED
    _check(sq.QWEN3_8B, w_cpu, w, S - 3, S, 2)


def test_qwen3_8b_long_context(qwen3_8b):
    """32768 pre-filled positions: the split-K attention path at full size."""
    w_cpu, w = qwen3_8b
    P = 32768
    _check(sq.QWEN3_8B, w_cpu, w, P, P + 128, 2)


def test_qwen3_8b_batch8(qwen3_8b):
    """The batched workload's shape: 8 requests (prompt lengths U[32,512]) half
    way through their 256 generated tokens, each at its own position: tensor-core
    projections over the batch, split-K attention per request.  Compared with
    the plain (unrounded) reading of the oracle."""
    from persistent_megakernel_decode_02_b200 import build_decoder

    w_cpu, w = qwen3_8b
    shape, R, S = sq.QWEN3_8B, 8, 1024
    lens = sq.make_prompt_lengths(R, 32, 512, seed=0)
    p0 = (lens - 1 + 128).numpy().astype(np.int32)
    kc, vc = sq.make_kv_prefill(shape, R, S, int(p0.max()), seed=21)
    tokens = sq.make_tokens(shape, R, S, [S] * R, seed=22, teacher_forced=True)
    dec = build_decoder(shape, w, requests=R, max_seq=S, k_cache=kc.cuda(), v_cache=vc.cuda())
    gpu, gtok, gstep = gpu_teacher_forced(dec, tokens, 2, step0=p0)
    ref, _, rkc, _ = oracle_teacher_forced(shape, w_cpu, tokens, 2, _u16(kc), _u16(vc), step0=p0)
    wl, wh = compare_captures(gpu, ref)
    print(f"{shape.name} x{R}: worst logits rel-L2 {wl:.2e}, hidden {wh:.2e}")
    assert np.array_equal(gstep.numpy(), p0 + 2)
    assert torch.equal(gtok, tokens)
    for r in range(R):
        a = int(p0[r])
        gk = dec.k_cache[:, r, :, a:a + 2].float().cpu().numpy()
        rk = (rkc[:, r, :, a:a + 2].astype(np.uint32) << 16).view(np.float32)
        assert np.linalg.norm(gk - rk) <= 1e-2 * np.linalg.norm(rk)
    dec.kernel.close()


def test_fused_attention_near_its_ceiling():
    """The fused projections + attention operation at the top of its range
    (4096 cached positions): an 8B-width, two-layer model over 4090 pre-filled
    positions, so each kv head's eight chunks hold about 512 positions and the
    attention loops run many rounds of loads.  Teacher-forced against the
    oracle at positions 4090 and 4091."""
    import dataclasses
    from persistent_megakernel_decode_02_b200.qwen3 import FUSED_ATTENTION_MAX_SEQ

    shape = dataclasses.replace(sq.QWEN3_8B, name="qwen3-8b-width-L2-V8192", layers=2, vocab=8192)
    w_cpu = sq.make_weights(shape, seed=0)
    w = to_cuda(w_cpu)
    S = FUSED_ATTENTION_MAX_SEQ
    _check(shape, w_cpu, w, S - 6, S, 2, fused_attention=True)


def _check_prefill(shape, w_cpu, w, P, T):
    """One prefill iteration of T columns (positions P..P+T-1) over a seeded
    pre-filled cache, per column against the oracle's per-position values."""
    from persistent_megakernel_decode_02_b200 import build_decoder
    from tests.gpu_util import HIDDEN_TOL, LOGITS_TOL, rel_l2

    S = P + T + 1
    kc, vc = sq.make_kv_prefill(shape, 1, S, P, seed=41)
    tokens = sq.make_tokens(shape, 1, S, [S], seed=42, teacher_forced=True)
    pre = build_decoder(shape, w, requests=1, max_seq=S, prefill_tokens=T, k_cache=kc.cuda(), v_cache=vc.cuda())
    lg = torch.full((T, shape.vocab), float("nan"), device="cuda")
    hd = torch.full((shape.layers + 1, T, shape.hidden), float("nan"), device="cuda")
    pre.kernel.set_capture(0, lg, hd)
    step = torch.full((1,), P, dtype=torch.int32, device="cuda")
    pre.run(step, tokens.cuda(), torch.full((1,), P + T, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    pre.kernel.check_status()
    assert int(step.item()) == P + T
    ref, _, rkc, _ = oracle_teacher_forced(shape, w_cpu, tokens, T, _u16(kc), _u16(vc), step0=P)
    gl, gh = lg.double().cpu().numpy(), hd.double().cpu().numpy()
    wl = wh = 0.0
    for c in range(T):
        rl, rh = ref[c]
        e = rel_l2(gl[c], rl[0])
        wl = max(wl, e)
        assert e <= LOGITS_TOL, (c, e)
        for layer in range(shape.layers + 1):
            e = rel_l2(gh[layer, c], rh[layer, 0])
            wh = max(wh, e)
            assert e <= HIDDEN_TOL, (c, layer, e)
    gk = pre.k_cache[:, :, :, P:P + T].float().cpu().numpy()
    rk = (rkc[:, :, :, P:P + T].astype(np.uint32) << 16).view(np.float32)
    assert np.linalg.norm(gk - rk) <= 1e-2 * np.linalg.norm(rk)
    print(f"{shape.name} prefill T={T} at {P}: worst logits rel-L2 {wl:.2e}, hidden {wh:.2e}")
    pre.kernel.close()


def test_qwen3_0_6b_prefill(qwen3_0_6b):
    w_cpu, w = qwen3_0_6b
    _check_prefill(sq.QWEN3_0_6B, w_cpu, w, 31, 8)


def test_qwen3_8b_prefill(qwen3_8b):
    w_cpu, w = qwen3_8b
    _check_prefill(sq.QWEN3_8B, w_cpu, w, 24, 8)
