"""The split-K attention operation on the tensor cores for every supported
query-heads-per-kv-head count G and head dim d ("Mirage Persistent Kernel:
Fusing Multi-GPU LLM Inference into One Kernel Launch", "How MPK Works": the
attention of a decode step over the request's KV cache; grouped-query
attention as in the Qwen3 configurations the pages benchmark).

Each case is a small two-layer decoder over a pre-filled cache whose length is
no multiple of the 16-position tiles or of a stage (64 positions at d = 128,
128 at d = 64), split into chunks of ragged sizes, teacher-forced against the
oracle: per-layer residual streams and logits within the tests' tolerances,
and the appended cache rows.  One request (the long-context graph) and three
(the tensor-core projection graph)."""
import numpy as np
import pytest
import torch

from synth import qwen3 as sq
from tests.gpu_util import compare_captures, gpu_teacher_forced, oracle_teacher_forced, to_cuda

pytestmark = pytest.mark.gpu


def _u16(t):
    return t.view(torch.int16).numpy().view(np.uint16)


CASES = [(1, 64), (2, 64), (4, 64), (1, 128), (2, 128), (4, 128)]


@pytest.mark.parametrize("requests", [1, 3])
@pytest.mark.parametrize("G,D", CASES, ids=[f"G{g}-d{d}" for g, d in CASES])
def test_split_attention_heads_and_dims(G, D, requests):
    from persistent_megakernel_decode_02_b200 import build_decoder
    kv = max(2, 256 // (G * D))  # the projections' reductions are multiples of 256
    shape = sq.Qwen3Shape(f"attn-g{G}-d{D}", 2, 256, G * kv, kv, D, 512, 512, tied=False)
    P = 301  # cached positions of request 0 before the first step
    S = 420
    w_cpu = sq.make_weights(shape, seed=40 + G + D)
    w = to_cuda(w_cpu)
    p0 = np.array([P + 17 * r for r in range(requests)], np.int32)
    kc, vc = sq.make_kv_prefill(shape, requests, S, int(p0.max()), seed=41)
    tokens = sq.make_tokens(shape, requests, S, [S] * requests, seed=42, teacher_forced=True)
    dec = build_decoder(shape, w, requests=requests, max_seq=S, k_cache=kc.cuda(), v_cache=vc.cuda(),
                        attn_chunks=3, fused_attention=False)
    gpu, gtok, gstep = gpu_teacher_forced(dec, tokens, 3, step0=p0)
    ref, _, rkc, _ = oracle_teacher_forced(shape, w_cpu, tokens, 3, _u16(kc), _u16(vc), step0=p0)
    wl, wh = compare_captures(gpu, ref)
    print(f"G={G} d={D} requests={requests}: worst logits rel-L2 {wl:.2e}, hidden {wh:.2e}")
    assert np.array_equal(gstep.numpy(), p0 + 3)
    for r in range(requests):
        a = int(p0[r])
        gk = dec.k_cache[:, r, :, a:a + 3].float().cpu().numpy()
        rk = (rkc[:, r, :, a:a + 3].astype(np.uint32) << 16).view(np.float32)
        assert np.linalg.norm(gk - rk) <= 1e-2 * np.linalg.norm(rk)
    dec.kernel.close()


def test_split_attention_short_contexts():
    """From position 0: chunks with no cached position at all, a single
    position, and the first tiles that are mostly past the valid count."""
    from persistent_megakernel_decode_02_b200 import build_decoder
    shape = sq.TINY
    S = 40
    w_cpu = sq.make_weights(shape, seed=0)
    w = to_cuda(w_cpu)
    tokens = sq.make_tokens(shape, 1, S, [S], seed=43, teacher_forced=True)
    dec = build_decoder(shape, w, requests=1, max_seq=S, attn_chunks=5, fused_attention=False)
    gpu, _, _ = gpu_teacher_forced(dec, tokens, 20)
    ref, _, _, _ = oracle_teacher_forced(shape, w_cpu, tokens, 20)
    compare_captures(gpu, ref)
    dec.kernel.close()


def test_split_attention_more_chunks_than_workers():
    """More chunk tasks than workers (several per worker, each streamed through
    the ring after the previous one): the chunk partials are merged in chunk
    order whoever computed them, so the result is bit-identical to op-by-op
    execution (one block per task) and matches the oracle."""
    from persistent_megakernel_decode_02_b200 import build_decoder
    shape = sq.TINY
    S = 300
    w_cpu = sq.make_weights(shape, seed=0)
    w = to_cuda(w_cpu)
    p0 = np.array([230], np.int32)
    kc, vc = sq.make_kv_prefill(shape, 1, S, int(p0.max()), seed=44)
    tokens = sq.make_tokens(shape, 1, S, [S], seed=45, teacher_forced=True)
    outs = []
    for mode in ("run", "run_op_by_op"):
        dec = build_decoder(shape, w, requests=1, max_seq=S, k_cache=kc.cuda(), v_cache=vc.cuda(),
                            attn_chunks=100, fused_attention=False)
        assert dec.kernel.num_workers < 100 * shape.kv_heads
        tok = tokens.cuda()
        step = torch.from_numpy(p0.copy()).cuda()
        getattr(dec, mode)(step, tok, step + 4)
        torch.cuda.synchronize()
        dec.kernel.check_status()
        outs.append((step.cpu(), dec.pred.cpu(), dec.k_cache.cpu().view(torch.int16)))
        dec.kernel.close()
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    dec = build_decoder(shape, w, requests=1, max_seq=S, k_cache=kc.cuda(), v_cache=vc.cuda(), attn_chunks=100,
                        fused_attention=False)
    gpu, _, _ = gpu_teacher_forced(dec, tokens, 3, step0=p0)
    ref, _, _, _ = oracle_teacher_forced(shape, w_cpu, tokens, 3, _u16(kc), _u16(vc), step0=p0)
    compare_captures(gpu, ref)
    dec.kernel.close()
