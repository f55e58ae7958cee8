"""Paged KV caches (mpk_options.kv_page_size): the caches are pages of
kv_page_size positions shared by all requests, and an int32 page table
"kv_pages" [requests, max_pages] maps each request's logical pages to cache
pages ("Mirage Persistent Kernel: Fusing Multi-GPU LLM Inference into One
Kernel Launch" leaves the KV layout open; paged caches are how serving systems
share one cache between requests of different lengths).

The split-K attention reads a request's positions through its page table and
appends there.  Checked against the oracle, which keeps one contiguous cache
per request: the pages are filled from a contiguous pre-filled cache through a
shuffled page table, the run is teacher-forced or greedy, and the pages are
gathered back for the comparison.  A page index outside the cache ends the run
with a device error and touches nothing."""
import numpy as np
import pytest
import torch

import oracle
from synth import qwen3 as sq
from tests.gpu_util import compare_captures, gpu_teacher_forced, oracle_teacher_forced, to_cuda

pytestmark = pytest.mark.gpu

PAGE = 128


def _u16(t):
    return t.view(torch.int16).numpy().view(np.uint16)


def _scatter(cont, table, num_pages):
    """Contiguous [L, R, Hkv, S, d] -> pages [L, num_pages, Hkv, PAGE, d]."""
    L, R, Hkv, S, d = cont.shape
    pages = torch.zeros((L, num_pages, Hkv, PAGE, d), dtype=cont.dtype)
    for r in range(R):
        for i in range(table.shape[1]):
            lo = i * PAGE
            n = min(PAGE, S - lo)
            if n > 0:
                pages[:, int(table[r, i]), :, :n] = cont[:, r, :, lo:lo + n]
    return pages


def _gather(pages, table, S):
    """Pages [L, P, Hkv, PAGE, d] -> contiguous [L, R, Hkv, S, d]."""
    L, _, Hkv, _, d = pages.shape
    R = table.shape[0]
    cont = torch.zeros((L, R, Hkv, S, d), dtype=pages.dtype)
    for r in range(R):
        for i in range(table.shape[1]):
            lo = i * PAGE
            n = min(PAGE, S - lo)
            if n > 0:
                cont[:, r, :, lo:lo + n] = pages[:, int(table[r, i]), :, :n]
    return cont


def _table(requests, max_pages, num_pages, seed):
    perm = np.random.default_rng(seed).permutation(num_pages)[:requests * max_pages]
    return torch.from_numpy(perm.reshape(requests, max_pages).astype(np.int32))


@pytest.mark.parametrize("shape", [sq.TINY, sq.Qwen3Shape("paged-d128", 2, 256, 8, 2, 128, 512, 512, tied=False)],
                         ids=["d64", "d128"])
def test_paged_cache_teacher_forced_matches_oracle(shape):
    """One request over a pre-filled cache (230 positions, crossing a page
    boundary inside a chunk) whose pages are scattered: per-layer residual
    streams, logits and the appended rows agree with the oracle's contiguous
    cache."""
    from persistent_megakernel_decode_02_b200 import build_decoder
    S = 300
    max_pages = -(-S // PAGE)
    num_pages = 7
    w_cpu = sq.make_weights(shape, seed=3)
    w = to_cuda(w_cpu)
    p0 = np.array([230], np.int32)
    kc, vc = sq.make_kv_prefill(shape, 1, S, int(p0[0]), seed=51)
    table = _table(1, max_pages, num_pages, seed=52)
    tokens = sq.make_tokens(shape, 1, S, [S], seed=53, teacher_forced=True)
    dec = build_decoder(shape, w, requests=1, max_seq=S, kv_page_size=PAGE, kv_pages=table.cuda(),
                        num_pages=num_pages, k_cache=_scatter(kc, table, num_pages).cuda(),
                        v_cache=_scatter(vc, table, num_pages).cuda(), attn_chunks=3)
    gpu, _, gstep = gpu_teacher_forced(dec, tokens, 3, step0=p0)
    ref, _, rkc, rvc = oracle_teacher_forced(shape, w_cpu, tokens, 3, _u16(kc), _u16(vc), step0=p0)
    compare_captures(gpu, ref)
    assert int(gstep[0]) == int(p0[0]) + 3
    gk = _gather(dec.k_cache.cpu(), table, S).float().numpy()[:, :, :, :int(p0[0]) + 3]
    rk = (rkc[:, :, :, :int(p0[0]) + 3].astype(np.uint32) << 16).view(np.float32)
    assert np.linalg.norm(gk - rk) <= 1e-2 * np.linalg.norm(rk)
    dec.kernel.close()


def test_paged_prefill_then_batched_decode_matches_oracle():
    """Three requests sharing a cache of shuffled pages: the prefill graph
    ingests their prompts, the batched decode graph continues them; every
    generated token is the oracle's."""
    from persistent_megakernel_decode_02_b200 import build_decoder
    shape = sq.TINY
    w_cpu = sq.make_weights(shape, seed=0)
    w = to_cuda(w_cpu)
    prompts = [150, 9, 131]
    R, S = len(prompts), 180
    max_pages = -(-S // PAGE)
    num_pages = R * max_pages + 3
    table = _table(R, max_pages, num_pages, seed=54).cuda()
    tokens = sq.make_tokens(shape, R, S, prompts, seed=55)
    kv = (shape.layers, num_pages, shape.kv_heads, PAGE, shape.head_dim)
    kc = torch.zeros(kv, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros(kv, dtype=torch.bfloat16, device="cuda")
    dec = build_decoder(shape, w, requests=R, max_seq=S, kv_page_size=PAGE, kv_pages=table, num_pages=num_pages,
                        k_cache=kc, v_cache=vc)
    pre = build_decoder(shape, w, requests=R, max_seq=S, prefill_tokens=6, kv_page_size=PAGE, kv_pages=table,
                        num_pages=num_pages, k_cache=kc, v_cache=vc)
    tok = tokens.cuda()
    step = torch.zeros(R, dtype=torch.int32, device="cuda")
    pre.run(step, tok, torch.tensor([p - 1 for p in prompts], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    pre.kernel.check_status()
    dec.run(step, tok, torch.full((R,), S - 1, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    dec.kernel.check_status()
    ref = oracle.Decoder(shape, w_cpu)
    out, st, rkc, _, _ = ref.generate(tokens.numpy(), np.zeros(R, np.int32), np.full(R, S - 1, np.int32))
    got = tok.cpu().numpy()
    assert np.array_equal(got, out), f"\n gpu    {got.tolist()}\n oracle {out.tolist()}"
    gk = _gather(kc.cpu(), table.cpu(), S).float().numpy()[:, :, :, :S - 1]
    rk = (rkc[:, :, :, :S - 1].astype(np.uint32) << 16).view(np.float32)
    assert np.linalg.norm(gk - rk) <= 1e-2 * np.linalg.norm(rk)
    pre.kernel.close()
    dec.kernel.close()


def test_paged_cache_bad_page_index_is_a_device_error():
    """A page table entry outside the cache ends the run with MPK_ERR_DEVICE
    before anything is read or written there; the pages stay as they were and
    the context runs again once the table is fixed."""
    from persistent_megakernel_decode_02_b200 import MpkError, build_decoder
    shape = sq.TINY
    w = to_cuda(sq.make_weights(shape, seed=0))
    S, num_pages = 200, 4
    table = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    kv = (shape.layers, num_pages, shape.kv_heads, PAGE, shape.head_dim)
    kc = torch.zeros(kv, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros(kv, dtype=torch.bfloat16, device="cuda")
    dec = build_decoder(shape, w, requests=1, max_seq=S, kv_page_size=PAGE, kv_pages=table, num_pages=num_pages,
                        k_cache=kc, v_cache=vc)
    tok = sq.make_tokens(shape, 1, S, [S], seed=56, teacher_forced=True).cuda()
    table[0, 1] = num_pages  # positions 128.. map to a page the cache does not have
    step = torch.full((1,), 140, dtype=torch.int32, device="cuda")
    dec.run(step, tok, step + 2)
    torch.cuda.synchronize()
    with pytest.raises(MpkError) as e:
        dec.kernel.check_status()
    assert e.value.name == "DEVICE" and "KV page" in str(e.value)
    assert int(step.item()) == 140
    assert not bool(kc[:, 2:].any()) and not bool(vc[:, 2:].any())
    table[0, 1] = 2
    dec.run(step, tok, step + 2)
    torch.cuda.synchronize()
    dec.kernel.check_status()
    assert int(step.item()) == 142 and bool(kc[:, 2, :, 140 - PAGE:142 - PAGE].any())
    dec.kernel.close()


def test_paged_cache_options_are_checked():
    from persistent_megakernel_decode_02_b200 import MpkError, build_decoder
    shape = sq.TINY
    w = to_cuda(sq.make_weights(shape, seed=0))
    with pytest.raises(MpkError) as e:
        build_decoder(shape, w, requests=1, max_seq=200, kv_page_size=96)
    assert e.value.name == "INVALID_ARG"
    with pytest.raises(ValueError):
        build_decoder(shape, w, requests=1, max_seq=200, kv_page_size=PAGE, fused_attention=True)
