"""Pins of the CPU oracle to facts outside itself.

Each block of the decoder is checked against a closed form, an invariant, a
brute-force exact computation or a library routine; the whole decoder against
special-case models whose output is known by construction and against an
independent restatement through PyTorch's own library routines.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from synth import qwen3


def bf(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def rb_exact(x):
    """Round float64 values to the nearest bf16 (8 significant bits, ties to even)
    in one step, without passing through fp32."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


# ---------------------------------------------------------------- bf16 rounding

def test_round_bf16_ties_to_even_and_library_cast():
    assert oracle.round_bf16(1.0 + 2 ** -8) == 1.0                # halfway -> even (1.0)
    assert oracle.round_bf16(1.0 + 3 * 2 ** -8) == 1.0 + 2 ** -6  # halfway -> even
    assert oracle.round_bf16(1.0 + 2 ** -8 + 2 ** -30) == 1.0 + 2 ** -7
    assert oracle.round_bf16(-0.0) == 0.0
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        [1e-40, -3e-39, 3.3e38]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.round_bf16(float(v)) for v in x])
    assert np.array_equal(ref, got)


# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_unit_rms_closed_form():
    rng = np.random.default_rng(1)
    for n in (7, 64, 4096):
        x = rng.standard_normal(n) * 3.0
        eps = 1e-6
        y = oracle.rmsnorm(x, torch.ones(n, dtype=torch.bfloat16), eps)
        m = np.mean(x * x)
        assert np.mean(y * y) == pytest.approx(m / (m + eps), rel=1e-12)
        # direction unchanged
        assert np.allclose(y / np.linalg.norm(y), x / np.linalg.norm(x), rtol=1e-12)


def test_rmsnorm_weight_scales_elementwise_and_library():
    rng = np.random.default_rng(2)
    x = rng.standard_normal(256)
    w = bf(rng.uniform(0.5, 2.0, 256))
    y = oracle.rmsnorm(x, w, 1e-6)
    y1 = oracle.rmsnorm(x, torch.ones(256, dtype=torch.bfloat16), 1e-6)
    assert np.allclose(y, y1 * w.double().numpy(), rtol=1e-14)
    ref = F.rms_norm(torch.from_numpy(x), (256,), w.double(), eps=1e-6).numpy()
    assert np.allclose(y, ref, rtol=1e-12, atol=0)


def test_rmsnorm_of_zero_is_zero():
    y = oracle.rmsnorm(np.zeros(16), torch.ones(16, dtype=torch.bfloat16), 1e-6)
    assert np.all(y == 0)


# ---------------------------------------------------------------- GEMV

def test_gemv_exact_on_integers_nonsquare():
    rng = np.random.default_rng(3)
    N, K = 37, 91
    Wi = rng.integers(-8, 9, size=(N, K))
    xi = rng.integers(-100, 101, size=K)
    y = oracle.gemv(bf(Wi), xi.astype(np.float64))
    exact = [sum(int(Wi[n, k]) * int(xi[k]) for k in range(K)) for n in range(N)]
    assert np.array_equal(y, np.array(exact, dtype=np.float64))


def test_gemv_row_major_out_in_orientation():
    # W[out, in]: y_n = sum_k W[n, k] x_k; the one-hot input picks column k.
    W = bf(np.arange(12).reshape(3, 4))
    for k in range(4):
        x = np.zeros(4)
        x[k] = 1.0
        assert np.array_equal(oracle.gemv(W, x), np.arange(12).reshape(3, 4)[:, k].astype(float))


# ---------------------------------------------------------------- RoPE

def test_rope_identity_at_zero():
    v = np.random.default_rng(4).standard_normal(64)
    assert np.array_equal(oracle.rope(v, 0, 1e6), v)


def test_rope_d2_is_rotation_by_position():
    for p in (1, 2, 5, 1000):
        out = oracle.rope(np.array([1.0, 0.0]), p, 1e6)
        assert out[0] == pytest.approx(math.cos(p), abs=1e-15)
        assert out[1] == pytest.approx(math.sin(p), abs=1e-15)
        # counter-clockwise: (0,1) -> (-sin, cos)
        out = oracle.rope(np.array([0.0, 1.0]), p, 1e6)
        assert out[0] == pytest.approx(-math.sin(p), abs=1e-15)
        assert out[1] == pytest.approx(math.cos(p), abs=1e-15)


def test_rope_pair_frequencies_and_rotate_half_pairing():
    d, theta, p = 8, 1e6, 7
    for i in range(d // 2):
        v = np.zeros(d)
        v[i] = 1.0
        out = oracle.rope(v, p, theta)
        ang = p * theta ** (-2.0 * i / d)
        exp = np.zeros(d)
        exp[i], exp[i + d // 2] = math.cos(ang), math.sin(ang)
        assert np.allclose(out, exp, atol=1e-15)


def test_rope_norm_and_relative_position():
    rng = np.random.default_rng(5)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    for m, n in ((3, 1), (100, 37), (32000, 31990)):
        a = oracle.rope(q, m, 1e6) @ oracle.rope(k, n, 1e6)
        b = oracle.rope(q, m + 11, 1e6) @ oracle.rope(k, n + 11, 1e6)
        assert a == pytest.approx(b, rel=1e-9, abs=1e-9)
        r = oracle.rope(q, m, 1e6)
        assert np.allclose(r[:64] ** 2 + r[64:] ** 2, q[:64] ** 2 + q[64:] ** 2, rtol=1e-12)


# ---------------------------------------------------------------- SiLU

def test_silu_special_values():
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu(1.0) == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    assert oracle.silu(1.0) == pytest.approx(0.7310585786300049, rel=1e-15)
    assert oracle.silu(-1.0) == pytest.approx(-0.2689414213699951, rel=1e-15)
    assert oracle.silu(60.0) == pytest.approx(60.0, rel=1e-15)
    assert abs(oracle.silu(-60.0)) < 1e-24
    xs = torch.linspace(-20, 20, 401, dtype=torch.float64)
    assert np.allclose([oracle.silu(float(x)) for x in xs], F.silu(xs).numpy(), rtol=1e-14)


# ---------------------------------------------------------------- attention

def test_attention_single_position_returns_value():
    rng = np.random.default_rng(6)
    v = bf(rng.standard_normal((1, 64)))
    o = oracle.attend(rng.standard_normal(64), bf(rng.standard_normal((1, 64))), v)
    assert np.array_equal(o, v.double().numpy()[0])


def test_attention_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(7)
    K = bf(np.tile(rng.standard_normal(64), (9, 1)))
    V = bf(rng.standard_normal((9, 64)))
    o = oracle.attend(rng.standard_normal(64), K, V)
    assert np.allclose(o, V.double().numpy().mean(0), rtol=1e-13, atol=1e-15)


def test_attention_weights_sum_to_one():
    rng = np.random.default_rng(8)
    K = bf(rng.standard_normal((33, 64)) * 4)
    o = oracle.attend(rng.standard_normal(64) * 4, K, bf(np.ones((33, 64))))
    assert np.allclose(o, 1.0, rtol=1e-13)


def test_attention_selects_matching_key_and_scale():
    d = 64
    K = np.zeros((5, d))
    for t in range(5):
        K[t, t] = 1.0
    V = np.arange(5 * d, dtype=float).reshape(5, d) / 64.0
    q = np.zeros(d)
    q[3] = 400.0  # score 400/8 = 50 against 0: weight e^-50 elsewhere
    o = oracle.attend(q, bf(K), bf(V))
    assert np.allclose(o, V[3], rtol=1e-12, atol=1e-18)
    # exact two-position softmax with the 1/sqrt(d) scale
    q = np.zeros(d)
    q[0] = 2.0
    o = oracle.attend(q, bf(K[:2]), bf(np.array([[1.0] * d, [0.0] * d])))
    p0 = math.exp(2.0 / 8.0) / (math.exp(2.0 / 8.0) + 1.0)
    assert o[0] == pytest.approx(p0, rel=1e-14)


def test_attention_matches_library_sdpa():
    rng = np.random.default_rng(9)
    q, K, V = rng.standard_normal(128), bf(rng.standard_normal((50, 128))), bf(rng.standard_normal((50, 128)))
    o = oracle.attend(q, K, V)
    ref = F.scaled_dot_product_attention(torch.from_numpy(q)[None, None, None], K.double()[None, None],
                                         V.double()[None, None])[0, 0, 0].numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- argmax

def test_argmax_lowest_index_on_ties_in_fp32():
    z = np.array([0.5, 2.0, 1.0, 2.0, -3.0])
    assert oracle.argmax_f32(z) == 1
    # 1 + 1e-12 and 1.0 are equal in fp32: a tie -> lowest index
    z = np.array([0.0, 1.0, 1.0 + 1e-12])
    assert oracle.argmax_f32(z) == 1
    z = np.array([-1.0, -0.5, -0.5000001])
    assert oracle.argmax_f32(z) == 1
    z = np.random.default_rng(10).standard_normal(151936)
    assert oracle.argmax_f32(z) == int(torch.argmax(torch.from_numpy(z).float()))


# ---------------------------------------------------------------- special-case decoders

SMALL = qwen3.Qwen3Shape("pin", 2, 32, 4, 2, 16, 48, 96, tied=True)


def _zero(w, names):
    for n in names:
        w[n] = torch.zeros_like(w[n])


def test_decoder_without_blocks_reads_embedding_through_final_norm():
    """Zero o_proj/down_proj: every block adds nothing, the residual stream stays
    the embedding row, and the logits are LM head x bf16(rmsnorm(embedding))."""
    s = qwen3.Qwen3Shape("pin-u", 2, 32, 4, 2, 16, 48, 96, tied=False)
    w = qwen3.make_weights(s, seed=11)
    _zero(w, [f"layers.{l}.{p}" for l in range(2) for p in ("o_proj", "down_proj")])
    dec = oracle.Decoder(s, w)
    tok = np.array([[17, -1]], dtype=np.int64)
    step = np.zeros(1, np.int32)
    kc, vc = dec.new_cache(1, 2)
    lg = np.zeros((1, s.vocab))
    hd = np.zeros((s.layers + 1, 1, s.hidden))
    assert dec.iteration(kc, vc, step, tok, None, oracle.ROUND_BF16, lg, hd) == 1
    e = w["embed_tokens"].double().numpy()[17]
    for l in range(s.layers + 1):
        assert np.array_equal(hd[l, 0], e)
    h = rb_exact(e * (1.0 / math.sqrt(np.mean(e * e) + s.eps)))
    exact = w["lm_head"].double().numpy() @ h
    assert np.allclose(lg[0], exact, rtol=1e-12, atol=1e-14)
    assert tok[0, 1] == int(np.argmax(exact.astype(np.float32))) and step[0] == 1


def test_decoder_greedy_feedback_with_one_hot_tied_embedding():
    """E[t] = e_(t mod H): the final-normed state of token t is sqrt(H)-ish times a
    one-hot, so the tied LM head's argmax is the lowest v = t (mod H), i.e. t mod H.
    Greedy decoding must write t mod H into the next -1 slot, keep pre-filled
    slots, advance step by one per iteration and stop at step_end."""
    s = SMALL
    w = qwen3.make_weights(s, seed=12)
    E = np.zeros((s.vocab, s.hidden), np.float32)
    for t in range(s.vocab):
        E[t, t % s.hidden] = 1.0
    w["embed_tokens"] = bf(E)
    _zero(w, [f"layers.{l}.{p}" for l in range(2) for p in ("o_proj", "down_proj")])
    dec = oracle.Decoder(s, w)
    S = 8
    tokens = np.full((2, S), -1, np.int64)
    tokens[0, 0] = 70          # -> 70 mod 32 = 6, then 6 forever
    tokens[1, :3] = [90, 5, 40]  # prompt of 3: no overwrite of slots 1, 2
    out, step, _, _, _ = dec.generate(tokens, np.zeros(2, np.int32), np.array([5, 6], np.int32))
    assert list(out[0]) == [70, 6, 6, 6, 6, 6, -1, -1]
    assert list(out[1]) == [90, 5, 40, 8, 8, 8, 8, -1]
    assert list(step) == [5, 6]


def test_decoder_uniform_attention_averages_cached_values():
    """Zero q_proj: q = 0, every score is 0 and attention is the plain mean of the
    cached values at positions 0..s (the new one included).  With o_proj = I
    (hidden = q_dim) and zero down_proj, the residual after layer 0 is
    E[t_s] + bf16(mean_t v_t) per head, v_t = bf16(W_v bf16(rmsnorm(E[t_t])))."""
    s = qwen3.Qwen3Shape("pin-a", 1, 64, 4, 2, 16, 48, 96, tied=True)
    w = qwen3.make_weights(s, seed=13)
    _zero(w, ["layers.0.q_proj", "layers.0.down_proj"])
    w["layers.0.o_proj"] = torch.eye(64, dtype=torch.bfloat16)
    dec = oracle.Decoder(s, w)
    S = 6
    toks = np.array([[3, 50, 7, 91, 22, 60]], np.int64)
    kc, vc = dec.new_cache(1, S)
    step = np.zeros(1, np.int32)
    E = w["embed_tokens"].double().numpy()
    Wv = w["layers.0.v_proj"].double().numpy()
    vs = []
    for it in range(S - 1):
        hd = np.zeros((2, 1, 64))
        dec.iteration(kc, vc, step, toks, None, oracle.ROUND_BF16, None, hd)
        e = E[toks[0, it]]
        h = rb_exact(e * (1.0 / math.sqrt(np.mean(e * e) + s.eps)))
        vs.append(rb_exact(Wv @ h))
        mean = np.mean(vs, axis=0)  # [kv_dim]: kv head j occupies [16j, 16j+16)
        # q heads 0,1 read kv head 0; q heads 2,3 read kv head 1 (contiguous groups)
        o = np.concatenate([mean[0:16], mean[0:16], mean[16:32], mean[16:32]])
        o = rb_exact(o)
        assert np.allclose(hd[1, 0], e + o, rtol=1e-12, atol=1e-15), it
    # the cache holds bf16(v) at every written position, in order
    got_v = torch.from_numpy(vc[0, 0].astype(np.int16)).view(torch.bfloat16).double().numpy()
    for t in range(S - 1):
        assert np.array_equal(np.concatenate([got_v[0, t], got_v[1, t]]), vs[t])
    assert np.all(vc[0, 0, :, S - 1] == 0)


def test_decoder_gqa_maps_contiguous_groups():
    """One-hot keys per kv head and values constant j+1 on kv head j: with a sharp
    query every q head h must return the value of kv head floor(h * Hkv / Hq)."""
    d = 16
    rng = np.random.default_rng(14)
    for Hq, Hkv in ((4, 2), (8, 2), (6, 3), (4, 4)):
        S = 3
        K = np.zeros((Hkv, S, d))
        V = np.zeros((Hkv, S, d))
        for j in range(Hkv):
            K[j, :, :] = rng.standard_normal((S, d))
            V[j] = j + 1.0
        for h in range(Hq):
            j = (h * Hkv) // Hq
            o = oracle.attend(rng.standard_normal(d), bf(K[j]), bf(V[j]))
            assert np.allclose(o, j + 1.0)


# ---------------------------------------------------------------- independent restatement

def _torch_reference(shape, w, tokens_row, steps, round_mode=oracle.ROUND_BF16):
    """Teacher-forced logits of the decoder written with PyTorch library routines
    (F.rms_norm, F.linear, F.scaled_dot_product_attention with GQA, F.silu) in
    float64.  The KV cache is bf16 in both modes; with ROUND_BF16 the inputs of
    the projections are rounded to bf16 too, with ROUND_NONE they are not."""
    s = shape
    rkv = lambda t: torch.from_numpy(rb_exact(t.numpy()))
    rb = rkv if round_mode == oracle.ROUND_BF16 else (lambda t: t)
    W = {k: v.double() for k, v in w.items()}
    d = s.head_dim
    inv = 1.0 / (s.rope_theta ** (torch.arange(0, d // 2, dtype=torch.float64) * 2.0 / d))
    Kc = [[] for _ in range(s.layers)]
    Vc = [[] for _ in range(s.layers)]
    out = []
    for pos in range(steps):
        x = W["embed_tokens"][int(tokens_row[pos])]
        ang = pos * inv
        cos, sin = torch.cos(ang), torch.sin(ang)

        def rot(t):
            a, b = t[..., : d // 2], t[..., d // 2:]
            return torch.cat([a * cos - b * sin, b * cos + a * sin], dim=-1)

        for l in range(s.layers):
            p = f"layers.{l}."
            h = rb(F.rms_norm(x, (s.hidden,), W[p + "input_layernorm"], eps=s.eps))
            q = F.linear(h, W[p + "q_proj"]).view(s.q_heads, d)
            k = F.linear(h, W[p + "k_proj"]).view(s.kv_heads, d)
            v = F.linear(h, W[p + "v_proj"]).view(s.kv_heads, d)
            q = rot(F.rms_norm(q, (d,), W[p + "q_norm"], eps=s.eps))
            k = rot(F.rms_norm(k, (d,), W[p + "k_norm"], eps=s.eps))
            Kc[l].append(rkv(k))
            Vc[l].append(rkv(v))
            Ks = torch.stack(Kc[l], dim=1)[None]  # [1, Hkv, T, d]
            Vs = torch.stack(Vc[l], dim=1)[None]
            o = F.scaled_dot_product_attention(q[None, :, None, :], Ks, Vs, enable_gqa=True)
            o = rb(o[0, :, 0, :].reshape(-1))
            x = x + F.linear(o, W[p + "o_proj"])
            h = rb(F.rms_norm(x, (s.hidden,), W[p + "post_attention_layernorm"], eps=s.eps))
            a = rb(F.silu(F.linear(h, W[p + "gate_proj"])) * F.linear(h, W[p + "up_proj"]))
            x = x + F.linear(a, W[p + "down_proj"])
        h = rb(F.rms_norm(x, (s.hidden,), W["norm"], eps=s.eps))
        lm = W["embed_tokens"] if s.tied else W["lm_head"]
        out.append(F.linear(h, lm).numpy())
    return np.stack(out)


@pytest.mark.parametrize("mode", [oracle.ROUND_NONE, oracle.ROUND_BF16], ids=["round-none", "round-bf16"])
@pytest.mark.parametrize("shape", [qwen3.TINY, qwen3.Qwen3Shape("pin-t", 2, 64, 4, 2, 16, 96, 200, tied=True)])
def test_decoder_matches_library_restatement(shape, mode):
    w = qwen3.make_weights(shape, seed=0)
    dec = oracle.Decoder(shape, w)
    S = 10
    toks = qwen3.make_prompts(shape, 1, S, seed=4).numpy().copy()
    kc, vc = dec.new_cache(1, S)
    step = np.zeros(1, np.int32)
    got = []
    for _ in range(S - 1):
        lg = np.zeros((1, shape.vocab))
        dec.iteration(kc, vc, step, toks, None, mode, lg, None)
        got.append(lg[0].copy())
    ref = _torch_reference(shape, w, toks[0], S - 1, mode)
    err = np.linalg.norm(np.stack(got) - ref) / np.linalg.norm(ref)
    assert err < 1e-9, err


@pytest.mark.parametrize("R", [3, 16])
def test_decoder_requests_are_independent(R):
    """Several requests decoded together (different prompt lengths, start and
    end positions, some finishing while the others go on) give, request by
    request, exactly what each gives decoded alone: tokens, final step, cache
    rows and the logits of every iteration it was active.  Pins the oracle's
    per-request bookkeeping (cache and token indexing by request, inactive
    requests left untouched) that the batched GPU parity tests rely on, up to
    the 16 requests of the widest contraction."""
    shape = qwen3.TINY
    w = qwen3.make_weights(shape, seed=0)
    dec = oracle.Decoder(shape, w)
    S = 20
    if R == 3:
        lens, step0, end = [5, 2, 8], np.array([0, 1, 3], np.int32), np.array([12, 6, 17], np.int32)
    else:
        lens = [2 + (5 * r) % 9 for r in range(R)]
        step0 = np.array([min(r % 4, lens[r] - 1) for r in range(R)], np.int32)  # each starts on a prompt token
        end = np.array([8 + (7 * r) % 11 for r in range(R)], np.int32)
    toks = qwen3.make_tokens(shape, R, S, lens, seed=9).numpy().copy()
    bt, bs, bk, bv, bcaps = dec.generate(toks, step0, end, capture=True)
    assert np.array_equal(bs, end)
    for r in range(R):
        t, s, k, v, caps = dec.generate(toks[r:r + 1], step0[r:r + 1], end[r:r + 1], capture=True)
        assert np.array_equal(bt[r], t[0]) and int(bs[r]) == int(s[0])
        assert np.array_equal(bk[:, r], k[:, 0]) and np.array_equal(bv[:, r], v[:, 0])
        n = int(end[r] - step0[r])
        assert len(caps) == n
        for i in range(n):
            assert np.array_equal(bcaps[i][0][r], caps[i][0][0])
            assert np.array_equal(bcaps[i][1][:, r], caps[i][1][:, 0])
        # the cache rows past the request's last position are untouched
        assert not bk[:, r, :, int(end[r]):].any()
