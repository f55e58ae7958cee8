"""The seeded input generator: reproducible, distribution as stated, shapes right."""
import numpy as np
import torch

import synth
from synth import qwen3


def test_reproducible_and_stream_independent():
    a = synth.normal_bf16((1000,), 0, "w", 0.02)
    b = synth.normal_bf16((1000,), 0, "w", 0.02)
    c = synth.normal_bf16((1000,), 0, "w2", 0.02)
    d = synth.normal_bf16((1000,), 1, "w", 0.02)
    assert torch.equal(a, b)
    assert not torch.equal(a, c) and not torch.equal(a, d)
    # a prefix of a longer draw is the shorter draw (counter-based)
    e = synth.normal_bf16((4000,), 0, "w", 0.02)
    assert torch.equal(e[:1000], a)


def test_normal_moments():
    x = synth.normal_f64(2_000_000, 3, "moments")
    assert abs(x.mean()) < 3e-3
    assert abs(x.std() - 1.0) < 3e-3
    # Irwin-Hall(8): excess kurtosis -6/(5*8) = -0.15
    k = ((x - x.mean()) ** 4).mean() / x.var() ** 2 - 3.0
    assert abs(k + 0.15) < 0.02


def test_bf16_is_rounded_f64_draw():
    x = synth.normal_f64(10000, 5, "t", std=0.02)
    b = synth.normal_bf16((10000,), 5, "t", 0.02)
    ref = torch.from_numpy(x).to(torch.float32).to(torch.bfloat16)
    assert torch.equal(ref, b)


def test_uniform_ids_range():
    ids = synth.uniform_ids(100000, 0, "ids", 0, 1023)
    assert int(ids.min()) == 0 and int(ids.max()) == 1023
    counts = torch.bincount(ids, minlength=1024).double()
    assert (counts.std() / counts.mean()) < 0.13  # Poisson: about 1/sqrt(97.7) = 0.101
    lens = qwen3.make_prompt_lengths(8, 32, 512)
    assert int(lens.min()) >= 32 and int(lens.max()) <= 512


def test_shapes_and_bytes():
    s = qwen3.QWEN3_8B
    # 8B-shaped weights: about 16 GB of bf16 (MPK blog excerpt, Figure 1: "16 GB of weights")
    assert 15.5e9 < s.weight_bytes() < 16.5e9
    # every weight but the embedding table, norms included, plus one embedding row
    assert s.streamed_weight_bytes() == 15_136_819_200
    assert qwen3.QWEN3_0_6B.streamed_weight_bytes() == 1_192_101_888  # tied: table read once + one row
    assert s.kv_bytes_per_position() == 147_456
    w = qwen3.make_weights(qwen3.TINY)
    assert set(w) == set(qwen3.TINY.weight_shapes())
    assert all(w[n].dtype == torch.bfloat16 for n in w)
    assert torch.all(w["norm"] == 1)
    assert abs(float(w["embed_tokens"].float().std()) - 0.02) < 1e-3
