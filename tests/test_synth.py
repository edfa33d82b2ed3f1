"""The synthetic-input recipe every parity test and the benchmark draw from:
seeded, deterministic, and distributed as stated (uniform codes, scales in
[0.5, 1.5] * 2^-8, biases centred at -128 * scale, N(0, 1) activations),
with every BF16 value the RNE rounding of its draw."""
from __future__ import annotations

import numpy as np

import synth


def test_same_seed_same_problem_different_seed_different_problem():
    a = synth.decode_pair(7, 64, 256, 64)
    b = synth.decode_pair(7, 64, 256, 64)
    c = synth.decode_pair(8, 64, 256, 64)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    assert not np.array_equal(a[0], c[0])


def test_weight_distribution():
    g = synth.rng(3)
    packed, scales, biases = synth.weight(g, 512, 1024, 64)
    q = packed.view(np.uint8)                      # little-endian bytes of the words
    assert q.min() == 0 and q.max() == 255 and abs(q.mean() - 127.5) < 1.0
    s = synth.bf16_bits_to_f32(scales).astype(np.float64)
    assert s.min() >= 0.5 * 2 ** -8 * (1 - 2 ** -8) and s.max() <= 1.5 * 2 ** -8 * (1 + 2 ** -8)
    b = synth.bf16_bits_to_f32(biases).astype(np.float64)
    noise = (b + 128 * s) / 2 ** -10               # bias = -128 s + N(0,1) 2^-10, before BF16 rounding
    assert abs(noise.mean()) < 0.2 and 0.5 < noise.std() < 2.0


def test_bf16_conversion_is_round_to_nearest_even():
    # 1 + 2^-8 is halfway between BF16 1 and 1 + 2^-7: ties go to the even 1
    v = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 1 + 2 ** -8 + 2 ** -20], np.float32)
    assert synth.to_bf16_bits(v).tolist() == [0x3F80, 0x3F82, 0xBF80, 0x3F81]
    x = synth.activations(synth.rng(4), 4096)
    f = synth.bf16_bits_to_f32(x)
    assert np.array_equal(synth.to_bf16_bits(f), x)   # activations are exactly BF16
    assert abs(f.mean()) < 0.1 and 0.9 < f.std() < 1.1
