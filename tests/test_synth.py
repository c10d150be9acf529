"""The seeded input generators: determinism, independence of streams and the
distributions they promise (they hold none of the method's arithmetic)."""
import math

import numpy as np
import torch

from ternary_neural_net_b200 import synth


def test_splitmix64_known_answer():
    """SplitMix64 with state 0: the first outputs of the published generator
    (state += 0x9E3779B97F4A7C15, then the output mix)."""
    z = synth._mix(np.arange(1, 4, dtype=np.uint64) * np.uint64(0x9E3779B97F4A7C15))
    assert [int(v) for v in z] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_deterministic_and_streams_differ():
    a = synth.u64(1, 5, 1000)
    assert np.array_equal(a, synth.u64(1, 5, 1000))
    assert not np.array_equal(a, synth.u64(1, 6, 1000))
    assert not np.array_equal(a, synth.u64(2, 5, 1000))
    assert np.array_equal(synth.u64(1, 5, 10), a[:10])


def test_fair_coin_pad_bits_cleared():
    w = synth.fair_coin_words(1, 1, 50, 1000)
    assert w.shape == (50, 16)
    assert np.all((w[:, 15] >> np.uint64(40)) == 0)
    frac = np.bitwise_count(w[:, :15]).sum() / (50 * 15 * 64)
    assert abs(frac - 0.5) < 0.01


def test_normal_and_uniform_moments():
    z = synth.normal_f32(1, 3, (1 << 18,)).astype(np.float64)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    assert abs(np.abs(z).mean() - math.sqrt(2 / math.pi)) < 0.01
    u = synth.uniform_f32(1, 4, (1 << 16,), 0.5, 1.5)
    assert u.min() >= 0.5 and u.max() <= 1.5 and abs(u.mean() - 1.0) < 0.01


def test_bf16_rounding_matches_torch():
    x = synth.normal_f32(2, 1, (4096,))
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.bf16_bits_from_f32(x), want)
    back = synth.bf16_bits_to_f32(want)
    assert np.array_equal(back, torch.from_numpy(want.view(np.int16)).view(torch.bfloat16).float().numpy())
