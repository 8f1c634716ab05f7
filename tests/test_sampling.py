"""Pins of the oracle's temperature sampler (oracle/sampling.py), CPU only.

The generator is pinned by values derived by hand from its published round function and key
schedule, and by statistics of its output; the sampler by the distribution it must draw
from (softmax(logits / T), a chi-square test over many positions) and its limits."""

import numpy as np
import pytest

from oracle import sampling as S


def _one(counter, key, rounds):
    out = S.philox4x32(tuple(np.array([c], np.uint32) for c in counter), key, rounds)
    return tuple(int(x[0]) for x in out)


def test_one_round_places_the_products_as_defined():
    # (c0, c1, c2, c3) -> (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0))
    assert _one((1, 0, 0, 0), (0, 0), 1) == (0, 0, 0, 0xD2511F53)
    assert _one((0, 0, 1, 0), (5, 7), 1) == (5, 0xCD9E8D57, 7, 0)
    assert _one((0, 9, 0, 3), (5, 7), 1) == (9 ^ 5, 0, 3 ^ 7, 0)
    # a product with a high half: 0xFFFFFFFF * M0 = (M0 - 1) << 32 | (2^32 - M0)
    assert _one((0xFFFFFFFF, 0, 0, 0), (0, 0), 1) == (0, 0, 0xD2511F53 - 1, (1 << 32) - 0xD2511F53)


def test_key_is_bumped_between_rounds():
    # zero counter and key: the first Philox round leaves zeros, the second sees the key bumped once
    assert _one((0, 0, 0, 0), (0, 0), 1) == (0, 0, 0, 0)
    assert _one((0, 0, 0, 0), (0, 0), 2) == (0x9E3779B9, 0, 0xBB67AE85, 0)


def test_uniforms_are_in_the_open_interval_and_uniform():
    u = S.uniforms(seed=12345, pos=77, n=1 << 16)
    assert u.dtype == np.float32
    assert np.all(u > 0) and np.all(u < 1)
    # every u sits on the lattice (k + 1/2) / 2^23, k an integer in [0, 2^23): exact in fp32,
    # never 0 or 1, so -log(-log(u)) is always finite
    k = u.astype(np.float64) * 2.0 ** 23 - 0.5
    assert np.all(k == np.round(k)) and k.min() >= 0 and k.max() < 2 ** 23
    top = S.uniforms(seed=0, pos=0, n=1)  # the largest word maps strictly below 1
    w = np.array([0xFFFFFFFF], np.uint32)
    assert ((w >> np.uint32(9)).astype(np.float32) + np.float32(0.5)) * np.float32(2.0 ** -23) < 1
    assert top.dtype == np.float32
    assert abs(float(u.mean()) - 0.5) < 0.005
    counts = np.bincount(np.minimum((u * 64).astype(np.int64), 63), minlength=64)
    expect = u.size / 64
    chi2 = float(((counts - expect) ** 2 / expect).sum())
    assert chi2 < 120, chi2  # 63 degrees of freedom: p < 1e-5 beyond this


def test_output_bits_are_balanced_and_streams_differ():
    i = np.arange(4096, dtype=np.uint32)
    z = np.zeros_like(i)
    out = np.stack(S.philox4x32((i, z, z, z), (1, 2)), axis=1).reshape(-1)
    bits = np.unpackbits(out.view(np.uint8))
    assert abs(float(bits.mean()) - 0.5) < 0.01
    assert len(np.unique(out)) == out.size  # no repeat among 16384 words
    a = S.uniforms(seed=1, pos=5, n=4096)
    b = S.uniforms(seed=2, pos=5, n=4096)
    c = S.uniforms(seed=1, pos=6, n=4096)
    assert not np.array_equal(a, b) and not np.array_equal(a, c)


@pytest.mark.parametrize("temperature", [0.7, 1.5])
def test_gumbel_max_draws_from_the_tempered_softmax(temperature):
    logits = np.array([1.0, 0.5, 0.0, -1.0, 2.0], np.float32)
    n = 20000
    draws = np.array([S.sample(logits, pos, temperature, seed=99) for pos in range(n)])
    p = np.exp(logits / temperature - np.max(logits / temperature))
    p /= p.sum()
    counts = np.bincount(draws, minlength=logits.size)
    chi2 = float(((counts - n * p) ** 2 / (n * p)).sum())
    assert chi2 < 25, (counts, n * p)  # 4 degrees of freedom: p < 1e-4 beyond this


def test_zero_temperature_is_greedy_and_ties_go_low():
    y = np.array([0.1, 3.0, -2.0, 3.0], np.float32)
    assert S.sample(y, 10, 0.0, seed=5) == 1
    # a very low temperature makes the noise negligible against a clear gap
    y2 = np.array([0.0, 1.0, 5.0, 2.0], np.float32)
    assert all(S.sample(y2, p, 1e-3, seed=3) == 2 for p in range(50))
