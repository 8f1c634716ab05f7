"""The sampler's pins are sharp: plant a plausible mistake in a copy of oracle/sampling.py and
at least one pin of tests/test_sampling.py must fail. The committed module is never
modified; each mutant is loaded from a rewritten copy under its own module name."""

import importlib.util
import os

import numpy as np
import pytest

from oracle import sampling
from tests import test_sampling as pins

SRC = sampling.__file__

# (name, text in sampling.py, replacement)
MUTANTS = [
    ("multipliers_swapped", "hi0, lo0 = _mulhilo(M0, c[0])\n    hi1, lo1 = _mulhilo(M1, c[2])",
     "hi0, lo0 = _mulhilo(M1, c[0])\n    hi1, lo1 = _mulhilo(M0, c[2])"),
    ("round_outputs_rotated", "return (hi1 ^ c[1] ^ np.uint32(k[0]), lo1, hi0 ^ c[3] ^ np.uint32(k[1]), lo0)",
     "return (lo1, hi1 ^ c[1] ^ np.uint32(k[0]), lo0, hi0 ^ c[3] ^ np.uint32(k[1]))"),
    ("key_never_bumped", "k0, k1 = (k0 + W0) & MASK, (k1 + W1) & MASK", "k0, k1 = k0, k1"),
    ("key_bumped_before_first_round", "        if r > 0:\n            k0, k1", "        if r >= 0:\n            k0, k1"),
    ("uniform_can_reach_one", "(w >> np.uint32(9)).astype(np.float32) + np.float32(0.5)",
     "(w >> np.uint32(9)).astype(np.float32) + np.float32(1.0)"),
    ("uniform_24_bits", "((w >> np.uint32(9)).astype(np.float32) + np.float32(0.5)) * np.float32(2.0 ** -23)",
     "((w >> np.uint32(8)).astype(np.float32) + np.float32(0.5)) * np.float32(2.0 ** -24)"),
    ("gumbel_sign", "return -np.log(-np.log(u))", "return np.log(-np.log(u))"),
    ("temperature_multiplies", "z = y * (np.float32(1.0) / np.float32(temperature)) + gumbel(seed, pos, y.size)",
     "z = y * np.float32(temperature) + gumbel(seed, pos, y.size)"),
    ("same_word_for_every_index", "w = words[np.arange(n), (i & np.uint64(3)).astype(np.int64)]",
     "w = words[np.arange(n), 0]"),
]

PINS = [
    pins.test_one_round_places_the_products_as_defined,
    pins.test_key_is_bumped_between_rounds,
    pins.test_uniforms_are_in_the_open_interval_and_uniform,
    pins.test_output_bits_are_balanced_and_streams_differ,
    lambda: pins.test_gumbel_max_draws_from_the_tempered_softmax(0.7),
    lambda: pins.test_gumbel_max_draws_from_the_tempered_softmax(1.5),
    pins.test_zero_temperature_is_greedy_and_ties_go_low,
]


def _load(path, name):
    spec = importlib.util.spec_from_file_location(name, path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_unmutated_module_passes_all_listed_pins():
    for f in PINS:
        f()


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(tmp_path, monkeypatch, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not found once: %s" % name
    path = tmp_path / ("sampling_%s.py" % name)
    path.write_text(src.replace(old, new))
    mutant = _load(str(path), "sampling_mutant_%s" % name)
    monkeypatch.setattr(pins, "S", mutant)
    failed = 0
    for f in PINS:
        try:
            with np.errstate(all="ignore"):
                f()
        except AssertionError:
            failed += 1
    assert failed >= 1, "no pin caught mutant %s" % name
