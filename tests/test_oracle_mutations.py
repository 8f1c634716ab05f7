"""The oracle's pins are sharp: plant a plausible mistake in a copy of the oracle source
and at least one pin must fail. The committed oracle is never modified; each mutant is
compiled from a rewritten copy in a temporary directory and loaded on its own."""

import os

import pytest

import oracle
import synth
from tests import test_oracle as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, text in oracle.c, replacement)
MUTANTS = [
    ("rope_sign", "v[i] = a * c - b * s;", "v[i] = a * c + b * s;"),
    ("rope_frequency", "-2.0 * (double)i / (double)hd", "-1.0 * (double)i / (double)hd"),
    ("gqa_interleaved", "int32_t g = h * c->n_kv_heads / c->n_heads;", "int32_t g = h % c->n_kv_heads;"),
    ("attention_scale", "float scale = 1.0f / sqrtf((float)hd);", "float scale = 1.0f / (float)hd;"),
    ("softmax_no_max_shift", "scratch[j] = expf(scratch[j] - mx);", "scratch[j] = expf(scratch[j]);"),
    ("eps_outside_sqrt", "sqrtf(ss / (float)n + eps)", "(sqrtf(ss / (float)n) + eps)"),
    ("norm_gain_dropped", "out[i] = (x[i] * inv) * orc_bf16_to_f32(g[i]);", "out[i] = x[i] * inv;"),
    ("attn_residual_dropped", "o->x[i] += o->tmp[i];\n\n        /* feed-forward block */",
     "o->x[i] = o->tmp[i];\n\n        /* feed-forward block */"),
    ("swiglu_swapped", "orc_silu(o->g[i]) * o->u[i]", "orc_silu(o->u[i]) * o->g[i]"),
    ("silu_sign", "z / (1.0f + expf(-z))", "z / (1.0f + expf(z))"),
    ("argmax_highest_index_on_tie", "if (v[i] > v[best]) best = i;", "if (v[i] >= v[best]) best = i;"),
    ("bf16_truncation", "u += 0x7fffu + lsb;", "u += 0u * lsb;"),
    ("kv_bytes_per_q_head", "nb += 2.0 * 2.0 * (double)Hkv * T * hd;", "nb += 2.0 * 2.0 * (double)Hq * T * hd;"),
    ("cache_misses_current_position", "att_job aj = {o, l, T};", "att_job aj = {o, l, T > 1 ? T - 1 : 1};"),
]

PIN_FUNCS = [
    lambda w, W: pins.test_bf16_round_matches_library_including_ties(),
    lambda w, W: pins.test_rmsnorm_closed_form_constant_vector(),
    lambda w, W: pins.test_rope_matches_library_rotate_half(),
    lambda w, W: pins.test_attend_matches_library_sdpa(),
    lambda w, W: pins.test_attend_large_scores_select_the_top_key(),
    lambda w, W: pins.test_silu_special_values_and_library(),
    lambda w, W: pins.test_argmax_brute_force_with_planted_ties(),
    lambda w, W: pins.test_decode_steps_reproduce_full_causal_forward(w, W),
    lambda w, W: pins.test_counted_bytes_equal_closed_form(w, W, {}),
]


def test_unmutated_source_passes_all_listed_pins(tiny, tiny_weights):
    for f in PIN_FUNCS:
        f(tiny, tiny_weights)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(tmp_path, monkeypatch, tiny, tiny_weights, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not found once: %s" % name
    mpath = tmp_path / ("oracle_%s.c" % name)
    mpath.write_text(src.replace(old, new))
    so = oracle.build(force=True, src=str(mpath), out=str(tmp_path / ("lib_%s.so" % name)))
    monkeypatch.setattr(oracle, "_lib", oracle.load(so))
    failed = []
    for i, f in enumerate(PIN_FUNCS):
        try:
            f(tiny, tiny_weights)
        except Exception:
            failed.append(i)
    assert failed, "mutant %s passed every pin" % name
