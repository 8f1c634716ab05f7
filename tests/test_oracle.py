"""Pins for the CPU oracle: each part checked against something other than itself.

Closed forms, invariants, special cases that reduce to a library routine, brute force on
tiny inputs, an independent fp64 full-sequence causal forward, and a library Llama-style
model. All CPU; no GPU needed.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import exact, naive
import synth


def rng(seed=0):
    return np.random.default_rng(seed)


def bf16_bits(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(
        np.uint16)


# ------------------------------------------------------------------ scalar stages

def test_bf16_round_matches_library_including_ties():
    r = rng(1)
    vals = list(r.standard_normal(2000).astype(np.float32) * 3)
    # exact halfway cases: lower 16 bits 0x8000 with even and odd upper halves, both signs
    for hi in (0x3F80, 0x3F81, 0x4000, 0x4001, 0xBF80, 0xBF81, 0x0001, 0x7F7F):
        vals.append(np.array([(hi << 16) | 0x8000], np.uint32).view(np.float32)[0])
        vals.append(np.array([(hi << 16) | 0x7FFF], np.uint32).view(np.float32)[0])
        vals.append(np.array([(hi << 16) | 0x8001], np.uint32).view(np.float32)[0])
    vals += [0.0, -0.0, 1e-40, -1e-40, 3.3895314e38, np.inf, -np.inf]
    v = np.array(vals, np.float32)
    assert np.array_equal(oracle.bf16_round(v), bf16_bits(v))
    # widening back is exact
    assert np.array_equal(oracle.bf16_to_f32(bf16_bits(v)),
                          torch.tensor(v).to(torch.bfloat16).float().numpy())


def test_rmsnorm_closed_form_constant_vector():
    eps = 1e-5
    for c in (2.5, -0.75, 1e-3):
        x = np.full(64, c, np.float32)
        g = np.linspace(0.5, 2.0, 64).astype(np.float32)
        out = oracle.rmsnorm(x, bf16_bits(g), eps)
        gb = torch.tensor(g).to(torch.bfloat16).double().numpy()
        want = gb * np.sign(c) * abs(c) / np.sqrt(c * c + eps)
        assert np.allclose(out, want, rtol=2e-6, atol=0)


def test_rmsnorm_matches_library():
    r = rng(2)
    x = r.standard_normal(2048).astype(np.float32)
    g = (1 + 0.1 * r.standard_normal(2048)).astype(np.float32)
    gb = torch.tensor(g).to(torch.bfloat16).double()
    want = torch.nn.functional.rms_norm(torch.tensor(x, dtype=torch.float64), (2048,), gb, 1e-5)
    out = oracle.rmsnorm(x, bf16_bits(g), 1e-5)
    assert np.allclose(out, want.numpy(), rtol=5e-5, atol=1e-6)


def test_rmsnorm_scale_invariance():
    r = rng(3)
    x = (r.standard_normal(256) * 10).astype(np.float32)
    g = bf16_bits(np.ones(256, np.float32))
    a = oracle.rmsnorm(x, g, 1e-5)
    b = oracle.rmsnorm(x * 8.0, g, 1e-5)   # exact power-of-two scaling
    assert np.allclose(a, b, rtol=1e-6, atol=1e-7)


def test_rope_identity_at_position_zero():
    v = rng(4).standard_normal(128).astype(np.float32)
    assert np.array_equal(oracle.rope(v, 0, 10000.0), v)


def test_rope_preserves_pair_norms():
    v = rng(5).standard_normal(128).astype(np.float32)
    r = oracle.rope(v, 1234, 10000.0)
    n0 = v[:64] ** 2 + v[64:] ** 2
    n1 = r[:64].astype(np.float64) ** 2 + r[64:].astype(np.float64) ** 2
    assert np.allclose(n0, n1, rtol=1e-5)


@pytest.mark.parametrize("theta", [10000.0, 500000.0])
def test_rope_dot_depends_only_on_relative_position(theta):
    r = rng(6)
    q = r.standard_normal(128).astype(np.float32)
    k = r.standard_normal(128).astype(np.float32)
    base = float(np.dot(oracle.rope(q, 7, theta).astype(np.float64),
                        oracle.rope(k, 3, theta).astype(np.float64)))
    for shift in (1, 50, 999):
        s = float(np.dot(oracle.rope(q, 7 + shift, theta).astype(np.float64),
                         oracle.rope(k, 3 + shift, theta).astype(np.float64)))
        assert abs(s - base) < 2e-4 * (1 + abs(base))


def test_rope_matches_library_rotate_half():
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    r = rng(7)
    hd, pos, theta = 64, 37, 10000.0
    q = r.standard_normal(hd).astype(np.float32)
    inv = 1.0 / (theta ** (torch.arange(0, hd, 2, dtype=torch.float64) / hd))
    ang = pos * inv
    emb = torch.cat([ang, ang])
    cos, sin = emb.cos()[None, None, None, :], emb.sin()[None, None, None, :]
    qt = torch.tensor(q, dtype=torch.float64)[None, None, None, :]
    want, _ = apply_rotary_pos_emb(qt, qt, cos[0], sin[0], unsqueeze_dim=1)
    got = oracle.rope(q, pos, theta)
    assert np.allclose(got, want.reshape(-1).numpy(), rtol=1e-5, atol=1e-6)


def test_attend_single_entry_returns_v():
    r = rng(8)
    for hd in (64, 128):
        q = (r.standard_normal(hd) * 5).astype(np.float32)
        K = bf16_bits(r.standard_normal((1, hd)))
        V = bf16_bits(r.standard_normal((1, hd)))
        out = oracle.attend(q, K, V)
        assert np.array_equal(out, oracle.bf16_to_f32(V[0]))


def test_attend_equal_keys_gives_mean_of_v():
    r = rng(9)
    T, hd = 37, 64
    q = r.standard_normal(hd).astype(np.float32)
    K = np.repeat(bf16_bits(r.standard_normal((1, hd))), T, axis=0)
    V = bf16_bits(r.standard_normal((T, hd)))
    out = oracle.attend(q, K, V)
    want = oracle.bf16_to_f32(V).astype(np.float64).mean(axis=0)
    assert np.allclose(out, want, rtol=1e-5, atol=1e-6)


def test_attend_large_scores_select_the_top_key():
    """Scores in the thousands: softmax is one-hot on the best key and must not overflow."""
    r = rng(13)
    T, hd = 10, 64
    q = (r.standard_normal(hd) * 400).astype(np.float32)
    K = bf16_bits(r.standard_normal((T, hd)))
    V = bf16_bits(r.standard_normal((T, hd)))
    s = oracle.bf16_to_f32(K).astype(np.float64) @ q.astype(np.float64)
    top = int(np.argmax(s))
    assert np.sort(s)[-1] - np.sort(s)[-2] > 200 * np.sqrt(hd)   # the rest underflow to 0
    out = oracle.attend(q, K, V)
    assert np.array_equal(out, oracle.bf16_to_f32(V[top]))


def test_attend_matches_library_sdpa():
    r = rng(10)
    T, hd = 300, 128
    q = r.standard_normal(hd).astype(np.float32)
    Kb = bf16_bits(r.standard_normal((T, hd)))
    Vb = bf16_bits(r.standard_normal((T, hd)))
    Kf = torch.tensor(oracle.bf16_to_f32(Kb), dtype=torch.float64)
    Vf = torch.tensor(oracle.bf16_to_f32(Vb), dtype=torch.float64)
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q, dtype=torch.float64)[None, None, None], Kf[None, None], Vf[None, None])
    got = oracle.attend(q, Kb, Vb)
    assert np.allclose(got, want.reshape(-1).numpy(), rtol=1e-4, atol=1e-5)


def test_silu_special_values_and_library():
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(30.0) - 30.0) < 1e-5
    assert abs(oracle.silu(-30.0)) < 1e-10
    z = np.linspace(-12, 12, 97).astype(np.float32)
    want = torch.nn.functional.silu(torch.tensor(z, dtype=torch.float64)).numpy()
    got = np.array([oracle.silu(float(v)) for v in z])
    assert np.allclose(got, want, rtol=1e-6, atol=1e-7)


def test_argmax_brute_force_with_planted_ties():
    r = rng(11)
    for trial in range(200):
        n = int(r.integers(1, 40))
        v = r.integers(-3, 4, n).astype(np.float32)   # many ties
        want = min(i for i in range(n) if v[i] == v.max())
        assert oracle.argmax(v) == want


def test_matvec_within_fp32_summation_bound():
    r = rng(12)
    W = bf16_bits(r.standard_normal((64, 2048)) * 0.02)
    x = r.standard_normal(2048).astype(np.float32)
    y = oracle.matvec(W, x)
    Wf = oracle.bf16_to_f32(W).astype(np.float64)
    exact = Wf @ x.astype(np.float64)
    bound = 2048 * np.finfo(np.float32).eps * (np.abs(Wf) @ np.abs(x.astype(np.float64)))
    assert np.all(np.abs(y - exact) <= bound)


# ------------------------------------------------------------------ whole decode step

def _forced_run(w, weights, tokens, n_threads=1, pos0=0, kv=None):
    o = oracle.Oracle(w.dims(), weights, capacity=pos0 + len(tokens), n_threads=n_threads)
    if kv is not None:
        o.set_kv(*kv)
    return o.forced(tokens, pos0)


def test_decode_steps_reproduce_full_causal_forward(tiny, tiny_weights):
    """Decode step t with a KV cache equals row t of a full-sequence causal forward."""
    toks = np.concatenate([synth.make_prompt(tiny).numpy(), synth.make_tokens(tiny, 24).numpy()])
    got = _forced_run(tiny, tiny_weights, toks)
    want = naive.causal_forward(tiny.dims(), tiny_weights, toks, round_kv=True)
    err = np.abs(got - want).max()
    scale = np.abs(want).max()
    # fp32 vs fp64 arithmetic: ~1e-6 of scale, except where the two round a K/V element to
    # different bf16 neighbours (its fp32 value within fp32 error of a rounding boundary);
    # one such flip moves logits by up to ~2^-8 of one attention term, ~1e-4 of scale.
    # An algebra mistake moves them by O(1).
    assert err <= 1e-4 * scale, (err, scale)


def test_decode_with_prefilled_cache_reproduces_causal_forward(tiny, tiny_weights):
    P = 40
    K, V = synth.make_kv(tiny, seed=2, device="cpu", n_pos=P)
    toks = synth.make_tokens(tiny, 6).numpy()
    got = _forced_run(tiny, tiny_weights, toks, pos0=P, kv=(K, V))
    want = naive.causal_forward(tiny.dims(), tiny_weights, toks, pos0=P, kv_prefix=(K, V))
    assert np.abs(got - want).max() <= 1e-4 * np.abs(want).max()


@pytest.mark.parametrize("prefix", [0, 40])
def test_torch_fp64_forward_matches_numpy_fp64_forward(tiny, tiny_weights, prefix):
    """oracle.exact (torch, one layer widened at a time, used on a GPU for the large models)
    states the same float64 forward as naive.causal_forward (numpy): they agree to float64
    rounding on the tiny model, from position 0 and over a pre-filled cache. A transposed
    operand, a wrong group index or a dropped term in either moves logits by O(1)."""
    toks = synth.make_tokens(tiny, 12).numpy()
    kv = None
    if prefix:
        K, V = synth.make_kv(tiny, seed=2, device="cpu", n_pos=prefix)
        kv = (K, V)
    want = naive.causal_forward(tiny.dims(), tiny_weights, toks, pos0=prefix, kv_prefix=kv)
    got = exact.causal_forward(tiny.dims(), tiny_weights, toks, pos0=prefix, kv_prefix=kv)
    assert got.shape == want.shape
    assert np.abs(got - want).max() <= 1e-10 * np.abs(want).max()


def _llama(dims, weights):
    from transformers import LlamaConfig, LlamaForCausalLM
    cfg = LlamaConfig(vocab_size=dims["vocab"], hidden_size=dims["d_model"],
                      intermediate_size=dims["ffn_dim"], num_hidden_layers=dims["n_layers"],
                      num_attention_heads=dims["n_heads"], num_key_value_heads=dims["n_kv_heads"],
                      head_dim=dims["head_dim"], rms_norm_eps=dims["rms_eps"],
                      rope_theta=dims["rope_theta"], tie_word_embeddings=False,
                      attention_bias=False, mlp_bias=False, max_position_embeddings=4096)
    m = LlamaForCausalLM(cfg).to(torch.float64).eval()
    sd = {"model.embed_tokens.weight": weights["embed"], "model.norm.weight": weights["final_norm"],
          "lm_head.weight": weights["lm_head"]}
    names = {"attn_norm": "input_layernorm.weight", "ffn_norm": "post_attention_layernorm.weight",
             "wq": "self_attn.q_proj.weight", "wk": "self_attn.k_proj.weight",
             "wv": "self_attn.v_proj.weight", "wo": "self_attn.o_proj.weight",
             "wg": "mlp.gate_proj.weight", "wu": "mlp.up_proj.weight", "wd": "mlp.down_proj.weight"}
    for l in range(dims["n_layers"]):
        for k, n in names.items():
            sd["model.layers.%d.%s" % (l, n)] = weights[k][l]
    m.load_state_dict({k: v.to(torch.float64) for k, v in sd.items()}, strict=True)
    return m


def test_fp64_forward_matches_library_llama(tiny, tiny_weights):
    """The plain fp64 model (no KV rounding) equals a library Llama-style decoder."""
    toks = synth.make_tokens(tiny, 40).numpy()
    m = _llama(tiny.dims(), tiny_weights)
    with torch.no_grad():
        want = m(torch.tensor(toks, dtype=torch.int64)[None], use_cache=False).logits[0].numpy()
    got = naive.causal_forward(tiny.dims(), tiny_weights, toks, round_kv=False)
    # The library forms RoPE angles and their cos/sin in fp32 even in an fp64 model: at
    # positions < 40 the angles are off by at most 40 * 2^-23 rad (~5e-6), so logits may
    # move by ~1e-5 of their scale. Any algebra mistake moves them by O(1).
    assert np.abs(got - want).max() <= 1e-5 * np.abs(want).max()


def test_oracle_within_kv_rounding_bound_of_library_llama(tiny, tiny_weights):
    """The oracle differs from the unrounded library model only by its bf16 KV cache:
    each K/V element moves by at most 2^-9 relative, so logits move by well under 1%."""
    toks = synth.make_tokens(tiny, 40).numpy()
    m = _llama(tiny.dims(), tiny_weights)
    with torch.no_grad():
        want = m(torch.tensor(toks, dtype=torch.int64)[None], use_cache=False).logits[0].numpy()
    got = _forced_run(tiny, tiny_weights, toks)
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert rel < 1e-2, rel


def test_zero_mixing_weights_leave_embedding_path(tiny, tiny_weights):
    """With Wo = Wd = 0 no layer changes the residual stream: logits = W_lm rms(E[tok])."""
    w = dict(tiny_weights)
    w["wo"] = torch.zeros_like(w["wo"])
    w["wd"] = torch.zeros_like(w["wd"])
    toks = synth.make_tokens(tiny, 5).numpy()
    got = _forced_run(tiny, w, toks)
    E = naive._f64(w["embed"])[toks]
    xn = E / np.sqrt((E * E).mean(axis=1, keepdims=True) + tiny.rms_eps)
    want = xn @ naive._f64(w["lm_head"]).T
    assert np.abs(got - want).max() <= 1e-5 * np.abs(want).max()


def test_row_parallel_mode_is_bit_identical(tiny, tiny_weights):
    toks = synth.make_tokens(tiny, 12).numpy()
    a = _forced_run(tiny, tiny_weights, toks, n_threads=1)
    b = _forced_run(tiny, tiny_weights, toks, n_threads=5)
    assert np.array_equal(a, b)


def test_greedy_tokens_are_argmax_of_logits(tiny, tiny_weights):
    o = oracle.Oracle(tiny.dims(), tiny_weights, capacity=tiny.capacity)
    toks, logits = o.greedy(synth.make_prompt(tiny).numpy(), 0, 10)
    assert toks.shape == (10,)
    for t, lg in zip(toks, logits):
        assert t == int(np.argmax(lg))


# ------------------------------------------------------------------ bytes model

def closed_form_step_bytes(w, T, head=True):
    """Active weight bytes + KV bytes read for one step over T cached positions (bf16)."""
    L, d, Hq, Hkv, hd, F, V = (w.n_layers, w.d_model, w.n_heads, w.n_kv_heads, w.head_dim,
                               w.ffn_dim, w.vocab)
    per_layer = d * (Hq + 2 * Hkv) * hd + Hq * hd * d + 3 * d * F + 2 * d
    params = L * per_layer + d  # + one embedding row
    if head:
        params += d + V * d
    return 2 * params + L * 2 * Hkv * hd * 2 * T


@pytest.mark.parametrize("shape", [dict(), dict(n_heads=4, n_kv_heads=1),
                                   dict(n_heads=6, n_kv_heads=3, head_dim=32)])
def test_counted_bytes_equal_closed_form(tiny, tiny_weights, shape):
    w = tiny.replace(**shape)
    weights = synth.make_weights(w, seed=0, device="cpu") if shape else tiny_weights
    o = oracle.Oracle(w.dims(), weights, capacity=8)
    for pos in range(4):
        _, _, nb = o.step(5, pos, head=(pos != 1))
        assert nb == closed_form_step_bytes(w, pos + 1, head=(pos != 1))


def test_pages_two_billion_model_is_about_four_gigabytes():
    w = synth.get("2b-4k")
    wbytes = closed_form_step_bytes(w, 0)
    assert 3.5e9 < wbytes < 4.2e9   # the pages' "about 4 GB of active FP16 weights"
    # the figures derived for this shape: 1,827.26 M active params at T=0
    assert round(wbytes / 2 / 1e6, 2) == 1827.26
