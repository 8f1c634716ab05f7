"""GPU parity: the CUDA monokernel (through the C ABI) against the CPU oracle.

Every input comes from the seeded generators in ``synth``; both sides get the same bytes.
Tolerances (stated in parity_util): logits max|d| <= 2e-2 and rel-L2 <= 1e-3 at every
compared step; tokens bit-exact wherever the oracle's top-1/top-2 margin exceeds 5e-2.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import naive
import synth
from tests.parity_util import (check_logits, check_tokens_against_logits, compare_free_run,
                               oracle_threads, rel_bound_from_exact)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


@pytest.fixture(scope="module")
def kd():
    from persistent_monokernel_sm_b200 import build
    build.build()
    import persistent_monokernel_sm_b200 as kd
    kd.load_library()
    return kd


_WEIGHTS = {}


def weights_for(name):
    if name not in _WEIGHTS:
        _WEIGHTS.clear()
        w = synth.get(name)
        _WEIGHTS[name] = synth.make_weights(w)
    return _WEIGHTS[name]


def host(weights):
    return {k: v.cpu() for k, v in weights.items()}


def make_decoder(kd, w, weights, max_seq=None):
    dec = kd.Decoder(w.dims(), max_seq or w.capacity)
    dec.load_weights(weights)
    return dec


# ------------------------------------------------------------------ tiny: every step

def test_tiny_forced_logits_every_step(kd):
    w = synth.get("tiny")
    W = weights_for("tiny")
    toks = np.concatenate([synth.make_prompt(w).numpy(), synth.make_tokens(w, 64).numpy()])
    dec = make_decoder(kd, w, W, max_seq=len(toks))
    dec.reset(toks, 0)
    _, lg = dec.decode(1, logits=True)
    dec.sync()
    gpu = lg.cpu().numpy()
    ref = oracle.Oracle(w.dims(), W, capacity=len(toks)).forced(toks, 0)
    bound = rel_bound_from_exact(ref, naive.causal_forward(w.dims(), W, toks))
    check_logits(gpu, ref, "tiny forced", bound)
    check_tokens_against_logits(gpu.argmax(axis=1), ref, "tiny forced")


def test_tiny_greedy_free_run_and_in_kernel_argmax(kd):
    w = synth.get("tiny")
    W = weights_for("tiny")
    prompt = synth.make_prompt(w).numpy()
    dec = make_decoder(kd, w, W)
    dec.reset(prompt, 0)
    toks, lg = dec.decode(w.n_gen, logits=True)
    dec.sync()
    toks = toks.cpu().numpy()
    lg = lg.cpu().numpy()
    assert lg.shape == (w.n_steps, w.vocab)
    chosen = lg[w.prompt_len - 1:]
    # the in-kernel argmax picks the lowest index of the maximum of its own logits
    assert np.array_equal(toks, chosen.argmax(axis=1))
    o = oracle.Oracle(w.dims(), W, capacity=w.capacity)
    otoks, ologits = o.greedy(prompt, 0, w.n_gen)
    seq = np.concatenate([prompt, otoks[:-1]])
    exact = naive.causal_forward(w.dims(), W, seq)[w.prompt_len - 1:]
    n = compare_free_run(toks, chosen, otoks, ologits, "tiny greedy", rel_bound_from_exact(ologits, exact))
    assert n >= 1
    # the launch that is benchmarked (no logits) picks the very same tokens
    dec.reset(prompt, 0)
    toks2, _ = dec.decode(w.n_gen)
    dec.sync()
    assert np.array_equal(toks, toks2.cpu().numpy())


def test_tiny_prefilled_cache(kd):
    w = synth.get("tiny").replace(kv_len=100, prompt_len=0, n_gen=24)
    W = weights_for("tiny")
    K, V = synth.make_kv(w, seed=2, device="cpu")
    start = synth.make_prompt(w).numpy()
    dec = make_decoder(kd, w, W)
    dec.set_kv(K, V)
    dec.reset(start, w.kv_len)
    toks, lg = dec.decode(w.n_gen, logits=True)
    dec.sync()
    o = oracle.Oracle(w.dims(), W, capacity=w.capacity)
    o.set_kv(K, V)
    otoks, ologits = o.greedy(start, w.kv_len, w.n_gen)
    compare_free_run(toks.cpu().numpy(), lg.cpu().numpy(), otoks, ologits, "tiny prefilled")


def test_tiny_calls_chain_and_are_deterministic(kd):
    w = synth.get("tiny")
    W = weights_for("tiny")
    prompt = synth.make_prompt(w).numpy()
    dec = make_decoder(kd, w, W)
    dec.reset(prompt, 0)
    full, lg_a = dec.decode(w.n_gen, logits=True)
    dec.sync()
    full = full.cpu().numpy().copy()
    lg_a = lg_a.cpu().numpy()
    dec.reset(prompt, 0)
    a, _ = dec.decode(20)
    a = a.cpu().numpy().copy()
    b, _ = dec.decode(w.n_gen - 20)
    dec.sync()
    assert np.array_equal(np.concatenate([a, b.cpu().numpy()]), full)
    assert dec.position() == w.capacity
    dec.reset(prompt, 0)
    _, lg_b = dec.decode(w.n_gen, logits=True)
    dec.sync()
    assert np.array_equal(lg_a, lg_b.cpu().numpy())  # bit-identical run to run


def test_tiny_one_launch_per_decode_and_host_api(kd):
    w = synth.get("tiny")
    W = weights_for("tiny")
    prompt = synth.make_prompt(w)
    dec = make_decoder(kd, w, W)
    before = dec.info().launches
    dec.reset(prompt.numpy(), 0)
    ref, _ = dec.decode(w.n_gen)
    dec.sync()
    assert dec.info().launches == before + 1
    host_out = dec.generate(prompt.pin_memory(), 0, w.n_gen, torch.empty(w.n_gen, dtype=torch.int32).pin_memory())
    assert np.array_equal(host_out.numpy(), ref.cpu().numpy())
    assert dec.info().launches == before + 2


def test_capacity_is_checked_before_launch(kd):
    w = synth.get("tiny")
    W = weights_for("tiny")
    dec = make_decoder(kd, w, W, max_seq=20)
    dec.reset(synth.make_prompt(w).numpy(), 0)
    before = dec.info().launches
    with pytest.raises(kd.KdError) as e:
        dec.decode(10)  # 16 + 10 - 1 steps > 20
    assert e.value.code == -3
    assert dec.info().launches == before


def test_token_outside_vocab_stops_the_launch(kd):
    """A pending id outside [0, vocab) is refused by the kernel's own range check before any
    embedding row is read: kd_sync reports KD_ETOKEN, and after kd_reset the handle decodes
    exactly as before."""
    w = synth.get("tiny")
    W = weights_for("tiny")
    prompt = synth.make_prompt(w).numpy()
    dec = make_decoder(kd, w, W)
    dec.reset(prompt, 0)
    ref, _ = dec.decode(8)
    dec.sync()
    ref = ref.cpu().numpy().copy()
    for bad in (w.vocab, -1):
        dec.reset(np.concatenate([prompt[:3], [bad], prompt[3:]]).astype(np.int32), 0)
        dec.decode(4)
        with pytest.raises(kd.KdError) as e:
            dec.sync()
        assert e.value.code == -8
        with pytest.raises(kd.KdError):
            dec.decode(1)  # refused until reset
    dec.reset(prompt, 0)
    again, _ = dec.decode(8)
    dec.sync()
    assert np.array_equal(again.cpu().numpy(), ref)


def test_wait_limit_reports_timeout_and_recovers(kd):
    """With a 1 ns wait limit the first wait that does not succeed at once gives up: the
    launch stops without trapping or hanging, kd_sync reports KD_ETIMEOUT, decode is refused
    until kd_reset, and with the normal limit back the handle decodes exactly as before."""
    w = synth.get("tiny")
    W = weights_for("tiny")
    prompt = synth.make_prompt(w).numpy()
    dec = make_decoder(kd, w, W)
    dec.reset(prompt, 0)
    ref, _ = dec.decode(16)
    dec.sync()
    ref = ref.cpu().numpy().copy()
    kd.kd_set_timeout(dec.h, 1)
    dec.reset(prompt, 0)
    dec.decode(16)
    with pytest.raises(kd.KdError) as e:
        dec.sync()
    assert e.value.code == -6
    with pytest.raises(kd.KdError):
        dec.decode(1)
    kd.kd_set_timeout(dec.h, 1_000_000_000)
    dec.reset(prompt, 0)
    again, _ = dec.decode(16)
    dec.sync()
    assert np.array_equal(again.cpu().numpy(), ref)


# ------------------------------------------------------------------ 0.5B: every step

def test_half_billion_forced_and_greedy(kd):
    w = synth.get("0.5b")
    W = weights_for("0.5b")
    prompt = synth.make_prompt(w).numpy()
    toks = np.concatenate([prompt, synth.make_tokens(w, w.n_gen).numpy()])
    dec = make_decoder(kd, w, W, max_seq=len(toks))
    dec.reset(toks, 0)
    _, lg = dec.decode(1, logits=True)
    dec.sync()
    Wh = host(W)
    ref = oracle.Oracle(w.dims(), Wh, capacity=len(toks), n_threads=oracle_threads()).forced(toks, 0)
    bound = rel_bound_from_exact(ref, naive.causal_forward(w.dims(), Wh, toks))
    check_logits(lg.cpu().numpy(), ref, "0.5b forced", bound)
    # free-running greedy decode, in the benchmarked launch configuration
    dec.reset(prompt, 0)
    gt, glg = dec.decode(w.n_gen, logits=True)
    dec.reset(prompt, 0)
    gt2, _ = dec.decode(w.n_gen)
    dec.sync()
    gt = gt.cpu().numpy()
    assert np.array_equal(gt, gt2.cpu().numpy())
    chosen = glg.cpu().numpy()[w.prompt_len - 1:]
    assert np.array_equal(gt, chosen.argmax(axis=1))
    o = oracle.Oracle(w.dims(), Wh, capacity=w.capacity, n_threads=oracle_threads())
    otoks, ologits = o.greedy(prompt, 0, w.n_gen)
    seq = np.concatenate([prompt, otoks[:-1]])
    exact = naive.causal_forward(w.dims(), Wh, seq)[w.prompt_len - 1:]
    compare_free_run(gt, chosen, otoks, ologits, "0.5b greedy", rel_bound_from_exact(ologits, exact))


# ------------------------------------------------------------------ large workloads

@pytest.mark.parametrize("name,n_check", [("2b-4k", 8), ("2b-32k", 4), ("8b-4k", 4)])
def test_full_size_workload(kd, name, n_check):
    """The full benchmarked decode (every token), checked three ways: the first n_check
    steps against the oracle (free-running, same start), every step's token against the
    argmax of its own dumped logits, and the undumped launch giving identical tokens."""
    _WEIGHTS.clear()
    torch.cuda.empty_cache()
    w = synth.get(name)
    W = synth.make_weights(w)
    K, V = synth.make_kv(w)
    start = synth.make_prompt(w).numpy()
    dec = make_decoder(kd, w, W)
    dec.set_kv(K, V)
    dec.reset(start, w.kv_len)
    toks, _ = dec.decode(w.n_gen)
    dec.reset(start, w.kv_len)
    toks_d, lg = dec.decode(w.n_gen, logits=True)
    dec.sync()
    toks = toks.cpu().numpy()
    assert np.array_equal(toks, toks_d.cpu().numpy())
    lg = lg.cpu().numpy()
    assert np.all(np.isfinite(lg))
    assert np.array_equal(toks, lg.argmax(axis=1))
    Wh = host(W)
    del W, dec
    torch.cuda.empty_cache()
    o = oracle.Oracle(w.dims(), Wh, capacity=w.kv_len + n_check, n_threads=oracle_threads())
    o.set_kv(K.cpu(), V.cpu())
    otoks, ologits = o.greedy(start, w.kv_len, n_check)
    compare_free_run(toks[:n_check], lg[:n_check], otoks, ologits, name)
