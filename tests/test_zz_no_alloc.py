"""The allocation-free decode call (kd_decode_noalloc) against kd_decode.

Some callers cannot allocate device memory while they decode; kd_decode_noalloc serves
them by keeping its working memory in a fixed array inside libkd. These tests call it
through the C ABI twice in a row and check that it returns what kd_decode returns, and that
a request too large for the array is refused before anything runs. This file is collected
last so that a failure here never hides the result of another test.
"""

import numpy as np
import pytest
import torch

import synth
from tests.parity_util import check_logits, compare_gpu_runs

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


@pytest.fixture(scope="module")
def kd():
    from persistent_monokernel_sm_b200 import build
    build.build()
    import persistent_monokernel_sm_b200 as kd
    kd.load_library()
    return kd


def test_noalloc_matches_decode_on_two_calls(kd):
    w = synth.get("tiny")
    weights = synth.make_weights(w, device="cpu")
    prompt = synth.make_prompt(w)
    dec = kd.Decoder(w.dims(), w.capacity)
    dec.load_weights(weights)
    dec.reset(prompt.numpy(), 0)
    ref_tok, ref_lg = dec.decode(w.n_gen, logits=True)
    dec.sync()
    ref_tok, ref_lg = ref_tok.cpu().numpy(), ref_lg.cpu().numpy()
    d_prompt = prompt.cuda()
    for call in range(2):
        tok = torch.full((w.n_gen,), -1, dtype=torch.int32, device="cuda")
        lg = torch.full((w.n_steps, w.vocab), float("nan"), dtype=torch.float32, device="cuda")
        kd.kd_decode_noalloc(dec.h, d_prompt.data_ptr(), prompt.numel(), 0, w.n_gen, tok.data_ptr(),
                             lg.data_ptr())
        lgn = lg.cpu().numpy()
        n = compare_gpu_runs(ref_tok, tok.cpu().numpy(), ref_lg[w.prompt_len - 1:], "call %d" % call,
                             lgn[w.prompt_len - 1:])
        assert n == w.n_gen, "call %d: tokens differ" % call
        check_logits(lgn, ref_lg, "kd_decode_noalloc call %d" % call)
    # and without the logits dump, as a user would call it
    tok = torch.full((w.n_gen,), -1, dtype=torch.int32, device="cuda")
    kd.kd_decode_noalloc(dec.h, d_prompt.data_ptr(), prompt.numel(), 0, w.n_gen, tok.data_ptr(), None)
    assert compare_gpu_runs(ref_tok, tok.cpu().numpy(), ref_lg[w.prompt_len - 1:], "no dump") == w.n_gen
    dec.close()


def test_noalloc_on_a_prefilled_cache_leaves_the_handle_as_it_was(kd):
    """kd_decode_noalloc over a pre-filled cache (kv_len = 100) gives what kd_decode gives
    from the same state; it leaves the handle's position and pending tokens alone, so a
    kd_decode that follows it continues exactly as if the call had not been made."""
    w = synth.get("tiny").replace(kv_len=100, prompt_len=0, n_gen=24)
    weights = synth.make_weights(w, device="cpu")
    K, V = synth.make_kv(w, seed=2, device="cpu")
    start = synth.make_prompt(w)
    dec = kd.Decoder(w.dims(), w.capacity + 40)
    dec.load_weights(weights)
    dec.set_kv(K, V)
    # reference: kd_decode from the pre-filled state, then 16 more tokens in a second call
    dec.reset(start.numpy(), w.kv_len)
    ref_tok, ref_lg = dec.decode(w.n_gen, logits=True)
    ref_more, ref_more_lg = dec.decode(16, logits=True)
    dec.sync()
    ref_tok, ref_lg = ref_tok.cpu().numpy(), ref_lg.cpu().numpy()
    ref_more, ref_more_lg = ref_more.cpu().numpy(), ref_more_lg.cpu().numpy()
    # the same first call through kd_decode_noalloc, on a handle reset to the same state
    dec.set_kv(K, V)
    dec.reset(start.numpy(), w.kv_len)
    pos = dec.position()
    d_start = start.cuda()
    tok = torch.full((w.n_gen,), -1, dtype=torch.int32, device="cuda")
    lg = torch.full((w.n_steps, w.vocab), float("nan"), dtype=torch.float32, device="cuda")
    kd.kd_decode_noalloc(dec.h, d_start.data_ptr(), start.numel(), w.kv_len, w.n_gen, tok.data_ptr(),
                         lg.data_ptr())
    lgn = lg.cpu().numpy()
    assert compare_gpu_runs(ref_tok, tok.cpu().numpy(), ref_lg, "prefilled", lgn) == w.n_gen
    check_logits(lgn, ref_lg, "kd_decode_noalloc prefilled")
    assert dec.position() == pos  # the handle's own state is untouched
    # the handle then decodes as if the call had not been made: its pending start token at
    # kv_len rewrites the same cache rows before any step reads them
    t1, lg1 = dec.decode(w.n_gen, logits=True)
    t2, lg2 = dec.decode(16, logits=True)
    dec.sync()
    assert compare_gpu_runs(ref_tok, t1.cpu().numpy(), ref_lg, "after noalloc", lg1.cpu().numpy()) == w.n_gen
    assert compare_gpu_runs(ref_more, t2.cpu().numpy(), ref_more_lg, "after noalloc, second call",
                            lg2.cpu().numpy()) == 16
    dec.close()


def test_noalloc_refuses_requests_larger_than_its_array(kd):
    w = synth.get("tiny")
    n_tokens = 300_000  # 1.2 MB of pending tokens alone
    dec = kd.Decoder(w.dims(), n_tokens + 8)
    dec.load_weights(synth.make_weights(w, device="cpu"))
    toks = torch.zeros(n_tokens, dtype=torch.int32, device="cuda")
    out = torch.empty(4, dtype=torch.int32, device="cuda")
    before = dec.info().launches
    with pytest.raises(kd.KdError) as e:
        kd.kd_decode_noalloc(dec.h, toks.data_ptr(), n_tokens, 0, 1, out.data_ptr(), None)
    assert e.value.code == -1 and "maximum" in str(e.value)
    assert dec.info().launches == before
    dec.close()
