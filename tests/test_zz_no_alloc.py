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
from tests.parity_util import check_logits

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
        assert np.array_equal(tok.cpu().numpy(), ref_tok), "call %d: tokens differ" % call
        check_logits(lg.cpu().numpy(), ref_lg, "kd_decode_noalloc call %d" % call)
    # and without the logits dump, as a user would call it
    tok = torch.full((w.n_gen,), -1, dtype=torch.int32, device="cuda")
    kd.kd_decode_noalloc(dec.h, d_prompt.data_ptr(), prompt.numel(), 0, w.n_gen, tok.data_ptr(), None)
    assert np.array_equal(tok.cpu().numpy(), ref_tok)
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
