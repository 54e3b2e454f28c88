"""Kept states (the prompt cache) through the C ABI: lfm3_keep / lfm3_restore.

TensorFold PR #1508, prompt-cache paragraph: a state at `at` is the slot's conv states and its
keys and values at positions [0, at); it is copied behind the chunk that ends at the mark and
restored into the new stream's pages before its next chunk. The pages check "resumed against
fresh"; here resumed == fresh bit for bit, and both match the oracle (whose kept state is an
independent copy of its incremental state) to the parity tolerances.
"""
import numpy as np
import pytest
import torch

from lfm3_inputs import lfm3_1p7b, lfm3_slice3, make_weights, make_embeds, make_tokens, page_permutation
from oracle import Lfm3Oracle
from parity import assert_hidden, assert_logits, bf16_rows, f64_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_decoder_b200 import build
    build.build(verbose=False)
    from attention_decoder_b200.model import Lfm3Model
    return Lfm3Model


@pytest.fixture(scope="module")
def slice3():
    g = lfm3_slice3()
    W = make_weights(g, 0)
    return g, W, Lfm3Oracle(W, bf16=True)


@pytest.mark.parametrize("at", [320, 300, 64])
def test_resumed_equals_fresh_and_the_oracle(lib, slice3, at):
    """Mark at a page boundary past the ring's wrap (320), off a page boundary (300) and before
    the window fills (64); the resumed slot has shuffled pages and NaN-poisoned state."""
    g, W, o = slice3
    n = 420
    x = make_embeds(9, "keep", n, g.d_model)
    ref = o.forward_full(x0=f64_rows(x))["hidden"]
    xd = bf16_rows(x)
    S, mpp = 3, 8
    pt = page_permutation(9, "keep.pages", S * mpp).reshape(S, mpp)
    m = lib(W, max_streams=S, max_pages_per_stream=mpp)
    st = m.new_state(page_table=pt, poison=True)
    m.prefill(st, 0, embeds=xd[:at])                     # the chunk ends at the mark
    mark, buf = m.keep(st, 0)
    assert mark == at and buf.numel() == m.state_bytes(at)
    fresh = m.prefill(st, 0, embeds=xd[at:n - 2], hidden=True)["hidden"].clone()
    fresh_d = [m.decode(st, [0], embeds=xd[t:t + 1], hidden=True)["hidden"].clone() for t in (n - 2, n - 1)]
    m.restore(st, 1, at, buf)                            # the source has moved on; the kept copy has not
    assert st.h_seq_len.tolist()[1] == at and st.seq_len.cpu().tolist()[1] == at
    resumed = m.prefill(st, 1, embeds=xd[at:n - 2], hidden=True)["hidden"].clone()
    resumed_d = [m.decode(st, [1], embeds=xd[t:t + 1], hidden=True)["hidden"].clone() for t in (n - 2, n - 1)]
    torch.cuda.synchronize()
    assert torch.isfinite(resumed).all()
    assert torch.equal(fresh, resumed)
    for a, b in zip(fresh_d, resumed_d):
        assert torch.equal(a, b)
    assert_hidden(resumed, [h[at:n - 2] for h in ref], what=f"resumed prefill at {at}")
    for i, t in enumerate((n - 2, n - 1)):
        assert_hidden(resumed_d[i], [h[t:t + 1] for h in ref], what=f"resumed decode {t}")
    m.check_device_errors()


def test_resumed_greedy_decode_with_head(lib):
    g = lfm3_1p7b(layer_types=(0, 2, 1, 0))
    W = make_weights(g, 0)
    o = Lfm3Oracle(W, bf16=True)
    tok = make_tokens(3, "keep.head", 700, g.vocab)
    m = lib(W, max_streams=2, max_pages_per_stream=12, max_chunk=512)
    st = m.new_state()
    m.prefill(st, 0, tokens=torch.from_numpy(tok[:512]).cuda(), logits=False, argmax=False)
    at, buf = m.keep(st, 0)
    a = m.prefill(st, 0, tokens=torch.from_numpy(tok[512:]).cuda())
    m.restore(st, 1, at, buf)
    b = m.prefill(st, 1, tokens=torch.from_numpy(tok[512:]).cuda())
    torch.cuda.synchronize()
    assert torch.equal(a["logits"], b["logits"]) and torch.equal(a["argmax"], b["argmax"])
    ost = o.new_state()
    o.forward_chunk(ost, tokens=tok[:512], logits=None)
    kept = o.keep(ost)
    r = o.forward_chunk(kept, tokens=tok[512:])
    assert_logits(b["logits"], r["logits"], b["argmax"], what="resumed prompt")
    # greedy steps from both slots stay identical
    ta, tb = a["argmax"].clone(), b["argmax"].clone()
    for _ in range(3):
        oa = m.decode(st, [0], tokens=ta)
        ob = m.decode(st, [1], tokens=tb)
        torch.cuda.synchronize()
        assert torch.equal(oa["logits"], ob["logits"])
        ta, tb = oa["argmax"].clone(), ob["argmax"].clone()


def test_keep_and_restore_refusals_touch_nothing(lib, slice3):
    from attention_decoder_b200 import Lfm3Error
    g, W, o = slice3
    x = bf16_rows(make_embeds(9, "keep.refuse", 200, g.d_model))
    m = lib(W, max_streams=2, max_pages_per_stream=4)
    st = m.new_state()
    m.prefill(st, 0, embeds=x[:200])
    small = torch.empty(m.state_bytes(200) - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(Lfm3Error) as e:
        m.keep(st, 0, buf=small)
    assert e.value.status == -3
    at, buf = m.keep(st, 0)
    before = [t.clone() for t in (st.conv, st.ring_k, st.kv_k, st.seq_len)]
    with pytest.raises(Lfm3Error) as e:                  # 300 positions do not fit 4 pages of 64
        m.restore(st, 1, 300, torch.empty(m.state_bytes(300), dtype=torch.uint8, device="cuda"))
    assert e.value.status == -3
    with pytest.raises(Lfm3Error) as e:
        m.restore(st, 1, at, small)
    assert e.value.status == -3
    torch.cuda.synchronize()
    for a, b in zip(before, (st.conv, st.ring_k, st.kv_k, st.seq_len)):
        assert torch.equal(a, b)
    assert st.h_seq_len.tolist() == [200, 0]
