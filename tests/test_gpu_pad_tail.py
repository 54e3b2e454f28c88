"""A prompt chunk padded at its end (lfm3_prefill_padded) against the same rows unpadded.

coreai-model-zoo note "lfm3-1.7b-port", pad-tail paragraph: the padded rows go through the pass,
but the conv state is read after the real rows (columns [n, n + 6) of [state | Bx]) and nothing
else changes: "an engine that never pads computes exactly what" the padded one does. Here the
real rows' hidden states, the logits, the state and every later step are bit-identical to the
unpadded call's, and match the oracle.
"""
import numpy as np
import pytest
import torch

from lfm3_inputs import lfm3_1p7b, lfm3_slice3, make_weights, make_embeds, make_tokens
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


def _copy(m, src):
    dst = m.new_state()
    for t in ("conv", "ring_k", "ring_v", "kv_k", "kv_v", "seq_len"):
        getattr(dst, t).copy_(getattr(src, t))
    dst.h_seq_len[:] = src.h_seq_len
    return dst


@pytest.mark.parametrize("n_real,n_rows", [(37, 64), (1, 64), (5, 64), (64, 64), (200, 256)])
def test_padded_chunk_equals_the_unpadded_rows(lib, n_real, n_rows):
    g = lfm3_slice3()
    W = make_weights(g, 0)
    head = 250                      # rows before the padded chunk: the ring has wrapped
    n = head + n_real
    x = make_embeds(10, "padtail", n + 3, g.d_model)
    ref = Lfm3Oracle(W, bf16=True).forward_full(x0=f64_rows(x))["hidden"]
    xd = bf16_rows(x)
    m = lib(W, max_streams=1, max_pages_per_stream=(n + 3 + 63) // 64)
    a = m.new_state(poison=True)
    m.prefill(a, 0, embeds=xd[:head])
    b = _copy(m, a)
    pads = torch.zeros(n_rows - n_real, g.d_model, dtype=torch.bfloat16, device="cuda")
    ha = m.prefill(a, 0, embeds=xd[head:n], hidden=True)["hidden"].clone()
    hb = m.prefill_padded(b, 0, n_real, embeds=torch.cat([xd[head:n], pads]), hidden=True)["hidden"].clone()
    torch.cuda.synchronize()
    assert hb.shape[1] == n_rows
    assert torch.equal(ha, hb[:, :n_real])
    assert b.h_seq_len.tolist() == [n] and b.seq_len.cpu().tolist() == [n]
    for t in ("conv", "ring_k", "ring_v"):  # bitwise: slots the prompt has not reached still hold NaN poison
        assert torch.equal(getattr(a, t).view(torch.int16), getattr(b, t).view(torch.int16)), t
    for t in range(n, n + 3):  # later steps read the committed state
        da = m.decode(a, [0], embeds=xd[t:t + 1], hidden=True)["hidden"].clone()
        db = m.decode(b, [0], embeds=xd[t:t + 1], hidden=True)["hidden"].clone()
        torch.cuda.synchronize()
        assert torch.equal(da, db)
        assert_hidden(db, [h[t:t + 1] for h in ref], what=f"decode {t} after the padded chunk")
    assert_hidden(hb[:, :n_real], [h[head:n] for h in ref], what="padded chunk")
    m.check_device_errors()


def test_padded_chunk_logits_are_the_last_real_rows(lib):
    g = lfm3_1p7b(layer_types=(0, 2, 1, 0))
    W = make_weights(g, 0)
    tok = make_tokens(4, "padtail.head", 100, g.vocab)
    m = lib(W, max_streams=2, max_pages_per_stream=3)
    st = m.new_state()
    padded = np.concatenate([tok, np.zeros(28, np.int32)])      # the pages' engine pads with token 0
    a = m.prefill(st, 0, tokens=torch.from_numpy(tok).cuda())
    b = m.prefill_padded(st, 1, 100, tokens=torch.from_numpy(padded).cuda())
    torch.cuda.synchronize()
    assert torch.equal(a["logits"], b["logits"]) and torch.equal(a["argmax"], b["argmax"])
    r = Lfm3Oracle(W, bf16=True).forward_full(tokens=tok)
    assert_logits(b["logits"], r["logits"], b["argmax"], what="padded chunk logits")
    assert st.h_seq_len.tolist() == [100, 100]
