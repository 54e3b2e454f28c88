"""Whole-forward invariants of the CPU oracle (CPU only).

The full-sequence mode (explicit masks, zero-padded conv, no cache) and the
incremental mode (carried conv columns, growing KV list, W-slot ring) are two
separate computations; the pages' engine invariants tie them together:
prompt == one-row decode at every cut point and chunked == unchunked (TensorFold
PR #1508, "Verification"), and the ring equals masked full attention. The
negative controls of the coreai-model-zoo note "lfm3-1.7b-port" (drop the
gate, rotate every dimension, remove the window) must turn the check red.
"""
import numpy as np
import pytest

from lfm3_inputs import (CONV, FULL, SLIDING, lfm3_slice3, tiny_geometry, make_weights, make_tokens,
                         make_embeds, synthetic_state, context_lengths)
from oracle import Lfm3Oracle
from oracle.lfm3 import _bf16, top2_margin


@pytest.fixture(scope="module")
def tiny():
    g = tiny_geometry()
    W = make_weights(g, 0)
    tok = make_tokens(1, "tokens", 21, g.vocab)
    o = Lfm3Oracle(W)
    return g, W, tok, o, o.forward_full(tokens=tok, logits="all")


def _close(a, b, tol=1e-10):
    return np.allclose(a, b, rtol=tol, atol=tol)


@pytest.mark.parametrize("cut", list(range(0, 21, 2)) + [19, 20])
def test_prompt_equals_one_row_decode_at_every_cut(tiny, cut):
    g, W, tok, o, ref = tiny
    st = o.new_state()
    rows_hidden = []
    rows_logits = []
    if cut:
        out = o.forward_chunk(st, tokens=tok[:cut], logits="all")
        rows_hidden.append(out["hidden"])
        rows_logits.append(out["logits"])
    for t in range(cut, len(tok)):
        out = o.forward_chunk(st, tokens=tok[t:t + 1], logits="all")
        rows_hidden.append(out["hidden"])
        rows_logits.append(out["logits"])
    for li in range(g.n_layers + 1):
        got = np.concatenate([h[li] for h in rows_hidden])
        assert _close(got, ref["hidden"][li]), li
    assert _close(np.concatenate(rows_logits), ref["logits"])
    assert st.seq_len == len(tok)


@pytest.mark.parametrize("chunk", [1, 3, 5, 8, 9, 16, 21])
def test_chunked_equals_unchunked(tiny, chunk):
    g, W, tok, o, ref = tiny
    st = o.new_state()
    outs = [o.forward_chunk(st, tokens=tok[i:i + chunk], logits="all") for i in range(0, len(tok), chunk)]
    assert _close(np.concatenate([x["logits"] for x in outs]), ref["logits"])
    # the ring holds exactly the last W positions
    for rp in st.ring_pos:
        assert sorted(rp.tolist()) == list(range(len(tok) - g.window, len(tok)))


def test_negative_controls_turn_red(tiny):
    g, W, tok, o, ref = tiny
    base = ref["hidden"][-1]
    for kw in (dict(gate=False), dict(rope_all_dims=True), dict(window=False)):
        alt = Lfm3Oracle(W, **kw).forward_full(tokens=tok, logits="all")["hidden"][-1]
        # far outside the 1e-10 agreement of the two modes above
        assert np.abs(alt - base).max() > 1e-3, kw
    # with no more tokens than the window, removing it changes nothing
    short = tok[:g.window]
    a = o.forward_full(tokens=short, logits="all")["logits"]
    b = Lfm3Oracle(W, window=False).forward_full(tokens=short, logits="all")["logits"]
    assert np.array_equal(a, b)


def test_greedy_ties_go_to_lowest_id():
    lg = np.array([0.1, 0.7, 0.7, -1.0])
    assert int(np.argmax(lg)) == 1
    assert np.isclose(top2_margin(lg)[0], 0.0)


def test_synthetic_state_lays_out_ring_and_conv():
    g = tiny_geometry()
    o = Lfm3Oracle(make_weights(g, 0))
    ctx = context_lengths(1, "ctx", 3, 3, 20)
    syn = synthetic_state(g, 1, ctx)
    for s, c in enumerate(ctx):
        st = o.state_from_synthetic(syn, s, int(c))
        assert st.seq_len == c
        for j, rp in enumerate(st.ring_pos):
            live = sorted(p for p in rp.tolist() if p >= 0)
            assert live == list(range(max(0, c - g.window), c))
            for p in live:
                assert np.array_equal(st.ring_k[j][p % g.window],
                                      _bf16(syn["slide_k"][j][s][p - (c - len(live))]).astype(np.float64))
        for j in range(len(st.conv)):
            assert np.array_equal(st.conv[j], _bf16(syn["conv"][j][s]).astype(np.float64))
        assert all(k.shape[0] == c for k in st.full_k)
        # one step continues at position c
        o.forward_chunk(st, tokens=np.array([1]))
        assert st.seq_len == c + 1


@pytest.mark.slow
def test_three_block_slice_modes_agree():
    """The width-2048 three-block slice: 64 input vectors, then 8 one-row steps."""
    g = lfm3_slice3()
    W = make_weights(g, 0)
    x = _bf16(make_embeds(0, "inputs", 72, g.d_model)).astype(np.float64)
    o = Lfm3Oracle(W)
    ref = o.forward_full(x0=x)
    st = o.new_state()
    parts = [o.forward_chunk(st, x0=x[:64])] + [o.forward_chunk(st, x0=x[64 + i:65 + i]) for i in range(8)]
    for li in range(g.n_layers + 1):
        got = np.concatenate([p["hidden"][li] for p in parts])
        assert np.allclose(got, ref["hidden"][li], rtol=1e-9, atol=1e-9)
    # every block moves the residual stream by O(1)
    for li in range(1, g.n_layers + 1):
        dlt = ref["hidden"][li] - ref["hidden"][li - 1]
        assert 0.3 < np.sqrt(np.mean(dlt * dlt)) < 5.0


@pytest.mark.parametrize("at", [5, 8, 13])
def test_kept_state_resumes_like_the_fresh_pass(tiny, at):
    """Keep at a mark (a chunk that ends at position `at`), then continue both the original and
    the kept copy with the rest of the prompt: both equal the full-sequence pass, and continuing
    one does not disturb the other (TensorFold PR #1508: "resumed against fresh")."""
    g, W, tok, o, ref = tiny
    st = o.new_state()
    o.forward_chunk(st, tokens=tok[:at], logits="all")
    kept = o.keep(st)
    a = o.forward_chunk(st, tokens=tok[at:], logits="all")
    b = o.forward_chunk(kept, tokens=tok[at:], logits="all")
    assert np.array_equal(a["logits"], b["logits"])
    assert _close(b["logits"], ref["logits"][at:])
    for li in range(g.n_layers + 1):
        assert _close(b["hidden"][li], ref["hidden"][li][at:]), li
    # a second resume from a fresh keep of the same mark gives the same rows again
    st2 = o.new_state()
    o.forward_chunk(st2, tokens=tok[:at], logits="all")
    k2 = o.keep(st2)
    o.forward_chunk(st2, tokens=tok[at:at + 3], logits="all")   # the source moves on
    c = o.forward_chunk(k2, tokens=tok[at:], logits="all")
    assert np.array_equal(c["logits"], b["logits"])
