"""Pins of the oracle's token lookup, tied head and greedy loop, and of the whole decoder's
composition, against torch code written independently of the oracle (CPU only).

coreai-model-zoo note "lfm3-1.7b-port", "Unchanged" paragraph: the 128000-row head is tied to
the token embedding and reads the output of the final embedding_norm (an RMSNorm with eps
1e-5 whose gain multiplies directly). Greedy selection takes the largest logit; on an exact tie
the lowest id wins (the reading the pages' router gives: "ties to the lower id", TensorFold
PR #1508). Each pin is paired with planted mistakes - built here, on the CPU, as subclasses
of the oracle - that the same comparison must reject.
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

from lfm3_inputs import CONV, FULL, SLIDING, tiny_geometry, make_weights, make_tokens
from oracle import Lfm3Oracle, rms_norm


def _tb(bits):
    """bf16 bit patterns -> float64 torch tensor, through torch's own bf16 type."""
    a = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16)).view(np.int16)
    return torch.from_numpy(a).view(torch.bfloat16).to(torch.float64)


@pytest.fixture(scope="module")
def tiny():
    g = tiny_geometry()
    return g, make_weights(g, 0)


# ---------------------------------------------------------------- token lookup

def test_embed_tokens_is_a_row_lookup_of_the_bf16_table(tiny):
    g, W = tiny
    o = Lfm3Oracle(W)
    tok = np.array([0, g.vocab - 1, 5, 5, 17, 0, 96 % g.vocab])
    ref = Fn.embedding(torch.from_numpy(tok), _tb(W["embed"])).numpy()
    assert np.array_equal(o.embed_tokens(tok), ref)

    class OffByOne(Lfm3Oracle):
        def embed_tokens(self, tokens):
            return self.embed[(np.asarray(tokens) + 1) % self.g.vocab].astype(self.dtype)

    class Transposed(Lfm3Oracle):  # reads column t of a [D, V] view instead of row t
        def embed_tokens(self, tokens):
            return self.embed.reshape(self.g.d_model, self.g.vocab)[:, np.asarray(tokens)].T.astype(self.dtype)

    for bad in (OffByOne(W), Transposed(W)):
        assert np.abs(bad.embed_tokens(tok) - ref).max() > 1e-3, type(bad).__name__


# ---------------------------------------------------------------- final norm + tied head

def _torch_logits(W, g, x):
    xn = Fn.rms_norm(torch.from_numpy(x), (g.d_model,), weight=_tb(W["final_norm"]), eps=g.eps)
    return Fn.linear(xn, _tb(W["embed"])).numpy()


def test_logits_are_final_rmsnorm_then_the_tied_embedding(tiny):
    g, W = tiny
    o = Lfm3Oracle(W)
    x = np.random.default_rng(21).standard_normal((11, g.d_model)) * 3.0
    ref = _torch_logits(W, g, x)
    assert np.allclose(o.logits(x), ref, rtol=1e-12, atol=1e-12)

    class Untied(Lfm3Oracle):  # a separate random head instead of the embedding
        def logits(self, x):
            head = np.random.default_rng(3).standard_normal(self.embed.shape) * 0.02
            return rms_norm(x, self.final_norm, self.g.eps) @ head.T

    class NoFinalNorm(Lfm3Oracle):
        def logits(self, x):
            return x @ self.embed.T.astype(self.dtype)

    class OnePlusGain(Lfm3Oracle):  # the (1 + g) gain convention
        def logits(self, x):
            return rms_norm(x, 1.0 + self.final_norm, self.g.eps) @ self.embed.T.astype(self.dtype)

    class NormOverRows(Lfm3Oracle):  # the RMS taken over the wrong axis
        def logits(self, x):
            ms = np.mean(x * x, axis=0, keepdims=True)
            return (x / np.sqrt(ms + self.g.eps) * self.final_norm) @ self.embed.T.astype(self.dtype)

    for bad in (Untied(W), NoFinalNorm(W), OnePlusGain(W), NormOverRows(W)):
        assert np.abs(bad.logits(x) - ref).max() > 1e-3, type(bad).__name__


# ---------------------------------------------------------------- greedy loop

def test_greedy_feeds_back_each_argmax_and_breaks_ties_to_the_lowest_id(tiny):
    g, W = tiny
    o = Lfm3Oracle(W)
    script = [np.array([0.0, 2.0, 2.0, 1.0]),     # tie between 1 and 2 -> 1
              np.array([5.0, -1.0, 5.0, 5.0]),    # three-way tie -> 0
              np.array([-3.0, -2.0, -1.0, -1.0])]
    seen = []

    def scripted(st, tokens=None, x0=None, logits="last"):
        seen.append(int(np.asarray(tokens).reshape(-1)[0]))
        return {"hidden": [], "logits": script[len(seen) - 1]}

    o.forward_chunk = scripted
    fed, lg = o.greedy(None, 9, 3)
    assert fed.tolist() == [9, 1, 0] and seen == [9, 1, 0]
    assert np.array_equal(lg, np.stack(script))


def test_greedy_chain_equals_argmax_of_the_full_sequence_pass(tiny):
    g, W = tiny
    o = Lfm3Oracle(W)
    prompt = make_tokens(1, "greedy", 6, g.vocab)
    st = o.new_state()
    first = int(np.argmax(o.forward_chunk(st, tokens=prompt)["logits"]))
    fed, lg = o.greedy(st, first, 5)
    full = o.forward_full(tokens=np.concatenate([prompt, fed]), logits="all")["logits"]
    assert np.allclose(lg, full[len(prompt):], rtol=1e-10, atol=1e-10)
    chain = [first] + [int(np.argmax(full[len(prompt) + i])) for i in range(4)]
    assert fed.tolist() == chain


# ---------------------------------------------------------------- whole decoder in torch

def _torch_decoder(W, g, tokens):
    """The LFM3 decoder written with torch primitives (embedding, rms_norm, linear, depthwise
    conv1d, scaled_dot_product_attention with repeat-kv and a band mask, rotary as a complex
    rotation), full sequence, float64. Returns the logits of every row."""
    T, D, d = len(tokens), g.d_model, g.head_dim
    x = Fn.embedding(torch.from_numpy(np.asarray(tokens)), _tb(W["embed"]))
    pos = torch.arange(T, dtype=torch.float64)
    rms = lambda v, gain, n: Fn.rms_norm(v, (n,), weight=_tb(gain), eps=g.eps)
    for kind, L in zip(g.layer_types, W["layers"]):
        xn = rms(x, L["op_norm"], D)
        if kind == CONV:
            B, C, X = Fn.linear(xn, _tb(L["in_proj"])).T.chunk(3, dim=0)
            z = Fn.conv1d((B * X)[None], _tb(L["conv"])[:, None, :], padding=g.conv_taps - 1, groups=D)[0, :, :T]
            m = Fn.linear((C * z).T, _tb(L["out_proj"]))
        else:
            q = rms(Fn.linear(xn, _tb(L["q_proj"])).view(T, g.n_q, d), L["q_norm"], d)
            k = rms(Fn.linear(xn, _tb(L["k_proj"])).view(T, g.n_kv, d), L["k_norm"], d)
            v = Fn.linear(xn, _tb(L["v_proj"])).view(T, g.n_kv, d)
            gate = torch.sigmoid(Fn.linear(xn, _tb(L["gate_proj"])))
            theta = g.theta_full if kind == FULL else g.theta_sliding
            pairs = g.rope_pairs_full if kind == FULL else d // 2
            f = torch.tensor([theta ** (-2.0 * i / d) if i < pairs else 0.0 for i in range(d // 2)],
                             dtype=torch.float64)
            rot = torch.polar(torch.ones(T, 1, d // 2, dtype=torch.float64), pos[:, None, None] * f)

            def rope(a):
                c = torch.complex(a[..., :d // 2], a[..., d // 2:]) * rot
                return torch.cat([c.real, c.imag], dim=-1)
            rep = g.n_q // g.n_kv
            qh = rope(q).permute(1, 0, 2)
            kh = rope(k).repeat_interleave(rep, dim=1).permute(1, 0, 2)
            vh = v.repeat_interleave(rep, dim=1).permute(1, 0, 2)
            dq = torch.arange(T)[:, None] - torch.arange(T)[None, :]
            mask = dq >= 0
            if kind == SLIDING:
                mask &= dq < g.window
            o = Fn.scaled_dot_product_attention(qh, kh, vh, attn_mask=mask).permute(1, 0, 2)
            m = Fn.linear((o * gate[:, :, None]).reshape(T, -1), _tb(L["o_proj"]))
        h = x + rms(m, L["post_op_norm"], D)
        hn = rms(h, L["ffn_norm"], D)
        u = Fn.silu(Fn.linear(hn, _tb(L["w1"]))) * Fn.linear(hn, _tb(L["w3"]))
        x = h + rms(Fn.linear(u, _tb(L["w2"])), L["post_ffn_norm"], D)
    return Fn.linear(rms(x, W["final_norm"], D), _tb(W["embed"])).numpy()


def test_whole_decoder_logits_against_an_independent_torch_assembly(tiny):
    """20 tokens (more than the window of 8, so the sliding layers' band bites) through the
    tiny geometry's six layers of all three kinds: every row's logits agree to 1e-9."""
    g, W = tiny
    tok = make_tokens(1, "whole", 20, g.vocab)
    ref = _torch_decoder(W, g, tok)
    mine = Lfm3Oracle(W).forward_full(tokens=tok, logits="all")["logits"]
    assert np.allclose(mine, ref, rtol=1e-9, atol=1e-9), np.abs(mine - ref).max()
    # the same comparison rejects the planted whole-model mistakes (by far more than the 1e-9
    # agreement: the tiny model's logits are O(0.1), so a rotary slip moves them by ~1e-4)
    for kw in (dict(gate=False), dict(rope_all_dims=True), dict(window=False)):
        bad = Lfm3Oracle(W, **kw).forward_full(tokens=tok, logits="all")["logits"]
        assert np.abs(bad - ref).max() > 1e-6, kw
