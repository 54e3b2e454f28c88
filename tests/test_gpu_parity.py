"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the same seeded inputs.

The oracle runs in float64 with the bf16 activation boundaries the pages fix ("BF16 activation
boundaries, and FP32 reductions"; TensorFold issue #1491), as the reference's own float64
checker did with "the engine's bf16 rounding points" (TensorFold PR #1508, "Verification").
Sizes span several tiles and ragged tails; the full 24-layer model is checked at the 2048-token
prompt of the decode benchmark, then through teacher-forced greedy decode steps.
"""
import numpy as np
import pytest
import torch

from lfm3_inputs import (lfm3_1p7b, lfm3_slice3, make_weights, make_tokens, make_embeds, page_permutation,
                         synthetic_state, context_lengths)
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


# ------------------------------------------------------------------------------ three-block slice

@pytest.fixture(scope="module")
def slice3():
    g = lfm3_slice3()
    W = make_weights(g, 0)
    return g, W, Lfm3Oracle(W, bf16=True)


def test_slice3_prefill_64_then_8_decode_steps(lib, slice3):
    """The three-block slice: 64 input vectors ~N(0,1), then 8 decode steps (seed 0)."""
    g, W, o = slice3
    x = make_embeds(0, "inputs", 72, g.d_model)
    ref = o.forward_full(x0=f64_rows(x))
    m = lib(W, max_streams=1, max_pages_per_stream=4)
    st = m.new_state()
    xd = bf16_rows(x)
    out = m.prefill(st, 0, embeds=xd[:64], hidden=True)
    torch.cuda.synchronize()
    assert_hidden(out["hidden"], [h[:64] for h in ref["hidden"]], what="prefill")
    for i in range(8):
        o1 = m.decode(st, [0], embeds=xd[64 + i:65 + i], hidden=True)
        torch.cuda.synchronize()
        assert_hidden(o1["hidden"], [h[64 + i:65 + i] for h in ref["hidden"]], what=f"decode {i}")
    assert st.seq_len.cpu().tolist() == [72] and st.h_seq_len.tolist() == [72]
    m.check_device_errors()


def test_slice3_ragged_chunked_prefill_across_the_window(lib, slice3):
    """300 rows in chunks of 128 (ragged tail of 44) crosses the 256 window; then 37 more rows."""
    g, W, o = slice3
    x = make_embeds(1, "ragged", 337, g.d_model)
    ref = o.forward_full(x0=f64_rows(x))
    m = lib(W, max_streams=1, max_pages_per_stream=8, max_chunk=128)
    st = m.new_state(poison=True)
    xd = bf16_rows(x)
    a = m.prefill(st, 0, embeds=xd[:300], hidden=True)
    b = m.prefill(st, 0, embeds=xd[300:], hidden=True)
    torch.cuda.synchronize()
    assert_hidden(a["hidden"], [h[:300] for h in ref["hidden"]], what="first call")
    assert_hidden(b["hidden"], [h[300:] for h in ref["hidden"]], what="second call")
    m.check_device_errors()


def test_slice3_300_row_chunk_on_paired_gemm_tiles(lib, slice3):
    """One 300-row chunk: the 2-SM GEMM tiles cover rows 0..511, so the second tile's upper CTA
    reads only rows past the chunk (zero-filled) and its lower CTA stores a ragged 32-row group."""
    g, W, o = slice3
    x = make_embeds(1, "paired", 300, g.d_model)
    ref = o.forward_full(x0=f64_rows(x))
    m = lib(W, max_streams=1, max_pages_per_stream=8, max_chunk=512)
    st = m.new_state(poison=True)
    out = m.prefill(st, 0, embeds=bf16_rows(x), hidden=True)
    torch.cuda.synchronize()
    assert_hidden(out["hidden"], ref["hidden"], what="300-row chunk")
    m.check_device_errors()


def test_slice3_prompt_equals_one_row_decode_at_cuts(lib, slice3):
    g, W, o = slice3
    x = make_embeds(2, "cuts", 270, g.d_model)
    ref = o.forward_full(x0=f64_rows(x))
    xd = bf16_rows(x)
    m = lib(W, max_streams=1, max_pages_per_stream=8)
    for cut in (1, 63, 64, 255, 256, 262):
        st = m.new_state()
        m.prefill(st, 0, embeds=xd[:cut])
        for t in range(cut, min(cut + 8, 270)):
            out = m.decode(st, [0], embeds=xd[t:t + 1], hidden=True)
            torch.cuda.synchronize()
            assert_hidden(out["hidden"], [h[t:t + 1] for h in ref["hidden"]], what=f"cut {cut} row {t}")


def test_slice3_shuffled_pages_and_poisoned_state_are_exact(lib, slice3):
    g, W, o = slice3
    x = bf16_rows(make_embeds(3, "pages", 333, g.d_model))
    m = lib(W, max_streams=2, max_pages_per_stream=8, n_pages=16)
    outs = []
    for pt, poison in ((None, False), (page_permutation(3, "perm", 16).reshape(2, 8), True)):
        st = m.new_state(page_table=pt, poison=poison)
        a = m.prefill(st, 1, embeds=x[:300], hidden=True)["hidden"].clone()
        b = m.decode(st, [1], embeds=x[300:301], hidden=True)["hidden"].clone()
        outs.append((a, b))
    torch.cuda.synchronize()
    assert torch.isfinite(outs[1][0]).all() and torch.isfinite(outs[1][1]).all()
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1], outs[1][1])


def test_slice3_batched_decode_gemv_and_gemm_paths(lib, slice3):
    """20 streams with their own prompts: a batch of 8 (warp-MMA GEMV path) and of 20
    (tensor-core GEMM path) against the oracle, and batched == solo exactly."""
    g, W, o = slice3
    S = 20
    xs = [make_embeds(4, f"s{s}", 41 + s, g.d_model) for s in range(S)]
    m = lib(W, max_streams=S, max_pages_per_stream=2, max_batch=S)
    st = m.new_state()
    for s in range(S):
        m.prefill(st, s, embeds=bf16_rows(xs[s][:-1]))
    last = torch.cat([bf16_rows(xs[s][-1:]) for s in range(S)])
    # batch of 8 (GEMV) on a copy of the state, then each of those alone
    st8 = m.new_state()
    for t in ("conv", "ring_k", "ring_v", "kv_k", "kv_v", "seq_len"):
        getattr(st8, t).copy_(getattr(st, t))
    st8.h_seq_len[:] = st.h_seq_len
    batch8 = m.decode(st8, list(range(8)), embeds=last[:8], hidden=True)["hidden"].clone()
    st_solo = m.new_state()
    for t in ("conv", "ring_k", "ring_v", "kv_k", "kv_v", "seq_len"):
        getattr(st_solo, t).copy_(getattr(st, t))
    st_solo.h_seq_len[:] = st.h_seq_len
    solo = [m.decode(st_solo, [s], embeds=last[s:s + 1], hidden=True)["hidden"].clone() for s in range(8)]
    big = m.decode(st, list(range(S)), embeds=last, hidden=True)["hidden"].clone()
    torch.cuda.synchronize()
    for s in range(S):
        ref = o.forward_full(x0=f64_rows(xs[s]))
        assert_hidden(big[:, s:s + 1], [h[-1:] for h in ref["hidden"]], what=f"B=20 stream {s}")
        if s < 8:
            assert_hidden(batch8[:, s:s + 1], [h[-1:] for h in ref["hidden"]], what=f"B=8 stream {s}")
            assert torch.equal(batch8[:, s:s + 1], solo[s]), s


def test_capacity_refusal_leaves_state_untouched(lib, slice3):
    from attention_decoder_b200 import Lfm3Error
    g, W, o = slice3
    x = bf16_rows(make_embeds(5, "cap", 200, g.d_model))
    m = lib(W, max_streams=1, max_pages_per_stream=2)
    st = m.new_state()
    m.prefill(st, 0, embeds=x[:100])
    with pytest.raises(Lfm3Error) as e:
        m.prefill(st, 0, embeds=x[100:200])
    assert e.value.status == -3
    torch.cuda.synchronize()
    assert st.h_seq_len.tolist() == [100] and st.seq_len.cpu().tolist() == [100]
    m.decode(st, [0], embeds=x[100:101])
    assert st.h_seq_len.tolist() == [101]


# ------------------------------------------------------------------------------ full model, bf16

@pytest.fixture(scope="module")
def full_bf16():
    g = lfm3_1p7b()
    W = make_weights(g, 0)
    tok = make_tokens(1, "prompt", 2048, g.vocab)
    o = Lfm3Oracle(W, bf16=True)
    st = o.new_state()
    ref = o.forward_chunk(st, tokens=tok)
    fed, lg = o.greedy(st, int(np.argmax(ref["logits"])), 3)
    return g, W, tok, ref, fed, lg


def test_full_model_prefill_2048_and_greedy_decode(lib, full_bf16):
    g, W, tok, ref, fed, lg = full_bf16
    m = lib(W, max_streams=1, max_pages_per_stream=40)
    st = m.new_state(poison=True)
    out = m.prefill(st, 0, tokens=torch.from_numpy(tok).cuda(), hidden=True)
    torch.cuda.synchronize()
    assert_hidden(out["hidden"], ref["hidden"], what="prefill 2048")
    assert_logits(out["logits"], ref["logits"], out["argmax"], what="prefill logits")
    for i, t in enumerate(fed):
        o1 = m.decode(st, [0], tokens=torch.tensor([t], dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        assert_logits(o1["logits"][0], lg[i], o1["argmax"], what=f"decode {i}")
    m.check_device_errors()


# ------------------------------------------------------------------------------ full model, NVFP4 FFN

def test_nvfp4_model_prefill_and_batched_decode(lib):
    g = lfm3_1p7b()
    W = make_weights(g, 0, ffn="nvfp4")
    o = Lfm3Oracle(W, bf16=True)
    B, n = 4, 200
    toks = [make_tokens(1, f"nvfp4.s{s}", n + 1, g.vocab) for s in range(B)]
    m = lib(W, max_streams=B, max_pages_per_stream=4, max_batch=B)
    st = m.new_state()
    refs = []
    for s in range(B):
        ost = o.new_state()
        r = o.forward_chunk(ost, tokens=toks[s][:n])
        d = o.forward_chunk(ost, tokens=toks[s][n:])
        refs.append((r, d))
        out = m.prefill(st, s, tokens=torch.from_numpy(toks[s][:n]).cuda())
        torch.cuda.synchronize()
        assert_logits(out["logits"], r["logits"], out["argmax"], what=f"nvfp4 prefill {s}")
    last = torch.from_numpy(np.array([t[n] for t in toks], dtype=np.int32)).cuda()
    out = m.decode(st, list(range(B)), tokens=last)
    torch.cuda.synchronize()
    for s in range(B):
        assert_logits(out["logits"][s], refs[s][1]["logits"], out["argmax"][s:s + 1], what=f"nvfp4 decode {s}")


# ------------------------------------------------------------------------------ 64 streams, drawn state

def test_nvfp4_64_streams_on_drawn_state_sampled(lib):
    """64 NVFP4 streams with contexts uniform in [256, 8192] (the batched-decode workload), shuffled
    pages and drawn K/V, conv and ring state; eight streams checked, the shortest and the longest
    among them."""
    g = lfm3_1p7b()
    W = make_weights(g, 0, ffn="nvfp4")
    B = 64
    ctx = context_lengths(1, "ctx64", B, 256, 8192)
    syn = synthetic_state(g, 1, ctx)
    mpp = 8192 // 64 + 1
    m = lib(W, max_streams=B, max_pages_per_stream=mpp, max_batch=B)
    pt = page_permutation(1, "pages64", B * mpp).reshape(B, mpp)
    st = m.new_state(page_table=pt)
    st.load_synthetic(syn, ctx)
    tok = make_tokens(1, "tok64", B, g.vocab)
    out = m.decode(st, list(range(B)), tokens=torch.from_numpy(tok).cuda())
    torch.cuda.synchronize()
    o = Lfm3Oracle(W, bf16=True)
    order = np.argsort(ctx, kind="stable")
    picks = sorted({int(order[0]), int(order[-1]), 0, 13, 29, 37, 50, 63})
    for s in picks:
        ost = o.state_from_synthetic(syn, s, int(ctx[s]))
        r = o.forward_chunk(ost, tokens=tok[s:s + 1])
        assert_logits(out["logits"][s], r["logits"], out["argmax"][s:s + 1], what=f"B=64 stream {s} ctx {ctx[s]}")
    assert st.h_seq_len.tolist() == [int(c) + 1 for c in ctx]


def test_graph_replay_equals_direct_launches_and_profile_counts(lib, slice3, monkeypatch):
    """Decode steps replayed from the library's CUDA graph give bit-identical state and outputs to
    direct launches; the measurement brackets count the projection launches."""
    g, W, o = slice3
    x = bf16_rows(make_embeds(6, "graph", 80, g.d_model))
    runs = []
    for no_graph in (False, True):
        if no_graph:
            monkeypatch.setenv("LFM3_NO_GRAPH", "1")
        m = lib(W, max_streams=1, max_pages_per_stream=4)
        st = m.new_state()
        m.prefill(st, 0, embeds=x[:70])
        hs = [m.decode(st, [0], embeds=x[t:t + 1], hidden=True)["hidden"].clone() for t in range(70, 80)]
        torch.cuda.synchronize()
        runs.append((hs, st.conv.clone(), st.kv_k.clone(), st.ring_v.clone()))
        launches = m.last_launch_count()
        assert launches > 10
        if no_graph:
            m.profile(True, capacity=64)
            m.decode(st, [0], embeds=x[:1])
            p = m.profile_read()
            m.profile(False)
            # conv layer: in_proj+conv, out_proj, w1|w3, w2; attention layers: qkvg, o_proj, w1|w3, w2
            wbytes = 2 * (3 * 2048 * 2048 + 2048 * 2048 + 2 * 3088 * 2048 + 2 * 2048 * 2048 + 3 * 3 * 7680 * 2048)
            assert p["launches"] == 12 and p["ms"] > 0
            assert wbytes < p["bytes"] < wbytes * 1.01
    for a, b in zip(runs[0][0], runs[1][0]):
        assert torch.equal(a, b)
    for i in (1, 2, 3):
        assert torch.equal(runs[0][i], runs[1][i])
