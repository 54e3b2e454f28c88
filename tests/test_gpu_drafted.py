"""Drafted windows through the C ABI: lfm3_verify and lfm3_commit.

TensorFold PR #1508 verifies its engine with "drafted == plain": greedy decode that checks W drafted
tokens per pass and commits the accepted prefix must produce what one-token decode produces. Here
the drafts are the plain run's own continuation with planted wrong tokens, so windows are accepted
in full, in part and down to one row; the drafted tokens, logits and final state equal the plain
run's. The window rows are also checked against the oracle (a window is a chunk of the stream's
next rows), on both the weight-streaming path (<= 16 rows) and the GEMM path (> 16 rows).
"""
import numpy as np
import pytest
import torch

from lfm3_inputs import lfm3_1p7b, lfm3_slice3, make_weights, make_tokens, make_embeds
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
def head4():
    g = lfm3_1p7b(layer_types=(0, 2, 1, 0))   # conv, sliding, full, conv + the tied head
    W = make_weights(g, 0)
    return g, W


def _copy(m, src):
    dst = m.new_state()
    for t in ("conv", "ring_k", "ring_v", "kv_k", "kv_v", "seq_len"):
        getattr(dst, t).copy_(getattr(src, t))
    dst.h_seq_len[:] = src.h_seq_len
    return dst


def test_drafted_equals_plain(lib, head4):
    g, W = head4
    S, N, WIN = 2, 14, 4
    prompts = [make_tokens(5, "drafted.p0", 37, g.vocab), make_tokens(5, "drafted.p1", 300, g.vocab)]
    m = lib(W, max_streams=S, max_pages_per_stream=8, max_batch=S * WIN)
    st = m.new_state()
    first = []
    for s in range(S):
        first.append(int(m.prefill(st, s, tokens=torch.from_numpy(prompts[s]).cuda())["argmax"].item()))
    # plain: one token per step for both streams
    plain = _copy(m, st)
    toks = [[first[0]], [first[1]]]
    plain_logits = [[], []]
    for _ in range(N):
        o = m.decode(plain, [0, 1], tokens=torch.tensor([toks[0][-1], toks[1][-1]], dtype=torch.int32, device="cuda"))
        for s in range(S):
            plain_logits[s].append(o["logits"][s].clone())
            toks[s].append(int(o["argmax"][s].item()))
    # drafted: W rows per pass, drafts taken from the plain continuation, some planted wrong
    dr = _copy(m, st)
    got = [[first[0]], [first[1]]]
    got_logits = [[], []]
    wrong = make_tokens(5, "drafted.wrong", 64, g.vocab)
    it = 0
    while min(len(x) for x in got) <= N + 1:
        window = []
        for s in range(S):
            n = len(got[s])
            drafts = [toks[s][n + j] if n + j < len(toks[s]) else 0 for j in range(WIN - 1)]
            # plant a wrong draft: stream 1 every other pass at draft 1, stream 0 every third at draft 0
            if s == 1 and it % 2 == 0:
                drafts[1] = int(wrong[it]) if int(wrong[it]) != drafts[1] else (drafts[1] + 1) % g.vocab
            if s == 0 and it % 3 == 1:
                drafts[0] = int(wrong[it]) if int(wrong[it]) != drafts[0] else (drafts[0] + 1) % g.vocab
            window.append([got[s][-1]] + drafts)
        o = m.verify(dr, [0, 1], WIN, tokens=torch.tensor(np.array(window).reshape(-1), dtype=torch.int32).cuda())
        am = o["argmax"].view(S, WIN).cpu().numpy()
        accept = []
        for s in range(S):
            k = 1
            while k < WIN and window[s][k] == am[s][k - 1]:
                k += 1
            accept.append(k)
            for j in range(k):
                got[s].append(int(am[s][j]))
                got_logits[s].append(o["logits"][s * WIN + j].clone())
        m.commit(dr, [0, 1], accept)
        it += 1
    assert it < N, "every window was accepted only one row at a time"
    for s in range(S):
        assert got[s][:N + 1] == toks[s][:N + 1], s
        for j in range(N):
            assert torch.equal(got_logits[s][j], plain_logits[s][j]), (s, j)
    # every token but the last of each drafted run has been consumed, and the committed state goes
    # on like the plain one: one more plain step from each agrees exactly
    assert dr.h_seq_len.tolist() == [len(p) + len(x) - 1 for p, x in zip(prompts, got)]
    oa = m.decode(plain, [0, 1], tokens=torch.tensor([toks[0][N], toks[1][N]], dtype=torch.int32, device="cuda"))
    assert [int(v) for v in oa["argmax"].tolist()] == [got[0][N + 1], got[1][N + 1]]


def test_window_rows_match_the_oracle_on_both_paths(lib, head4):
    """5 streams x 4 rows (20 rows: the GEMM path) and 2 x 4 (the weight-streaming path)."""
    g, W = head4
    o = Lfm3Oracle(W, bf16=True)
    for S in (2, 5):
        WIN = 4
        prompts = [make_tokens(6, f"win{S}.p{s}", 50 + 67 * s, g.vocab) for s in range(S)]
        windows = [make_tokens(6, f"win{S}.w{s}", WIN, g.vocab) for s in range(S)]
        m = lib(W, max_streams=S, max_pages_per_stream=8, max_batch=S * WIN)
        st = m.new_state(poison=True)
        for s in range(S):
            m.prefill(st, s, tokens=torch.from_numpy(prompts[s]).cuda(), logits=False, argmax=False)
        out = m.verify(st, list(range(S)), WIN, tokens=torch.from_numpy(np.concatenate(windows)).cuda(), hidden=True)
        torch.cuda.synchronize()
        assert st.h_seq_len.tolist() == [len(p) for p in prompts]      # nothing committed yet
        for s in range(S):
            ost = o.new_state()
            o.forward_chunk(ost, tokens=prompts[s], logits=None)
            ref = o.forward_chunk(ost, tokens=windows[s], logits="all")
            rows = slice(s * WIN, (s + 1) * WIN)
            assert_hidden(out["hidden"][:, rows], ref["hidden"], what=f"S={S} stream {s}")
            for j in range(WIN):
                assert_logits(out["logits"][s * WIN + j], ref["logits"][j], out["argmax"][s * WIN + j:s * WIN + j + 1],
                              what=f"S={S} stream {s} row {j}")
        # commit two rows of every stream; the next step sees exactly those rows
        m.commit(st, list(range(S)), [2] * S)
        nxt = make_tokens(6, f"win{S}.next", S, g.vocab)
        d = m.decode(st, list(range(S)), tokens=torch.from_numpy(nxt).cuda())
        torch.cuda.synchronize()
        for s in range(S):
            ost = o.new_state()
            o.forward_chunk(ost, tokens=np.concatenate([prompts[s], windows[s][:2]]), logits=None)
            r = o.forward_chunk(ost, tokens=nxt[s:s + 1])
            assert_logits(d["logits"][s], r["logits"], d["argmax"][s:s + 1], what=f"S={S} after commit, stream {s}")


def test_slice_window_hidden_states_across_the_ring_wrap(lib):
    g = lfm3_slice3()
    W = make_weights(g, 0)
    x = make_embeds(11, "window.slice", 262, g.d_model)
    ref = Lfm3Oracle(W, bf16=True).forward_full(x0=f64_rows(x))["hidden"]
    xd = bf16_rows(x)
    m = lib(W, max_streams=1, max_pages_per_stream=6, max_batch=8)
    st = m.new_state(poison=True)
    m.prefill(st, 0, embeds=xd[:254])
    out = m.verify(st, [0], 8, embeds=xd[254:262], hidden=True)   # positions 254..261 cross slot 255 -> 0
    torch.cuda.synchronize()
    assert_hidden(out["hidden"], [h[254:262] for h in ref], what="window across the wrap")
    m.commit(st, [0], [5])
    d = m.decode(st, [0], embeds=xd[259:260], hidden=True)
    torch.cuda.synchronize()
    assert_hidden(d["hidden"], [h[259:260] for h in ref], what="decode after a 5-row commit")


def test_verify_and_commit_refusals(lib, head4):
    from attention_decoder_b200 import Lfm3Error
    g, W = head4
    m = lib(W, max_streams=2, max_pages_per_stream=2, max_batch=8)
    st = m.new_state()
    m.prefill(st, 0, tokens=torch.from_numpy(make_tokens(7, "refuse", 20, g.vocab)).cuda())
    with pytest.raises(Lfm3Error) as e:
        m.commit(st, [0], [1])
    assert e.value.status == -7                                    # no window
    t = torch.zeros(9, dtype=torch.int32, device="cuda")
    with pytest.raises(Lfm3Error) as e:
        m.verify(st, [0], 9, tokens=t)
    assert e.value.status == -1                                    # window longer than 8
    m.verify(st, [0], 4, tokens=t[:4])
    with pytest.raises(Lfm3Error) as e:
        m.commit(st, [0], [5])
    assert e.value.status == -1                                    # more rows than the window
    m.decode(st, [0], tokens=t[:1])
    with pytest.raises(Lfm3Error) as e:
        m.commit(st, [0], [2])
    assert e.value.status == -7                                    # the window was ended
    st.h_seq_len[0] = 126
    st.seq_len[0] = 126
    with pytest.raises(Lfm3Error) as e:
        m.verify(st, [0], 4, tokens=t[:4])                          # 126 + 4 > 2 pages of 64
    assert e.value.status == -3
