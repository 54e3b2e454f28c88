"""GPU parity of the persistent decode step (one launch per token step, up to four streams;
opt-in with LFM3_PERSISTENT=1, which every model here sets).

Each case runs the same prompts and decode rows through the persistent step and checks every
layer's hidden state against the bf16-boundary float64 oracle; batched == solo exactly; the
per-projection path (the default) is checked beside it on the same rows; the step's
measurement bracket counts one launch and the algorithmic bytes (every weight once plus the
cached keys and values read).
"""
import numpy as np
import pytest
import torch

from lfm3_inputs import lfm3_slice3, make_weights, make_embeds, page_permutation
from oracle import Lfm3Oracle
from parity import assert_hidden, bf16_rows, f64_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_decoder_b200 import build
    build.build(verbose=False)
    from attention_decoder_b200.model import Lfm3Model
    return Lfm3Model


@pytest.fixture(autouse=True)
def persistent(monkeypatch):
    monkeypatch.setenv("LFM3_PERSISTENT", "1")


@pytest.fixture(scope="module")
def slice3():
    g = lfm3_slice3()
    W = make_weights(g, 0)
    return g, W, Lfm3Oracle(W, bf16=True)


def _copy_state(m, src):
    st = m.new_state(page_table=src.h_page_table)
    for t in ("conv", "ring_k", "ring_v", "kv_k", "kv_v", "seq_len"):
        getattr(st, t).copy_(getattr(src, t))
    st.h_seq_len[:] = src.h_seq_len
    return st


def test_persistent_four_streams_ragged_contexts(lib, slice3):
    """Four streams whose contexts straddle the 256-slot window and several 128-key splits
    (37, 255, 300, 513 positions), shuffled pages: batch of 4, then each alone, 3 steps."""
    g, W, o = slice3
    lens = [37, 255, 300, 513]
    steps = 3
    xs = [make_embeds(7, f"p{s}", n + steps, g.d_model) for s, n in enumerate(lens)]
    mpp = 10
    pt = page_permutation(7, "pages", 4 * mpp).reshape(4, mpp)
    m = lib(W, max_streams=4, max_pages_per_stream=mpp, max_batch=4)
    st = m.new_state(page_table=pt, poison=True)
    for s, n in enumerate(lens):
        m.prefill(st, s, embeds=bf16_rows(xs[s][:n]))
    st_solo = _copy_state(m, st)
    refs = [o.forward_full(x0=f64_rows(x)) for x in xs]
    for t in range(steps):
        rows = torch.cat([bf16_rows(xs[s][lens[s] + t:lens[s] + t + 1]) for s in range(4)])
        hb = m.decode(st, [0, 1, 2, 3], embeds=rows, hidden=True)["hidden"].clone()
        solo = [m.decode(st_solo, [s], embeds=rows[s:s + 1], hidden=True)["hidden"].clone() for s in range(4)]
        torch.cuda.synchronize()
        assert m.last_launch_count() == 1
        for s in range(4):
            p = lens[s] + t
            assert_hidden(hb[:, s:s + 1], [h[p:p + 1] for h in refs[s]["hidden"]], what=f"step {t} stream {s}")
            assert torch.equal(hb[:, s:s + 1], solo[s]), (t, s)
    m.check_device_errors()
    assert st.h_seq_len.tolist() == [n + steps for n in lens]
    assert st.seq_len.cpu().tolist() == [n + steps for n in lens]
    for t in ("conv", "ring_k", "ring_v", "kv_k", "kv_v"):
        # bitwise (the poisoned, never-written rows are NaN on both sides)
        assert torch.equal(getattr(st, t).view(torch.int16), getattr(st_solo, t).view(torch.int16)), t


def test_persistent_matches_per_projection_path(lib, slice3, monkeypatch):
    """The same 6 decode steps after a 250-row prompt through both decode paths: both within the
    oracle's tolerance, and the state they leave close (bf16 rounding of the new keys may differ
    by one unit where the two summation orders straddle a rounding boundary)."""
    g, W, o = slice3
    x = make_embeds(8, "both", 256, g.d_model)
    ref = o.forward_full(x0=f64_rows(x))
    outs = []
    for off in (False, True):
        if off:
            monkeypatch.delenv("LFM3_PERSISTENT")
        m = lib(W, max_streams=1, max_pages_per_stream=4)
        st = m.new_state()
        m.prefill(st, 0, embeds=bf16_rows(x[:250]))
        hs = [m.decode(st, [0], embeds=bf16_rows(x[t:t + 1]), hidden=True)["hidden"].clone() for t in range(250, 256)]
        torch.cuda.synchronize()
        if not off:
            assert m.last_launch_count() == 1
        for i, h in enumerate(hs):
            assert_hidden(h, [r[250 + i:251 + i] for r in ref["hidden"]], what=f"{'multi' if off else 'persistent'} {i}")
        outs.append((st.kv_k.float(), st.ring_k.float(), st.conv.float()))
    for a, b in zip(outs[0], outs[1]):
        assert torch.allclose(a, b, rtol=2e-2, atol=2e-2)


def test_persistent_profile_counts_one_launch_and_its_bytes(lib, slice3):
    g, W, o = slice3
    x = bf16_rows(make_embeds(9, "prof", 101, g.d_model))
    m = lib(W, max_streams=1, max_pages_per_stream=4)
    st = m.new_state()
    m.prefill(st, 0, embeds=x[:100])
    m.profile(True, capacity=8)
    m.decode(st, [0], embeds=x[100:101])
    p = m.profile_read()
    m.profile(False)
    wbytes = 2 * (3 * 2048 * 2048 + 2048 * 2048 + 2 * 3088 * 2048 + 2 * 2048 * 2048 + 3 * 3 * 7680 * 2048)
    kv = 2 * 2 * 4 * 128 * (101 + 101)  # one full and one sliding layer, 101 keys each, K and V
    assert p["launches"] == 1 and p["ms"] > 0
    assert p["bytes"] == pytest.approx(wbytes + kv, rel=1e-9)
