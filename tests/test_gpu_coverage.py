"""GPU parity at the workloads' own sizes and on the paths the smaller tests do not reach.

* The long-prompt workload (8192 rows in 2048-row chunks over a shuffled page pool): the three-
  block slice, every layer's hidden state against the oracle's full-sequence pass. Later chunks
  run the paired 2-SM GEMM tiles and the tensor-core attention over 2k-6k keys of history read
  through the page table, and the sliding layer's ring across chunk seams.
* 9 to 16 streams: the weight-streaming kernels' two-column-tile form, bf16 and NVFP4.
* The failure path: a bounded device wait that runs out is reported as LFM3_E_TIMEOUT by
  lfm3_check_device_errors, and the context keeps giving exact results afterwards.

The 64-stream workload (contexts uniform in [256, 8192]) is in test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

from lfm3_inputs import lfm3_1p7b, lfm3_slice3, make_weights, make_tokens, make_embeds, page_permutation
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


def test_slice3_8192_rows_in_2048_row_chunks_over_shuffled_pages(lib):
    g = lfm3_slice3()
    W = make_weights(g, 0)
    n, mpp, pool = 8192, 8192 // 64, 160
    x = make_embeds(1, "long8k", n, g.d_model)
    ref = Lfm3Oracle(W, bf16=True).forward_full(x0=f64_rows(x))["hidden"]
    pt = page_permutation(1, "long8k.pages", pool)[:mpp].reshape(1, mpp)
    m = lib(W, max_streams=1, max_pages_per_stream=mpp, n_pages=pool, max_chunk=2048)
    st = m.new_state(page_table=pt, poison=True)
    out = m.prefill(st, 0, embeds=bf16_rows(x), hidden=True)
    torch.cuda.synchronize()
    got = out["hidden"]
    assert torch.isfinite(got).all()
    for c in range(4):
        rows = slice(2048 * c, 2048 * (c + 1))
        assert_hidden(got[:, rows], [h[rows] for h in ref], what=f"chunk {c}")
    assert st.seq_len.cpu().tolist() == [n]
    m.check_device_errors()


@pytest.mark.parametrize("ffn", ["bf16", "nvfp4"])
def test_twelve_streams_use_the_two_column_tiles(lib, ffn):
    """12 streams (more than one 8-column MMA tile) through the weight-streaming kernels with
    every epilogue: conv, q|k|v|gate and attention, SwiGLU, down-projection and the tied head."""
    g = lfm3_1p7b(layer_types=(0, 2, 1, 0))
    W = make_weights(g, 0, ffn=ffn)
    o = Lfm3Oracle(W, bf16=True)
    S = 12
    toks = [make_tokens(2, f"nt2.{ffn}.s{s}", 30 + 23 * s, g.vocab) for s in range(S)]
    m = lib(W, max_streams=S, max_pages_per_stream=6, max_batch=S)
    st = m.new_state(poison=True)
    refs = []
    for s in range(S):
        m.prefill(st, s, tokens=torch.from_numpy(toks[s][:-1]).cuda(), logits=False, argmax=False)
        ost = o.new_state()
        o.forward_chunk(ost, tokens=toks[s][:-1], logits=None)
        refs.append(o.forward_chunk(ost, tokens=toks[s][-1:]))
    last = torch.from_numpy(np.array([t[-1] for t in toks], dtype=np.int32)).cuda()
    out = m.decode(st, list(range(S)), tokens=last, hidden=True)
    torch.cuda.synchronize()
    for s in range(S):
        assert_hidden(out["hidden"][:, s:s + 1], [h for h in refs[s]["hidden"]], what=f"{ffn} stream {s}")
        assert_logits(out["logits"][s], refs[s]["logits"], out["argmax"][s:s + 1], what=f"{ffn} stream {s}")
    assert st.h_seq_len.tolist() == [len(t) for t in toks]


def test_bounded_wait_that_runs_out_is_reported_and_the_context_stays_usable(lib):
    from attention_decoder_b200 import Lfm3Error
    g = lfm3_slice3()
    W = make_weights(g, 0)
    x = bf16_rows(make_embeds(8, "timeout", 90, g.d_model))
    m = lib(W, max_streams=1, max_pages_per_stream=4)
    a, b = m.new_state(), m.new_state()
    for st in (a, b):
        m.prefill(st, 0, embeds=x[:88])
    ha = m.decode(a, [0], embeds=x[88:89], hidden=True)["hidden"].clone()
    m.check_device_errors()
    m.selftest_wait(rounds=4096)
    with pytest.raises(Lfm3Error) as e:
        m.check_device_errors()
    assert e.value.status == -6 and "gave up" in str(e.value)
    m.check_device_errors()  # the word was cleared
    assert b.h_seq_len.tolist() == [88] and b.seq_len.cpu().tolist() == [88]
    hb = m.decode(b, [0], embeds=x[88:89], hidden=True)["hidden"]
    torch.cuda.synchronize()
    assert torch.equal(ha, hb)
    for t in ("conv", "ring_k", "kv_k", "kv_v"):
        assert torch.equal(getattr(a, t), getattr(b, t)), t
    m.check_device_errors()
