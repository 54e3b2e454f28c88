"""lfm3_decode_step_noalloc: the decode step for callers that cannot allocate device memory.

Such callers (a host program that gives the library a finished arena and forbids allocation
afterwards, or code where an allocation would synchronise the device) get the same step with the
attention's scratch held in a fixed array inside the library. This file runs last so that a
failure here does not hide the other GPU tests; it must pass alone in a fresh process and after
them. Two consecutive calls are compared with lfm3_decode_step on identical copies of the state.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from lfm3_inputs import lfm3_1p7b, lfm3_slice3, make_weights, make_embeds, make_tokens
from parity import HIDDEN_REL_L2, LOGIT_ABS, bf16_rows, hidden_errors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mods():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_decoder_b200 import build
    build.build(verbose=False)
    from attention_decoder_b200 import _lib
    from attention_decoder_b200.model import Lfm3Model
    return _lib, Lfm3Model


def _copy_state(m, src):
    dst = m.new_state()
    for t in ("conv", "ring_k", "ring_v", "kv_k", "kv_v", "seq_len"):
        getattr(dst, t).copy_(getattr(src, t))
    dst.h_seq_len[:] = src.h_seq_len
    return dst


def _outputs(m, B, with_head=False):
    g = m.geom
    return {"hidden": torch.empty(g.n_layers + 1, B, g.d_model, dtype=torch.float32, device="cuda"),
            "logits": torch.empty(B, g.vocab, dtype=torch.float32, device="cuda") if with_head else None,
            "argmax": torch.empty(B, dtype=torch.int32, device="cuda") if with_head else None}


def _call(L, m, st, fn, slots, tokens=None, embeds=None, with_head=False, out=None):
    B = len(slots)
    h_slots = np.ascontiguousarray(slots, dtype=np.int32)
    d_slots = torch.from_numpy(h_slots).cuda()
    out = out if out is not None else _outputs(m, B, with_head)
    p = lambda t: None if t is None else C.c_void_p(t.data_ptr())
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    st_code = fn(m.ctx, C.byref(st.struct), B, h_slots.ctypes.data_as(C.POINTER(C.c_int32)), p(d_slots), p(tokens),
                 p(embeds), p(out["logits"]), p(out["argmax"]), p(out["hidden"]), stream)
    L.check(st_code, m.ctx)
    torch.cuda.synchronize()
    return out["hidden"], out["logits"], out["argmax"]


def test_noalloc_decode_matches_decode_step_on_two_calls(mods):
    L, Lfm3Model = mods
    g = lfm3_slice3()
    W = make_weights(g, 0)
    S = 3
    m = Lfm3Model(W, max_streams=S, max_pages_per_stream=6, max_batch=S)
    st = m.new_state()
    xs = [make_embeds(7, f"noalloc{s}", 300 + 20 * s, g.d_model) for s in range(S)]
    for s in range(S):
        m.prefill(st, s, embeds=bf16_rows(xs[s][:-2]))
    ref_st, new_st, warm_st = _copy_state(m, st), _copy_state(m, st), _copy_state(m, st)
    embeds = [torch.cat([bf16_rows(xs[s][-k:len(xs[s]) - k + 1]) for s in range(S)]) for k in (2, 1)]
    outs = [_outputs(m, S) for _ in range(2)]
    # one call on a spare copy looks the fixed array up; after it the calls must not change the
    # device's free memory (nothing allocated, lazily or otherwise)
    _call(L, m, warm_st, L.lib().lfm3_decode_step_noalloc, list(range(S)), embeds=embeds[0], out=_outputs(m, S))
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    h_new = [_call(L, m, new_st, L.lib().lfm3_decode_step_noalloc, list(range(S)), embeds=e, out=o)[0]
             for e, o in zip(embeds, outs)]
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    for e, hn in zip(embeds, h_new):  # two calls in a row, each advancing every stream by one row
        h_ref, _, _ = _call(L, m, ref_st, L.lib().lfm3_decode_step, list(range(S)), embeds=e)
        errs = hidden_errors(hn, [h.cpu().numpy().astype(np.float64) for h in h_ref])
        assert max(errs) <= HIDDEN_REL_L2, errs
        assert torch.equal(hn, h_ref)
    assert new_st.h_seq_len.tolist() == ref_st.h_seq_len.tolist()
    assert torch.equal(new_st.seq_len, ref_st.seq_len)
    for t in ("conv", "ring_k", "ring_v", "kv_k", "kv_v"):
        assert torch.equal(getattr(new_st, t), getattr(ref_st, t)), t


def test_noalloc_decode_with_head_and_size_refusal(mods):
    L, Lfm3Model = mods
    g = lfm3_1p7b(layer_types=(0, 2, 1, 0))  # conv, sliding, full, conv + the tied head
    W = make_weights(g, 0)
    m = Lfm3Model(W, max_streams=64, max_pages_per_stream=40, max_batch=64)
    st = m.new_state()
    tok = torch.from_numpy(make_tokens(1, "noalloc.head", 40, g.vocab)).cuda()
    m.prefill(st, 0, tokens=tok[:38])
    a, b = _copy_state(m, st), _copy_state(m, st)
    for t in (38, 39):
        _, lr, ar = _call(L, m, a, L.lib().lfm3_decode_step, [0], tokens=tok[t:t + 1], with_head=True)
        _, ln, an = _call(L, m, b, L.lib().lfm3_decode_step_noalloc, [0], tokens=tok[t:t + 1], with_head=True)
        assert float((ln - lr).abs().max()) <= LOGIT_ABS
        assert torch.equal(ln, lr) and torch.equal(an, ar)
    # 64 streams at a 2048-token context need 64 x 16 heads x 64 splits x 130 floats (34 MB):
    # more than the fixed array
    st.h_seq_len[:] = 2048
    st.seq_len.fill_(2048)
    before = st.h_seq_len.copy()
    with pytest.raises(L.Lfm3Error) as e:
        _call(L, m, st, L.lib().lfm3_decode_step_noalloc, list(range(64)), tokens=tok[:1].repeat(64),
              with_head=True)
    assert e.value.status == -3 and "scratch" in str(e.value)
    assert np.array_equal(st.h_seq_len, before)
