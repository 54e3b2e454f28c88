"""MLX affine FFN weights (4, 6 and 8 bits, groups of 64) through the C ABI, against the oracle.

TensorFold issue #1491, "Checkpoint handling": the text exports use affine groups of 64 (w = s * q
+ b per group). Decode streams the codes through the affine weight-streaming kernel, which keeps
the dot product exact (s * sum(q x) + b * sum(x)); prefill and batches of more than 16 streams
expand the weights to bf16 for the tensor-core GEMM (each weight rounded once).
"""
import numpy as np
import pytest
import torch

from lfm3_inputs import lfm3_1p7b, make_weights, make_tokens
from oracle import Lfm3Oracle
from parity import assert_hidden, assert_logits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_decoder_b200 import build
    build.build(verbose=False)
    from attention_decoder_b200.model import Lfm3Model
    return Lfm3Model


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_affine_ffn_prefill_and_decode_on_every_path(lib, bits):
    g = lfm3_1p7b(layer_types=(0, 2, 1, 0))
    W = make_weights(g, 0, ffn=f"affine{bits}")
    o = Lfm3Oracle(W, bf16=True)
    S = 20
    prompts = [make_tokens(9, f"aff{bits}.s{s}", 40 + 11 * s, g.vocab) for s in range(S)]
    m = lib(W, max_streams=S, max_pages_per_stream=6, max_batch=S)
    st = m.new_state()
    refs = []
    for s in range(S):
        out = m.prefill(st, s, tokens=torch.from_numpy(prompts[s][:-1]).cuda(), logits=(s == 0), argmax=(s == 0))
        ost = o.new_state()
        r = o.forward_chunk(ost, tokens=prompts[s][:-1])
        if s == 0:
            torch.cuda.synchronize()
            assert_logits(out["logits"], r["logits"], out["argmax"], what=f"affine{bits} prefill")
        refs.append((ost, o.forward_chunk(o.keep(ost), tokens=prompts[s][-1:])))
    last = np.array([p[-1] for p in prompts], dtype=np.int32)
    for B in (1, 12, S):  # one stream; two-column tiles; the GEMM path
        snap = [m.keep(st, s) for s in range(B)]
        out = m.decode(st, list(range(B)), tokens=torch.from_numpy(last[:B]).cuda(), hidden=True)
        torch.cuda.synchronize()
        for s in range(B):
            ref = refs[s][1]
            assert_hidden(out["hidden"][:, s:s + 1], ref["hidden"], what=f"affine{bits} B={B} stream {s}")
            assert_logits(out["logits"][s], ref["logits"], out["argmax"][s:s + 1], what=f"affine{bits} B={B} stream {s}")
        for s in range(B):  # back to the prompt's state for the next batch
            m.restore(st, s, snap[s][0], snap[s][1])
    m.check_device_errors()
