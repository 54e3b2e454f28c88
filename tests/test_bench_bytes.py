"""The decode-step byte count the bench's roofline divides by the device time, pinned to numbers it
does not compute itself: the published NVFP4 export total, the element counts of the weight arrays
the generator draws, and the cache growth one more position costs."""
import hashlib
import json
import os
import re

import numpy as np

import bench
from lfm3_inputs import make_weights
from lfm3_inputs.gen import CONV, lfm3_1p7b, tiny_geometry

HERE = os.path.dirname(os.path.abspath(__file__))


def _export_total():
    txt = open(os.path.join(HERE, "golden", "nvfp4_export_header.txt")).read()
    return int(re.search(r"^total_bytes\s*=\s*(\d+)", txt, re.M).group(1))


def test_nvfp4_weight_bytes_equal_the_published_export_total():
    # TensorFold PR #1508, NVFP4 admission commit: 502 text tensors, 1,829,689,408 bytes. The step
    # reads every one of them once except the two fp32 scalars per NVFP4 matrix (the tensor scale,
    # folded into the GEMV, and the static input scale, which is not applied): 24 layers x 3 x 8 B.
    g = lfm3_1p7b()
    weights = bench.decode_step_bytes(g, [], nvfp4=True, logits=False)
    assert weights + len(g.layer_types) * 3 * 2 * 4 == _export_total()


def test_bf16_weight_bytes_equal_the_drawn_arrays():
    # the generator's arrays for a small geometry, counted element by element (bf16 = 2 bytes);
    # the tied head is the embedding, read once
    g = tiny_geometry()
    W = make_weights(g, 0)
    elems = W["embed"].size + W["final_norm"].size
    for L in W["layers"]:
        elems += sum(np.asarray(v).size for k, v in L.items() if isinstance(v, np.ndarray) and v.dtype != np.int32)
    assert bench.decode_step_bytes(g, [], nvfp4=False, logits=False) == 2 * elems


def test_cache_and_logit_bytes_per_stream():
    g = lfm3_1p7b()
    row = 2 * 2 * g.n_kv * g.head_dim  # K and V of one position, bf16
    from lfm3_inputs.gen import FULL, SLIDING
    n_full = sum(t == FULL for t in g.layer_types)
    n_sl = sum(t == SLIDING for t in g.layer_types)
    n_conv = sum(t == CONV for t in g.layer_types)
    base = bench.decode_step_bytes(g, [], logits=False)
    # one more visible position: every attention layer inside the window, full layers only past it
    assert bench.decode_step_bytes(g, [11], logits=False) - bench.decode_step_bytes(g, [10], logits=False) == \
        (n_full + n_sl) * row
    assert bench.decode_step_bytes(g, [3001], logits=False) - bench.decode_step_bytes(g, [3000], logits=False) == \
        n_full * row
    # position 0: one key read and the new row written per attention layer; six conv columns read
    # and written per conv layer
    assert bench.decode_step_bytes(g, [0], logits=False) - base == \
        (n_full + n_sl) * 2 * row + n_conv * 2 * 2 * (g.conv_taps - 1) * g.d_model
    # fp32 logits of every stream
    assert bench.decode_step_bytes(g, [5, 6]) - bench.decode_step_bytes(g, [5, 6], logits=False) == 2 * 4 * g.vocab
    # streams add up
    assert bench.decode_step_bytes(g, [100, 2000]) - base == \
        (bench.decode_step_bytes(g, [100]) - base) + (bench.decode_step_bytes(g, [2000]) - base)


def test_traffic_record_is_dropped_once_a_source_changes(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    (tmp_path / "profiles").mkdir()
    rec = {"decode_step_b1": {"sources": {"k.cu": hashlib.sha256(b"kernel v1\n").hexdigest()},
                              "dram_per_algorithmic": 1.001, "note": "n"}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("decode_step_b1")["dram_per_algorithmic"] == 1.001
    src.write_text("kernel v2\n")
    assert bench.traffic_record("decode_step_b1") is None
    assert bench.traffic_record("missing") is None


def test_committed_traffic_record_names_existing_sources():
    rec = json.load(open(os.path.join(os.path.dirname(HERE), "profiles", "traffic.json")))["decode_step_b1"]
    for path in rec["sources"]:
        assert os.path.exists(os.path.join(os.path.dirname(HERE), path)), path
    assert 0.9 < rec["dram_per_algorithmic"] < 1.5
