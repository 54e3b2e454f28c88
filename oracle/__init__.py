"""CPU oracle for the LFM3-1.7B hybrid decoder forward (prefill and decode).

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs (``cpu_baseline`` and ``--impl reference``) may import or run it. The
CUDA path in ``attention_decoder_b200`` shares no code with it; the two meet
only through the seeded generators in ``lfm3_inputs``.

It is plain NumPy in float64 (fp32 optional for long timing runs), written
from the method's definition, optionally with the bf16 activation boundaries
the pages fix (``bf16=True``; see lfm3.py):

* ``lfm3.py`` - RMSNorm, the gated 7-tap short conv and its state, partial /
  full rotary, full and sliding-window GQA attention with the per-head sigmoid
  gate, sandwich norms, SwiGLU, tied head and greedy pick; a full-sequence
  mode (no cache: explicit masks, zero-padded conv) and an independent
  incremental mode (conv columns, a growing KV list, a 256-slot ring).
* ``nvfp4.py`` - E2M1 / E4M3 decoding from the OCP definitions and exact
  NVFP4 dequantisation.
* ``affine.py`` - MLX affine (4/6/8-bit, groups of 64) unpacking and
  dequantisation.

Every function is pinned by the ``-m "not gpu"`` tests (library routines,
brute force, closed forms, invariants and the pages' own totals). The pages
print no worked numbers for a whole forward pass; whole-model values are pinned
instead against an independent torch assembly of the decoder on a small
geometry (tests/test_oracle_head_pins.py), beside the invariants above.
"""
from .lfm3 import Lfm3Oracle, OracleState, rms_norm, rope_inv_freq, apply_rope, round_bf16  # noqa: F401
from .nvfp4 import e2m1_value, e4m3_value, nvfp4_dequant  # noqa: F401
from .affine import affine_unpack, affine_dequant  # noqa: F401
