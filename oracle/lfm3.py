"""The LFM3 hybrid decoder forward as a plain, slow CPU computation.

TEST INFRASTRUCTURE ONLY (see the package docstring). float64 by default.

Sources (coreai-model-zoo note "lfm3-1.7b-port" unless stated):
* diff table row 1 - gated short-conv mixer, 7 taps, state = the last 6 columns
  of B*x, 13 conv layers;
* row 2 - 6 full + 5 sliding (window 256) attention layers, 16 q / 4 kv heads,
  head_dim 128;
* row 3 - rotary: full layers theta 1e6 on half the head_dim with a zero tail,
  sliding layers theta 1e4 on the whole head_dim; the partial-rotary paragraph
  fixes the pairs (i, i + 64), i < 32, and the pass-through of 32-63 / 96-127;
* row 4 - output gate sigmoid(gate_proj(x)), one scalar per head, x = the
  mixer's normed input, multiplied into each head before o_proj;
* row 5 - sandwich norms: operator_norm -> mixer -> post_operator_norm ->
  + residual -> ffn_norm -> SwiGLU -> post_ffn_norm -> + residual; final
  embedding_norm;
* "Unchanged" paragraph - width 2048, vocab 128000 tied head, SwiGLU 7680,
  RMSNorm eps 1e-5, per-head q/k RMSNorm;
* "window_size, with no mask input" - key allowed iff query position - key
  position < 256 (and causal);
* chunked-prefill / pad-tail paragraphs - the new conv state is columns
  [n, n+6) of [state | Bx] for a chunk of n rows.

Precision. TensorFold issue #1491 ("Goal and current state") keeps "BF16 activation
boundaries, and FP32 reductions", and PR #1508 ("Verification") checks the engine against a
float64 reference with "the engine's bf16 rounding points" added. With ``bf16=True`` this
oracle does the same: arithmetic stays float64, and a value is rounded to bf16 exactly where it
becomes a stored operand of a matrix product or attention, or persistent state - the normed
inputs of every projection (and of the head), Bx (the conv state), y = C * conv, q and k after
norm and rotary, v, the gated attention output and the SwiGLU product. Projection accumulators,
gate logits, norms, softmax and the residual stream are reductions and stay unrounded. With
``bf16=False`` (default) nothing is rounded: the plain float64 definition.

Readings where the pages are silent:
in_proj rows are B, C, x in that order; the conv is causal with tap 6 on the
current column and zero history at sequence start; no biases; q/k RMSNorm
before rotary, gains of length head_dim shared by all heads; q head h reads kv
head h // (n_q / n_kv); softmax scale 1/sqrt(head_dim); masked keys are
excluded exactly; RMSNorm gain multiplies directly (g * x_hat); greedy ties go
to the lowest id.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from lfm3_inputs import CONV, FULL, SLIDING
from .affine import affine_dequant
from .nvfp4 import nvfp4_block_values


def _bf16(bits) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_bf16(x):
    """Nearest bf16 value (8 significant bits, ties to even) of each float, as float64."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                 # x = m * 2^e, |m| in [0.5, 1)
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def rms_norm(x, g, eps):
    """y = g * x / sqrt(mean(x^2) + eps) over the last axis."""
    x = np.asarray(x)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


def sigmoid(x):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def silu(x):
    return x * sigmoid(x)


def causal_conv_full(bx, w):
    """Depthwise causal conv of bx[T, C] with w[C, taps] from zero history:
    z[t] = sum over lags l of w[:, taps-1-l] * bx[t-l] (bx before t = 0 is zero)."""
    T = bx.shape[0]
    taps = w.shape[1]
    z = np.zeros_like(bx)
    for lag in range(min(taps, T)):
        z[lag:] += w[:, taps - 1 - lag] * bx[:T - lag]
    return z


def causal_conv_chunk(state, bx, w):
    """The same conv over carried columns: win = [state | bx] (state[taps-1, C], oldest
    first), z[t] = sum_k w[:, k] * win[t + k]; returns (z, win[n : n + taps - 1])."""
    n = bx.shape[0]
    taps = w.shape[1]
    win = np.concatenate([state, bx], axis=0)
    z = np.zeros_like(bx)
    for t in range(n):
        z[t] = np.sum(w.T * win[t:t + taps], axis=0)
    return z, win[n:n + taps - 1].copy()


def rope_inv_freq(theta: float, head_dim: int, rotated_pairs: int) -> np.ndarray:
    """inv_freq[i] = theta^(-2i/head_dim) for i < rotated_pairs, 0 after (the zero tail)."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    f = np.power(float(theta), -2.0 * i / head_dim)
    f[rotated_pairs:] = 0.0
    return f


def apply_rope(x, pos, inv_freq):
    """rotate_half rotary on x[..., T, H, d] at integer positions pos[T]: pair (i, i+d/2)
    turns by angle pos * inv_freq[i]."""
    x = np.asarray(x)
    half = x.shape[-1] // 2
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv_freq[None, :]   # [T, half]
    c = np.cos(ang)[:, None, :].astype(x.dtype)
    s = np.sin(ang)[:, None, :].astype(x.dtype)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


@dataclass
class OracleState:
    """Incremental state of one stream: conv columns (oldest first) per conv layer, the
    whole K/V history per full layer, and a W-slot ring (slot = position mod W, with the
    position each slot holds, -1 if empty) per sliding layer."""
    conv: list = field(default_factory=list)
    full_k: list = field(default_factory=list)
    full_v: list = field(default_factory=list)
    ring_k: list = field(default_factory=list)
    ring_v: list = field(default_factory=list)
    ring_pos: list = field(default_factory=list)
    seq_len: int = 0


class Lfm3Oracle:
    """Forward of one decoder on seeded weights from ``lfm3_inputs.make_weights``."""

    def __init__(self, weights: dict, dtype=np.float64, gate=True, rope_all_dims=False, window=True, bf16=False):
        self.g = weights["geometry"]
        self.dtype = dtype
        self._rb = round_bf16 if bf16 else (lambda x: x)
        # negative controls (planted mistakes for the tests): drop the gate, rotate every
        # dimension on full layers, remove the window
        self.use_gate = gate
        self.rope_all_dims = rope_all_dims
        self.use_window = window
        g = self.g
        self.embed = _bf16(weights["embed"]) if g.has_head else None
        self.final_norm = _bf16(weights["final_norm"]).astype(dtype) if g.has_head else None
        self.layers = []
        for L in weights["layers"]:
            O = {"kind": L["kind"]}
            for nm in ("op_norm", "post_op_norm", "ffn_norm", "post_ffn_norm"):
                O[nm] = _bf16(L[nm]).astype(dtype)
            if L["kind"] == CONV:
                O["in_proj"] = _bf16(L["in_proj"])
                O["conv"] = _bf16(L["conv"]).astype(dtype)
                O["out_proj"] = _bf16(L["out_proj"])
            else:
                O["q_proj"] = _bf16(L["q_proj"])
                O["k_proj"] = _bf16(L["k_proj"])
                O["v_proj"] = _bf16(L["v_proj"])
                O["gate_proj"] = _bf16(L["gate_proj"])
                O["q_norm"] = _bf16(L["q_norm"]).astype(dtype)
                O["k_norm"] = _bf16(L["k_norm"]).astype(dtype)
                O["o_proj"] = _bf16(L["o_proj"])
            if "w1" in L:
                O["w1"], O["w3"], O["w2"] = _bf16(L["w1"]), _bf16(L["w3"]), _bf16(L["w2"])
                O["s13"] = O["s2"] = 1.0
            elif "affine_bits" in L:
                # MLX affine groups of 64: w = s * q + b, exact in float64
                bits = L["affine_bits"]
                for nm in ("w1", "w3", "w2"):
                    cols = g.d_model if nm != "w2" else g.d_ffn
                    O[nm] = affine_dequant(L[nm + "_codes"], L[nm + "_scales"], L[nm + "_biases"], bits, cols)
                O["s13"] = O["s2"] = 1.0
            else:
                # exact E2M1 x E4M3 products in float32; the fp32 tensor scale is applied
                # to the float64 product below (same value as scaling each weight)
                O["w1"] = nvfp4_block_values(L["w1_codes"], L["w1_scales"])
                O["w3"] = nvfp4_block_values(L["w3_codes"], L["w3_scales"])
                O["w2"] = nvfp4_block_values(L["w2_codes"], L["w2_scales"])
                O["s13"] = float(np.float32(L["w13_scale2"]))
                O["s2"] = float(np.float32(L["w2_scale2"]))
            self.layers.append(O)
        d = g.head_dim
        pairs_full = d // 2 if rope_all_dims else g.rope_pairs_full
        self.inv_freq = {FULL: rope_inv_freq(g.theta_full, d, pairs_full),
                         SLIDING: rope_inv_freq(g.theta_sliding, d, d // 2)}

    # ------------------------------------------------------------------ pieces

    def _lin(self, x, w):
        """x @ w.T in the oracle's precision (w is float32 storage of exact values)."""
        return x @ w.T.astype(self.dtype, copy=False)

    def _ffn(self, hn, O):
        hn = self._rb(hn)
        a = O["s13"] * self._lin(hn, O["w1"])
        b = O["s13"] * self._lin(hn, O["w3"])
        u = self._rb(silu(a) * b)
        return O["s2"] * self._lin(u, O["w2"])

    def _qkvg(self, xn, O):
        g = self.g
        xn = self._rb(xn)
        T = xn.shape[0]
        q = self._lin(xn, O["q_proj"]).reshape(T, g.n_q, g.head_dim)
        k = self._lin(xn, O["k_proj"]).reshape(T, g.n_kv, g.head_dim)
        v = self._lin(xn, O["v_proj"]).reshape(T, g.n_kv, g.head_dim)
        gate = self._lin(xn, O["gate_proj"])                       # [T, n_q]
        q = rms_norm(q, O["q_norm"], g.eps)
        k = rms_norm(k, O["k_norm"], g.eps)
        return q, k, self._rb(v), gate

    def _attend(self, q, qpos, k, v, kpos, window, gate):
        """Softmax attention of queries q[Tq, Hq, d] at qpos over keys k/v[Tk, Hkv, d] at
        kpos; key j is allowed for query i iff kpos_j <= qpos_i and, with a window W,
        qpos_i - kpos_j < W. Masked keys are excluded exactly."""
        g = self.g
        group = g.n_q // g.n_kv
        scale = 1.0 / math.sqrt(g.head_dim)
        diff = qpos[:, None] - kpos[None, :]
        allowed = diff >= 0
        if window is not None:
            allowed &= diff < window
        o = np.zeros(q.shape, dtype=self.dtype)
        for h in range(g.n_q):
            kvh = h // group
            s = (q[:, h, :] @ k[:, kvh, :].T) * scale
            s = np.where(allowed, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p = p / p.sum(axis=1, keepdims=True)
            o[:, h, :] = p @ v[:, kvh, :]
        if self.use_gate:
            o = o * sigmoid(gate)[:, :, None]
        return self._rb(o.reshape(q.shape[0], -1))

    def _window(self, kind):
        return self.g.window if (kind == SLIDING and self.use_window) else None

    # ------------------------------------------------------------------ full-sequence mode

    def _conv_full(self, xn, O):
        """Whole sequence from zero history: z[t] = sum over lags l = 0..taps-1 of
        w[:, taps-1-l] * bx[t-l], with bx[t<0] = 0."""
        D = self.g.d_model
        bcx = self._lin(self._rb(xn), O["in_proj"])
        b, c, xc = bcx[:, :D], bcx[:, D:2 * D], bcx[:, 2 * D:]
        z = causal_conv_full(self._rb(b * xc), O["conv"])
        return self._lin(self._rb(c * z), O["out_proj"])

    def _attn_full(self, xn, O, pos, kind):
        q, k, v, gate = self._qkvg(xn, O)
        q = self._rb(apply_rope(q, pos, self.inv_freq[kind]))
        k = self._rb(apply_rope(k, pos, self.inv_freq[kind]))
        o = self._attend(q, pos, k, v, pos, self._window(kind), gate)
        return self._lin(o, O["o_proj"])

    def _block(self, x, O, mixer):
        eps = self.g.eps
        xn = rms_norm(x, O["op_norm"], eps)
        m = mixer(xn)
        h = x + rms_norm(m, O["post_op_norm"], eps)
        hn = rms_norm(h, O["ffn_norm"], eps)
        f = self._ffn(hn, O)
        return h + rms_norm(f, O["post_ffn_norm"], eps)

    def embed_tokens(self, tokens):
        return self.embed[np.asarray(tokens)].astype(self.dtype)

    def logits(self, x):
        xn = self._rb(rms_norm(x, self.final_norm, self.g.eps))
        return xn @ self.embed.T.astype(self.dtype, copy=False)

    def forward_full(self, tokens=None, x0=None, logits="last"):
        """One call over the whole sequence, positions 0..T-1, no cache.
        Returns {'hidden': [L+1] arrays [T, D], 'logits': [V] (last row), [T, V] or None}."""
        x = self.embed_tokens(tokens) if x0 is None else np.asarray(x0, dtype=self.dtype)
        pos = np.arange(x.shape[0])
        hidden = [x]
        for O in self.layers:
            kind = O["kind"]
            if kind == CONV:
                mixer = lambda xn, O=O: self._conv_full(xn, O)
            else:
                mixer = lambda xn, O=O, kind=kind: self._attn_full(xn, O, pos, kind)
            x = self._block(x, O, mixer)
            hidden.append(x)
        out = {"hidden": hidden, "logits": None}
        if self.g.has_head and logits == "last":
            out["logits"] = self.logits(x[-1:])[0]
        elif self.g.has_head and logits == "all":
            out["logits"] = self.logits(x)
        return out

    # ------------------------------------------------------------------ incremental mode

    def new_state(self) -> OracleState:
        g = self.g
        st = OracleState()
        for kind in g.layer_types:
            if kind == CONV:
                st.conv.append(np.zeros((g.conv_taps - 1, g.d_model), dtype=self.dtype))
            elif kind == FULL:
                st.full_k.append(np.zeros((0, g.n_kv, g.head_dim), dtype=self.dtype))
                st.full_v.append(np.zeros((0, g.n_kv, g.head_dim), dtype=self.dtype))
            else:
                st.ring_k.append(np.zeros((g.window, g.n_kv, g.head_dim), dtype=self.dtype))
                st.ring_v.append(np.zeros((g.window, g.n_kv, g.head_dim), dtype=self.dtype))
                st.ring_pos.append(np.full(g.window, -1, dtype=np.int64))
        return st

    def state_from_synthetic(self, syn: dict, stream: int, context: int) -> OracleState:
        """Stream ``stream`` of ``lfm3_inputs.synthetic_state`` as an oracle state."""
        g = self.g
        st = self.new_state()
        st.seq_len = int(context)
        for j in range(len(st.conv)):
            st.conv[j] = _bf16(syn["conv"][j][stream]).astype(self.dtype)
        for j in range(len(st.full_k)):
            st.full_k[j] = _bf16(syn["full_k"][j][stream]).astype(self.dtype)
            st.full_v[j] = _bf16(syn["full_v"][j][stream]).astype(self.dtype)
        for j in range(len(st.ring_k)):
            ks = _bf16(syn["slide_k"][j][stream]).astype(self.dtype)
            vs = _bf16(syn["slide_v"][j][stream]).astype(self.dtype)
            m = ks.shape[0]
            for r in range(m):
                p = context - m + r
                st.ring_k[j][p % g.window] = ks[r]
                st.ring_v[j][p % g.window] = vs[r]
                st.ring_pos[j][p % g.window] = p
        return st

    def _conv_chunk(self, xn, O, st, j):
        """Chunk of n rows over the carried columns: win = [state | bx],
        z[t] = sum_k w[:, k] * win[t + k]; the new state is win[n : n + taps - 1]."""
        D = self.g.d_model
        bcx = self._lin(self._rb(xn), O["in_proj"])
        b, c, xc = bcx[:, :D], bcx[:, D:2 * D], bcx[:, 2 * D:]
        z, st.conv[j] = causal_conv_chunk(st.conv[j], self._rb(b * xc), O["conv"])
        return self._lin(self._rb(c * z), O["out_proj"])

    def _attn_chunk(self, xn, O, kind, st, j, pos):
        g = self.g
        q, k, v, gate = self._qkvg(xn, O)
        q = self._rb(apply_rope(q, pos, self.inv_freq[kind]))
        k = self._rb(apply_rope(k, pos, self.inv_freq[kind]))
        if kind == FULL:
            st.full_k[j] = np.concatenate([st.full_k[j], k], axis=0)
            st.full_v[j] = np.concatenate([st.full_v[j], v], axis=0)
            kk, vv = st.full_k[j], st.full_v[j]
            kpos = np.arange(kk.shape[0])
            o = self._attend(q, pos, kk, vv, kpos, None, gate)
        else:
            live = st.ring_pos[j] >= 0
            kk = np.concatenate([st.ring_k[j][live], k], axis=0)
            vv = np.concatenate([st.ring_v[j][live], v], axis=0)
            kpos = np.concatenate([st.ring_pos[j][live], pos])
            window = g.window if self.use_window else None
            if not self.use_window:
                raise ValueError("the incremental ring cannot hold an unwindowed history")
            o = self._attend(q, pos, kk, vv, kpos, window, gate)
            for r, p in enumerate(pos):
                slot = int(p) % g.window
                st.ring_k[j][slot] = k[r]
                st.ring_v[j][slot] = v[r]
                st.ring_pos[j][slot] = int(p)
        return self._lin(o, O["o_proj"])

    def forward_chunk(self, st: OracleState, tokens=None, x0=None, logits="last"):
        """Consume n rows at positions st.seq_len .. st.seq_len+n-1, updating ``st``.
        Returns {'hidden': [L+1] arrays [n, D], 'logits': as in forward_full}."""
        x = self.embed_tokens(tokens) if x0 is None else np.asarray(x0, dtype=self.dtype)
        n = x.shape[0]
        pos = np.arange(st.seq_len, st.seq_len + n)
        hidden = [x]
        ci = fi = si = 0
        for O in self.layers:
            kind = O["kind"]
            if kind == CONV:
                mixer = lambda xn, O=O, j=ci: self._conv_chunk(xn, O, st, j)
                ci += 1
            elif kind == FULL:
                mixer = lambda xn, O=O, j=fi: self._attn_chunk(xn, O, FULL, st, j, pos)
                fi += 1
            else:
                mixer = lambda xn, O=O, j=si: self._attn_chunk(xn, O, SLIDING, st, j, pos)
                si += 1
            x = self._block(x, O, mixer)
            hidden.append(x)
        st.seq_len += n
        out = {"hidden": hidden, "logits": None}
        if self.g.has_head and logits == "last":
            out["logits"] = self.logits(x[-1:])[0]
        elif self.g.has_head and logits == "all":
            out["logits"] = self.logits(x)
        return out

    def keep(self, st: OracleState) -> OracleState:
        """The state at the mark at = st.seq_len, as an independent copy: the conv columns, the
        sliding rings and the keys / values of positions [0, at) of the full layers (TensorFold
        PR #1508, prompt-cache paragraph: "a state at `at` is the slot's conv states and its keys
        and values at positions [0, at)"). Restoring is continuing from the copy."""
        return OracleState(conv=[a.copy() for a in st.conv],
                           full_k=[a[:st.seq_len].copy() for a in st.full_k],
                           full_v=[a[:st.seq_len].copy() for a in st.full_v],
                           ring_k=[a.copy() for a in st.ring_k], ring_v=[a.copy() for a in st.ring_v],
                           ring_pos=[a.copy() for a in st.ring_pos], seq_len=st.seq_len)

    def greedy(self, st: OracleState, first_token: int, steps: int):
        """Greedy decode: feed ``first_token``, then each argmax (ties -> lowest id).
        Returns (tokens fed [steps], logits [steps, V])."""
        fed, lg = [], []
        tok = int(first_token)
        for _ in range(steps):
            out = self.forward_chunk(st, tokens=np.array([tok]))
            fed.append(tok)
            lg.append(out["logits"])
            tok = int(np.argmax(out["logits"]))
        return np.array(fed, dtype=np.int32), np.stack(lg)


def top2_margin(logits) -> np.ndarray:
    """Top-1 minus top-2 logit per row."""
    lg = np.atleast_2d(np.asarray(logits, dtype=np.float64))
    part = np.partition(lg, -2, axis=1)
    return part[:, -1] - part[:, -2]
