"""Device memory for the C ABI: uploads weights, allocates state and workspace with torch and calls
liblfm3.so through the ctypes binding. No arithmetic of the forward happens here; torch is only
the allocator and the stream provider."""
from __future__ import annotations

import ctypes as C

import numpy as np
import torch

from . import _lib as L
from ._lib import check

CONV, FULL, SLIDING = L.LFM3_LAYER_CONV, L.LFM3_LAYER_FULL, L.LFM3_LAYER_SLIDING


def _bf16(bits: np.ndarray, device) -> torch.Tensor:
    """bf16 bit patterns (uint16) -> a device bf16 tensor holding the same bits."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def _u8(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(device)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


class Lfm3Model:
    """One decoder on one GPU. ``weights`` is ``lfm3_inputs.make_weights(...)``'s dict."""

    def __init__(self, weights: dict, device="cuda", max_streams=1, max_pages_per_stream=64, n_pages=None,
                 max_chunk=2048, max_batch=None):
        g = weights["geometry"]
        self.geom = g
        self.device = torch.device(device)
        self.nvfp4 = weights["ffn"] == "nvfp4"
        self.affine = weights["ffn"].startswith("affine")
        max_batch = max_batch or max_streams
        if n_pages is None:
            n_pages = max_streams * max_pages_per_stream
        cfg = L.lfm3_config()
        cfg.n_layers = g.n_layers
        for i, t in enumerate(g.layer_types):
            cfg.layer_type[i] = t
        cfg.d_model, cfg.d_ffn, cfg.n_q, cfg.n_kv = g.d_model, g.d_ffn, g.n_q, g.n_kv
        cfg.head_dim, cfg.conv_taps, cfg.window, cfg.vocab = g.head_dim, g.conv_taps, g.window, g.vocab
        cfg.theta_full, cfg.theta_sliding = g.theta_full, g.theta_sliding
        cfg.rope_pairs_full, cfg.eps = g.rope_pairs_full, g.eps
        cfg.has_head = 1 if g.has_head else 0
        cfg.ffn_format = L.LFM3_FFN_NVFP4 if self.nvfp4 else (L.LFM3_FFN_AFFINE if self.affine else L.LFM3_FFN_BF16)
        cfg.ffn_bits = int(weights["ffn"][6:]) if self.affine else 0
        cfg.page_size = 64
        cfg.n_pages = n_pages
        cfg.max_streams = max_streams
        cfg.max_pages_per_stream = max_pages_per_stream
        cfg.max_chunk = max_chunk
        cfg.max_batch = max_batch
        self.cfg = cfg
        dev = self.device
        keep = []

        def up(bits):
            t = _bf16(bits, dev)
            keep.append(t)
            return C.c_void_p(t.data_ptr())

        def up8(a):
            t = _u8(a, dev)
            keep.append(t)
            return C.c_void_p(t.data_ptr())

        layers = (L.lfm3_layer_weights * g.n_layers)()
        for i, Lw in enumerate(weights["layers"]):
            lw = layers[i]
            for nm in ("op_norm", "post_op_norm", "ffn_norm", "post_ffn_norm"):
                setattr(lw, nm, up(Lw[nm]))
            if Lw["kind"] == CONV:
                lw.in_proj, lw.conv, lw.out_proj = up(Lw["in_proj"]), up(Lw["conv"]), up(Lw["out_proj"])
            else:
                # q | k | v | gate rows as one projection weight
                lw.qkvg = up(np.concatenate([Lw["q_proj"], Lw["k_proj"], Lw["v_proj"], Lw["gate_proj"]], axis=0))
                lw.q_norm, lw.k_norm, lw.o_proj = up(Lw["q_norm"]), up(Lw["k_norm"]), up(Lw["o_proj"])
            if self.affine:
                for nm in ("w1", "w3", "w2"):
                    setattr(lw, nm + "_codes", up8(Lw[nm + "_codes"].view(np.uint8)))
                    setattr(lw, nm + "_scales", up(Lw[nm + "_scales"]))
                    setattr(lw, nm + "_biases", up(Lw[nm + "_biases"]))
            elif self.nvfp4:
                lw.w1_codes, lw.w1_scales = up8(Lw["w1_codes"]), up8(Lw["w1_scales"])
                lw.w3_codes, lw.w3_scales = up8(Lw["w3_codes"]), up8(Lw["w3_scales"])
                lw.w2_codes, lw.w2_scales = up8(Lw["w2_codes"]), up8(Lw["w2_scales"])
                lw.w13_scale, lw.w2_scale = float(Lw["w13_scale2"]), float(Lw["w2_scale2"])
            else:
                lw.w1, lw.w3, lw.w2 = up(Lw["w1"]), up(Lw["w3"]), up(Lw["w2"])
        w = L.lfm3_weights()
        if g.has_head:
            w.embed, w.final_norm = up(weights["embed"]), up(weights["final_norm"])
        w.layers = C.cast(layers, C.POINTER(L.lfm3_layer_weights))
        self._keep, self._layers, self._w = keep, layers, w
        ctx = C.c_void_p()
        ws = C.c_size_t()
        st = L.lfm3_create(C.byref(cfg), C.byref(w), C.byref(ws), C.byref(ctx))
        check(st, None)
        self.ctx = ctx
        self.workspace = torch.empty(ws.value, dtype=torch.uint8, device=dev)
        check(L.lfm3_bind_workspace(ctx, C.c_void_p(self.workspace.data_ptr()), ws.value), ctx)

    @property
    def weight_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self._keep)

    def new_state(self, page_table=None, poison=False) -> "Lfm3State":
        return Lfm3State(self, page_table=page_table, poison=poison)

    def profile(self, on: bool, capacity: int = 4096):
        check(L.lfm3_profile_enable(self.ctx, 1 if on else 0, capacity), self.ctx)

    def profile_read(self) -> dict:
        n, ms, b, f = C.c_int(), C.c_double(), C.c_double(), C.c_double()
        check(L.lfm3_profile_read(self.ctx, C.byref(n), C.byref(ms), C.byref(b), C.byref(f)), self.ctx)
        return {"launches": n.value, "ms": ms.value, "bytes": b.value, "flops": f.value}

    def last_launch_count(self) -> int:
        return L.lfm3_last_launch_count(self.ctx)

    def check_device_errors(self, stream=None):
        check(L.lfm3_check_device_errors(self.ctx, _stream(stream)), self.ctx)

    def state_bytes(self, at: int) -> int:
        return int(L.lfm3_state_bytes(self.ctx, at))

    def keep(self, st, slot, buf=None, stream=None):
        """Keeps slot's state at its current position; returns (mark, device buffer)."""
        at = int(st.h_seq_len[slot])
        n = self.state_bytes(at)
        if buf is None:
            buf = torch.empty(n, dtype=torch.uint8, device=self.device)
        out = C.c_int()
        check(L.lfm3_keep(self.ctx, C.byref(st.struct), slot, _ptr(buf), buf.numel(), C.byref(out), _stream(stream)),
              self.ctx)
        return out.value, buf

    def restore(self, st, slot, at, buf, stream=None):
        check(L.lfm3_restore(self.ctx, C.byref(st.struct), slot, _ptr(buf), buf.numel(), at, _stream(stream)), self.ctx)

    def selftest_wait(self, rounds=4096, stream=None):
        check(L.lfm3_selftest_wait(self.ctx, rounds, _stream(stream)), self.ctx)

    # ------------------------------------------------------------------ calls
    def prefill(self, st, slot, tokens=None, embeds=None, logits=True, argmax=True, hidden=False, stream=None,
                out=None):
        """Consume rows for one slot. tokens: device int32 [n]; embeds: device bf16 [n, D].
        Returns a dict of device tensors (logits [V] fp32, argmax [1] int32, hidden [L+1, n, D] fp32)."""
        g = self.geom
        n = int(tokens.shape[0] if tokens is not None else embeds.shape[0])
        out = {} if out is None else out
        if g.has_head and logits and "logits" not in out:
            out["logits"] = torch.empty(g.vocab, dtype=torch.float32, device=self.device)
        if g.has_head and argmax and "argmax" not in out:
            out["argmax"] = torch.empty(1, dtype=torch.int32, device=self.device)
        if hidden and "hidden" not in out:
            out["hidden"] = torch.empty(g.n_layers + 1, n, g.d_model, dtype=torch.float32, device=self.device)
        check(L.lfm3_prefill(self.ctx, C.byref(st.struct), slot, _ptr(tokens), _ptr(embeds), n, _ptr(out.get("logits")),
                             _ptr(out.get("argmax")), _ptr(out.get("hidden")), _stream(stream)), self.ctx)
        return out

    def prefill_padded(self, st, slot, n_real, tokens=None, embeds=None, logits=True, argmax=True, hidden=False,
                       stream=None):
        """One chunk whose rows past n_real are padding (see lfm3_prefill_padded)."""
        g = self.geom
        n = int(tokens.shape[0] if tokens is not None else embeds.shape[0])
        out = {}
        if g.has_head and logits:
            out["logits"] = torch.empty(g.vocab, dtype=torch.float32, device=self.device)
        if g.has_head and argmax:
            out["argmax"] = torch.empty(1, dtype=torch.int32, device=self.device)
        if hidden:
            out["hidden"] = torch.empty(g.n_layers + 1, n, g.d_model, dtype=torch.float32, device=self.device)
        check(L.lfm3_prefill_padded(self.ctx, C.byref(st.struct), slot, _ptr(tokens), _ptr(embeds), n, n_real,
                                    _ptr(out.get("logits")), _ptr(out.get("argmax")), _ptr(out.get("hidden")),
                                    _stream(stream)), self.ctx)
        return out

    def decode(self, st, slots, tokens=None, embeds=None, logits=True, argmax=True, hidden=False, stream=None,
               d_slots=None, out=None):
        """One step for the listed slots (host list); tokens: device int32 [B]; embeds: bf16 [B, D]."""
        g = self.geom
        h_slots = np.ascontiguousarray(slots, dtype=np.int32)
        B = len(h_slots)
        if d_slots is None:
            d_slots = torch.from_numpy(h_slots).to(self.device)
        out = {} if out is None else out
        if g.has_head and logits and "logits" not in out:
            out["logits"] = torch.empty(B, g.vocab, dtype=torch.float32, device=self.device)
        if g.has_head and argmax and "argmax" not in out:
            out["argmax"] = torch.empty(B, dtype=torch.int32, device=self.device)
        if hidden and "hidden" not in out:
            out["hidden"] = torch.empty(g.n_layers + 1, B, g.d_model, dtype=torch.float32, device=self.device)
        check(L.lfm3_decode_step(self.ctx, C.byref(st.struct), B, h_slots.ctypes.data_as(C.POINTER(C.c_int32)),
                                 _ptr(d_slots), _ptr(tokens), _ptr(embeds), _ptr(out.get("logits")),
                                 _ptr(out.get("argmax")), _ptr(out.get("hidden")), _stream(stream)), self.ctx)
        return out

    def verify(self, st, slots, W, tokens=None, embeds=None, hidden=False, stream=None):
        """One verify window of W rows per listed slot (see lfm3_verify); nothing is committed.
        tokens: device int32 [len(slots) * W], stream-major. Returns logits [n*W, V], argmax [n*W]."""
        g = self.geom
        h_slots = np.ascontiguousarray(slots, dtype=np.int32)
        rows = len(h_slots) * W
        d_slots = torch.from_numpy(h_slots).to(self.device)
        out = {}
        if g.has_head:
            out["logits"] = torch.empty(rows, g.vocab, dtype=torch.float32, device=self.device)
            out["argmax"] = torch.empty(rows, dtype=torch.int32, device=self.device)
        if hidden:
            out["hidden"] = torch.empty(g.n_layers + 1, rows, g.d_model, dtype=torch.float32, device=self.device)
        out["_slots"] = d_slots  # kept alive until the window has run
        check(L.lfm3_verify(self.ctx, C.byref(st.struct), len(h_slots), h_slots.ctypes.data_as(C.POINTER(C.c_int32)),
                            _ptr(d_slots), W, _ptr(tokens), _ptr(embeds), _ptr(out.get("logits")),
                            _ptr(out.get("argmax")), _ptr(out.get("hidden")), _stream(stream)), self.ctx)
        return out

    def commit(self, st, slots, accept, stream=None):
        h_slots = np.ascontiguousarray(slots, dtype=np.int32)
        h_acc = np.ascontiguousarray(accept, dtype=np.int32)
        check(L.lfm3_commit(self.ctx, C.byref(st.struct), len(h_slots), h_slots.ctypes.data_as(C.POINTER(C.c_int32)),
                            h_acc.ctypes.data_as(C.POINTER(C.c_int32)), _stream(stream)), self.ctx)

    def close(self):
        if getattr(self, "ctx", None):
            L.lfm3_free(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Lfm3State:
    """Caller-owned decode state of ``model.cfg.max_streams`` slots (see include/lfm3.h)."""

    def __init__(self, model: Lfm3Model, page_table=None, poison=False):
        g, cfg, dev = model.geom, model.cfg, model.device
        S, P, mpp = cfg.max_streams, cfg.n_pages, cfg.max_pages_per_stream
        fill = float("nan") if poison else 0.0
        bf = torch.bfloat16
        self.model = model
        self.conv = torch.zeros(max(g.count(CONV), 1), S, g.conv_taps - 1, g.d_model, dtype=bf, device=dev)
        nsl, nfu = g.count(SLIDING), g.count(FULL)
        self.ring_k = torch.full((max(nsl, 1), S, g.n_kv, g.window, g.head_dim), fill, dtype=bf, device=dev)
        self.ring_v = torch.full_like(self.ring_k, fill)
        self.kv_k = torch.full((max(nfu, 1), P, g.n_kv, 64, g.head_dim), fill, dtype=bf, device=dev)
        self.kv_v = torch.full_like(self.kv_k, fill)
        if page_table is None:
            if P >= S * mpp:
                page_table = np.arange(S * mpp, dtype=np.int32).reshape(S, mpp)
            else:
                page_table = np.full((S, mpp), -1, dtype=np.int32)
        self.h_page_table = np.ascontiguousarray(page_table, dtype=np.int32)
        assert self.h_page_table.shape == (S, mpp)
        self.page_table = torch.from_numpy(self.h_page_table).to(dev)
        self.h_seq_len = np.zeros(S, dtype=np.int32)
        self.seq_len = torch.zeros(S, dtype=torch.int32, device=dev)
        s = L.lfm3_state()
        s.conv_state, s.ring_k, s.ring_v = _ptr(self.conv), _ptr(self.ring_k), _ptr(self.ring_v)
        s.kv_k, s.kv_v, s.page_table, s.seq_len = _ptr(self.kv_k), _ptr(self.kv_v), _ptr(self.page_table), _ptr(self.seq_len)
        s.h_seq_len = self.h_seq_len.ctypes.data_as(C.POINTER(C.c_int32))
        s.h_page_table = self.h_page_table.ctypes.data_as(C.POINTER(C.c_int32))
        self.struct = s

    def load_synthetic(self, syn: dict, contexts):
        """Lay a drawn state (``lfm3_inputs.synthetic_state``) out in pages, rings and conv columns:
        position p of slot s goes to page page_table[s][p // 64], row p % 64, and ring slot p % W."""
        g, dev = self.model.geom, self.model.device
        W = g.window
        for s, c in enumerate(contexts):
            c = int(c)
            for j in range(g.count(CONV)):
                self.conv[j, s] = _bf16(syn["conv"][j][s], dev)
            for j in range(g.count(FULL)):
                k = _bf16(syn["full_k"][j][s], dev)   # [c, kv, d]
                v = _bf16(syn["full_v"][j][s], dev)
                for p0 in range(0, c, 64):
                    pg = int(self.h_page_table[s, p0 // 64])
                    m = min(64, c - p0)
                    self.kv_k[j, pg, :, :m] = k[p0:p0 + m].transpose(0, 1)
                    self.kv_v[j, pg, :, :m] = v[p0:p0 + m].transpose(0, 1)
            for j in range(g.count(SLIDING)):
                k = _bf16(syn["slide_k"][j][s], dev)
                v = _bf16(syn["slide_v"][j][s], dev)
                m = k.shape[0]
                pos = torch.arange(c - m, c, device=dev) % W
                self.ring_k[j, s][:, pos] = k.transpose(0, 1)
                self.ring_v[j, s][:, pos] = v.transpose(0, 1)
            self.h_seq_len[s] = c
        self.seq_len.copy_(torch.from_numpy(self.h_seq_len))
