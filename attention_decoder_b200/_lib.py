"""ctypes binding of liblfm3.so: the structs and entry points of include/lfm3.h, marshalling only.

Loading fails loudly when the library has not been built: there is no fallback path.
"""
import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblfm3.so")

LFM3_MAX_LAYERS = 64
LFM3_LAYER_CONV, LFM3_LAYER_FULL, LFM3_LAYER_SLIDING = 0, 1, 2
LFM3_FFN_BF16, LFM3_FFN_NVFP4, LFM3_FFN_AFFINE = 0, 1, 2

STATUS = {0: "LFM3_OK", -1: "LFM3_E_ARG", -2: "LFM3_E_CONFIG", -3: "LFM3_E_CAPACITY", -4: "LFM3_E_CUDA",
          -5: "LFM3_E_UNSUPPORTED", -6: "LFM3_E_TIMEOUT", -7: "LFM3_E_STATE"}

# exported entry points (every one declared in include/lfm3.h)
SYMBOLS = ("lfm3_create", "lfm3_bind_workspace", "lfm3_prefill", "lfm3_prefill_padded", "lfm3_decode_step",
           "lfm3_verify", "lfm3_commit", "lfm3_decode_step_noalloc", "lfm3_state_bytes", "lfm3_keep", "lfm3_restore", "lfm3_check_device_errors",
           "lfm3_selftest_wait", "lfm3_profile_enable", "lfm3_profile_read", "lfm3_last_launch_count",
           "lfm3_last_error", "lfm3_free")


class lfm3_config(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("layer_type", C.c_int8 * LFM3_MAX_LAYERS),
                ("d_model", C.c_int), ("d_ffn", C.c_int), ("n_q", C.c_int), ("n_kv", C.c_int),
                ("head_dim", C.c_int), ("conv_taps", C.c_int), ("window", C.c_int), ("vocab", C.c_int),
                ("theta_full", C.c_float), ("theta_sliding", C.c_float), ("rope_pairs_full", C.c_int),
                ("eps", C.c_float), ("has_head", C.c_int), ("ffn_format", C.c_int), ("page_size", C.c_int),
                ("n_pages", C.c_int), ("max_streams", C.c_int), ("max_pages_per_stream", C.c_int),
                ("max_chunk", C.c_int), ("max_batch", C.c_int), ("ffn_bits", C.c_int)]


class lfm3_layer_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("op_norm", "post_op_norm", "ffn_norm", "post_ffn_norm", "in_proj", "conv",
                                          "out_proj", "qkvg", "q_norm", "k_norm", "o_proj", "w1", "w3", "w2",
                                          "w1_codes", "w1_scales", "w3_codes", "w3_scales", "w2_codes",
                                          "w2_scales")] + [("w13_scale", C.c_float), ("w2_scale", C.c_float)] + \
        [(n, C.c_void_p) for n in ("w1_biases", "w3_biases", "w2_biases")]


class lfm3_weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("final_norm", C.c_void_p), ("layers", C.POINTER(lfm3_layer_weights))]


class lfm3_state(C.Structure):
    _fields_ = [("conv_state", C.c_void_p), ("ring_k", C.c_void_p), ("ring_v", C.c_void_p), ("kv_k", C.c_void_p),
                ("kv_v", C.c_void_p), ("page_table", C.c_void_p), ("seq_len", C.c_void_p),
                ("h_seq_len", C.POINTER(C.c_int32)), ("h_page_table", C.POINTER(C.c_int32))]


_lib = None


def lib():
    """The loaded library; raises if liblfm3.so is missing (build it with attention_decoder_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run python -m attention_decoder_b200.build")
    L = C.CDLL(LIB_PATH)
    vp, i32p = C.c_void_p, C.POINTER(C.c_int32)
    L.lfm3_create.argtypes = [C.POINTER(lfm3_config), C.POINTER(lfm3_weights), C.POINTER(C.c_size_t), C.POINTER(vp)]
    L.lfm3_bind_workspace.argtypes = [vp, vp, C.c_size_t]
    L.lfm3_prefill.argtypes = [vp, C.POINTER(lfm3_state), C.c_int, vp, vp, C.c_int, vp, vp, vp, vp]
    L.lfm3_prefill_padded.argtypes = [vp, C.POINTER(lfm3_state), C.c_int, vp, vp, C.c_int, C.c_int, vp, vp, vp, vp]
    L.lfm3_decode_step.argtypes = [vp, C.POINTER(lfm3_state), C.c_int, i32p, vp, vp, vp, vp, vp, vp, vp]
    L.lfm3_decode_step_noalloc.argtypes = L.lfm3_decode_step.argtypes
    L.lfm3_verify.argtypes = [vp, C.POINTER(lfm3_state), C.c_int, i32p, vp, C.c_int, vp, vp, vp, vp, vp, vp]
    L.lfm3_commit.argtypes = [vp, C.POINTER(lfm3_state), C.c_int, i32p, i32p, vp]
    L.lfm3_check_device_errors.argtypes = [vp, vp]
    L.lfm3_selftest_wait.argtypes = [vp, C.c_uint, vp]
    L.lfm3_state_bytes.argtypes = [vp, C.c_int]
    L.lfm3_state_bytes.restype = C.c_size_t
    L.lfm3_keep.argtypes = [vp, C.POINTER(lfm3_state), C.c_int, vp, C.c_size_t, C.POINTER(C.c_int), vp]
    L.lfm3_restore.argtypes = [vp, C.POINTER(lfm3_state), C.c_int, vp, C.c_size_t, C.c_int, vp]
    L.lfm3_profile_enable.argtypes = [vp, C.c_int, C.c_int]
    dp = C.POINTER(C.c_double)
    L.lfm3_profile_read.argtypes = [vp, C.POINTER(C.c_int), dp, dp, dp]
    L.lfm3_last_launch_count.argtypes = [vp]
    L.lfm3_last_error.argtypes = [vp]
    L.lfm3_last_error.restype = C.c_char_p
    L.lfm3_free.argtypes = [vp]
    L.lfm3_free.restype = None
    for name in ("lfm3_create", "lfm3_bind_workspace", "lfm3_prefill", "lfm3_prefill_padded", "lfm3_decode_step",
                 "lfm3_verify", "lfm3_commit", "lfm3_decode_step_noalloc", "lfm3_keep", "lfm3_restore", "lfm3_check_device_errors",
                 "lfm3_selftest_wait", "lfm3_profile_enable", "lfm3_profile_read", "lfm3_last_launch_count"):
        getattr(L, name).restype = C.c_int
    _lib = L
    return L


class Lfm3Error(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


def check(status, ctx=None):
    if status != 0:
        msg = lib().lfm3_last_error(ctx)
        raise Lfm3Error(status, msg.decode() if msg else "")
    return status


# Same names as the C ABI; arguments are passed through unchanged.
def lfm3_create(cfg, weights, ws_bytes, out):
    return lib().lfm3_create(cfg, weights, ws_bytes, out)


def lfm3_bind_workspace(ctx, d_ws, nbytes):
    return lib().lfm3_bind_workspace(ctx, d_ws, nbytes)


def lfm3_prefill(ctx, st, slot, d_tokens, d_embeds, n, d_logits, d_argmax, d_hidden, stream):
    return lib().lfm3_prefill(ctx, st, slot, d_tokens, d_embeds, n, d_logits, d_argmax, d_hidden, stream)


def lfm3_prefill_padded(ctx, st, slot, d_tokens, d_embeds, n_rows, n_real, d_logits, d_argmax, d_hidden, stream):
    return lib().lfm3_prefill_padded(ctx, st, slot, d_tokens, d_embeds, n_rows, n_real, d_logits, d_argmax, d_hidden,
                                     stream)


def lfm3_decode_step(ctx, st, n_streams, h_slots, d_slots, d_tokens, d_embeds, d_logits, d_argmax, d_hidden, stream):
    return lib().lfm3_decode_step(ctx, st, n_streams, h_slots, d_slots, d_tokens, d_embeds, d_logits, d_argmax,
                                  d_hidden, stream)


def lfm3_verify(ctx, st, n_streams, h_slots, d_slots, W, d_tokens, d_embeds, d_logits, d_argmax, d_hidden, stream):
    return lib().lfm3_verify(ctx, st, n_streams, h_slots, d_slots, W, d_tokens, d_embeds, d_logits, d_argmax, d_hidden,
                             stream)


def lfm3_commit(ctx, st, n_streams, h_slots, h_accept, stream):
    return lib().lfm3_commit(ctx, st, n_streams, h_slots, h_accept, stream)


def lfm3_decode_step_noalloc(ctx, st, n_streams, h_slots, d_slots, d_tokens, d_embeds, d_logits, d_argmax, d_hidden,
                             stream):
    return lib().lfm3_decode_step_noalloc(ctx, st, n_streams, h_slots, d_slots, d_tokens, d_embeds, d_logits,
                                          d_argmax, d_hidden, stream)


def lfm3_state_bytes(ctx, at):
    return lib().lfm3_state_bytes(ctx, at)


def lfm3_keep(ctx, st, slot, d_snap, nbytes, at_out, stream):
    return lib().lfm3_keep(ctx, st, slot, d_snap, nbytes, at_out, stream)


def lfm3_restore(ctx, st, slot, d_snap, nbytes, at, stream):
    return lib().lfm3_restore(ctx, st, slot, d_snap, nbytes, at, stream)


def lfm3_check_device_errors(ctx, stream):
    return lib().lfm3_check_device_errors(ctx, stream)


def lfm3_selftest_wait(ctx, rounds, stream):
    return lib().lfm3_selftest_wait(ctx, rounds, stream)


def lfm3_profile_enable(ctx, on, capacity):
    return lib().lfm3_profile_enable(ctx, on, capacity)


def lfm3_profile_read(ctx, launches, ms, nbytes, flops):
    return lib().lfm3_profile_read(ctx, launches, ms, nbytes, flops)


def lfm3_last_launch_count(ctx):
    return lib().lfm3_last_launch_count(ctx)


def lfm3_last_error(ctx):
    return lib().lfm3_last_error(ctx)


def lfm3_free(ctx):
    return lib().lfm3_free(ctx)
