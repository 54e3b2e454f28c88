/*
 * lfm3.h - C ABI of the LFM3-1.7B hybrid decoder forward on one NVIDIA B200 (sm_100a).
 *
 * What it computes (coreai-model-zoo note "lfm3-1.7b-port", LFM2.5 -> LFM3 diff table, and
 * TensorFold issue #1491, "Architecture"): a 24-layer decoder at width 2048 made of
 *   - 13 gated short-conv blocks: in_proj 2048 -> B | C | x, Bx = B * x, a 7-tap causal
 *     depthwise conv over Bx whose state keeps the last 6 columns, y = C * conv, out_proj;
 *   - 6 full-attention and 5 sliding-window (256) GQA blocks: 16 q / 4 kv heads of 128,
 *     per-head q/k RMSNorm, rotary theta 1e6 on 32 of 64 pairs (full) or theta 1e4 on all
 *     pairs (sliding), a sigmoid(gate_proj(x)) scalar per head multiplied in before o_proj;
 *   - sandwich RMSNorms (eps 1e-5) around every mixer and FFN;
 *   - a SwiGLU FFN of 7680, bf16 or NVFP4 weight-only (TensorFold PR #1508, "What");
 *   - a tied 128000-row head with greedy (argmax, ties to the lowest id) selection.
 *
 * Conventions for every entry point
 *   - Ownership: the CALLER owns all device memory (weights, state, workspace, outputs) and
 *     every host array passed in. The library owns only its host-side context. The per-slot
 *     state the pages' engine keeps for itself (TensorFold PR #1508, "What": a 6-row conv state
 *     per slot, a per-slot ring for the sliding layers, pages of a pool for the full layers;
 *     pool-leasing commit: the tables and conv states of the slots) is here a caller-allocated
 *     lfm3_state whose layout this header fixes and which only this library writes.
 *   - All pointers named d_* or documented "device" are device pointers; h_* are host.
 *   - bf16 tensors are IEEE bfloat16 bit patterns, row-major, densely packed.
 *   - Calls enqueue work on the given CUDA stream (a cudaStream_t passed as void*; NULL =
 *     legacy default stream) and return without synchronising.
 *   - Errors: arguments, configuration and capacity are checked on the host BEFORE anything
 *     is enqueued; on any error nothing is launched and no state is modified. CUDA launch
 *     errors map to LFM3_E_CUDA. lfm3_last_error() gives a message naming the refusal
 *     (TensorFold PR #1508, NVFP4 admission commit: an unsupported layout is refused by name,
 *     e.g. "Lfm3UnsupportedGeometry: d_model = 4096").
 *   - The library never allocates device memory and never reads /writes device memory from
 *     the host, except lfm3_bind_workspace (which uploads constant tables into the workspace)
 *     and lfm3_check_device_errors (which reads one status word).
 */
#ifndef LFM3_H
#define LFM3_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct lfm3_ctx lfm3_ctx; /* opaque; created by lfm3_create, freed by lfm3_free */

typedef enum {
  LFM3_OK = 0,
  LFM3_E_ARG = -1,         /* a NULL or out-of-range argument                        */
  LFM3_E_CONFIG = -2,      /* an inconsistent configuration                           */
  LFM3_E_CAPACITY = -3,    /* rows past a slot's pages, or more rows than the workspace */
  LFM3_E_CUDA = -4,        /* a CUDA runtime/driver call failed                       */
  LFM3_E_UNSUPPORTED = -5, /* a geometry the kernels do not implement (named in the message) */
  LFM3_E_TIMEOUT = -6,     /* a device-side bounded wait gave up (see lfm3_check_device_errors) */
  LFM3_E_STATE = -7        /* workspace not bound, or the context was used after an error */
} lfm3_status;

enum { LFM3_LAYER_CONV = 0, LFM3_LAYER_FULL = 1, LFM3_LAYER_SLIDING = 2 };
enum { LFM3_FFN_BF16 = 0, LFM3_FFN_NVFP4 = 1, LFM3_FFN_AFFINE = 2 };
#define LFM3_MAX_LAYERS 64

/* Geometry and capacity. The kernels implement d_model 2048, d_ffn 7680, 16 q / 4 kv heads of
 * 128, 7 conv taps, window 256 and page size 64; other values are refused with
 * LFM3_E_UNSUPPORTED. n_layers and the layer pattern are free (1..64 layers). */
typedef struct {
  int n_layers;
  int8_t layer_type[LFM3_MAX_LAYERS]; /* LFM3_LAYER_* per layer, in order                 */
  int d_model, d_ffn, n_q, n_kv, head_dim, conv_taps, window, vocab;
  float theta_full, theta_sliding; /* rotary bases: full layers, sliding layers           */
  int rope_pairs_full;             /* rotated (i, i + head_dim/2) pairs on full layers (32) */
  float eps;                       /* RMSNorm epsilon (1e-5)                              */
  int has_head;                    /* 1: token ids in, embedding + tied head + argmax out; 0: vectors in/out */
  int ffn_format;                  /* LFM3_FFN_BF16, LFM3_FFN_NVFP4 or LFM3_FFN_AFFINE    */
  int page_size;                   /* positions per KV page (64)                          */
  int n_pages;                     /* pages in the pool, per full-attention layer         */
  int max_streams;                 /* slots in the state                                  */
  int max_pages_per_stream;        /* page-table width; a slot holds at most this x page_size positions */
  int max_chunk;                   /* rows per prefill pass (1..2048); longer prompts run in chunks */
  int max_batch;                   /* rows per decode step (1..64): streams, or streams x window rows in lfm3_verify */
  int ffn_bits;                    /* LFM3_FFN_AFFINE: code width, 4, 6 or 8 (ignored otherwise) */
} lfm3_config;

/* One layer's weights: device pointers, bf16 unless stated; unused fields may be NULL. */
typedef struct {
  const void* op_norm;       /* [d_model] operator_norm gain                              */
  const void* post_op_norm;  /* [d_model] post_operator_norm gain                         */
  const void* ffn_norm;      /* [d_model]                                                 */
  const void* post_ffn_norm; /* [d_model]                                                 */
  /* conv layers */
  const void* in_proj;  /* [3*d_model][d_model], output rows B | C | x                    */
  const void* conv;     /* [d_model][conv_taps], tap conv_taps-1 multiplies the newest column */
  const void* out_proj; /* [d_model][d_model]                                              */
  /* attention layers */
  const void* qkvg;   /* [n_q*hd + 2*n_kv*hd + n_q][d_model]: q rows, k rows, v rows, gate rows */
  const void* q_norm; /* [head_dim], shared by all q heads                                 */
  const void* k_norm; /* [head_dim], shared by all k heads                                 */
  const void* o_proj; /* [d_model][n_q*head_dim]                                           */
  /* bf16 FFN */
  const void* w1; /* [d_ffn][d_model] */
  const void* w3; /* [d_ffn][d_model] */
  const void* w2; /* [d_model][d_ffn] */
  /* NVFP4 FFN: E2M1 codes packed two per byte along the input dimension (element 2b in the low
   * nibble), one E4M3 scale byte per 16 inputs, row-major; w = e2m1 * e4m3 * tensor scale.   */
  const uint8_t* w1_codes;  /* [d_ffn][d_model/2]  */
  const uint8_t* w1_scales; /* [d_ffn][d_model/16] */
  const uint8_t* w3_codes;
  const uint8_t* w3_scales;
  const uint8_t* w2_codes;  /* [d_model][d_ffn/2]  */
  const uint8_t* w2_scales; /* [d_model][d_ffn/16] */
  float w13_scale;          /* fp32 tensor scale shared by w1 and w3 */
  float w2_scale;
  /* Affine FFN (MLX affine groups of 64; TensorFold issue #1491, "Checkpoint handling"): w = s * q + b
   * with q an unsigned ffn_bits-bit code, s and b bf16 per group of 64 inputs. The codes of a row
   * are one little-endian bit stream (code k at bits [k * bits, k * bits + bits)) in the *_codes
   * fields, [rows][cols * bits / 8] bytes; the scales in the *_scales fields and the biases here
   * are bf16 [rows][cols / 64]. */
  const uint8_t* w1_biases;
  const uint8_t* w3_biases;
  const uint8_t* w2_biases;
} lfm3_layer_weights;

typedef struct {
  const void* embed;                /* [vocab][d_model] (tied head); NULL when has_head == 0 */
  const void* final_norm;           /* [d_model] embedding_norm gain; NULL when has_head == 0 */
  const lfm3_layer_weights* layers; /* HOST array [n_layers], copied by lfm3_create          */
} lfm3_weights;

/* Decode state, caller-owned device memory (bf16 unless stated). Layouts:
 *   conv_state  [n_conv][max_streams][conv_taps-1][d_model]   oldest column first
 *   ring_k/v    [n_sliding][max_streams][n_kv][window][head_dim]   slot = position % window
 *   kv_k/v      [n_full][n_pages][n_kv][page_size][head_dim]      position p of slot s lives in
 *               page page_table[s][p / page_size], row p % page_size
 *   page_table  device int32 [max_streams][max_pages_per_stream] (values in [0, n_pages))
 *   seq_len     device int32 [max_streams]: tokens already consumed by each slot; the next row
 *               of a slot sits at position seq_len[slot]
 *   h_seq_len   HOST int32 [max_streams]: the same values; the library reads it to check
 *               capacity and updates it when it enqueues work (the device copy is updated by
 *               the enqueued kernels).
 *   h_page_table HOST int32 [max_streams][max_pages_per_stream]: mirror used only to check that
 *               every page a call writes is in range. */
typedef struct {
  void* conv_state;
  void* ring_k;
  void* ring_v;
  void* kv_k;
  void* kv_v;
  const int32_t* page_table;
  int32_t* seq_len;
  int32_t* h_seq_len;
  const int32_t* h_page_table;
} lfm3_state;

/* Validates cfg and w (no device access, no launches) and returns the number of workspace
 * bytes the context needs. On success *out owns a context (free with lfm3_free); on failure
 * *out is NULL and lfm3_last_error(NULL) names the refusal: LFM3_E_UNSUPPORTED for a geometry or
 * FFN format the kernels do not implement, named in the message as the pages' admission does
 * (TensorFold PR #1508, NVFP4 admission commit: "refuse the other by name"), LFM3_E_CONFIG for an
 * inconsistent configuration, LFM3_E_ARG for a NULL or misaligned weight pointer. The geometry is
 * the pages' LFM3-1.7B one (coreai-model-zoo note "lfm3-1.7b-port", LFM2.5 -> LFM3 diff table and
 * "Unchanged" paragraph). */
lfm3_status lfm3_create(const lfm3_config* cfg, const lfm3_weights* w, size_t* workspace_bytes,
                        lfm3_ctx** out);

/* Binds caller-owned device workspace (>= the size lfm3_create reported, 256-byte aligned) and
 * uploads the rotary tables into it (synchronous). Must precede prefill/decode. The tables hold
 * cos/sin of p * theta^(-2i/128) per position p and pair i, built in double precision and stored
 * fp32 (coreai-model-zoo note "lfm3-1.7b-port", partial-rotary paragraph: theta 1e6 on pairs
 * i < 32 of full layers, theta 1e4 on all 64 pairs of sliding layers). Errors: LFM3_E_ARG for a
 * NULL, misaligned or short workspace; LFM3_E_CUDA if a copy or a tensor-map encoding fails. */
lfm3_status lfm3_bind_workspace(lfm3_ctx* ctx, void* d_workspace, size_t bytes);

/* Prompt pass for one slot: consumes n rows at positions h_seq_len[slot] .. +n-1, in chunks
 * of at most max_chunk rows, updating conv state, ring, pages and seq_len in place.
 * Positions come from the state alone and there is no mask input: a key is visible to a query
 * iff its position is not later and, on sliding layers, fewer than 256 positions earlier
 * (coreai-model-zoo note "lfm3-1.7b-port", "window_size, with no mask input"). The conv state
 * after a chunk of n rows is columns [n, n + 6) of [state | Bx] (same note, chunked-prefill
 * paragraph).
 *   d_tokens    device int32 [n] (has_head == 1) or NULL
 *   d_embeds    device bf16 [n][d_model] input vectors (has_head == 0) or NULL
 *   d_logits    device fp32 [vocab]: logits of the LAST row (has_head == 1), or NULL
 *   d_argmax    device int32 [1]: greedy id of the last row, or NULL
 *   d_hidden    device fp32 [n_layers+1][n][d_model]: the residual stream entering layer 0 and
 *               leaving every layer (the per-layer parity tap), or NULL
 * Refuses with LFM3_E_CAPACITY, before anything is enqueued, if the slot's pages cannot hold
 * seq_len + n positions or a page-table entry it would write is outside the pool (TensorFold
 * PR #1508, pool-leasing commit: "forward refuses rows past a slot's pages"); LFM3_E_ARG for a bad
 * slot, an empty call, or inputs that do not match has_head; LFM3_E_STATE before
 * lfm3_bind_workspace. */
lfm3_status lfm3_prefill(lfm3_ctx* ctx, const lfm3_state* st, int slot, const int32_t* d_tokens,
                         const void* d_embeds, int n, float* d_logits, int32_t* d_argmax,
                         float* d_hidden, void* stream);

/* A prompt chunk padded at its end (coreai-model-zoo note "lfm3-1.7b-port", pad-tail paragraph):
 * n_rows rows (1..max_chunk) of which the first n_real (>= 1) are the prompt and the rest are
 * padding (the pages' engine writes token 0 there). Every row goes through the row-wise steps (the
 * projections, norms and FFN), so a caller can keep one fixed chunk shape; but no real row sees a
 * pad, the pads' keys and values are not stored, the conv state is columns [n_real, n_real + 6)
 * of [state | Bx] ("n = the number of query position ids >= 0") rather than the last 6, d_logits
 * and d_argmax belong to row n_real - 1, and seq_len advances by n_real. The real rows' results
 * and the state equal those of lfm3_prefill on the n_real rows alone. d_hidden, if given, holds
 * n_rows rows; the pad rows' values there are unspecified. Capacity is checked for the real rows
 * only. Errors: as lfm3_prefill, and LFM3_E_ARG for n_rows or n_real out of range. */
lfm3_status lfm3_prefill_padded(lfm3_ctx* ctx, const lfm3_state* st, int slot, const int32_t* d_tokens,
                                const void* d_embeds, int n_rows, int n_real, float* d_logits, int32_t* d_argmax,
                                float* d_hidden, void* stream);

/* One decode step for n_streams distinct slots (one row each, at position seq_len[slot]; as for
 * lfm3_prefill the position comes from the state and there is no mask input - coreai-model-zoo
 * note "lfm3-1.7b-port", "window_size, with no mask input"). Streams share no state; the pages'
 * engine checks that concurrent == solo (TensorFold PR #1508, "Verification"), which holds here
 * bit for bit at up to 16 streams. Up to 16 rows stream every weight through the weight-streaming
 * GEMVs; larger batches run the projections as tensor-core GEMMs (fp32 outputs split along K and
 * summed in split order), so their results match those of smaller batches to fp32 rounding, not
 * bit for bit. An NVFP4 FFN multiplies f16 copies of its bf16 activations: a value above 65504 in
 * magnitude there would not be representable.
 *   h_slots     HOST int32 [n_streams] slot ids (checked; must equal d_slots)
 *   d_slots     device int32 [n_streams]
 *   d_tokens    device int32 [n_streams] (has_head == 1) or NULL; may alias d_argmax of the
 *               previous step for a device-resident greedy loop
 *   d_embeds    device bf16 [n_streams][d_model] (has_head == 0) or NULL
 *   d_logits    device fp32 [n_streams][vocab] or NULL
 *   d_argmax    device int32 [n_streams] greedy ids, or NULL
 *   d_hidden    device fp32 [n_layers+1][n_streams][d_model] or NULL
 * Errors (nothing enqueued, no state touched): LFM3_E_CAPACITY if a slot's pages cannot hold one
 * more position (TensorFold PR #1508, pool-leasing commit: "forward refuses rows past a slot's
 * pages"); LFM3_E_ARG for a slot out of range or listed twice, n_streams outside 1..max_batch,
 * or inputs that do not match has_head; LFM3_E_STATE before lfm3_bind_workspace. */
lfm3_status lfm3_decode_step(lfm3_ctx* ctx, const lfm3_state* st, int n_streams, const int32_t* h_slots,
                             const int32_t* d_slots, const int32_t* d_tokens, const void* d_embeds,
                             float* d_logits, int32_t* d_argmax, float* d_hidden, void* stream);

/* Drafted windows (TensorFold PR #1508, lfm2_moe.cu paragraph: "the short conv over each stream's
 * state with every window row's snapshot, the commit of an accepted row's conv state"; its check
 * is "drafted == plain"). lfm3_verify runs, for each listed slot, W rows (1..8: the stream's next
 * token and W - 1 drafted ones) at positions seq_len[slot] .. + W - 1 in one pass and returns every
 * row's logits and greedy id; it commits nothing. The full layers' keys and values of the window
 * are written to the slot's pages past its cursor (where a later row overwrites them), the
 * sliding layers' go to the workspace, and so does the conv state after every window row.
 * lfm3_commit then makes the first accept[i] rows (1..W) of stream i the slot's state: the conv
 * state after row accept[i] - 1, those rows' keys and values in the rings, and seq_len advanced by
 * accept[i]. The result equals plain decode of the accepted tokens.
 *   d_tokens  device int32 [n_streams][W] (row i*W + j is stream i's j-th row), or NULL
 *   d_embeds  device bf16 [n_streams * W][d_model] (has_head == 0), or NULL
 *   d_logits  device fp32 [n_streams * W][vocab] or NULL;  d_argmax  device int32 [n_streams * W]
 *   d_hidden  device fp32 [n_layers+1][n_streams * W][d_model] or NULL
 * Errors (nothing enqueued): those of lfm3_decode_step for the listed slots; LFM3_E_ARG if W is
 * outside 1..8 or n_streams * W > max_batch; LFM3_E_CAPACITY if a slot's pages cannot hold the
 * window. Only the last window can be committed, and only before any other call touches its
 * slots: lfm3_commit refuses with LFM3_E_STATE otherwise (a decode step or another window ends
 * it), and with LFM3_E_ARG for slots that differ from the window's or accept counts out of range. */
lfm3_status lfm3_verify(lfm3_ctx* ctx, const lfm3_state* st, int n_streams, const int32_t* h_slots,
                        const int32_t* d_slots, int W, const int32_t* d_tokens, const void* d_embeds, float* d_logits,
                        int32_t* d_argmax, float* d_hidden, void* stream);

/* Commits the last verify window (see lfm3_verify). h_slots: the window's slots, in its order;
 * h_accept: HOST int32 [n_streams], rows accepted per stream (1..W). */
lfm3_status lfm3_commit(lfm3_ctx* ctx, const lfm3_state* st, int n_streams, const int32_t* h_slots,
                        const int32_t* h_accept, void* stream);

/* The same decode step as lfm3_decode_step, for callers that cannot allocate device memory at
 * the point of the call - a host program that hands this library a finished arena and forbids
 * later allocation, or code running where an allocation would synchronise the device. The
 * pages have no counterpart: it is a service of this library, not part of the method.
 *   Arguments, checks, state updates and results are those of lfm3_decode_step (a context with
 *   a bound workspace is still required). The difference: the attention's per-split partial
 *   results go to a fixed 4 MiB array inside the library's own device image instead of the
 *   workspace, and the step is launched kernel by kernel (no captured graph).
 *   Limit: n_streams x 16 heads x splits x 130 floats must fit in the 4 MiB, where splits is the
 *   smallest power of two >= 4 with 64 x splits >= (longest context + 1); larger calls are
 *   refused with LFM3_E_CAPACITY and a message giving both sizes. One stream fits any context
 *   below 16384 positions; 64 streams fit contexts below 256.
 *   Nothing in the array has to start at zero: every call writes all the partials it reads.
 *   The array is one per GPU for the whole process and every call shares it, so calls that can
 *   overlap on the GPU (different streams, different contexts) race on it; serialise them.
 *   The first call in each CUDA context looks the array's address up (cudaGetSymbolAddress) with
 *   that context current; make that first call before any stream capture. A context destroyed
 *   and created again (cudaDeviceReset) is a new context: its first call looks the address up
 *   again. No device memory is allocated or freed by this call. */
lfm3_status lfm3_decode_step_noalloc(lfm3_ctx* ctx, const lfm3_state* st, int n_streams, const int32_t* h_slots,
                                     const int32_t* d_slots, const int32_t* d_tokens, const void* d_embeds,
                                     float* d_logits, int32_t* d_argmax, float* d_hidden, void* stream);

/* Kept states (the prompt cache; TensorFold PR #1508, prompt-cache paragraph): "a state at `at` is
 * the slot's conv states and its keys and values at positions [0, at)"; on LFM3 it also holds
 * every sliding layer's ring, the model's other fixed region (same PR, "One backend" paragraph).
 * A state is kept behind a prompt chunk that ends at the mark and restored into another slot (its
 * own pages) before that slot's next chunk, so the later pass starts at its history; resumed ==
 * fresh, bit for bit. The buffer is caller-owned device memory, 16-byte aligned, laid out as
 *   [n_conv][conv_taps-1][d_model] | [n_sliding][K, V][n_kv][window][head_dim] |
 *   [n_full][K, V][ceil(at / page_size)][n_kv][page_size][head_dim]            (bf16)
 * Both calls enqueue one copy kernel on `stream` and allocate nothing. A mark inside a chunk
 * (the pages' "taps") is not offered: on LFM3 it needs the rings as they stood at the mark. */

/* Bytes of a state kept at mark `at` (0 for a NULL context or a negative mark). */
size_t lfm3_state_bytes(const lfm3_ctx* ctx, int at);

/* Keeps the state of `slot` at its current position: *at_out = h_seq_len[slot], and d_snap
 * (>= lfm3_state_bytes(at) bytes) receives its conv columns, rings and pages [0, at).
 * Errors: LFM3_E_CAPACITY if the buffer is too small; LFM3_E_ARG for a bad slot or buffer;
 * LFM3_E_STATE before lfm3_bind_workspace. Nothing is enqueued on error. */
lfm3_status lfm3_keep(lfm3_ctx* ctx, const lfm3_state* st, int slot, void* d_snap, size_t bytes, int* at_out,
                      void* stream);

/* Restores a state kept at mark `at` into `slot`: conv columns and rings are overwritten, the
 * kept pages are written into the slot's own pages (through its page table), and seq_len[slot]
 * and h_seq_len[slot] become `at`. The slot's previous contents are discarded. Errors:
 * LFM3_E_CAPACITY if the slot's pages cannot hold [0, at) or the buffer is too small (TensorFold
 * PR #1508, pool-leasing commit: "forward refuses rows past a slot's pages"); LFM3_E_ARG for a
 * bad slot, buffer or mark. Nothing is enqueued and no state is touched on error. */
lfm3_status lfm3_restore(lfm3_ctx* ctx, const lfm3_state* st, int slot, const void* d_snap, size_t bytes, int at,
                         void* stream);

/* Synchronises the stream and reads the device status word that bounded device-side waits set
 * when they give up (every wait on a copy or a peer block in the kernels has an iteration limit
 * and then records the failure and returns instead of spinning). Returns LFM3_OK or
 * LFM3_E_TIMEOUT; on LFM3_E_TIMEOUT it clears the word and the attention's split counters, so
 * the context stays usable, but the results of the calls since the last check are invalid. The
 * pages have no counterpart: a service of this library. */
lfm3_status lfm3_check_device_errors(lfm3_ctx* ctx, void* stream);

/* Self-test of the failure path (no counterpart on the pages): enqueues one kernel whose single
 * bounded wait can never complete - a fresh barrier that nothing arrives on - so that after at
 * most `rounds` polls (1..65536) it gives up and sets the status word exactly as the kernels' own
 * waits do. A following lfm3_check_device_errors returns LFM3_E_TIMEOUT and clears the word; the
 * state and the context are untouched and stay usable. Nothing faults, traps or hangs. */
lfm3_status lfm3_selftest_wait(lfm3_ctx* ctx, unsigned rounds, void* stream);

/* Kernel timing for measurement (no counterpart on the pages). While enabled, every projection
 * kernel that prefill/decode enqueue (the weight-streaming GEMVs of decode and the tensor-core
 * GEMMs of prefill) is bracketed by two CUDA events recorded on the call's stream; decode steps
 * then run launch by launch rather than from their captured graph. Event handles are host objects
 * created here (up to `capacity` brackets between reads); no device memory is allocated. */
lfm3_status lfm3_profile_enable(lfm3_ctx* ctx, int on, int capacity);

/* Synchronises on the recorded events and returns, summed over the brackets since the last
 * read: the number of launches, their device time in ms, their algorithmic bytes (weights +
 * activations in + results out) and their algorithmic FLOPs (2 * rows * N * K). Clears the
 * record. Returns LFM3_E_CAPACITY if more brackets were requested than `capacity` (the
 * excess launches ran unbracketed). */
lfm3_status lfm3_profile_read(lfm3_ctx* ctx, int* launches, double* ms, double* bytes, double* flops);

/* Number of kernels the last prefill/decode call enqueued. */
int lfm3_last_launch_count(const lfm3_ctx* ctx);

/* Message for the last error on this context (never NULL; "" after success). With ctx == NULL:
 * the message of the last failed lfm3_create on the calling thread. */
const char* lfm3_last_error(const lfm3_ctx* ctx);

/* Frees the host context. Device memory is the caller's and is not touched. */
void lfm3_free(lfm3_ctx* ctx);

#ifdef __cplusplus
}
#endif
#endif /* LFM3_H */
