// Internal launch interface of the LFM3 kernels (host side). Not part of the C ABI.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <utility>

#include "common.cuh"

namespace lfm3 {

// Geometry the kernels implement (the LFM3-1.7B decoder).
constexpr int D = 2048;        // d_model
constexpr int F = 7680;        // d_ffn
constexpr int HQ = 16;         // query heads
constexpr int HKV = 4;         // kv heads
constexpr int HD = 128;        // head_dim
constexpr int TAPS = 7;        // conv taps
constexpr int CST = TAPS - 1;  // conv state columns
constexpr int WIN = 256;       // sliding window
constexpr int PAGE = 64;       // positions per KV page
constexpr int NQKVG = HQ * HD + 2 * HKV * HD + HQ;  // 3088 fused projection rows
constexpr int GQA = HQ / HKV;

// Launch counter of the calling thread (reset by the API at each call).
extern thread_local int g_launches;
#ifdef LFM3_TRACE
extern unsigned long long* g_trace;  // timeline buffer of the diagnostic build (lfm3_trace_set)
#endif

// Every kernel is launched with programmatic stream serialisation (see pdl_wait()).
template <typename... KArgs, typename... Args>
inline cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  ++g_launches;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Where the rows of a call sit: row r belongs to slot row_slot[r] at position row_pos[r].
struct Rows {
  const int32_t* slot;
  const int32_t* pos;
  int n;
};

// ---------------------------------------------------------------- elementwise / small kernels
// decode: `win` consecutive rows per listed slot (1, or a verify window) at seq_len[slot] + r % win
cudaError_t setup_rows(int prefill, int slot, const int32_t* d_slots, const int32_t* seq_len, int rows, int win,
                       int32_t* row_slot, int32_t* row_pos, unsigned long long* amax, cudaStream_t s);
cudaError_t embed_rows(const int32_t* tokens, const bf16* table, const bf16* vecs, int rows, float* x_res,
                       float* dump, cudaStream_t s);
// x_res[r] += g_post * RMS(sum_s part[s][r]) (if n_part > 0); dump x_res; xn = g_next * RMS(x_res),
// rounded to bf16 and stored as bf16, or (xn_f16) as the f16 of that bf16 value
cudaError_t resid_norm(float* x_res, const float* part, int n_part, long part_stride, const bf16* g_post,
                       const bf16* g_next, bf16* xn, int rows, float eps, float* dump, int xn_f16, cudaStream_t s);
// one row per stream (win 1: the state shifts), or verify windows of `win` rows per stream (the
// state is left alone; the state after each row goes to snap [rows][CST][D])
// bcx: the in_proj rows as the sum of n_parts K-split partials, part_stride floats apart
cudaError_t conv_decode(const float* bcx, int n_parts, long part_stride, const bf16* conv_w, bf16* state_layer,
                        const int32_t* row_slot, int rows, int win, bf16* snap, bf16* y, cudaStream_t s);
// n rows; the new state is columns [n_state, n_state + 6) of [state | bx] (n_state <= n)
cudaError_t conv_prefill(const float* bcx, const bf16* conv_w, bf16* state_slot, int n, int n_state, bf16* y,
                         cudaStream_t s);

enum KvDst { KV_PAGES = 0, KV_SCRATCH = 1 };
struct KvWrite {
  int mode;
  bf16* k;               // pages: pool base of this layer; scratch: sliding scratch base
  bf16* v;
  const int32_t* page_table;
  int max_pages;         // page-table width
  int max_streams;
  int scratch_rows;      // WIN + max_chunk (scratch mode)
};
cudaError_t qk_norm_rope_kv(const float* part, int n_part, long part_stride, const bf16* q_norm,
                            const bf16* k_norm, const float* rope_cos, const float* rope_sin, Rows rows,
                            float eps, bf16* q_out, float* gate_out, KvWrite kv, cudaStream_t s);
cudaError_t ring_to_scratch(const bf16* ring_k, const bf16* ring_v, int slot, int max_streams, int p0,
                            bf16* sk, bf16* sv, int scratch_rows, cudaStream_t s);
cudaError_t scratch_to_ring(const bf16* sk, const bf16* sv, int scratch_rows, int n, int p0, bf16* ring_k,
                            bf16* ring_v, int slot, int max_streams, cudaStream_t s);
// advance = 0 leaves seq_len alone (a verify window)
cudaError_t finish_step(int32_t* seq_len, const int32_t* row_slot, int rows, int add_prefill, int prefill_slot,
                        const unsigned long long* amax, int32_t* argmax_out, int advance, cudaStream_t s);

// Commit of verify windows: per stream, the first k of its W rows become state.
struct CommitArgs {
  int n, W, n_conv, n_sliding, max_streams, max_batch;
  int slot[64], pos[64], k[64];      // slot, position of the window's first row, rows accepted
  const bf16* snap;                  // [n_conv][max_batch][CST][D]
  const bf16* side_k; const bf16* side_v;  // [n_sliding][max_batch][HKV][HD]
  bf16* conv; bf16* ring_k; bf16* ring_v;
  int32_t* seq_len;
};
cudaError_t commit_windows(const CommitArgs& a, cudaStream_t s);
// One bounded wait that can never complete (at most `rounds` polls), then the status word is set.
cudaError_t wait_selftest(int* err, unsigned rounds, cudaStream_t s);

// Kept state of one slot at mark `at` (see k_state_copy): state -> snapshot (keep) or back.
struct SnapArgs {
  int restore, slot, at, npg;          // npg = ceil(at / PAGE) pages per full layer
  int n_conv, n_sliding, n_full, max_streams, n_pages, max_pages;
  void* snap;
  bf16* conv; bf16* ring_k; bf16* ring_v; bf16* kv_k; bf16* kv_v;
  const int32_t* page_table;
  int32_t* seq_len;
};
size_t snapshot_bytes(int n_conv, int n_sliding, int n_full, int at);
cudaError_t state_copy(const SnapArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- decode projection epilogues
enum GemvEpi { GEMV_PARTIAL = 0, GEMV_SWIGLU = 1, GEMV_CONV = 2, GEMV_HEAD = 3 };

// ---------------------------------------------------------------- decode weight streaming (persistent)
enum WsPro { WS_PRO_LOAD = 0, WS_PRO_NORM = 1 };
struct WsArgs {
  const bf16* w; const bf16* w3;                   // bf16 weights [N][K] (SwiGLU: w1, w3)
  const uint8_t* codes; const uint8_t* scales;     // NVFP4 (SwiGLU: w1)
  const uint8_t* codes3; const uint8_t* scales3;   // NVFP4 w3
  int bits;                                        // affine: code width (4, 6, 8); scales and biases bf16
  float tscale;
  int K, N, rows, splits;
  int pro;                                         // WS_PRO_LOAD: x bf16 [rows][K]; WS_PRO_NORM: see below
  const bf16* x;
  // WS_PRO_NORM (K == d_model): x' = x_in + g_post * RMS(sum_s parts[s]) (no parts: x' = x_in),
  // written to x_out (+ dump) by block (0,0); activations = bf16(g_next * RMS(x'))
  const float* x_in; float* x_out; const float* parts; int n_parts; long part_stride;
  const bf16* g_post; const bf16* g_next; float eps; float* dump;
  float* part_out;                                 // PARTIAL: [splits][rows][N]
  bf16* out;                                       // SWIGLU: [rows][N]
  const bf16* conv_w; bf16* conv_state; const int32_t* row_slot; bf16* y;  // CONV
  int win; bf16* conv_snap;                        // CONV in a verify window (win > 1), see conv_decode
  unsigned long long* amax; float* logits;         // HEAD (logits may be null)
  int* err;
  int stages;                                      // set by the launcher
#ifdef LFM3_TRACE
  unsigned long long* trace;
  int trace_id;
#endif
};
struct WsMaps {
  CUtensorMap w, w3, s, s3;  // weights (SwiGLU: w1, w3) or quantised codes; NVFP4 / affine scales
  CUtensorMap b, b3;         // affine biases
};
bool make_ws_map(CUtensorMap* m, const void* w, int N, int K, int fp4, int br, int kch);
bool make_ws_scale_map(CUtensorMap* m, const void* sc, int N, int K, int br, int kch);
int ws_kch(int epi, int fp4);
int ws_br(int epi, int fp4);
enum WsFormat { WS_BF16 = 0, WS_NVFP4 = 1, WS_AFFINE = 2 };
cudaError_t wstream(int epi, int format, const WsMaps& mp, const WsArgs& a, cudaStream_t s);
// Affine code maps ([N][K * bits / 8] bytes as 64- or 96-byte blocks) and bf16 scale / bias maps.
bool make_aff_map(CUtensorMap* m, const void* codes, int N, int K, int bits, int br);
bool make_aff_sb_map(CUtensorMap* m, const void* sb, int N, int K, int br);
int aff_br(int epi);
// Affine weights expanded to bf16 for the tensor-core GEMM: w = bf16(s * q + b).
cudaError_t affine_to_bf16(const uint8_t* codes, const void* scales, const void* biases, int bits, int N, int K, bf16* out,
                           cudaStream_t s);
cudaError_t wstream_init();

// ---------------------------------------------------------------- attention
constexpr int DEC_KEYS = 64;  // keys per decode split: one 64-position page, or a quarter of the ring
constexpr int MAX_WIN = 8;    // rows per stream in one verify window
struct AttnLayer {
  int full;               // 1 full (pages), 0 sliding
  const bf16* k; const bf16* v;   // pages: this layer's pool; ring: this layer's ring base
  const int32_t* page_table;
  int max_pages, max_streams;
};
// Decode attention in one launch from the raw q|k|v|gate rows (see k_attn_decode_fused).
struct AttnDecodeArgs {
  const bf16* q_norm;
  const bf16* k_norm;
  const float* rope_cos;   // [pos][64] of this layer kind
  const float* rope_sin;
  float eps;
  unsigned* counters;      // [streams][HKV], zero between calls
  int* err;                // status word (a bounded wait that gave up)
  // verify windows: rows come in groups of `win` consecutive positions of one stream (1 when
  // decoding); a sliding layer's window rows go to side_k / side_v [rows][HKV][HD], not the ring
  int win;
  bf16* side_k;
  bf16* side_v;
  // the q|k|v|gate rows are the sum of n_parts K-split partials, part_stride floats apart (>= 1)
  int n_parts;
  long part_stride;
#ifdef LFM3_TRACE
  unsigned long long* trace;
  int trace_id;
#endif
};
// Split slots a decode step reserves per (stream, head) in the partials buffer: the smallest
// power of two >= the splits of the longest context (and >= the ring's WIN / DEC_KEYS).
int attn_decode_splits(int max_pos);
cudaError_t attn_decode_fused(const float* qkvg, Rows rows, AttnLayer L, const AttnDecodeArgs& A, int splits,
                              float* part, bf16* y, cudaStream_t s);
cudaError_t attn_init();
// Device address and size (floats) of the library's fixed attention scratch on the current device.
cudaError_t attn_static_scratch(float** ptr, size_t* nfloats);

// Prefill attention on tcgen05: maps over q [rows][16][128] and K/V stores viewed as [rows][128].
struct AttnTcArgs {
  int n, p0, slot, full, row0;
  const int32_t* page_table;
  int max_pages, scratch_rows;
  const float* gate;
  bf16* y;
  int* err;
};
cudaError_t attn_tc_init();
bool make_tmap_q(CUtensorMap* m, const void* q, uint64_t rows);
bool make_tmap_kv(CUtensorMap* m, const void* base, uint64_t rows);
cudaError_t attn_prefill_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnTcArgs& a,
                            cudaStream_t s);

// ---------------------------------------------------------------- tensor-core GEMM (prefill)
// GEMM_HEAD: fp32 logits (optional) and the per-row argmax of the tied head, as the packed key
// of the weight-streaming head (see the HEAD epilogue there).
enum GemmEpi { GEMM_F32 = 0, GEMM_BF16 = 1, GEMM_SWIGLU = 2, GEMM_HEAD = 3 };
struct GemmPlan {
  CUtensorMap a;      // activations [M][K] bf16, box 64 x 128
  CUtensorMap b;      // weights [N][K] bf16 (SwiGLU: w1)
  CUtensorMap b3;     // SwiGLU: w3
  CUtensorMap bh, b3h;  // SwiGLU with 128-column tiles: w1 and w3 in 64-row boxes
  CUtensorMap o;      // output [M][ld] (fp32, or bf16), 32-row boxes of 128 bytes for TMA stores
  int epi, M, N, K;
  void* out;          // fp32 or bf16 [M][ld]; GEMM_HEAD: logits [M][N] or null
  int ld;
  float alpha;        // scales the accumulator (NVFP4 tensor scale; 1 otherwise)
  // set per call (defaults 1 / 0 / null): K splits of an fp32 output, written as partial sums to
  // out + s * M * ld (plain stores); the argmax keys of GEMM_HEAD
  int splits;
  unsigned long long* amax;
  int w_const;        // 1: weights no kernel writes (read before the wait on the previous kernel)
  // NVFP4 weights (q4 = 1): codes [N][K/2] in 64-row (SwiGLU: w1 and w3) or 128-row boxes of one
  // K block, E4M3 scales [N][K/16]; the activations (a) are f16 and the SwiGLU output is f16
  int q4;
  CUtensorMap q, q3;
  const uint8_t* sc;
  const uint8_t* sc3;
};
bool make_tmap_codes(CUtensorMap* m, const void* codes, uint64_t rows, uint64_t K, uint32_t box_rows);
bool tma_init();
bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);
// Output map of a GEMM: [rows][cols] with row pitch ld elements, fp32 (32-column boxes) or bf16
// (64-column boxes), 32 rows per box, 128-byte swizzle.
bool make_tmap_out(CUtensorMap* m, void* base, bool fp32, uint64_t rows, uint64_t cols, uint64_t ld);
cudaError_t gemm(const GemmPlan& p, int M, int* err, cudaStream_t s);
bool gemm_wide(int N);  // 256-column tiles for this output width
cudaError_t gemm_init();

}  // namespace lfm3
