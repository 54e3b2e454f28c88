// C ABI of the LFM3 decoder forward: host-side validation, workspace layout and the launch
// sequence of a prompt pass (lfm3_prefill) and of a decode step (lfm3_decode_step).
// The declarations and conventions are in include/lfm3.h.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "kernels.cuh"
#include "lfm3.h"

using namespace lfm3;

namespace {

// Decode GEMV K splits (partial sums are added by the consumer).
constexpr int SPLIT_DD = 2, SPLIT_W2 = 5, SPLIT_MAX = 8;
constexpr int GEMV_MAX_ROWS = 16;

struct LayerPlan {
  GemmPlan in_proj, out_proj, qkvg, o_proj, w13, w2;   // prefill (tensor-core GEMM)
  WsMaps ws_in, ws_out, ws_qkvg, ws_o, ws_w13, ws_w2;  // decode (weight streaming)
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

struct lfm3_ctx {
  lfm3_config cfg;
  std::vector<lfm3_layer_weights> L;
  const bf16* embed = nullptr;
  const bf16* final_norm = nullptr;
  int n_conv = 0, n_full = 0, n_sliding = 0;
  std::vector<int> kidx;
  int max_pos = 0, R = 0, max_splits = 0, scratch_rows = 0;
  size_t ws_bytes = 0;
  bool bound = false;
  // workspace carve
  int* err = nullptr;
  int32_t* row_slot = nullptr;
  int32_t* row_pos = nullptr;
  unsigned long long* amax = nullptr;
  float* x_res = nullptr;
  float* x_res2 = nullptr;  // decode: the residual stream ping-pongs between x_res and x_res2
  bf16* xn = nullptr;
  bf16* big = nullptr;
  bf16* y = nullptr;
  float* part = nullptr;
  float* part2 = nullptr;   // decode: FFN down-projection partials
  float* part3 = nullptr;   // decode: q|k|v|gate projection
  bf16* q = nullptr;
  float* gate = nullptr;
  bf16* sk = nullptr;
  bf16* sv = nullptr;
  float* attn_part = nullptr;
  float* rope_cos[2] = {nullptr, nullptr};  // [0] full layers, [1] sliding layers
  float* rope_sin[2] = {nullptr, nullptr};
  bf16* deq = nullptr;
  std::vector<LayerPlan> plans;
  GemmPlan deq_w13, deq_w2;  // affine: maps over the expanded bf16 weights (b, b3)
  GemmPlan head_gemm;        // decode batches over 16 rows: the tied head with the argmax epilogue
  CUtensorMap tm_q, tm_sk, tm_sv;  // prefill attention: q rows, sliding scratch K / V
  WsMaps ws_head;                  // decode: tied head
  unsigned* attn_cnt = nullptr;    // workspace: decode attention split counts [max_batch][n_kv]
  bf16* conv_snap = nullptr;       // workspace: verify windows' conv states [n_conv][max_batch][6][D]
  bf16* side_k = nullptr;          // workspace: verify windows' sliding keys [n_sliding][max_batch][n_kv][hd]
  bf16* side_v = nullptr;
  // the last verify window, which lfm3_commit applies
  int vw_n = 0, vw_W = 0;
  std::vector<int> vw_slots, vw_pos;
  std::string msg;
  int launches = 0;
  // decode-step CUDA graphs, keyed by batch, split count and every device pointer the step reads
  struct GraphEntry {
    std::vector<const void*> key;
    cudaGraphExec_t exec;
    int launches;
  };
  std::vector<GraphEntry> graphs;
  cudaStream_t cap_stream = nullptr;  // capture only; graphs launch on the caller's stream
  bool graphs_on = true;
  // measurement brackets (lfm3_profile_*)
  bool prof = false;
  std::vector<cudaEvent_t> ev;
  std::vector<double> ev_bytes, ev_flops;
  int ev_used = 0, ev_overflow = 0;
};

namespace {

thread_local std::string g_create_msg;  // message of the last failed lfm3_create on this thread

lfm3_status fail(lfm3_ctx* c, lfm3_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  if (c) c->msg = buf;
  return s;
}

#define CK(x)                                                                                     \
  do {                                                                                            \
    cudaError_t e_ = (x);                                                                         \
    if (e_ != cudaSuccess) return fail(ctx, LFM3_E_CUDA, "%s: %s", #x, cudaGetErrorString(e_));   \
  } while (0)

// Workspace layout; with base == nullptr only sizes it.
size_t layout(lfm3_ctx* c, char* base) {
  const lfm3_config& g = c->cfg;
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    off = align_up(off, 256);
    char* p = base ? base + off : nullptr;
    off += bytes;
    return p;
  };
  const size_t R = c->R;
  c->err = reinterpret_cast<int*>(take(256));
  c->row_slot = reinterpret_cast<int32_t*>(take(4 * R));
  c->row_pos = reinterpret_cast<int32_t*>(take(4 * R));
  c->amax = reinterpret_cast<unsigned long long*>(take(8 * R));
  c->x_res = reinterpret_cast<float*>(take(4 * R * D));
  c->x_res2 = reinterpret_cast<float*>(take(4 * (size_t)g.max_batch * D));
  c->xn = reinterpret_cast<bf16*>(take(2 * R * D));
  c->big = reinterpret_cast<bf16*>(take(2 * R * F));
  c->y = reinterpret_cast<bf16*>(take(2 * R * D));
  // fp32 projection outputs: the conv in_proj [R][3D], qkvg [R][3088], or decode K-split partials
  c->part = reinterpret_cast<float*>(take(4 * std::max(R * 3 * D, (size_t)SPLIT_MAX * g.max_batch * NQKVG)));
  c->part2 = reinterpret_cast<float*>(take(4 * (size_t)SPLIT_MAX * g.max_batch * D));
  c->part3 = reinterpret_cast<float*>(take(4 * (size_t)g.max_batch * NQKVG));  // decode q|k|v|gate projection
  c->q = reinterpret_cast<bf16*>(take(2 * R * HQ * HD));
  c->gate = reinterpret_cast<float*>(take(4 * R * HQ));
  c->sk = reinterpret_cast<bf16*>(take(2 * (size_t)HKV * c->scratch_rows * HD));
  c->sv = reinterpret_cast<bf16*>(take(2 * (size_t)HKV * c->scratch_rows * HD));
  c->attn_part = reinterpret_cast<float*>(take(4 * (size_t)g.max_batch * HQ * c->max_splits * (HD + 2)));
  for (int k = 0; k < 2; ++k) {
    c->rope_cos[k] = reinterpret_cast<float*>(take(4 * (size_t)c->max_pos * (HD / 2)));
    c->rope_sin[k] = reinterpret_cast<float*>(take(4 * (size_t)c->max_pos * (HD / 2)));
  }
  c->deq = g.ffn_format == LFM3_FFN_AFFINE ? reinterpret_cast<bf16*>(take(2 * (size_t)2 * F * D)) : nullptr;
  c->attn_cnt = reinterpret_cast<unsigned*>(take(4 * (size_t)g.max_batch * HKV));
  c->conv_snap = reinterpret_cast<bf16*>(take(2 * (size_t)c->n_conv * g.max_batch * CST * D));
  c->side_k = reinterpret_cast<bf16*>(take(2 * (size_t)c->n_sliding * g.max_batch * HKV * HD));
  c->side_v = reinterpret_cast<bf16*>(take(2 * (size_t)c->n_sliding * g.max_batch * HKV * HD));
  return align_up(off, 256);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

lfm3_status check_config(lfm3_ctx* c, const lfm3_config* g) {
  if (g->n_layers < 1 || g->n_layers > LFM3_MAX_LAYERS)
    return fail(c, LFM3_E_CONFIG, "n_layers %d outside 1..%d", g->n_layers, LFM3_MAX_LAYERS);
  for (int i = 0; i < g->n_layers; ++i)
    if (g->layer_type[i] < 0 || g->layer_type[i] > 2)
      return fail(c, LFM3_E_CONFIG, "layer_type[%d] = %d is not conv/full/sliding", i, (int)g->layer_type[i]);
  struct { const char* name; long got, want; } fixed[] = {
      {"d_model", g->d_model, D}, {"d_ffn", g->d_ffn, F}, {"n_q", g->n_q, HQ}, {"n_kv", g->n_kv, HKV},
      {"head_dim", g->head_dim, HD}, {"conv_taps", g->conv_taps, TAPS}, {"window", g->window, WIN},
      {"page_size", g->page_size, PAGE}};
  for (auto& f : fixed)
    if (f.got != f.want)
      return fail(c, LFM3_E_UNSUPPORTED, "Lfm3UnsupportedGeometry: %s = %ld (the kernels implement %ld)", f.name,
                  f.got, f.want);
  if (g->rope_pairs_full < 0 || g->rope_pairs_full > HD / 2)
    return fail(c, LFM3_E_CONFIG, "rope_pairs_full %d outside 0..%d", g->rope_pairs_full, HD / 2);
  if (!(g->theta_full > 0.f) || !(g->theta_sliding > 0.f) || !(g->eps > 0.f))
    return fail(c, LFM3_E_CONFIG, "rotary bases and eps must be positive");
  if (g->ffn_format != LFM3_FFN_BF16 && g->ffn_format != LFM3_FFN_NVFP4 && g->ffn_format != LFM3_FFN_AFFINE)
    return fail(c, LFM3_E_UNSUPPORTED, "Lfm3UnsupportedFfnFormat: %d", g->ffn_format);
  if (g->ffn_format == LFM3_FFN_AFFINE && g->ffn_bits != 4 && g->ffn_bits != 6 && g->ffn_bits != 8)
    return fail(c, LFM3_E_UNSUPPORTED, "Lfm3UnsupportedAffineBits: %d (the kernels implement 4, 6 and 8)", g->ffn_bits);
  if (g->has_head && (g->vocab <= 0 || g->vocab % 16))
    return fail(c, LFM3_E_UNSUPPORTED, "Lfm3UnsupportedVocab: vocab %d must be a positive multiple of 16", g->vocab);
  if (g->max_streams < 1) return fail(c, LFM3_E_CONFIG, "max_streams %d < 1", g->max_streams);
  if (g->max_pages_per_stream < 1) return fail(c, LFM3_E_CONFIG, "max_pages_per_stream < 1");
  if ((long)g->max_pages_per_stream * PAGE > (1 << 20))
    return fail(c, LFM3_E_CONFIG, "a slot of %d pages exceeds 2^20 positions", g->max_pages_per_stream);
  if (g->max_chunk < 1 || g->max_chunk > 2048) return fail(c, LFM3_E_CONFIG, "max_chunk %d outside 1..2048", g->max_chunk);
  if (g->max_batch < 1 || g->max_batch > 64) return fail(c, LFM3_E_CONFIG, "max_batch %d outside 1..64", g->max_batch);
  int nf = 0;
  for (int i = 0; i < g->n_layers; ++i) nf += g->layer_type[i] == LFM3_LAYER_FULL;
  if (nf && g->n_pages < 1) return fail(c, LFM3_E_CONFIG, "full-attention layers need n_pages >= 1");
  return LFM3_OK;
}

lfm3_status check_weights(lfm3_ctx* c, const lfm3_config* g, const lfm3_weights* w) {
  if (!w->layers) return fail(c, LFM3_E_ARG, "weights.layers is NULL");
  if (g->has_head && (!w->embed || !w->final_norm)) return fail(c, LFM3_E_ARG, "has_head needs embed and final_norm");
  if (g->has_head && (!aligned16(w->embed) || !aligned16(w->final_norm)))
    return fail(c, LFM3_E_ARG, "embed/final_norm must be 16-byte aligned");
  for (int i = 0; i < g->n_layers; ++i) {
    const lfm3_layer_weights& L = w->layers[i];
    const void* need[16];
    int n = 0;
    need[n++] = L.op_norm; need[n++] = L.post_op_norm; need[n++] = L.ffn_norm; need[n++] = L.post_ffn_norm;
    if (g->layer_type[i] == LFM3_LAYER_CONV) {
      need[n++] = L.in_proj; need[n++] = L.conv; need[n++] = L.out_proj;
    } else {
      need[n++] = L.qkvg; need[n++] = L.q_norm; need[n++] = L.k_norm; need[n++] = L.o_proj;
    }
    if (g->ffn_format == LFM3_FFN_BF16) {
      need[n++] = L.w1; need[n++] = L.w3; need[n++] = L.w2;
    } else if (g->ffn_format == LFM3_FFN_AFFINE) {
      need[n++] = L.w1_codes; need[n++] = L.w1_scales; need[n++] = L.w1_biases;
      need[n++] = L.w3_codes; need[n++] = L.w3_scales; need[n++] = L.w3_biases;
      need[n++] = L.w2_codes; need[n++] = L.w2_scales;
      if (!L.w2_biases) return fail(c, LFM3_E_ARG, "layer %d: w2_biases is NULL", i);
    } else {
      need[n++] = L.w1_codes; need[n++] = L.w1_scales; need[n++] = L.w3_codes; need[n++] = L.w3_scales;
      need[n++] = L.w2_codes; need[n++] = L.w2_scales;
    }
    for (int j = 0; j < n; ++j) {
      if (!need[j]) return fail(c, LFM3_E_ARG, "layer %d: a required weight pointer is NULL (field %d)", i, j);
      if (!aligned16(need[j])) return fail(c, LFM3_E_ARG, "layer %d: weight field %d is not 16-byte aligned", i, j);
    }
  }
  return LFM3_OK;
}

const bf16* B(const void* p) { return reinterpret_cast<const bf16*>(p); }

// Brackets one projection launch with events when measurement is on.
struct Bracket {
  lfm3_ctx* c;
  cudaStream_t s;
  int i = -1;
  Bracket(lfm3_ctx* c_, cudaStream_t s_, double bytes, double flops) : c(c_), s(s_) {
    if (!c->prof) return;
    if (c->ev_used >= (int)c->ev_bytes.size()) { ++c->ev_overflow; return; }
    i = c->ev_used++;
    c->ev_bytes[i] = bytes;
    c->ev_flops[i] = flops;
    cudaEventRecord(c->ev[2 * i], s);
  }
  ~Bracket() {
    if (i >= 0) cudaEventRecord(c->ev[2 * i + 1], s);
  }
};

double gemm_flops(const GemmPlan& p, int M) {
  return 2.0 * M * (double)p.N * p.K * (p.epi == GEMM_SWIGLU ? 2 : 1);
}
double gemm_bytes(const GemmPlan& p, int M) {
  const int nw = p.epi == GEMM_SWIGLU ? 2 : 1;
  return 2.0 * nw * p.N * (double)p.K + 2.0 * M * p.K + (p.epi == GEMM_F32 ? 4.0 : 2.0) * M * p.N;
}

// format: WS_BF16, WS_NVFP4 or WS_AFFINE (a.bits wide codes)
cudaError_t run_ws(lfm3_ctx* c, int epi, int format, const WsMaps& mp, const WsArgs& a, cudaStream_t s) {
  const double mats = (a.w3 || a.codes3) ? 2.0 : 1.0;
  const double rows = epi == GEMV_CONV ? 3.0 * D : (double)a.N;
  const double w = format == WS_NVFP4    ? rows * a.K / 2 + rows * a.K / 16
                   : format == WS_AFFINE ? rows * a.K * a.bits / 8.0 + 2.0 * 2 * rows * a.K / 64
                                         : 2.0 * rows * a.K;
  const double bytes = mats * w + 2.0 * a.rows * a.K + 4.0 * a.rows * a.N;
  Bracket b(c, s, bytes, 2.0 * a.rows * rows * a.K * mats);
  return wstream(epi, format, mp, a, s);
}
cudaError_t run_gemm(lfm3_ctx* c, const GemmPlan& p, int M, cudaStream_t s) {
  Bracket b(c, s, gemm_bytes(p, M), gemm_flops(p, M));
  return gemm(p, M, c->err, s);
}

bool plan_gemm(GemmPlan* p, int epi, const void* a, int a_rows, const void* b, const void* b3, int N, int K, void* out,
               int ld, float alpha) {
  p->epi = epi;
  p->N = N;
  p->K = K;
  p->M = a_rows;
  p->out = out;
  p->ld = ld;
  p->alpha = alpha;
  p->splits = 1;
  p->amax = nullptr;
  p->w_const = 1;
  p->q4 = 0;
  p->sc = p->sc3 = nullptr;
  const uint32_t box_b = 128;  // weight boxes: 128 rows (wide and paired tiles issue several)
  if (!make_tmap_bf16(&p->a, a, a_rows, K, 128)) return false;
  if (!make_tmap_bf16(&p->b, b, N, K, box_b)) return false;
  if (b3 && !make_tmap_bf16(&p->b3, b3, N, K, box_b)) return false;
  if (!b3) p->b3 = p->b;
  p->bh = p->b;
  p->b3h = p->b3;
  if (epi == GEMM_SWIGLU && (!make_tmap_bf16(&p->bh, b, N, K, 64) || !make_tmap_bf16(&p->b3h, b3, N, K, 64)))
    return false;
  if (epi == GEMM_HEAD) return true;  // logits take plain stores
  return make_tmap_out(&p->o, out, epi == GEMM_F32, a_rows, N, ld);
}

// NVFP4 weights expanded on the chip (k_gemm_q4): activations a are f16 [a_rows][K].
bool plan_gemm_q4(GemmPlan* p, int epi, const void* a, int a_rows, const uint8_t* codes, const uint8_t* scales,
                  const uint8_t* codes3, const uint8_t* scales3, int N, int K, void* out, int ld, float alpha) {
  p->epi = epi;
  p->N = N;
  p->K = K;
  p->M = a_rows;
  p->out = out;
  p->ld = ld;
  p->alpha = alpha;
  p->splits = 1;
  p->amax = nullptr;
  p->w_const = 1;
  p->q4 = 1;
  p->sc = scales;
  p->sc3 = scales3 ? scales3 : scales;
  const uint32_t box = epi == GEMM_SWIGLU ? 64 : 128;
  if (!make_tmap_bf16(&p->a, a, a_rows, K, 128)) return false;
  if (!make_tmap_codes(&p->q, codes, N, K, box)) return false;
  p->q3 = p->q;
  if (codes3 && !make_tmap_codes(&p->q3, codes3, N, K, box)) return false;
  p->b = p->b3 = p->bh = p->b3h = p->a;  // unused
  return make_tmap_out(&p->o, out, epi == GEMM_F32, a_rows, N, ld);
}

// K splits for an fp32 projection of a decode batch (one 128-row tile): enough 128-column tiles x
// splits to give every SM one, at most SPLIT_MAX and one 64-column K block per split.
int batch_splits(int N, int K) {
  const int tiles = (N + 127) / 128;
  return std::max(1, std::min({SPLIT_MAX, K / 64, 148 / tiles}));
}
GemmPlan split_plan(const GemmPlan& p, int splits) {
  GemmPlan q = p;
  q.splits = splits;
  return q;
}

// Host check that every position a call writes or reads in slot s, [0, end), has a page.
lfm3_status check_pages(lfm3_ctx* ctx, const lfm3_state* st, int slot, long end) {
  const lfm3_config& g = ctx->cfg;
  if (end > ctx->max_pos)
    return fail(ctx, LFM3_E_CAPACITY, "slot %d: %ld positions exceed the slot's %d pages of %d", slot, end,
                g.max_pages_per_stream, PAGE);
  if (ctx->n_full == 0) return LFM3_OK;
  if (!st->h_page_table) return fail(ctx, LFM3_E_ARG, "h_page_table is NULL");
  const long npg = (end + PAGE - 1) / PAGE;
  for (long p = 0; p < npg; ++p) {
    const int32_t pg = st->h_page_table[(size_t)slot * g.max_pages_per_stream + p];
    if (pg < 0 || pg >= g.n_pages)
      return fail(ctx, LFM3_E_CAPACITY, "slot %d: page %ld of its table is %d, outside the pool of %d", slot, p, pg,
                  g.n_pages);
  }
  return LFM3_OK;
}

lfm3_status check_state(lfm3_ctx* ctx, const lfm3_state* st) {
  if (!st) return fail(ctx, LFM3_E_ARG, "state is NULL");
  if (!st->seq_len || !st->h_seq_len) return fail(ctx, LFM3_E_ARG, "seq_len / h_seq_len is NULL");
  if (ctx->n_conv && !st->conv_state) return fail(ctx, LFM3_E_ARG, "conv_state is NULL");
  if (ctx->n_sliding && (!st->ring_k || !st->ring_v)) return fail(ctx, LFM3_E_ARG, "ring_k / ring_v is NULL");
  if (ctx->n_full && (!st->kv_k || !st->kv_v || !st->page_table)) return fail(ctx, LFM3_E_ARG, "kv_k/kv_v/page_table is NULL");
  return LFM3_OK;
}

// ---------------------------------------------------------------- per-layer pieces
struct Views {
  bf16* conv_layer;  // conv state of this conv layer, all slots
  bf16* ring_k; bf16* ring_v;
  bf16* kv_k; bf16* kv_v;
};

Views views(lfm3_ctx* ctx, const lfm3_state* st, int l) {
  const lfm3_config& g = ctx->cfg;
  Views v{};
  const int j = ctx->kidx[l];
  switch (g.layer_type[l]) {
    case LFM3_LAYER_CONV:
      v.conv_layer = reinterpret_cast<bf16*>(st->conv_state) + (size_t)j * g.max_streams * CST * D;
      break;
    case LFM3_LAYER_SLIDING: {
      const size_t per = (size_t)g.max_streams * HKV * WIN * HD;
      v.ring_k = reinterpret_cast<bf16*>(st->ring_k) + j * per;
      v.ring_v = reinterpret_cast<bf16*>(st->ring_v) + j * per;
      break;
    }
    default: {
      const size_t per = (size_t)g.n_pages * HKV * PAGE * HD;
      v.kv_k = reinterpret_cast<bf16*>(st->kv_k) + j * per;
      v.kv_v = reinterpret_cast<bf16*>(st->kv_v) + j * per;
    }
  }
  return v;
}

AttnLayer attn_layer(lfm3_ctx* ctx, const lfm3_state* st, int l, const Views& v) {
  const lfm3_config& g = ctx->cfg;
  AttnLayer a{};
  a.full = g.layer_type[l] == LFM3_LAYER_FULL;
  a.k = a.full ? v.kv_k : v.ring_k;
  a.v = a.full ? v.kv_v : v.ring_v;
  a.page_table = st->page_table;
  a.max_pages = g.max_pages_per_stream;
  a.max_streams = g.max_streams;
  return a;
}

// FFN of n rows (prefill or large-batch decode) on the tensor-core GEMM: u = SwiGLU -> big, w2 ->
// part (as w2_splits K-split partials, n rows apart).
lfm3_status ffn_gemm(lfm3_ctx* ctx, int l, int n, int w2_splits, cudaStream_t s) {
  const lfm3_layer_weights& W = ctx->L[l];
  if (ctx->cfg.ffn_format == LFM3_FFN_AFFINE) {
    const int bits = ctx->cfg.ffn_bits;
    CK(affine_to_bf16(W.w1_codes, W.w1_scales, W.w1_biases, bits, F, D, ctx->deq, s));
    CK(affine_to_bf16(W.w3_codes, W.w3_scales, W.w3_biases, bits, F, D, ctx->deq + (size_t)F * D, s));
    CK(run_gemm(ctx, ctx->deq_w13, n, s));
    CK(affine_to_bf16(W.w2_codes, W.w2_scales, W.w2_biases, bits, D, F, ctx->deq, s));
    CK(run_gemm(ctx, split_plan(ctx->deq_w2, w2_splits), n, s));
  } else {  // bf16, or NVFP4 expanded inside the GEMM (f16 activations)
    CK(run_gemm(ctx, ctx->plans[l].w13, n, s));
    CK(run_gemm(ctx, split_plan(ctx->plans[l].w2, w2_splits), n, s));
  }
  return LFM3_OK;
}

}  // namespace

// ======================================================================================== ABI

extern "C" lfm3_status lfm3_create(const lfm3_config* cfg, const lfm3_weights* w, size_t* workspace_bytes,
                                   lfm3_ctx** out) {
  if (!cfg || !w || !workspace_bytes || !out) return LFM3_E_ARG;
  *out = nullptr;
  lfm3_ctx* c = new lfm3_ctx();
  lfm3_status st = check_config(c, cfg);
  if (st == LFM3_OK) st = check_weights(c, cfg, w);
  if (st != LFM3_OK) {
    g_create_msg = c->msg;
    delete c;
    return st;
  }
  g_create_msg.clear();
  c->cfg = *cfg;
  c->L.assign(w->layers, w->layers + cfg->n_layers);
  c->embed = B(w->embed);
  c->final_norm = B(w->final_norm);
  for (int i = 0; i < cfg->n_layers; ++i) {
    const int t = cfg->layer_type[i];
    c->kidx.push_back(t == LFM3_LAYER_CONV ? c->n_conv++ : t == LFM3_LAYER_FULL ? c->n_full++ : c->n_sliding++);
  }
  c->max_pos = cfg->max_pages_per_stream * PAGE;
  c->R = std::max(cfg->max_chunk, cfg->max_batch);
  c->max_splits = attn_decode_splits(c->max_pos);
  c->scratch_rows = WIN + cfg->max_chunk;
  c->ws_bytes = layout(c, nullptr);
  *workspace_bytes = c->ws_bytes;
  *out = c;
  return LFM3_OK;
}

extern "C" lfm3_status lfm3_bind_workspace(lfm3_ctx* ctx, void* d_ws, size_t bytes) {
  if (!ctx) return LFM3_E_ARG;
  if (!d_ws || (reinterpret_cast<uintptr_t>(d_ws) & 255))
    return fail(ctx, LFM3_E_ARG, "workspace must be non-NULL and 256-byte aligned");
  if (bytes < ctx->ws_bytes)
    return fail(ctx, LFM3_E_ARG, "workspace of %zu bytes is smaller than the %zu required", bytes, ctx->ws_bytes);
  if (!tma_init()) return fail(ctx, LFM3_E_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  CK(wstream_init());
  CK(gemm_init());
  CK(attn_init());
  CK(attn_tc_init());
  layout(ctx, reinterpret_cast<char*>(d_ws));
  const lfm3_config& g = ctx->cfg;
  const int R = ctx->R;
  // rotary tables in double precision, stored fp32: [pos][i] for pairs (i, i + 64)
  {
    std::vector<float> cs((size_t)ctx->max_pos * (HD / 2)), sn(cs.size());
    for (int k = 0; k < 2; ++k) {
      const double theta = k == 0 ? g.theta_full : g.theta_sliding;
      const int pairs = k == 0 ? g.rope_pairs_full : HD / 2;
      for (int i = 0; i < HD / 2; ++i) {
        const double inv = i < pairs ? std::pow(theta, -2.0 * i / HD) : 0.0;
        for (int p = 0; p < ctx->max_pos; ++p) {
          cs[(size_t)p * (HD / 2) + i] = (float)std::cos(p * inv);
          sn[(size_t)p * (HD / 2) + i] = (float)std::sin(p * inv);
        }
      }
      CK(cudaMemcpy(ctx->rope_cos[k], cs.data(), cs.size() * 4, cudaMemcpyHostToDevice));
      CK(cudaMemcpy(ctx->rope_sin[k], sn.data(), sn.size() * 4, cudaMemcpyHostToDevice));
    }
  }
  CK(cudaMemset(ctx->err, 0, 256));
  CK(cudaMemset(ctx->attn_cnt, 0, 4 * (size_t)g.max_batch * HKV));
  // GEMM plans (tensor maps over the weights and the workspace activations)
  ctx->plans.assign(g.n_layers, LayerPlan{});
  for (int l = 0; l < g.n_layers; ++l) {
    const lfm3_layer_weights& W = ctx->L[l];
    LayerPlan& P = ctx->plans[l];
    bool ok = true;
    if (g.layer_type[l] == LFM3_LAYER_CONV) {
      ok &= plan_gemm(&P.in_proj, GEMM_F32, ctx->xn, R, W.in_proj, nullptr, 3 * D, D, ctx->part, 3 * D, 1.f);
      ok &= plan_gemm(&P.out_proj, GEMM_F32, ctx->y, R, W.out_proj, nullptr, D, D, ctx->part, D, 1.f);
    } else {
      ok &= plan_gemm(&P.qkvg, GEMM_F32, ctx->xn, R, W.qkvg, nullptr, NQKVG, D, ctx->part, NQKVG, 1.f);
      ok &= plan_gemm(&P.o_proj, GEMM_F32, ctx->y, R, W.o_proj, nullptr, D, HQ * HD, ctx->part, D, 1.f);
    }
    if (g.ffn_format == LFM3_FFN_BF16) {
      ok &= plan_gemm(&P.w13, GEMM_SWIGLU, ctx->xn, R, W.w1, W.w3, F, D, ctx->big, F, 1.f);
      ok &= plan_gemm(&P.w2, GEMM_F32, ctx->big, R, W.w2, nullptr, D, F, ctx->part, D, 1.f);
    } else if (g.ffn_format == LFM3_FFN_NVFP4) {  // f16 activations (xn, big) for these two
      ok &= plan_gemm_q4(&P.w13, GEMM_SWIGLU, ctx->xn, R, W.w1_codes, W.w1_scales, W.w3_codes, W.w3_scales, F, D,
                         ctx->big, F, W.w13_scale);
      ok &= plan_gemm_q4(&P.w2, GEMM_F32, ctx->big, R, W.w2_codes, W.w2_scales, nullptr, nullptr, D, F, ctx->part, D,
                         W.w2_scale);
    }
    if (!ok) return fail(ctx, LFM3_E_CUDA, "layer %d: tensor map encoding failed", l);
  }
  // decode weight-streaming maps
  for (int l = 0; l < g.n_layers; ++l) {
    const lfm3_layer_weights& W = ctx->L[l];
    LayerPlan& P = ctx->plans[l];
    bool ok = true;
    auto bf = [&](CUtensorMap* m, const void* w, int N, int K, int epi) {
      ok &= make_ws_map(m, w, N, K, 0, ws_br(epi, 0), ws_kch(epi, 0));
    };
    if (g.layer_type[l] == LFM3_LAYER_CONV) {
      bf(&P.ws_in.w, W.in_proj, 3 * D, D, GEMV_CONV);
      bf(&P.ws_out.w, W.out_proj, D, D, GEMV_PARTIAL);
      P.ws_in.w3 = P.ws_in.s = P.ws_in.s3 = P.ws_in.w;
      P.ws_out.w3 = P.ws_out.s = P.ws_out.s3 = P.ws_out.w;
    } else {
      bf(&P.ws_qkvg.w, W.qkvg, NQKVG, D, GEMV_PARTIAL);
      bf(&P.ws_o.w, W.o_proj, D, HQ * HD, GEMV_PARTIAL);
      P.ws_qkvg.w3 = P.ws_qkvg.s = P.ws_qkvg.s3 = P.ws_qkvg.w;
      P.ws_o.w3 = P.ws_o.s = P.ws_o.s3 = P.ws_o.w;
    }
    if (g.ffn_format == LFM3_FFN_AFFINE) {
      const int bits = g.ffn_bits;
      ok &= make_aff_map(&P.ws_w13.w, W.w1_codes, F, D, bits, aff_br(GEMV_SWIGLU));
      ok &= make_aff_map(&P.ws_w13.w3, W.w3_codes, F, D, bits, aff_br(GEMV_SWIGLU));
      ok &= make_aff_sb_map(&P.ws_w13.s, W.w1_scales, F, D, aff_br(GEMV_SWIGLU));
      ok &= make_aff_sb_map(&P.ws_w13.s3, W.w3_scales, F, D, aff_br(GEMV_SWIGLU));
      ok &= make_aff_sb_map(&P.ws_w13.b, W.w1_biases, F, D, aff_br(GEMV_SWIGLU));
      ok &= make_aff_sb_map(&P.ws_w13.b3, W.w3_biases, F, D, aff_br(GEMV_SWIGLU));
      ok &= make_aff_map(&P.ws_w2.w, W.w2_codes, D, F, bits, aff_br(GEMV_PARTIAL));
      ok &= make_aff_sb_map(&P.ws_w2.s, W.w2_scales, D, F, aff_br(GEMV_PARTIAL));
      ok &= make_aff_sb_map(&P.ws_w2.b, W.w2_biases, D, F, aff_br(GEMV_PARTIAL));
      P.ws_w2.w3 = P.ws_w2.w;
      P.ws_w2.s3 = P.ws_w2.s;
      P.ws_w2.b3 = P.ws_w2.b;
    } else if (g.ffn_format == LFM3_FFN_NVFP4) {
      const int kch = ws_kch(GEMV_PARTIAL, 1);
      ok &= make_ws_map(&P.ws_w13.w, W.w1_codes, F, D, 1, ws_br(GEMV_SWIGLU, 1), kch);
      ok &= make_ws_map(&P.ws_w13.w3, W.w3_codes, F, D, 1, ws_br(GEMV_SWIGLU, 1), kch);
      ok &= make_ws_scale_map(&P.ws_w13.s, W.w1_scales, F, D, ws_br(GEMV_SWIGLU, 1), kch);
      ok &= make_ws_scale_map(&P.ws_w13.s3, W.w3_scales, F, D, ws_br(GEMV_SWIGLU, 1), kch);
      ok &= make_ws_map(&P.ws_w2.w, W.w2_codes, D, F, 1, ws_br(GEMV_PARTIAL, 1), kch);
      ok &= make_ws_scale_map(&P.ws_w2.s, W.w2_scales, D, F, ws_br(GEMV_PARTIAL, 1), kch);
      P.ws_w2.w3 = P.ws_w2.w;
      P.ws_w2.s3 = P.ws_w2.s;
    } else {
      bf(&P.ws_w13.w, W.w1, F, D, GEMV_SWIGLU);
      bf(&P.ws_w13.w3, W.w3, F, D, GEMV_SWIGLU);
      bf(&P.ws_w2.w, W.w2, D, F, GEMV_PARTIAL);
      P.ws_w13.s = P.ws_w13.s3 = P.ws_w13.w;
      P.ws_w2.w3 = P.ws_w2.s = P.ws_w2.s3 = P.ws_w2.w;
    }
    if (!ok) return fail(ctx, LFM3_E_CUDA, "layer %d: weight-streaming tensor map encoding failed", l);
  }
  if (g.has_head) {
    if (!make_ws_map(&ctx->ws_head.w, ctx->embed, g.vocab, D, 0, ws_br(GEMV_HEAD, 0), ws_kch(GEMV_HEAD, 0)))
      return fail(ctx, LFM3_E_CUDA, "head weight-streaming tensor map encoding failed");
    ctx->ws_head.w3 = ctx->ws_head.s = ctx->ws_head.s3 = ctx->ws_head.w;
  }
  if (g.has_head && !plan_gemm(&ctx->head_gemm, GEMM_HEAD, ctx->xn, R, ctx->embed, nullptr, g.vocab, D, nullptr,
                                g.vocab, 1.f))
    return fail(ctx, LFM3_E_CUDA, "head GEMM tensor map encoding failed");
  if (g.ffn_format == LFM3_FFN_AFFINE) {
    bool ok = plan_gemm(&ctx->deq_w13, GEMM_SWIGLU, ctx->xn, R, ctx->deq, ctx->deq + (size_t)F * D, F, D, ctx->big, F, 1.f);
    ok &= plan_gemm(&ctx->deq_w2, GEMM_F32, ctx->big, R, ctx->deq, nullptr, D, F, ctx->part, D, 1.f);
    ctx->deq_w13.w_const = ctx->deq_w2.w_const = 0;  // expanded into scratch by the kernel before
    if (!ok) return fail(ctx, LFM3_E_CUDA, "NVFP4 tensor map encoding failed");
  }
  CK(cudaDeviceSynchronize());
  ctx->graphs_on = getenv("LFM3_NO_GRAPH") == nullptr;
  if (!make_tmap_q(&ctx->tm_q, ctx->q, (uint64_t)R) ||
      !make_tmap_kv(&ctx->tm_sk, ctx->sk, (uint64_t)HKV * ctx->scratch_rows) ||
      !make_tmap_kv(&ctx->tm_sv, ctx->sv, (uint64_t)HKV * ctx->scratch_rows))
    return fail(ctx, LFM3_E_CUDA, "attention tensor map encoding failed");
  ctx->bound = true;
  ctx->msg.clear();
  return LFM3_OK;
}

namespace {

// The prompt pass of lfm3_prefill; the last n_pad rows (of the last chunk) are padding: they go
// through the row-independent steps but not into attention, the caches, the conv state, the head
// or seq_len.
lfm3_status prefill_rows(lfm3_ctx* ctx, const lfm3_state* st, int slot, const int32_t* d_tokens,
                         const void* d_embeds, int n, int n_pad, float* d_logits, int32_t* d_argmax, float* d_hidden,
                         void* stream) {
  if (!ctx->bound) return fail(ctx, LFM3_E_STATE, "workspace not bound");
  const lfm3_config& g = ctx->cfg;
  lfm3_status vs = check_state(ctx, st);
  if (vs != LFM3_OK) return vs;
  if (slot < 0 || slot >= g.max_streams) return fail(ctx, LFM3_E_ARG, "slot %d outside 0..%d", slot, g.max_streams - 1);
  if (n < 1) return fail(ctx, LFM3_E_ARG, "n = %d rows", n);
  if (g.has_head && !d_tokens) return fail(ctx, LFM3_E_ARG, "has_head needs d_tokens");
  if (!g.has_head && !d_embeds) return fail(ctx, LFM3_E_ARG, "a model without embedding needs d_embeds");
  if (!g.has_head && (d_logits || d_argmax)) return fail(ctx, LFM3_E_ARG, "a model without head has no logits");
  const long p_start = st->h_seq_len[slot];
  if (p_start < 0) return fail(ctx, LFM3_E_ARG, "h_seq_len[%d] = %ld", slot, p_start);
  const int n_real = n - n_pad;
  vs = check_pages(ctx, st, slot, p_start + n_real);
  if (vs != LFM3_OK) return vs;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  g_launches = 0;
  const float eps = g.eps;
  for (int c0 = 0; c0 < n; c0 += g.max_chunk) {
    const int nc = std::min(g.max_chunk, n - c0);
    const int p0 = (int)p_start + c0;
    const bool last = c0 + nc == n;
    const int nr = last ? nc - n_pad : nc;  // real rows of this chunk
    CK(setup_rows(1, slot, nullptr, st->seq_len, nc, 1, ctx->row_slot, ctx->row_pos, ctx->amax, s));
    const Rows rows{ctx->row_slot, ctx->row_pos, nr};
    CK(embed_rows(d_tokens ? d_tokens + c0 : nullptr, ctx->embed,
                  d_embeds ? B(d_embeds) + (size_t)c0 * D : nullptr, nc, ctx->x_res,
                  d_hidden ? d_hidden + (size_t)c0 * D : nullptr, s));
    CK(resid_norm(ctx->x_res, nullptr, 0, 0, nullptr, B(ctx->L[0].op_norm), ctx->xn, nc, eps, nullptr, 0, s));
    for (int l = 0; l < g.n_layers; ++l) {
      const lfm3_layer_weights& W = ctx->L[l];
      const LayerPlan& P = ctx->plans[l];
      const Views v = views(ctx, st, l);
      if (g.layer_type[l] == LFM3_LAYER_CONV) {
        CK(run_gemm(ctx, P.in_proj, nc, s));
        CK(conv_prefill(ctx->part, B(W.conv), v.conv_layer + (size_t)slot * CST * D, nc, nr, ctx->y, s));
        CK(run_gemm(ctx, P.out_proj, nc, s));
      } else {
        const bool full = g.layer_type[l] == LFM3_LAYER_FULL;
        CK(run_gemm(ctx, P.qkvg, nc, s));
        if (!full)
          CK(ring_to_scratch(v.ring_k, v.ring_v, slot, g.max_streams, p0, ctx->sk, ctx->sv, ctx->scratch_rows, s));
        KvWrite kw{};
        kw.mode = full ? KV_PAGES : KV_SCRATCH;
        kw.k = full ? v.kv_k : ctx->sk;
        kw.v = full ? v.kv_v : ctx->sv;
        kw.page_table = st->page_table;
        kw.max_pages = g.max_pages_per_stream;
        kw.max_streams = g.max_streams;
        kw.scratch_rows = ctx->scratch_rows;
        const int k = full ? 0 : 1;
        CK(qk_norm_rope_kv(ctx->part, 1, 0, B(W.q_norm), B(W.k_norm), ctx->rope_cos[k], ctx->rope_sin[k], rows, eps,
                           ctx->q, ctx->gate, kw, s));
        CUtensorMap tk, tv;
        if (full) {
          const uint64_t rows = (uint64_t)g.n_pages * HKV * PAGE;
          if (!make_tmap_kv(&tk, v.kv_k, rows) || !make_tmap_kv(&tv, v.kv_v, rows))
            return fail(ctx, LFM3_E_CUDA, "layer %d: K/V pool tensor map encoding failed", l);
        }
        AttnTcArgs ta{};
        ta.n = nr;
        ta.p0 = p0;
        ta.slot = slot;
        ta.full = full;
        ta.row0 = 0;
        ta.page_table = st->page_table;
        ta.max_pages = g.max_pages_per_stream;
        ta.scratch_rows = ctx->scratch_rows;
        ta.gate = ctx->gate;
        ta.y = ctx->y;
        ta.err = ctx->err;
        CK(attn_prefill_tc(ctx->tm_q, full ? tk : ctx->tm_sk, full ? tv : ctx->tm_sv, ta, s));
        if (!full)
          CK(scratch_to_ring(ctx->sk, ctx->sv, ctx->scratch_rows, nr, p0, v.ring_k, v.ring_v, slot, g.max_streams, s));
        CK(run_gemm(ctx, P.o_proj, nc, s));
      }
      CK(resid_norm(ctx->x_res, ctx->part, 1, 0, B(W.post_op_norm), B(W.ffn_norm), ctx->xn, nc, eps, nullptr,
                    g.ffn_format == LFM3_FFN_NVFP4, s));
      lfm3_status fs = ffn_gemm(ctx, l, nc, 1, s);
      if (fs != LFM3_OK) return fs;
      const bf16* gnext = l + 1 < g.n_layers ? B(ctx->L[l + 1].op_norm) : (g.has_head ? ctx->final_norm : nullptr);
      CK(resid_norm(ctx->x_res, ctx->part, 1, 0, B(W.post_ffn_norm), gnext, ctx->xn, nc, eps,
                    d_hidden ? d_hidden + ((size_t)(l + 1) * n + c0) * D : nullptr, 0, s));
    }
    const bool head = last && g.has_head && (d_logits || d_argmax);
    if (head) {
      WsArgs a{};
      a.w = ctx->embed;
      a.pro = WS_PRO_LOAD;
      a.x = ctx->xn + (size_t)(nr - 1) * D;
      a.K = D;
      a.N = g.vocab;
      a.rows = 1;
      a.splits = 1;
      a.logits = d_logits;
      a.amax = ctx->amax;
      a.err = ctx->err;
      CK(run_ws(ctx, GEMV_HEAD, WS_BF16, ctx->ws_head, a, s));
    }
    CK(finish_step(st->seq_len, ctx->row_slot, nc, nr, slot, head ? ctx->amax : nullptr, head ? d_argmax : nullptr, 1,
                   s));
  }
  st->h_seq_len[slot] += n_real;
  ctx->launches = g_launches;
  return LFM3_OK;
}

}  // namespace

extern "C" lfm3_status lfm3_prefill(lfm3_ctx* ctx, const lfm3_state* st, int slot, const int32_t* d_tokens,
                                    const void* d_embeds, int n, float* d_logits, int32_t* d_argmax, float* d_hidden,
                                    void* stream) {
  if (!ctx) return LFM3_E_ARG;
  return prefill_rows(ctx, st, slot, d_tokens, d_embeds, n, 0, d_logits, d_argmax, d_hidden, stream);
}

extern "C" lfm3_status lfm3_prefill_padded(lfm3_ctx* ctx, const lfm3_state* st, int slot, const int32_t* d_tokens,
                                           const void* d_embeds, int n_rows, int n_real, float* d_logits,
                                           int32_t* d_argmax, float* d_hidden, void* stream) {
  if (!ctx) return LFM3_E_ARG;
  if (n_rows < 1 || n_rows > ctx->cfg.max_chunk)
    return fail(ctx, LFM3_E_ARG, "a padded chunk has 1..%d rows, not %d", ctx->cfg.max_chunk, n_rows);
  if (n_real < 1 || n_real > n_rows) return fail(ctx, LFM3_E_ARG, "n_real %d outside 1..%d", n_real, n_rows);
  return prefill_rows(ctx, st, slot, d_tokens, d_embeds, n_rows, n_rows - n_real, d_logits, d_argmax, d_hidden,
                      stream);
}

namespace {

// Every launch of one decode step, in order, on stream s.
AttnDecodeArgs attn_args(lfm3_ctx* ctx, int l, int win) {
  const lfm3_layer_weights& W = ctx->L[l];
  const int k = ctx->cfg.layer_type[l] == LFM3_LAYER_FULL ? 0 : 1;
  AttnDecodeArgs A{};
  A.q_norm = B(W.q_norm);
  A.k_norm = B(W.k_norm);
  A.rope_cos = ctx->rope_cos[k];
  A.rope_sin = ctx->rope_sin[k];
  A.eps = ctx->cfg.eps;
  A.counters = ctx->attn_cnt;
  A.err = ctx->err;
  A.win = win;
  A.n_parts = 1;
  A.part_stride = 0;
  if (k == 1) {
    const size_t per = (size_t)ctx->cfg.max_batch * HKV * HD;
    A.side_k = ctx->side_k + (size_t)ctx->kidx[l] * per;
    A.side_v = ctx->side_v + (size_t)ctx->kidx[l] * per;
  }
  return A;
}

// win > 1: nb rows are verify windows of win rows per stream (nothing committed, see lfm3_verify).
lfm3_status enqueue_decode_large(lfm3_ctx* ctx, const lfm3_state* st, int nb, int win, const int32_t* d_slots,
                           const int32_t* d_tokens, const void* d_embeds, float* d_logits, int32_t* d_argmax,
                           float* d_hidden, int splits_full, float* attn_part, cudaStream_t s) {
  const lfm3_config& g = ctx->cfg;
  const float eps = g.eps;
  CK(setup_rows(0, 0, d_slots, st->seq_len, nb, win, ctx->row_slot, ctx->row_pos, ctx->amax, s));
  const Rows rows{ctx->row_slot, ctx->row_pos, nb};
  CK(embed_rows(d_tokens, ctx->embed, B(d_embeds), nb, ctx->x_res, d_hidden, s));
  CK(resid_norm(ctx->x_res, nullptr, 0, 0, nullptr, B(ctx->L[0].op_norm), ctx->xn, nb, eps, nullptr, 0, s));
  for (int l = 0; l < g.n_layers; ++l) {
    const lfm3_layer_weights& W = ctx->L[l];
    const LayerPlan& P = ctx->plans[l];
    const Views v = views(ctx, st, l);
    // a batch that fits one 128-row tile splits the projections along K (partials nb rows apart)
    const bool one = nb <= 128;
    int sp_o = 1;
    if (g.layer_type[l] == LFM3_LAYER_CONV) {
      const int sp = one ? batch_splits(3 * D, D) : 1;
      sp_o = one ? batch_splits(D, D) : 1;
      CK(run_gemm(ctx, split_plan(P.in_proj, sp), nb, s));
      CK(conv_decode(ctx->part, sp, (long)nb * 3 * D, B(W.conv), v.conv_layer, ctx->row_slot, nb, win,
                     ctx->conv_snap + (size_t)ctx->kidx[l] * g.max_batch * CST * D, ctx->y, s));
      CK(run_gemm(ctx, split_plan(P.out_proj, sp_o), nb, s));
    } else {
      const bool full = g.layer_type[l] == LFM3_LAYER_FULL;
      // q|k|v|gate is not split: every attention split block reads its rows (a sum of partials
      // there costs more than the unsplit projection)
      const int sp = 1;
      sp_o = one ? batch_splits(D, HQ * HD) : 1;
      CK(run_gemm(ctx, split_plan(P.qkvg, sp), nb, s));
      AttnDecodeArgs A = attn_args(ctx, l, win);
      A.n_parts = sp;
      A.part_stride = (long)nb * NQKVG;
      CK(attn_decode_fused(ctx->part, rows, attn_layer(ctx, st, l, v), A, full ? splits_full : WIN / DEC_KEYS,
                           attn_part, ctx->y, s));
      CK(run_gemm(ctx, split_plan(P.o_proj, sp_o), nb, s));
    }
    CK(resid_norm(ctx->x_res, ctx->part, sp_o, (long)nb * D, B(W.post_op_norm), B(W.ffn_norm), ctx->xn, nb, eps,
                  nullptr, g.ffn_format == LFM3_FFN_NVFP4, s));
    const int sp_2 = one ? batch_splits(D, F) : 1;
    lfm3_status fs = ffn_gemm(ctx, l, nb, sp_2, s);
    if (fs != LFM3_OK) return fs;
    const bf16* gnext = l + 1 < g.n_layers ? B(ctx->L[l + 1].op_norm) : (g.has_head ? ctx->final_norm : nullptr);
    CK(resid_norm(ctx->x_res, ctx->part, sp_2, (long)nb * D, B(W.post_ffn_norm), gnext, ctx->xn, nb, eps,
                  d_hidden ? d_hidden + (size_t)(l + 1) * nb * D : nullptr, 0, s));
  }
  const bool head = g.has_head && (d_logits || d_argmax);
  if (head) {
    GemmPlan h = ctx->head_gemm;  // logits (if asked for) and the argmax keys in one pass
    h.out = d_logits;
    h.amax = ctx->amax;
    CK(run_gemm(ctx, h, nb, s));
  }
  CK(finish_step(st->seq_len, ctx->row_slot, nb, 0, 0, head ? ctx->amax : nullptr, head ? d_argmax : nullptr,
                 win == 1, s));
  return LFM3_OK;
}

// Decode for up to 16 streams: the weight-streaming kernel, whose prologue also applies the
// previous projection's residual add + post-norm and this projection's input norm.
lfm3_status enqueue_decode_stream(lfm3_ctx* ctx, const lfm3_state* st, int nb, int win, const int32_t* d_slots,
                                  const int32_t* d_tokens, const void* d_embeds, float* d_logits, int32_t* d_argmax,
                                  float* d_hidden, int splits_full, float* attn_part, cudaStream_t s) {
  const lfm3_config& g = ctx->cfg;
  const float eps = g.eps;
  const bool fp4 = g.ffn_format == LFM3_FFN_NVFP4;
  const bool aff = g.ffn_format == LFM3_FFN_AFFINE;
  const int ffmt = fp4 ? WS_NVFP4 : aff ? WS_AFFINE : WS_BF16;
  CK(setup_rows(0, 0, d_slots, st->seq_len, nb, win, ctx->row_slot, ctx->row_pos, ctx->amax, s));
  const Rows rows{ctx->row_slot, ctx->row_pos, nb};
  CK(embed_rows(d_tokens, ctx->embed, B(d_embeds), nb, ctx->x_res, d_hidden, s));
  float* cur = ctx->x_res;
  float* nxt = ctx->x_res2;
  // partial sums still to be added into the residual (with their post-norm gain)
  const float* pend = nullptr;
  int pend_n = 0;
  const bf16* pend_g = nullptr;
  auto base = [&](WsArgs& a, int K, int N, int splits) {
    a.rows = nb;
    a.K = K;
    a.N = N;
    a.splits = splits;
    a.err = ctx->err;
    a.eps = eps;
  };
  auto norm_in = [&](WsArgs& a, const bf16* g_next, float* dump) {
    a.pro = WS_PRO_NORM;
    a.x_in = cur;
    a.x_out = nxt;
    a.parts = pend;
    a.n_parts = pend_n;
    a.part_stride = (long)nb * D;
    a.g_post = pend_g;
    a.g_next = g_next;
    a.dump = dump;
  };
  auto advance = [&]() { std::swap(cur, nxt); };
  for (int l = 0; l < g.n_layers; ++l) {
    const lfm3_layer_weights& W = ctx->L[l];
    const Views v = views(ctx, st, l);
    float* dump_l = (d_hidden && l > 0) ? d_hidden + (size_t)l * nb * D : nullptr;
    if (g.layer_type[l] == LFM3_LAYER_CONV) {
      WsArgs c{};
      base(c, D, 3 * D, 1);
      c.w = B(W.in_proj);
      c.conv_w = B(W.conv);
      c.conv_state = v.conv_layer;
      c.row_slot = ctx->row_slot;
      c.y = ctx->y;
      c.win = win;
      c.conv_snap = ctx->conv_snap + (size_t)ctx->kidx[l] * g.max_batch * CST * D;
      norm_in(c, B(W.op_norm), dump_l);
      CK(run_ws(ctx, GEMV_CONV, WS_BF16, ctx->plans[l].ws_in, c, s));
      advance();
      WsArgs o{};
      base(o, D, D, SPLIT_DD);
      o.pro = WS_PRO_LOAD;
      o.x = ctx->y;
      o.w = B(W.out_proj);
      o.part_out = ctx->part;
      CK(run_ws(ctx, GEMV_PARTIAL, WS_BF16, ctx->plans[l].ws_out, o, s));
    } else {
      const bool full = g.layer_type[l] == LFM3_LAYER_FULL;
      WsArgs q{};
      base(q, D, NQKVG, 1);
      q.w = B(W.qkvg);
      q.part_out = ctx->part3;
      norm_in(q, B(W.op_norm), dump_l);
      CK(run_ws(ctx, GEMV_PARTIAL, WS_BF16, ctx->plans[l].ws_qkvg, q, s));
      advance();
      AttnDecodeArgs A = attn_args(ctx, l, win);
      CK(attn_decode_fused(ctx->part3, rows, attn_layer(ctx, st, l, v), A, full ? splits_full : WIN / DEC_KEYS,
                           attn_part, ctx->y, s));
      WsArgs o{};
      base(o, HQ * HD, D, SPLIT_DD);
      o.pro = WS_PRO_LOAD;
      o.x = ctx->y;
      o.w = B(W.o_proj);
      o.part_out = ctx->part;
      CK(run_ws(ctx, GEMV_PARTIAL, WS_BF16, ctx->plans[l].ws_o, o, s));
    }
    pend = ctx->part;
    pend_n = SPLIT_DD;
    pend_g = B(W.post_op_norm);
    WsArgs f{};
    base(f, D, F, 1);
    f.out = ctx->big;
    if (fp4 || aff) {
      f.codes = W.w1_codes; f.scales = W.w1_scales; f.codes3 = W.w3_codes; f.scales3 = W.w3_scales;
      f.tscale = W.w13_scale;
      f.bits = g.ffn_bits;
    } else {
      f.w = B(W.w1);
      f.w3 = B(W.w3);
    }
    norm_in(f, B(W.ffn_norm), nullptr);
    CK(run_ws(ctx, GEMV_SWIGLU, ffmt, ctx->plans[l].ws_w13, f, s));
    advance();
    WsArgs d{};
    base(d, F, D, SPLIT_W2);
    d.pro = WS_PRO_LOAD;
    d.x = ctx->big;
    d.part_out = ctx->part2;
    if (fp4 || aff) {
      d.codes = W.w2_codes; d.scales = W.w2_scales; d.tscale = W.w2_scale;
      d.bits = g.ffn_bits;
    } else {
      d.w = B(W.w2);
    }
    CK(run_ws(ctx, GEMV_PARTIAL, ffmt, ctx->plans[l].ws_w2, d, s));
    pend = ctx->part2;
    pend_n = SPLIT_W2;
    pend_g = B(W.post_ffn_norm);
  }
  float* dump_last = d_hidden ? d_hidden + (size_t)g.n_layers * nb * D : nullptr;
  const bool head = g.has_head && (d_logits || d_argmax);
  if (head) {
    WsArgs h{};
    base(h, D, g.vocab, 1);
    h.w = ctx->embed;
    h.logits = d_logits;
    h.amax = ctx->amax;
    norm_in(h, ctx->final_norm, dump_last);
    CK(run_ws(ctx, GEMV_HEAD, WS_BF16, ctx->ws_head, h, s));
    advance();
  } else if (dump_last) {
    CK(resid_norm(cur, pend, pend_n, (long)nb * D, pend_g, nullptr, nullptr, nb, eps, dump_last, 0, s));
  }
  CK(finish_step(st->seq_len, ctx->row_slot, nb, 0, 0, head ? ctx->amax : nullptr, head ? d_argmax : nullptr,
                 win == 1, s));
  return LFM3_OK;
}

lfm3_status enqueue_decode(lfm3_ctx* ctx, const lfm3_state* st, int nb, int win, const int32_t* d_slots,
                           const int32_t* d_tokens, const void* d_embeds, float* d_logits, int32_t* d_argmax,
                           float* d_hidden, int splits_full, float* attn_part, cudaStream_t s) {
  if (nb <= GEMV_MAX_ROWS)
    return enqueue_decode_stream(ctx, st, nb, win, d_slots, d_tokens, d_embeds, d_logits, d_argmax, d_hidden,
                                 splits_full, attn_part, s);
  return enqueue_decode_large(ctx, st, nb, win, d_slots, d_tokens, d_embeds, d_logits, d_argmax, d_hidden, splits_full,
                              attn_part, s);
}

}  // namespace

namespace {

// Host checks of a decode step and its full-layer split count (quantised to a power of two so
// that one captured graph serves a range of contexts).
lfm3_status validate_decode(lfm3_ctx* ctx, const lfm3_state* st, int nb, const int32_t* h_slots,
                            const int32_t* d_slots, const int32_t* d_tokens, const void* d_embeds,
                            const float* d_logits, const int32_t* d_argmax, int* splits_out) {
  if (!ctx->bound) return fail(ctx, LFM3_E_STATE, "workspace not bound");
  const lfm3_config& g = ctx->cfg;
  lfm3_status vs = check_state(ctx, st);
  if (vs != LFM3_OK) return vs;
  if (nb < 1 || nb > g.max_batch) return fail(ctx, LFM3_E_ARG, "n_streams %d outside 1..%d", nb, g.max_batch);
  if (!h_slots || !d_slots) return fail(ctx, LFM3_E_ARG, "h_slots / d_slots is NULL");
  if (g.has_head && !d_tokens) return fail(ctx, LFM3_E_ARG, "has_head needs d_tokens");
  if (!g.has_head && !d_embeds) return fail(ctx, LFM3_E_ARG, "a model without embedding needs d_embeds");
  if (!g.has_head && (d_logits || d_argmax)) return fail(ctx, LFM3_E_ARG, "a model without head has no logits");
  int maxpos = 0;
  for (int b = 0; b < nb; ++b) {
    const int s = h_slots[b];
    if (s < 0 || s >= g.max_streams) return fail(ctx, LFM3_E_ARG, "slot %d outside 0..%d", s, g.max_streams - 1);
    for (int c = 0; c < b; ++c)
      if (h_slots[c] == s) return fail(ctx, LFM3_E_ARG, "slot %d listed twice", s);
    vs = check_pages(ctx, st, s, (long)st->h_seq_len[s] + 1);
    if (vs != LFM3_OK) return vs;
    maxpos = std::max(maxpos, (int)st->h_seq_len[s]);
  }
  *splits_out = std::min(attn_decode_splits(maxpos + 1), ctx->max_splits);
  return LFM3_OK;
}

}  // namespace

namespace {

// Enqueues nr rows (win per stream) on stream s, from the step's captured graph when graphs are on.
lfm3_status run_decode(lfm3_ctx* ctx, const lfm3_state* st, int nr, int win, int splits_full, const int32_t* d_slots,
                       const int32_t* d_tokens, const void* d_embeds, float* d_logits, int32_t* d_argmax,
                       float* d_hidden, cudaStream_t s) {
  g_launches = 0;
  if (!ctx->graphs_on || ctx->prof) {
    lfm3_status es = enqueue_decode(ctx, st, nr, win, d_slots, d_tokens, d_embeds, d_logits, d_argmax, d_hidden,
                                    splits_full, ctx->attn_part, s);
    if (es != LFM3_OK) return es;
    ctx->launches = g_launches;
    return LFM3_OK;
  }
  std::vector<const void*> key = {reinterpret_cast<const void*>((intptr_t)nr), reinterpret_cast<const void*>((intptr_t)win),
                                  reinterpret_cast<const void*>((intptr_t)splits_full), d_slots, d_tokens, d_embeds,
                                  d_logits, d_argmax, d_hidden, st->conv_state, st->ring_k, st->ring_v, st->kv_k,
                                  st->kv_v, st->page_table, st->seq_len};
  lfm3_ctx::GraphEntry* hit = nullptr;
  for (auto& e : ctx->graphs)
    if (e.key == key) hit = &e;
  if (!hit) {
    if (!ctx->cap_stream) CK(cudaStreamCreateWithFlags(&ctx->cap_stream, cudaStreamNonBlocking));
    if (ctx->graphs.size() >= 32) {
      for (auto& e : ctx->graphs) cudaGraphExecDestroy(e.exec);
      ctx->graphs.clear();
    }
    cudaGraph_t graph = nullptr;
    CK(cudaStreamBeginCapture(ctx->cap_stream, cudaStreamCaptureModeThreadLocal));
    lfm3_status es = enqueue_decode(ctx, st, nr, win, d_slots, d_tokens, d_embeds, d_logits, d_argmax, d_hidden,
                                    splits_full, ctx->attn_part, ctx->cap_stream);
    cudaError_t ce = cudaStreamEndCapture(ctx->cap_stream, &graph);
    if (es != LFM3_OK) {
      if (graph) cudaGraphDestroy(graph);
      return es;
    }
    CK(ce);
    cudaGraphExec_t exec = nullptr;
    ce = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    CK(ce);
    ctx->graphs.push_back({key, exec, g_launches});
    hit = &ctx->graphs.back();
  }
  CK(cudaGraphLaunch(hit->exec, s));
  ctx->launches = hit->launches;
  return LFM3_OK;
}

}  // namespace

extern "C" lfm3_status lfm3_decode_step(lfm3_ctx* ctx, const lfm3_state* st, int nb, const int32_t* h_slots,
                                        const int32_t* d_slots, const int32_t* d_tokens, const void* d_embeds,
                                        float* d_logits, int32_t* d_argmax, float* d_hidden, void* stream) {
  if (!ctx) return LFM3_E_ARG;
  int splits_full = 1;
  lfm3_status vs = validate_decode(ctx, st, nb, h_slots, d_slots, d_tokens, d_embeds, d_logits, d_argmax,
                                   &splits_full);
  if (vs != LFM3_OK) return vs;
  vs = run_decode(ctx, st, nb, 1, splits_full, d_slots, d_tokens, d_embeds, d_logits, d_argmax, d_hidden,
                  reinterpret_cast<cudaStream_t>(stream));
  if (vs != LFM3_OK) return vs;
  ctx->vw_n = 0;  // a decode step ends any verify window
  for (int b = 0; b < nb; ++b) st->h_seq_len[h_slots[b]] += 1;
  return LFM3_OK;
}

extern "C" lfm3_status lfm3_verify(lfm3_ctx* ctx, const lfm3_state* st, int n_streams, const int32_t* h_slots,
                                   const int32_t* d_slots, int W, const int32_t* d_tokens, const void* d_embeds,
                                   float* d_logits, int32_t* d_argmax, float* d_hidden, void* stream) {
  if (!ctx) return LFM3_E_ARG;
  if (W < 1 || W > MAX_WIN) return fail(ctx, LFM3_E_ARG, "window of %d rows outside 1..%d", W, MAX_WIN);
  if (n_streams < 1 || (long)n_streams * W > ctx->cfg.max_batch)
    return fail(ctx, LFM3_E_ARG, "%d streams x %d rows outside 1..max_batch (%d)", n_streams, W, ctx->cfg.max_batch);
  int splits_full = 1;
  // the row checks of a decode step, per stream; then room for the window's last row
  lfm3_status vs = validate_decode(ctx, st, n_streams, h_slots, d_slots, d_tokens, d_embeds, d_logits, d_argmax,
                                   &splits_full);
  if (vs != LFM3_OK) return vs;
  int maxpos = 0;
  for (int i = 0; i < n_streams; ++i) {
    vs = check_pages(ctx, st, h_slots[i], (long)st->h_seq_len[h_slots[i]] + W);
    if (vs != LFM3_OK) return vs;
    maxpos = std::max(maxpos, (int)st->h_seq_len[h_slots[i]] + W - 1);
  }
  splits_full = std::min(attn_decode_splits(maxpos + 1), ctx->max_splits);
  vs = run_decode(ctx, st, n_streams * W, W, splits_full, d_slots, d_tokens, d_embeds, d_logits, d_argmax, d_hidden,
                  reinterpret_cast<cudaStream_t>(stream));
  if (vs != LFM3_OK) return vs;
  ctx->vw_n = n_streams;
  ctx->vw_W = W;
  ctx->vw_slots.assign(h_slots, h_slots + n_streams);
  ctx->vw_pos.resize(n_streams);
  for (int i = 0; i < n_streams; ++i) ctx->vw_pos[i] = st->h_seq_len[h_slots[i]];
  return LFM3_OK;
}

extern "C" lfm3_status lfm3_commit(lfm3_ctx* ctx, const lfm3_state* st, int n_streams, const int32_t* h_slots,
                                   const int32_t* h_accept, void* stream) {
  if (!ctx) return LFM3_E_ARG;
  if (!ctx->bound) return fail(ctx, LFM3_E_STATE, "workspace not bound");
  lfm3_status vs = check_state(ctx, st);
  if (vs != LFM3_OK) return vs;
  if (!h_slots || !h_accept) return fail(ctx, LFM3_E_ARG, "h_slots / h_accept is NULL");
  if (ctx->vw_n == 0) return fail(ctx, LFM3_E_STATE, "no verify window to commit");
  if (n_streams != ctx->vw_n) return fail(ctx, LFM3_E_ARG, "%d streams, the window had %d", n_streams, ctx->vw_n);
  CommitArgs a{};
  a.n = n_streams;
  a.W = ctx->vw_W;
  for (int i = 0; i < n_streams; ++i) {
    if (h_slots[i] != ctx->vw_slots[i])
      return fail(ctx, LFM3_E_ARG, "stream %d is slot %d, the window's was slot %d", i, h_slots[i], ctx->vw_slots[i]);
    if (st->h_seq_len[h_slots[i]] != ctx->vw_pos[i])
      return fail(ctx, LFM3_E_STATE, "slot %d moved since its verify window", h_slots[i]);
    if (h_accept[i] < 1 || h_accept[i] > a.W)
      return fail(ctx, LFM3_E_ARG, "slot %d: %d rows accepted, outside 1..%d", h_slots[i], h_accept[i], a.W);
    a.slot[i] = h_slots[i];
    a.pos[i] = ctx->vw_pos[i];
    a.k[i] = h_accept[i];
  }
  const lfm3_config& g = ctx->cfg;
  a.n_conv = ctx->n_conv;
  a.n_sliding = ctx->n_sliding;
  a.max_streams = g.max_streams;
  a.max_batch = g.max_batch;
  a.snap = ctx->conv_snap;
  a.side_k = ctx->side_k;
  a.side_v = ctx->side_v;
  a.conv = reinterpret_cast<bf16*>(st->conv_state);
  a.ring_k = reinterpret_cast<bf16*>(st->ring_k);
  a.ring_v = reinterpret_cast<bf16*>(st->ring_v);
  a.seq_len = st->seq_len;
  g_launches = 0;
  CK(commit_windows(a, reinterpret_cast<cudaStream_t>(stream)));
  ctx->launches = g_launches;
  for (int i = 0; i < n_streams; ++i) st->h_seq_len[h_slots[i]] += h_accept[i];
  ctx->vw_n = 0;
  return LFM3_OK;
}

// A decode step that allocates nothing: the split-KV attention keeps its per-split partial
// results in the library's own fixed device array (see attn_static_scratch) instead of the
// bound workspace, and the step is launched directly rather than through a captured graph.
extern "C" lfm3_status lfm3_decode_step_noalloc(lfm3_ctx* ctx, const lfm3_state* st, int nb,
                                                const int32_t* h_slots, const int32_t* d_slots,
                                                const int32_t* d_tokens, const void* d_embeds, float* d_logits,
                                                int32_t* d_argmax, float* d_hidden, void* stream) {
  if (!ctx) return LFM3_E_ARG;
  int splits_full = 1;
  lfm3_status vs = validate_decode(ctx, st, nb, h_slots, d_slots, d_tokens, d_embeds, d_logits, d_argmax,
                                   &splits_full);
  if (vs != LFM3_OK) return vs;
  float* scratch = nullptr;
  size_t cap = 0;
  CK(attn_static_scratch(&scratch, &cap));
  const size_t need = (size_t)nb * HQ * splits_full * (HD + 2);
  if (need > cap)
    return fail(ctx, LFM3_E_CAPACITY,
                "lfm3_decode_step_noalloc: %d streams x %d key splits need %zu bytes of attention scratch, more "
                "than the fixed %zu bytes",
                nb, splits_full, need * sizeof(float), cap * sizeof(float));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  g_launches = 0;
  lfm3_status es = enqueue_decode(ctx, st, nb, 1, d_slots, d_tokens, d_embeds, d_logits, d_argmax, d_hidden,
                                  splits_full, scratch, s);
  if (es != LFM3_OK) return es;
  ctx->launches = g_launches;
  ctx->vw_n = 0;
  for (int b = 0; b < nb; ++b) st->h_seq_len[h_slots[b]] += 1;
  return LFM3_OK;
}

extern "C" lfm3_status lfm3_check_device_errors(lfm3_ctx* ctx, void* stream) {
  if (!ctx) return LFM3_E_ARG;
  if (!ctx->bound) return fail(ctx, LFM3_E_STATE, "workspace not bound");
  CK(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  int e = 0;
  CK(cudaMemcpy(&e, ctx->err, sizeof e, cudaMemcpyDeviceToHost));
  if (e) {
    CK(cudaMemset(ctx->err, 0, sizeof e));
    // a step that gave up can leave the attention's split counts mid-way
    CK(cudaMemset(ctx->attn_cnt, 0, 4 * (size_t)ctx->cfg.max_batch * HKV));
    return fail(ctx, LFM3_E_TIMEOUT, "a device-side bounded wait gave up (status %d)", e);
  }
  return LFM3_OK;
}

// ---------------------------------------------------------------- kept states (prompt cache)
namespace {

lfm3_status snap_args(lfm3_ctx* ctx, const lfm3_state* st, int slot, const void* d_snap, size_t bytes, int at,
                      SnapArgs* a) {
  if (!ctx->bound) return fail(ctx, LFM3_E_STATE, "workspace not bound");
  lfm3_status vs = check_state(ctx, st);
  if (vs != LFM3_OK) return vs;
  const lfm3_config& g = ctx->cfg;
  if (slot < 0 || slot >= g.max_streams) return fail(ctx, LFM3_E_ARG, "slot %d outside 0..%d", slot, g.max_streams - 1);
  if (!d_snap || (reinterpret_cast<uintptr_t>(d_snap) & 15))
    return fail(ctx, LFM3_E_ARG, "the kept-state buffer must be non-NULL and 16-byte aligned");
  if (at < 0) return fail(ctx, LFM3_E_ARG, "mark %d < 0", at);
  const size_t need = snapshot_bytes(ctx->n_conv, ctx->n_sliding, ctx->n_full, at);
  if (bytes < need)
    return fail(ctx, LFM3_E_CAPACITY, "a state at %d needs %zu bytes, the buffer has %zu", at, need, bytes);
  vs = check_pages(ctx, st, slot, at);
  if (vs != LFM3_OK) return vs;
  *a = SnapArgs{};
  a->slot = slot;
  a->at = at;
  a->npg = (at + PAGE - 1) / PAGE;
  a->n_conv = ctx->n_conv;
  a->n_sliding = ctx->n_sliding;
  a->n_full = ctx->n_full;
  a->max_streams = g.max_streams;
  a->n_pages = g.n_pages;
  a->max_pages = g.max_pages_per_stream;
  a->snap = const_cast<void*>(d_snap);
  a->conv = reinterpret_cast<bf16*>(st->conv_state);
  a->ring_k = reinterpret_cast<bf16*>(st->ring_k);
  a->ring_v = reinterpret_cast<bf16*>(st->ring_v);
  a->kv_k = reinterpret_cast<bf16*>(st->kv_k);
  a->kv_v = reinterpret_cast<bf16*>(st->kv_v);
  a->page_table = st->page_table;
  a->seq_len = st->seq_len;
  return LFM3_OK;
}

}  // namespace

extern "C" size_t lfm3_state_bytes(const lfm3_ctx* ctx, int at) {
  if (!ctx || at < 0) return 0;
  return snapshot_bytes(ctx->n_conv, ctx->n_sliding, ctx->n_full, at);
}

extern "C" lfm3_status lfm3_keep(lfm3_ctx* ctx, const lfm3_state* st, int slot, void* d_snap, size_t bytes,
                                 int* at_out, void* stream) {
  if (!ctx || !at_out) return LFM3_E_ARG;
  if (!st || !st->h_seq_len) return fail(ctx, LFM3_E_ARG, "state / h_seq_len is NULL");
  if (slot < 0 || slot >= ctx->cfg.max_streams) return fail(ctx, LFM3_E_ARG, "slot %d outside 0..%d", slot,
                                                            ctx->cfg.max_streams - 1);
  SnapArgs a;
  const int at = st->h_seq_len[slot];
  lfm3_status vs = snap_args(ctx, st, slot, d_snap, bytes, at, &a);
  if (vs != LFM3_OK) return vs;
  g_launches = 0;
  a.restore = 0;
  CK(state_copy(a, reinterpret_cast<cudaStream_t>(stream)));
  ctx->launches = g_launches;
  *at_out = at;
  return LFM3_OK;
}

extern "C" lfm3_status lfm3_restore(lfm3_ctx* ctx, const lfm3_state* st, int slot, const void* d_snap, size_t bytes,
                                    int at, void* stream) {
  if (!ctx) return LFM3_E_ARG;
  SnapArgs a;
  lfm3_status vs = snap_args(ctx, st, slot, d_snap, bytes, at, &a);
  if (vs != LFM3_OK) return vs;
  g_launches = 0;
  a.restore = 1;
  CK(state_copy(a, reinterpret_cast<cudaStream_t>(stream)));
  ctx->launches = g_launches;
  st->h_seq_len[slot] = at;
  return LFM3_OK;
}

extern "C" lfm3_status lfm3_selftest_wait(lfm3_ctx* ctx, unsigned rounds, void* stream) {
  if (!ctx) return LFM3_E_ARG;
  if (!ctx->bound) return fail(ctx, LFM3_E_STATE, "workspace not bound");
  if (rounds < 1 || rounds > (1u << 16)) return fail(ctx, LFM3_E_ARG, "rounds %u outside 1..65536", rounds);
  CK(wait_selftest(ctx->err, rounds, reinterpret_cast<cudaStream_t>(stream)));
  return LFM3_OK;
}

extern "C" lfm3_status lfm3_profile_enable(lfm3_ctx* ctx, int on, int capacity) {
  if (!ctx) return LFM3_E_ARG;
  if (on && capacity < 1) return fail(ctx, LFM3_E_ARG, "capacity %d", capacity);
  for (cudaEvent_t e : ctx->ev) cudaEventDestroy(e);
  ctx->ev.clear();
  ctx->ev_bytes.clear();
  ctx->ev_flops.clear();
  ctx->ev_used = ctx->ev_overflow = 0;
  ctx->prof = on != 0;
  if (!on) return LFM3_OK;
  ctx->ev.resize(2 * (size_t)capacity);
  for (auto& e : ctx->ev) CK(cudaEventCreate(&e));
  ctx->ev_bytes.assign(capacity, 0.0);
  ctx->ev_flops.assign(capacity, 0.0);
  return LFM3_OK;
}

extern "C" lfm3_status lfm3_profile_read(lfm3_ctx* ctx, int* launches, double* ms, double* bytes, double* flops) {
  if (!ctx || !launches || !ms || !bytes || !flops) return LFM3_E_ARG;
  *launches = 0;
  *ms = *bytes = *flops = 0.0;
  for (int i = 0; i < ctx->ev_used; ++i) {
    CK(cudaEventSynchronize(ctx->ev[2 * i + 1]));
    float t = 0.f;
    CK(cudaEventElapsedTime(&t, ctx->ev[2 * i], ctx->ev[2 * i + 1]));
    *ms += t;
    *bytes += ctx->ev_bytes[i];
    *flops += ctx->ev_flops[i];
  }
  *launches = ctx->ev_used;
  const int over = ctx->ev_overflow;
  ctx->ev_used = ctx->ev_overflow = 0;
  if (over) return fail(ctx, LFM3_E_CAPACITY, "%d launches ran unbracketed (capacity exceeded)", over);
  return LFM3_OK;
}

#ifdef LFM3_TRACE
// Diagnostic builds only: the device buffer [256 launches][512 blocks][8] uint64 the kernels stamp.
extern "C" void lfm3_trace_set(void* d_buf) { g_trace = static_cast<unsigned long long*>(d_buf); }
#endif

extern "C" int lfm3_last_launch_count(const lfm3_ctx* ctx) { return ctx ? ctx->launches : 0; }

extern "C" const char* lfm3_last_error(const lfm3_ctx* ctx) { return ctx ? ctx->msg.c_str() : g_create_msg.c_str(); }

extern "C" void lfm3_free(lfm3_ctx* ctx) {
  if (!ctx) return;
  for (cudaEvent_t e : ctx->ev) cudaEventDestroy(e);
  for (auto& e : ctx->graphs) cudaGraphExecDestroy(e.exec);
  if (ctx->cap_stream) cudaStreamDestroy(ctx->cap_stream);
  delete ctx;
}
