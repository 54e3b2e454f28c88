// Small memory-bound kernels of the LFM3 forward: row bookkeeping, embedding, the fused
// sandwich-norm/residual step, the gated short conv with its state, q/k RMSNorm + rotary +
// KV placement, and the sliding-ring copies.
#include "kernels.cuh"

namespace lfm3 {

thread_local int g_launches = 0;
#ifdef LFM3_TRACE
unsigned long long* g_trace = nullptr;
#endif

// ------------------------------------------------------------------------------------------
// Row bookkeeping: prefill rows are consecutive positions of one slot; decode rows are one
// position of each listed slot. Also clears the per-row greedy cells.
__global__ void k_setup_rows(int prefill, int slot, const int32_t* __restrict__ d_slots,
                             const int32_t* __restrict__ seq_len, int rows, int win, int32_t* row_slot,
                             int32_t* row_pos, unsigned long long* amax) {
  pdl_wait();
  pdl_launch_dependents();
  int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  if (prefill) {
    row_slot[r] = slot;
    row_pos[r] = seq_len[slot] + r;
  } else {
    int s = d_slots[r / win];
    row_slot[r] = s;
    row_pos[r] = seq_len[s] + r % win;
  }
  if (amax) amax[r] = 0ull;
}

cudaError_t setup_rows(int prefill, int slot, const int32_t* d_slots, const int32_t* seq_len, int rows, int win,
                       int32_t* row_slot, int32_t* row_pos, unsigned long long* amax, cudaStream_t s) {
  return launch(k_setup_rows, dim3((rows + 127) / 128), dim3(128), 0, s, prefill, slot, d_slots, seq_len, rows,
                win < 1 ? 1 : win, row_slot, row_pos, amax);
}

// ------------------------------------------------------------------------------------------
// Embedding (tied table) or input vectors -> fp32 residual stream.
__global__ void __launch_bounds__(256) k_embed(const int32_t* __restrict__ tokens, const bf16* __restrict__ table,
                                               const bf16* __restrict__ vecs, float* __restrict__ x_res,
                                               float* __restrict__ dump) {
  pdl_wait();
  pdl_launch_dependents();
  const int r = blockIdx.x;
  const bf16* src = tokens ? table + (size_t)tokens[r] * D : vecs + (size_t)r * D;
  const int i = threadIdx.x * 8;
  uint4 w = ldg16(src + i);
  float4 a = make_float4(bflo(w.x), bfhi(w.x), bflo(w.y), bfhi(w.y));
  float4 b = make_float4(bflo(w.z), bfhi(w.z), bflo(w.w), bfhi(w.w));
  float4* dst = reinterpret_cast<float4*>(x_res + (size_t)r * D + i);
  dst[0] = a;
  dst[1] = b;
  if (dump) {
    float4* dd = reinterpret_cast<float4*>(dump + (size_t)r * D + i);
    dd[0] = a;
    dd[1] = b;
  }
}

cudaError_t embed_rows(const int32_t* tokens, const bf16* table, const bf16* vecs, int rows, float* x_res,
                       float* dump, cudaStream_t s) {
  return launch(k_embed, dim3(rows), dim3(256), 0, s, tokens, table, vecs, x_res, dump);
}

// ------------------------------------------------------------------------------------------
// Sandwich-norm step on one row (d_model = 2048, 256 threads x 8):
//   if n_part > 0:  m = sum_s part[s][r];  x += g_post * m * rsqrt(mean(m^2) + eps)
//   dump[r] = x (optional);  xn = bf16(g_next * x * rsqrt(mean(x^2) + eps)) (optional)
__global__ void __launch_bounds__(256) k_resid_norm(float* __restrict__ x_res, const float* __restrict__ part,
                                                    int n_part, long part_stride, const bf16* __restrict__ g_post,
                                                    const bf16* __restrict__ g_next, bf16* __restrict__ xn, float eps,
                                                    float* __restrict__ dump, int xn_f16) {
  __shared__ float red[8];
  pdl_wait();
  pdl_launch_dependents();
  const int r = blockIdx.x;
  const int i = threadIdx.x * 8;
  float* xr = x_res + (size_t)r * D + i;
  float x[8];
  {
    float4 a = reinterpret_cast<float4*>(xr)[0], b = reinterpret_cast<float4*>(xr)[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
  if (n_part > 0) {
    float m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int s = 0; s < n_part; ++s) {
      const float* p = part + s * part_stride + (size_t)r * D + i;
      float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
      m[0] += a.x; m[1] += a.y; m[2] += a.z; m[3] += a.w; m[4] += b.x; m[5] += b.y; m[6] += b.z; m[7] += b.w;
    }
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) ss += m[j] * m[j];
    ss = block_sum<8>(ss, red);
    const float inv = rsqrtf(ss * (1.0f / D) + eps);
    uint4 gw = ldg16(g_post + i);
    float g[8] = {bflo(gw.x), bfhi(gw.x), bflo(gw.y), bfhi(gw.y), bflo(gw.z), bfhi(gw.z), bflo(gw.w), bfhi(gw.w)};
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] += g[j] * (m[j] * inv);
    reinterpret_cast<float4*>(xr)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4*>(xr)[1] = make_float4(x[4], x[5], x[6], x[7]);
  }
  if (dump) {
    float4* dd = reinterpret_cast<float4*>(dump + (size_t)r * D + i);
    dd[0] = make_float4(x[0], x[1], x[2], x[3]);
    dd[1] = make_float4(x[4], x[5], x[6], x[7]);
  }
  if (g_next) {
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) ss += x[j] * x[j];
    ss = block_sum<8>(ss, red);
    const float inv = rsqrtf(ss * (1.0f / D) + eps);
    uint4 gw = ldg16(g_next + i);
    float g[8] = {bflo(gw.x), bfhi(gw.x), bflo(gw.y), bfhi(gw.y), bflo(gw.z), bfhi(gw.z), bflo(gw.w), bfhi(gw.w)};
    uint4 o;
    o.x = pack_bf2(g[0] * (x[0] * inv), g[1] * (x[1] * inv));
    o.y = pack_bf2(g[2] * (x[2] * inv), g[3] * (x[3] * inv));
    o.z = pack_bf2(g[4] * (x[4] * inv), g[5] * (x[5] * inv));
    o.w = pack_bf2(g[6] * (x[6] * inv), g[7] * (x[7] * inv));
    if (xn_f16) o = make_uint4(bf2_to_h2(o.x), bf2_to_h2(o.y), bf2_to_h2(o.z), bf2_to_h2(o.w));
    stg16(xn + (size_t)r * D + i, o);
  }
}

cudaError_t resid_norm(float* x_res, const float* part, int n_part, long part_stride, const bf16* g_post,
                       const bf16* g_next, bf16* xn, int rows, float eps, float* dump, int xn_f16, cudaStream_t s) {
  return launch(k_resid_norm, dim3(rows), dim3(256), 0, s, x_res, part, n_part, part_stride, g_post, g_next, xn,
                eps, dump, xn_f16);
}

// ------------------------------------------------------------------------------------------
// Gated short conv (coreai-model-zoo "lfm3-1.7b-port", diff table row 1): with [B|C|x] the
// in_proj output (fp32 accumulators), bx = bf16(B * x); over win = [state(6) | bx], z_t = sum_k w[c][k] win[t+k]
// (tap 6 on the newest column); y = bf16(C * z); the new state is win[n : n + 6].
// Decode: one row per stream, state [slot][6][D] shifts by one column.
__global__ void __launch_bounds__(256) k_conv_decode(const float* __restrict__ bcx, int n_parts, long part_stride,
                                                     const bf16* __restrict__ conv_w, bf16* __restrict__ state,
                                                     const int32_t* __restrict__ row_slot, int win,
                                                     bf16* __restrict__ snap, bf16* __restrict__ y) {
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.y;
  const int c = blockIdx.x * 256 + threadIdx.x;
  auto at = [&](int r, int i) {  // column i of in_proj row r: the partials summed in split order
    const float* e = bcx + (size_t)r * 3 * D + i;
    float v = e[0];
    for (int p = 1; p < n_parts; ++p) v += e[p * part_stride];
    return v;
  };
  const float Cv = at(b, D + c);
  bf16* st = state + (size_t)row_slot[b] * CST * D + c;
  const bf16* w = conv_w + (size_t)c * TAPS;
  if (win <= 1) {
    const float bx = round_bf(at(b, c) * at(b, 2 * D + c));
    float win6[CST];
#pragma unroll
    for (int j = 0; j < CST; ++j) win6[j] = bf2f(st[(size_t)j * D]);
    float z = 0.f;
#pragma unroll
    for (int k = 0; k < CST; ++k) z += bf2f(w[k]) * win6[k];
    z += bf2f(w[CST]) * bx;
    y[(size_t)b * D + c] = f2bf(Cv * z);
#pragma unroll
    for (int j = 0; j < CST - 1; ++j) st[(size_t)j * D] = f2bf(win6[j + 1]);
    st[(size_t)(CST - 1) * D] = f2bf(bx);
    return;
  }
  // verify window: row wi of its stream sees [state | bx of the window's rows 0..wi]
  const int wi = b % win, b0 = b - wi;
  float wnd[CST + MAX_WIN];
#pragma unroll
  for (int j = 0; j < CST; ++j) wnd[j] = bf2f(st[(size_t)j * D]);
  for (int i = 0; i <= wi; ++i) wnd[CST + i] = round_bf(at(b0 + i, c) * at(b0 + i, 2 * D + c));
  float z = 0.f;
#pragma unroll
  for (int k = 0; k < TAPS; ++k) z += bf2f(w[k]) * wnd[wi + k];
  y[(size_t)b * D + c] = f2bf(Cv * z);
#pragma unroll
  for (int j = 0; j < CST; ++j) snap[((size_t)b * CST + j) * D + c] = f2bf(wnd[wi + 1 + j]);
}

cudaError_t conv_decode(const float* bcx, int n_parts, long part_stride, const bf16* conv_w, bf16* state_layer,
                        const int32_t* row_slot, int rows, int win, bf16* snap, bf16* y, cudaStream_t s) {
  return launch(k_conv_decode, dim3(D / 256, rows), dim3(256), 0, s, bcx, n_parts, part_stride, conv_w, state_layer,
                row_slot, win, snap, y);
}

// Prefill: n consecutive rows of one slot. Block (channel group, row group of 32). Only the
// first row group reads the carried state (rows < 6), and it also writes the new state, so
// the read precedes the write within one thread. The new state is columns [n_state, n_state + 6)
// of [state | bx]: n_state = n, or the real rows of a chunk padded at its end (coreai-model-zoo
// note "lfm3-1.7b-port", pad-tail paragraph: "columns [n, n + 6) of [state | Bx], n = the
// number of query position ids >= 0").
constexpr int CONV_RG = 32;
__global__ void __launch_bounds__(128) k_conv_prefill(const float* __restrict__ bcx, const bf16* __restrict__ conv_w,
                                                      bf16* __restrict__ state, int n, int n_state,
                                                      bf16* __restrict__ y) {
  pdl_wait();
  pdl_launch_dependents();
  const int c = blockIdx.x * 128 + threadIdx.x;
  const int r0 = blockIdx.y * CONV_RG;
  const int r1 = min(n, r0 + CONV_RG);
  float w[TAPS];
#pragma unroll
  for (int k = 0; k < TAPS; ++k) w[k] = bf2f(conv_w[(size_t)c * TAPS + k]);
  auto bx_at = [&](int t) -> float {  // bx of row t of this chunk (stored state precision: bf16)
    const float* row = bcx + (size_t)t * 3 * D;
    return round_bf(row[c] * row[2 * D + c]);
  };
  auto win_at = [&](int i) -> float {  // win[i] = state[i] for i < 6, bx[i - 6] after
    return i < CST ? bf2f(state[(size_t)i * D + c]) : bx_at(i - CST);
  };
  float win[TAPS];
#pragma unroll
  for (int k = 0; k < CST; ++k) win[k] = win_at(r0 + k);
  for (int t = r0; t < r1; ++t) {
    win[CST] = bx_at(t);
    float z = 0.f;
#pragma unroll
    for (int k = 0; k < TAPS; ++k) z += w[k] * win[k];
    y[(size_t)t * D + c] = f2bf(bcx[(size_t)t * 3 * D + D + c] * z);
#pragma unroll
    for (int k = 0; k < CST; ++k) win[k] = win[k + 1];
  }
  if (blockIdx.y == 0) {
    float ns[CST];
#pragma unroll
    for (int j = 0; j < CST; ++j) ns[j] = win_at(n_state + j);
#pragma unroll
    for (int j = 0; j < CST; ++j) state[(size_t)j * D + c] = f2bf(ns[j]);
  }
}

cudaError_t conv_prefill(const float* bcx, const bf16* conv_w, bf16* state_slot, int n, int n_state, bf16* y,
                         cudaStream_t s) {
  return launch(k_conv_prefill, dim3(D / 128, (n + CONV_RG - 1) / CONV_RG), dim3(128), 0, s, bcx, conv_w,
                state_slot, n, n_state, y);
}

// ------------------------------------------------------------------------------------------
// Per-head q/k RMSNorm (gain of length 128 shared across heads), rotary on pairs (i, i+64) with
// a per-position table (zero-tail pairs carry cos 1, sin 0), and placement of k/v.
// One warp per (row, head slot): slots 0..15 are q heads, 16..19 k heads, 20..23 v heads. Lane l
// holds dims l, l + 32, l + 64, l + 96, so each rotary pair (i, i + 64) sits in one lane; the head's
// RMS is a warp sum. q (and k) are normalised, rotated and rounded to bf16; v is rounded; the gate
// logits (q slots' lane 0) are summed over the partials.
__global__ void __launch_bounds__(256) k_qk_norm_rope_kv(const float* __restrict__ part, int n_part,
                                                         long part_stride, const bf16* __restrict__ q_norm,
                                                         const bf16* __restrict__ k_norm,
                                                         const float* __restrict__ rope_cos,
                                                         const float* __restrict__ rope_sin, Rows rows, float eps,
                                                         bf16* __restrict__ q_out, float* __restrict__ gate_out,
                                                         KvWrite kv) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x, hh = blockIdx.y * 8 + warp;  // head slot 0..23
  // gains and rotary rows do not depend on the previous kernel
  const bool qk = hh < HQ + HKV;
  float gn[4] = {1.f, 1.f, 1.f, 1.f};
  if (qk) {
    const bf16* g = hh < HQ ? q_norm : k_norm;
#pragma unroll
    for (int k = 0; k < 4; ++k) gn[k] = bf2f(g[lane + 32 * k]);
  }
  pdl_wait();
  pdl_launch_dependents();
  const int pos = rows.pos[r];
  const int col0 = hh * HD;  // q heads, then k heads, then v heads are consecutive in qkvg
  float x[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < n_part; ++s) {
    const float* p = part + s * part_stride + (size_t)r * NQKVG + col0;
#pragma unroll
    for (int k = 0; k < 4; ++k) x[k] += p[lane + 32 * k];
  }
  if (qk) {
    const float ss = warp_sum(x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3]);
    const float inv = rsqrtf(ss * (1.0f / HD) + eps);
#pragma unroll
    for (int k = 0; k < 4; ++k) x[k] = gn[k] * (x[k] * inv);
    // pairs (d, d + 64): dims lane + 32k for k = 0, 1 with k + 2
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int i = lane + 32 * k;
      const float c = rope_cos[(size_t)pos * (HD / 2) + i], sn = rope_sin[(size_t)pos * (HD / 2) + i];
      const float lo = x[k], hi = x[k + 2];
      x[k] = lo * c - hi * sn;
      x[k + 2] = hi * c + lo * sn;
    }
  }
  if (hh < HQ) {
    bf16* qo = q_out + ((size_t)r * HQ + hh) * HD;
#pragma unroll
    for (int k = 0; k < 4; ++k) qo[lane + 32 * k] = f2bf(x[k]);
    if (lane == 0) {
      float gsum = 0.f;
      for (int s = 0; s < n_part; ++s) gsum += part[s * part_stride + (size_t)r * NQKVG + HQ * HD + 2 * HKV * HD + hh];
      gate_out[r * HQ + hh] = gsum;
    }
    return;
  }
  const bool isk = hh < HQ + HKV;
  const int kvh = isk ? hh - HQ : hh - HQ - HKV;
  bf16* base = isk ? kv.k : kv.v;
  size_t off;
  if (kv.mode == KV_PAGES) {
    const int slot = rows.slot[r];
    const int page = kv.page_table[(size_t)slot * kv.max_pages + pos / PAGE];
    off = (((size_t)page * HKV + kvh) * PAGE + pos % PAGE) * HD;
  } else {
    off = ((size_t)kvh * kv.scratch_rows + WIN + r) * HD;
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) base[off + lane + 32 * k] = f2bf(x[k]);
}

cudaError_t qk_norm_rope_kv(const float* part, int n_part, long part_stride, const bf16* q_norm, const bf16* k_norm,
                            const float* rope_cos, const float* rope_sin, Rows rows, float eps, bf16* q_out,
                            float* gate_out, KvWrite kv, cudaStream_t s) {
  return launch(k_qk_norm_rope_kv, dim3(rows.n, (HQ + 2 * HKV) / 8), dim3(256), 0, s, part, n_part, part_stride,
                q_norm, k_norm, rope_cos, rope_sin, rows, eps, q_out, gate_out, kv);
}

// ------------------------------------------------------------------------------------------
// Sliding layers in a prompt pass: the ring's last WIN positions before the chunk are copied
// into scratch rows [0, WIN) (index i <-> position p0 - WIN + i; rows before position 0 are
// zero), the chunk's own k/v land in rows WIN + r, and after attention the chunk's last
// min(n, WIN) positions go back to their ring slots.
__global__ void __launch_bounds__(128) k_ring_to_scratch(const bf16* __restrict__ rk, const bf16* __restrict__ rv,
                                                         int slot, int p0, bf16* __restrict__ sk,
                                                         bf16* __restrict__ sv, int scratch_rows) {
  pdl_wait();
  pdl_launch_dependents();
  const int i = blockIdx.x, h = blockIdx.y, d = threadIdx.x;
  const int pos = p0 - WIN + i;
  bf16 kx = f2bf(0.f), vx = f2bf(0.f);
  if (pos >= 0) {
    const size_t o = (((size_t)slot * HKV + h) * WIN + pos % WIN) * HD + d;
    kx = rk[o];
    vx = rv[o];
  }
  const size_t so = ((size_t)h * scratch_rows + i) * HD + d;
  sk[so] = kx;
  sv[so] = vx;
}

cudaError_t ring_to_scratch(const bf16* ring_k, const bf16* ring_v, int slot, int max_streams, int p0, bf16* sk,
                            bf16* sv, int scratch_rows, cudaStream_t s) {
  (void)max_streams;
  return launch(k_ring_to_scratch, dim3(WIN, HKV), dim3(HD), 0, s, ring_k, ring_v, slot, p0, sk, sv, scratch_rows);
}

__global__ void __launch_bounds__(128) k_scratch_to_ring(const bf16* __restrict__ sk, const bf16* __restrict__ sv,
                                                         int scratch_rows, int n, int p0, bf16* __restrict__ rk,
                                                         bf16* __restrict__ rv, int slot) {
  pdl_wait();
  pdl_launch_dependents();
  const int m = min(n, WIN);
  const int r = n - m + blockIdx.x, h = blockIdx.y, d = threadIdx.x;
  const int pos = p0 + r;
  const size_t so = ((size_t)h * scratch_rows + WIN + r) * HD + d;
  const size_t o = (((size_t)slot * HKV + h) * WIN + pos % WIN) * HD + d;
  rk[o] = sk[so];
  rv[o] = sv[so];
}

cudaError_t scratch_to_ring(const bf16* sk, const bf16* sv, int scratch_rows, int n, int p0, bf16* ring_k,
                            bf16* ring_v, int slot, int max_streams, cudaStream_t s) {
  (void)max_streams;
  return launch(k_scratch_to_ring, dim3(n < WIN ? n : WIN, HKV), dim3(HD), 0, s, sk, sv, scratch_rows, n, p0, ring_k,
                ring_v, slot);
}

// ------------------------------------------------------------------------------------------
// End of a call: advance seq_len and publish greedy ids (the cells hold (ordered value << 32) |
// (0xffffffff - id), so the max is the largest logit with the lowest id among ties).
__global__ void k_finish(int32_t* seq_len, const int32_t* __restrict__ row_slot, int rows, int add_prefill,
                         int prefill_slot, const unsigned long long* __restrict__ amax, int32_t* argmax_out,
                         int advance) {
  pdl_wait();
  pdl_launch_dependents();
  const int r = threadIdx.x;
  if (add_prefill) {
    if (r == 0) {
      seq_len[prefill_slot] += add_prefill;
      if (argmax_out && amax) argmax_out[0] = (int32_t)(0xffffffffu - (uint32_t)(amax[0] & 0xffffffffull));
    }
    return;
  }
  if (r < rows) {
    if (advance) seq_len[row_slot[r]] += 1;
    if (argmax_out && amax) argmax_out[r] = (int32_t)(0xffffffffu - (uint32_t)(amax[r] & 0xffffffffull));
  }
}

cudaError_t finish_step(int32_t* seq_len, const int32_t* row_slot, int rows, int add_prefill, int prefill_slot,
                        const unsigned long long* amax, int32_t* argmax_out, int advance, cudaStream_t s) {
  return launch(k_finish, dim3(1), dim3(64), 0, s, seq_len, row_slot, rows, add_prefill, prefill_slot, amax,
                argmax_out, advance);
}

// ------------------------------------------------------------------------------------------
// Commit of verify windows (TensorFold PR #1508, lfm2_moe.cu paragraph: "the commit of an
// accepted row's conv state"): for stream i, with k = a.k[i] accepted rows of its window,
// the conv state becomes the snapshot after row k - 1, the sliding rings take the window's first
// k rows at their slots, and seq_len advances by k. Block (stream, unit): units 0 .. n_conv - 1
// copy one layer's conv columns, the rest one (sliding layer, accepted row).
__global__ void __launch_bounds__(256) k_commit(CommitArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int i = blockIdx.x, u = blockIdx.y;
  const int slot = a.slot[i], k = a.k[i];
  if (u < a.n_conv) {
    const uint4* src = reinterpret_cast<const uint4*>(
        a.snap + (((size_t)u * a.max_batch + (size_t)i * a.W + k - 1) * CST) * D);
    uint4* dst = reinterpret_cast<uint4*>(a.conv + (((size_t)u * a.max_streams + slot) * CST) * D);
    for (int e = threadIdx.x; e < CST * D / 8; e += blockDim.x) dst[e] = src[e];
  } else {
    const int j = (u - a.n_conv) / MAX_WIN, r = (u - a.n_conv) % MAX_WIN;
    if (r < k) {
      const int ringpos = (a.pos[i] + r) % WIN;
      for (int e = threadIdx.x; e < 2 * HKV * HD / 8; e += blockDim.x) {
        const int kv = e / (HKV * HD / 8), hc = e % (HKV * HD / 8), h = hc / (HD / 8), c8 = hc % (HD / 8);
        const bf16* sb = (kv ? a.side_v : a.side_k) + (((size_t)j * a.max_batch + (size_t)i * a.W + r) * HKV + h) * HD;
        bf16* rb = (kv ? a.ring_v : a.ring_k) + ((((size_t)j * a.max_streams + slot) * HKV + h) * WIN + ringpos) * HD;
        reinterpret_cast<uint4*>(rb)[c8] = reinterpret_cast<const uint4*>(sb)[c8];
      }
    }
  }
  if (u == 0 && threadIdx.x == 0) a.seq_len[slot] = a.pos[i] + k;
}

cudaError_t commit_windows(const CommitArgs& a, cudaStream_t s) {
  return launch(k_commit, dim3(a.n, a.n_conv + a.n_sliding * MAX_WIN), dim3(256), 0, s, a);
}

// ------------------------------------------------------------------------------------------
// Self-test of the failure path: one thread waits on a fresh mbarrier that nothing will ever
// arrive on, with the given iteration limit (the kernels' own waits use WAIT_LIMIT); when the
// limit runs out it records the failure in the status word, as every bounded wait does, and
// the kernel returns. Nothing is copied into the barrier's transaction, so nothing is in flight.
__global__ void k_wait_selftest(int* err, unsigned rounds) {
  __shared__ __align__(8) uint64_t bar;
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x != 0) return;
  mbar_init(su32(&bar), 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  for (unsigned i = 0; i < rounds; ++i)
    if (mbar_try(su32(&bar), 0)) return;
  atomicExch(err, 2);
}

cudaError_t wait_selftest(int* err, unsigned rounds, cudaStream_t s) {
  return launch(k_wait_selftest, dim3(1), dim3(32), 0, s, err, rounds);
}

// ------------------------------------------------------------------------------------------
// Kept state of one slot at a mark (TensorFold PR #1508, prompt-cache paragraph: the slot's
// conv states and its keys and values at positions [0, at); on LFM3 also the sliding rings).
// The snapshot is [conv: n_conv][6][D] | [ring: n_sliding][K, V][HKV][WIN][HD] |
// [pages: n_full][K, V][ceil(at / 64)][HKV][PAGE][HD], bf16. One block per 8 KB unit of it;
// pages are found through the slot's page table. keep: state -> snapshot; restore: snapshot ->
// state, and seq_len[slot] = at.
constexpr int SNAP_UNIT = 8192;
constexpr int SNAP_CONV_UNITS = CST * D * 2 / SNAP_UNIT;              // 3
constexpr int SNAP_RING_UNITS = HKV * WIN * HD * 2 / SNAP_UNIT;       // 32 per K or V
constexpr int SNAP_PAGE_UNITS = HKV * PAGE * HD * 2 / SNAP_UNIT;      // 8 per K or V
static_assert(CST * D * 2 % SNAP_UNIT == 0, "conv columns in whole units");

__global__ void __launch_bounds__(256) k_state_copy(SnapArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  int u = blockIdx.x;
  const char* src;
  char* dst;
  char* snap = reinterpret_cast<char*>(a.snap);
  size_t soff;
  char* st;
  if (u < a.n_conv * SNAP_CONV_UNITS) {
    const int j = u / SNAP_CONV_UNITS, part = u % SNAP_CONV_UNITS;
    soff = (size_t)j * CST * D * 2 + (size_t)part * SNAP_UNIT;
    st = reinterpret_cast<char*>(a.conv) + ((size_t)j * a.max_streams + a.slot) * CST * D * 2 + (size_t)part * SNAP_UNIT;
  } else if ((u -= a.n_conv * SNAP_CONV_UNITS) < a.n_sliding * 2 * SNAP_RING_UNITS) {
    const int j = u / (2 * SNAP_RING_UNITS), kv = (u / SNAP_RING_UNITS) & 1, part = u % SNAP_RING_UNITS;
    soff = (size_t)a.n_conv * CST * D * 2 + (((size_t)j * 2 + kv) * SNAP_RING_UNITS + part) * SNAP_UNIT;
    st = reinterpret_cast<char*>(kv ? a.ring_v : a.ring_k) + ((size_t)j * a.max_streams + a.slot) * HKV * WIN * HD * 2 +
         (size_t)part * SNAP_UNIT;
  } else {
    u -= a.n_sliding * 2 * SNAP_RING_UNITS;
    const int per = 2 * a.npg * SNAP_PAGE_UNITS;
    const int j = u / per, kv = (u / (a.npg * SNAP_PAGE_UNITS)) & 1, pg = (u / SNAP_PAGE_UNITS) % a.npg,
              part = u % SNAP_PAGE_UNITS;
    soff = (size_t)a.n_conv * CST * D * 2 + (size_t)a.n_sliding * 2 * SNAP_RING_UNITS * SNAP_UNIT +
           ((((size_t)j * 2 + kv) * a.npg + pg) * SNAP_PAGE_UNITS + part) * SNAP_UNIT;
    const int page = a.page_table[(size_t)a.slot * a.max_pages + pg];
    st = reinterpret_cast<char*>(kv ? a.kv_v : a.kv_k) + (((size_t)j * a.n_pages + page) * HKV * PAGE * HD) * 2 +
         (size_t)part * SNAP_UNIT;
  }
  if (a.restore) {
    src = snap + soff;
    dst = st;
  } else {
    src = st;
    dst = snap + soff;
  }
  for (int i = threadIdx.x; i < SNAP_UNIT / 16; i += blockDim.x)
    stg16(dst + 16 * i, ldg16(src + 16 * i));
  if (a.restore && blockIdx.x == 0 && threadIdx.x == 0) a.seq_len[a.slot] = a.at;
}

size_t snapshot_bytes(int n_conv, int n_sliding, int n_full, int at) {
  const size_t npg = ((size_t)at + PAGE - 1) / PAGE;
  return (size_t)n_conv * CST * D * 2 + (size_t)n_sliding * 2 * HKV * WIN * HD * 2 +
         (size_t)n_full * 2 * npg * HKV * PAGE * HD * 2;
}

cudaError_t state_copy(const SnapArgs& a, cudaStream_t s) {
  const int units = a.n_conv * SNAP_CONV_UNITS + a.n_sliding * 2 * SNAP_RING_UNITS +
                    a.n_full * 2 * a.npg * SNAP_PAGE_UNITS;
  if (units == 0) return cudaSuccess;
  return launch(k_state_copy, dim3(units), dim3(256), 0, s, a);
}

}  // namespace lfm3
