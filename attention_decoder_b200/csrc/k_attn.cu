// Decode-time GQA attention of the LFM3 decoder (16 q heads over 4 kv heads of 128;
// coreai-model-zoo note "lfm3-1.7b-port", diff table rows 2-4, and "window_size, with no mask
// input").
//
// A key at position k is visible to a query at position p iff k <= p and, on sliding layers,
// p - k < 256. Scores are q.k / sqrt(128), softmax in fp32, and the per-head gate sigmoid(g_h)
// multiplies each head's output before o_proj (fused into the merge here).
//
// One launch per layer, from the raw q|k|v|gate projection rows (fp32, one row per stream):
// block (split, kv head, stream) owns whole 64-key pages - on full layers one page, or 2..8 pages
// once the batch gives thousands of blocks; on sliding layers a quarter of the 256-slot ring - so
// its keys and values arrive as contiguous 16 KB tiles, two bulk copies per page into one of two
// buffers; the first two pages are requested before the block waits for the projection kernel
// (the cache does not depend on it). After the wait the block normalises and rotates its four
// query heads and the head's new key, rounds them to bf16, writes the new key and value to the
// cache (the block holding the current position does) and substitutes them for the stale row
// in its shared copy. Each warp owns 8 keys of every page: lane l holds dims 4l..4l+3 of the
// four queries, one transposing butterfly turns the 32 per-lane partial dots (8 keys x 4 heads)
// into 32 finished scores, one per lane, and the warp keeps its own online softmax (running max
// and sum per head, its P.V sums over dims 4l..4l+3 rescaled at a new max), so a page needs no
// block barrier between scores, softmax and P.V; the eight warps' states merge once per split.
// Each block writes its unnormalised partial (max, sum, o) per head; the last block of a
// (stream, kv head) - counted with an atomic - merges the splits with every warp loading a
// different subset of them, applies the gate and writes the bf16 output.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <utility>
#include <vector>

#include "kernels.cuh"

namespace lfm3 {

constexpr int DA_THREADS = 256;                  // 8 warps
constexpr int DA_WARPS = DA_THREADS / 32;
constexpr int DA_TILE = DEC_KEYS * HD * 2;       // bytes of one K or V tile
constexpr int DA_SMEM = 2 * DA_TILE;             // one page buffer: K and V tiles (two buffers)
static_assert(DEC_KEYS == PAGE, "a decode split is one page");
static_assert(DA_WARPS * 8 == DEC_KEYS, "eight keys per warp");

int attn_decode_splits(int max_pos) {
  int s = WIN / DEC_KEYS;
  while (s * DEC_KEYS < max_pos) s *= 2;
  return s;
}

// Partials of a step: o [rows][HQ][splits][HD] (float4 aligned), then (max, sum) [rows][HQ][splits][2].
DEVI size_t da_ml_offset(int nrows, int splits) { return (size_t)nrows * HQ * splits * HD; }

__global__ void __launch_bounds__(DA_THREADS) k_attn_decode_fused(const float* __restrict__ qkvg, Rows rows,
                                                                  AttnLayer L, AttnDecodeArgs A, int splits, int pps,
                                                                  float* __restrict__ part, bf16* __restrict__ y) {
  extern __shared__ __align__(128) unsigned char dsm[];  // two buffers of one page: K then V
  __shared__ __align__(16) float qs[GQA][HD];
  __shared__ float kb[HD];
  __shared__ __align__(16) float obuf[DA_WARPS][GQA][HD];  // the warps' P.V sums (then the merge's halves)
  __shared__ float wm[DA_WARPS][GQA], wl[DA_WARPS][GQA];     // the warps' running max and sum per head
  __shared__ float red[GQA + 1][4];
  __shared__ float lx[GQA];
  __shared__ __align__(16) bf16 wk[MAX_WIN][HD], wv[MAX_WIN][HD];  // earlier rows of a verify window
  __shared__ float kw[HD];
  __shared__ __align__(8) uint64_t kv_bar[2];
  __shared__ int last;

  const int sp = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
#ifdef LFM3_TRACE
  if (tid == 0) {
    TRACE(A.trace, A.trace_id, 0);
    TRACE(A.trace, A.trace_id, 7);
  }
#endif
  // rows were set by the first kernel of the step, which has completed (reads go to L2)
  const int slot = __ldcg(rows.slot + b), pos = __ldcg(rows.pos + b);
  const int nkeys = L.full ? pos + 1 : min(pos + 1, WIN);
  const int keys_per = pps * DEC_KEYS;                 // keys of one split: pps pages
  const int nact = (nkeys + keys_per - 1) / keys_per;  // splits with keys
  if (sp >= nact) {
    pdl_wait();
    pdl_launch_dependents();
    return;
  }
  const int cur = L.full ? pos : pos % WIN;  // key index of the current position
  const int j0 = sp * keys_per, cnt = min(nkeys - j0, keys_per);
  const int np = (cnt + DEC_KEYS - 1) / DEC_KEYS;  // pages of this split
  // the K / V tile of page i of the split (64 keys of this kv head, contiguous)
  auto tile_of = [&](int i) -> size_t {
    const int j = j0 + i * DEC_KEYS;
    return L.full ? ((size_t)L.page_table[(size_t)slot * L.max_pages + j / DEC_KEYS] * HKV + kvh) * PAGE * HD
                  : (((size_t)slot * HKV + kvh) * WIN + j) * HD;
  };
  auto fetch = [&](int i) {  // page i into buffer i & 1 (thread 0)
    const uint32_t buf = su32(dsm) + (uint32_t)(i & 1) * DA_SMEM, bar = su32(&kv_bar[i & 1]);
    const size_t t = tile_of(i);
    mbar_expect_tx(bar, DA_SMEM);
    bulk_g2s(buf, L.k + t, DA_TILE, bar);
    bulk_g2s(buf + DA_TILE, L.v + t, DA_TILE, bar);
  };
  if (tid == 0) {
    mbar_init(su32(&kv_bar[0]), 1);
    mbar_init(su32(&kv_bar[1]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fetch(0);
    if (np > 1) fetch(1);
  }
  // gains and rotary coefficients of dimension d = tid (threads < 128) are weights too
  const int d = tid & (HD - 1), pd = d < 64 ? d + 64 : d - 64, ir = d & 63;
  const float gq = bf2f(A.q_norm[d]), gk = bf2f(A.k_norm[d]);
  const float cr = A.rope_cos[(size_t)pos * (HD / 2) + ir], sr = A.rope_sin[(size_t)pos * (HD / 2) + ir];
  pdl_wait();
  pdl_launch_dependents();
#ifdef LFM3_TRACE
  if (tid == 0) TRACE(A.trace, A.trace_id, 2);
#endif

  // ---- queries and the new key / value (threads 0..127: thread = dimension d of each head)
  // element i of q|k|v|gate row r: the K-split partials summed in split order
  auto rawat = [&](int r, int i) {
    const float* e = qkvg + (size_t)r * NQKVG + i;
    float v = e[0];
    for (int p = 1; p < A.n_parts; ++p) v += e[p * A.part_stride];
    return v;
  };
  float qv[GQA], kv = 0.f, vv = 0.f;
  if (tid < HD) {
    float s2[GQA + 1];
#pragma unroll
    for (int hh = 0; hh < GQA; ++hh) {
      qv[hh] = rawat(b, (kvh * GQA + hh) * HD + d);
      s2[hh] = warp_sum(qv[hh] * qv[hh]);
    }
    kv = rawat(b, HQ * HD + kvh * HD + d);
    vv = rawat(b, HQ * HD + HKV * HD + kvh * HD + d);
    s2[GQA] = warp_sum(kv * kv);
    if (lane == 0)
#pragma unroll
      for (int hh = 0; hh <= GQA; ++hh) red[hh][warp] = s2[hh];
  }
  __syncthreads();
  if (tid < HD) {
#pragma unroll
    for (int hh = 0; hh < GQA; ++hh) {
      const float inv = rsqrtf((red[hh][0] + red[hh][1] + red[hh][2] + red[hh][3]) * (1.0f / HD) + A.eps);
      qs[hh][d] = gq * (qv[hh] * inv);
    }
    kb[d] = gk * (kv * rsqrtf((red[GQA][0] + red[GQA][1] + red[GQA][2] + red[GQA][3]) * (1.0f / HD) + A.eps));
  }
  __syncthreads();
  // rotary on pairs (i, i + 64); q and k rounded to bf16 (their stored precision)
  float qr[GQA], kr = 0.f;
  if (tid < HD) {
#pragma unroll
    for (int hh = 0; hh < GQA; ++hh)
      qr[hh] = round_bf(d < 64 ? qs[hh][d] * cr - qs[hh][pd] * sr : qs[hh][d] * cr + qs[hh][pd] * sr);
    kr = round_bf(d < 64 ? kb[d] * cr - kb[pd] * sr : kb[d] * cr + kb[pd] * sr);
  }
  __syncthreads();
  const float scale = rsqrtf((float)HD);
  const bool has_cur = cur >= j0 && cur < j0 + cnt;
  const int wi = b % A.win;  // this row's index in its stream's verify window (0 when decoding)
  if (tid < HD) {
#pragma unroll
    for (int hh = 0; hh < GQA; ++hh) qs[hh][d] = qr[hh] * scale;
    if (has_cur) {  // the new key and value into the cache, as every later step reads them
      if (L.full || A.win == 1) {
        const size_t row = tile_of((cur - j0) / DEC_KEYS) + (size_t)((cur - j0) % DEC_KEYS) * HD + d;
        const_cast<bf16*>(L.k)[row] = f2bf(kr);
        const_cast<bf16*>(L.v)[row] = f2bf(vv);
      } else {  // a verify window's sliding rows wait for the commit in the side buffer
        A.side_k[((size_t)b * HKV + kvh) * HD + d] = f2bf(kr);
        A.side_v[((size_t)b * HKV + kvh) * HD + d] = f2bf(vv);
      }
    }
  }
  // the window's earlier rows (positions pos - wi .. pos - 1) are not in the cache yet: compute
  // their keys and values here (norm, rotary at their own positions, bf16) for this split
  for (int ip = 0; ip < wi; ++ip) {
    const int pp = pos - wi + ip;
    const int kidx = L.full ? pp : pp % WIN;
    if (kidx < j0 || kidx >= j0 + cnt) continue;  // uniform over the block
    float k1 = 0.f, v1 = 0.f;
    if (tid < HD) {
      k1 = rawat(b - wi + ip, HQ * HD + kvh * HD + d);
      v1 = rawat(b - wi + ip, HQ * HD + HKV * HD + kvh * HD + d);
      const float s2 = warp_sum(k1 * k1);
      if (lane == 0) red[0][warp] = s2;
    }
    __syncthreads();
    if (tid < HD) kw[d] = gk * (k1 * rsqrtf((red[0][0] + red[0][1] + red[0][2] + red[0][3]) * (1.0f / HD) + A.eps));
    __syncthreads();
    if (tid < HD) {
      const float c1 = A.rope_cos[(size_t)pp * (HD / 2) + ir], s1 = A.rope_sin[(size_t)pp * (HD / 2) + ir];
      wk[ip][d] = f2bf(d < 64 ? kw[d] * c1 - kw[pd] * s1 : kw[d] * c1 + kw[pd] * s1);
      wv[ip][d] = f2bf(v1);
    }
    __syncthreads();
  }

  // ---- the split's pages, two buffers deep. Each warp keeps its own online softmax over its
  // eight keys of every page (running max and sum per head, its P.V sums rescaled at a new max):
  // no block barrier between scores, softmax and P.V; the eight warps' states merge once at the
  // end of the split.
  const size_t mloff = da_ml_offset(rows.n, splits);
  const size_t hbase = ((size_t)b * HQ + kvh * GQA) * splits;  // (stream, first head of the group) x splits
  float o[GQA][4] = {};                       // this lane's dims 4 lane .. 4 lane + 3 of each head
  float Mw = -INFINITY, Lw = 0.f;             // head lane >> 3: this warp's running max and sum
  float4 q4[GQA];                             // dims 4 lane .. of the four (scaled) queries
  bool ok = true;
  int issued = min(np, 2), done = 0;          // pages copied / pages landed
  for (int i = 0; i < np; ++i) {
    const bf16* ks = reinterpret_cast<const bf16*>(dsm + (size_t)(i & 1) * DA_SMEM);
    const bf16* vs = ks + DEC_KEYS * HD;
    const int pj0 = j0 + i * DEC_KEYS, pc = min(cnt - i * DEC_KEYS, DEC_KEYS);
    if (ok) ok = mbar_wait(su32(&kv_bar[i & 1]), (i >> 1) & 1, A.err);
    ok = __syncthreads_and(ok);  // the same for every thread of the block
    if (ok) done = i + 1;
    // the rows of the current position (and of the window's earlier ones) here are stale
    if (tid < HD) {
      bf16* kw2 = const_cast<bf16*>(ks);
      bf16* vw2 = const_cast<bf16*>(vs);
      if (cur >= pj0 && cur < pj0 + pc) {
        kw2[(cur - pj0) * HD + d] = f2bf(kr);
        vw2[(cur - pj0) * HD + d] = f2bf(vv);
      }
      for (int ip = 0; ip < wi; ++ip) {
        const int pp = pos - wi + ip;
        const int kidx = L.full ? pp : pp % WIN;
        if (kidx >= pj0 && kidx < pj0 + pc) {
          kw2[(kidx - pj0) * HD + d] = wk[ip][d];
          vw2[(kidx - pj0) * HD + d] = wv[ip][d];
        }
      }
    }
    __syncthreads();
    if (ok && 8 * warp < pc) {
      if (i == 0)
#pragma unroll
        for (int hh = 0; hh < GQA; ++hh) q4[hh] = *reinterpret_cast<const float4*>(&qs[hh][4 * lane]);
      // scores: this warp's keys 8w .. 8w+7; one transposing butterfly turns the 32 per-lane
      // partial dots into 32 finished scores, lane l holding (head l >> 3, key 8w + (l & 7))
      float v[32];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint2 kk = *reinterpret_cast<const uint2*>(ks + (8 * warp + k) * HD + 4 * lane);
        const float k0 = bflo(kk.x), k1 = bfhi(kk.x), k2 = bflo(kk.y), k3 = bfhi(kk.y);
#pragma unroll
        for (int hh = 0; hh < GQA; ++hh) v[hh * 8 + k] = q4[hh].x * k0 + q4[hh].y * k1 + q4[hh].z * k2 + q4[hh].w * k3;
      }
#pragma unroll
      for (int o2 = 16, c = 32; o2 >= 1; o2 >>= 1, c >>= 1) {
        const bool up = (lane & o2) != 0;
#pragma unroll
        for (int e = 0; e < c / 2; ++e) {
          const float send = up ? v[e] : v[e + c / 2];
          const float keep = up ? v[e + c / 2] : v[e];
          v[e] = keep + __shfl_xor_sync(0xffffffffu, send, o2);
        }
      }
      const float sj = 8 * warp + (lane & 7) < pc ? v[0] : -INFINITY;
      // online softmax of head lane >> 3 over the warp's keys (groups of eight lanes)
      float m8 = sj;
      m8 = fmaxf(m8, __shfl_xor_sync(0xffffffffu, m8, 1));
      m8 = fmaxf(m8, __shfl_xor_sync(0xffffffffu, m8, 2));
      m8 = fmaxf(m8, __shfl_xor_sync(0xffffffffu, m8, 4));
      const float mn = fmaxf(Mw, m8);  // finite: the warp's first key is valid
      const float p = __expf(sj - mn);
      const float a = __expf(Mw - mn);  // 0 on the warp's first page
      float ps = p;
      ps += __shfl_xor_sync(0xffffffffu, ps, 1);
      ps += __shfl_xor_sync(0xffffffffu, ps, 2);
      ps += __shfl_xor_sync(0xffffffffu, ps, 4);
      Lw = Lw * a + ps;
      Mw = mn;
      // P.V over the warp's valid keys: lane l accumulates dims 4l..4l+3 of the four heads
#pragma unroll
      for (int hh = 0; hh < GQA; ++hh) {
        const float ah = __shfl_sync(0xffffffffu, a, 8 * hh);
        o[hh][0] *= ah; o[hh][1] *= ah; o[hh][2] *= ah; o[hh][3] *= ah;
      }
      const int nk = min(8, pc - 8 * warp);
      for (int k = 0; k < nk; ++k) {
        const uint2 vw = *reinterpret_cast<const uint2*>(vs + (8 * warp + k) * HD + 4 * lane);
        const float v0 = bflo(vw.x), v1 = bfhi(vw.x), v2 = bflo(vw.y), v3 = bfhi(vw.y);
#pragma unroll
        for (int hh = 0; hh < GQA; ++hh) {
          const float ph = __shfl_sync(0xffffffffu, p, 8 * hh + k);
          o[hh][0] += ph * v0; o[hh][1] += ph * v1; o[hh][2] += ph * v2; o[hh][3] += ph * v3;
        }
      }
    }
    __syncthreads();  // the buffer is read; refill it with page i + 2
    if (ok && i + 2 < np) {
      if (tid == 0) fetch(i + 2);
      issued = i + 3;
    }
  }
  if (!ok && tid == 0)  // copies still in flight land before the block exits (bounded)
    for (int p = done; p < issued; ++p) mbar_wait(su32(&kv_bar[p & 1]), (p >> 1) & 1, A.err);
  if (ok) {
    // merge the eight warps: weights exp(M_w - M) per head (a warp that saw no key has M_w = -inf)
#pragma unroll
    for (int hh = 0; hh < GQA; ++hh)
      *reinterpret_cast<float4*>(&obuf[warp][hh][4 * lane]) = make_float4(o[hh][0], o[hh][1], o[hh][2], o[hh][3]);
    if ((lane & 7) == 0) {
      wm[warp][lane >> 3] = Mw;
      wl[warp][lane >> 3] = Lw;
    }
    __syncthreads();
    // thread: head hh = tid >> 6, dims 2 (tid & 63) .. +1
    const int hh = tid >> 6, d2 = 2 * (tid & 63);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < DA_WARPS; ++w) M = fmaxf(M, wm[w][hh]);
    float s0 = 0.f, s1 = 0.f, l = 0.f;
#pragma unroll
    for (int w = 0; w < DA_WARPS; ++w) {
      const float wt = wm[w][hh] == -INFINITY ? 0.f : __expf(wm[w][hh] - M);
      const float2 t = *reinterpret_cast<const float2*>(&obuf[w][hh][d2]);
      s0 += wt * t.x;
      s1 += wt * t.y;
      l += wt * wl[w][hh];
    }
    *reinterpret_cast<float2*>(part + (hbase + (size_t)hh * splits + sp) * HD + d2) = make_float2(s0, s1);
    if ((tid & 63) == 0) {
      part[mloff + 2 * (hbase + (size_t)hh * splits + sp)] = M;
      part[mloff + 2 * (hbase + (size_t)hh * splits + sp) + 1] = l;
    }
  } else {  // a copy that never landed: this split contributes nothing
    if (tid < GQA) {
      part[mloff + 2 * (hbase + (size_t)tid * splits + sp)] = -INFINITY;
      part[mloff + 2 * (hbase + (size_t)tid * splits + sp) + 1] = 0.f;
    }
    if (tid < GQA * HD / 4)
      *reinterpret_cast<float4*>(part + (hbase + (size_t)(tid >> 5) * splits + sp) * HD + 4 * lane) =
          make_float4(0.f, 0.f, 0.f, 0.f);
  }

  // ---- the last block of (stream, kv head) merges the splits and applies the gates. The count is
  // taken with acquire-release semantics after the block barrier: it releases every thread's
  // partial (ordered before it by the barrier) and, in the last block, acquires the others'.
  __syncthreads();
#ifdef LFM3_TRACE
  if (tid == 0) TRACE(A.trace, A.trace_id, 3);
#endif
  if (tid == 0) {
    unsigned old;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(old) : "l"(A.counters + b * HKV + kvh) : "memory");
    last = old == (unsigned)(nact - 1);
  }
  __syncthreads();
  if (!last) return;
  // warp w: head w & 3 over the splits s = half, half + 2, ... (half = w >> 2)
  const int hh = warp & 3, half = warp >> 2;
  const size_t hb = hbase + (size_t)hh * splits;
  const float2* ml = reinterpret_cast<const float2*>(part + mloff);
  float M = -INFINITY;
  for (int s = lane; s < nact; s += 32) M = fmaxf(M, __ldcg(&ml[hb + s].x));
  M = warp_max(M);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float lsum = 0.f;
  for (int s0 = 0; s0 < nact; s0 += 32) {
    const int s = s0 + lane;
    float wgt = 0.f;
    if (s < nact) {
      const float2 m2 = __ldcg(&ml[hb + s]);
      wgt = m2.x == -INFINITY ? 0.f : __expf(m2.x - M);
      if ((s & 1) == half) lsum += wgt * m2.y;
    }
    const int ns = min(32, nact - s0);
#pragma unroll 16
    for (int i = half; i < ns; i += 2) {
      const float wi = __shfl_sync(0xffffffffu, wgt, i);
      const float4 o = __ldcg(reinterpret_cast<const float4*>(part + (hb + s0 + i) * HD) + lane);
      acc.x += wi * o.x; acc.y += wi * o.y; acc.z += wi * o.z; acc.w += wi * o.w;
    }
  }
  lsum = warp_sum(lsum);
  if (half == 1) {
    *reinterpret_cast<float4*>(&obuf[0][hh][4 * lane]) = acc;
    if (lane == 0) lx[hh] = lsum;
  }
  __syncthreads();
  if (half == 0) {
    const float4 t = *reinterpret_cast<const float4*>(&obuf[0][hh][4 * lane]);
    const float l = lsum + lx[hh];
    const float gt = sigmoidf_(rawat(b, HQ * HD + 2 * HKV * HD + kvh * GQA + hh)) / l;
    bf16* yo = y + (size_t)b * HQ * HD + (kvh * GQA + hh) * HD + 4 * lane;
    uint2 w;
    w.x = pack_bf2(gt * (acc.x + t.x), gt * (acc.y + t.y));
    w.y = pack_bf2(gt * (acc.z + t.z), gt * (acc.w + t.w));
    *reinterpret_cast<uint2*>(yo) = w;
  }
  if (tid == 0) A.counters[b * HKV + kvh] = 0u;
#ifdef LFM3_TRACE
  if (tid == 0) TRACE(A.trace, A.trace_id, 5);
#endif
}

// Pages per split on full layers: one page while that keeps every SM busy, more (up to 8, each
// split then streams its pages through two buffers) once the batch x kv heads x splits give
// thousands of blocks; fewer, longer blocks spend less on their fixed work and on the merge.
int attn_pages_per_split(int rows, int splits) {
  int pps = 1;
  while (pps < 8 && splits % (2 * pps) == 0 && (long)rows * HKV * (splits / (2 * pps)) >= 2048) pps *= 2;
  return pps;
}

cudaError_t attn_decode_fused(const float* qkvg, Rows rows, AttnLayer L, const AttnDecodeArgs& A, int splits,
                              float* part, bf16* y, cudaStream_t s) {
  const int pps = L.full ? attn_pages_per_split(rows.n, splits) : 1;
  const int nsp = splits / pps;  // blocks (and partial slots) per (stream, kv head)
#ifdef LFM3_TRACE
  AttnDecodeArgs At = A;
  At.trace = g_trace;
  At.trace_id = g_launches;
  return launch(k_attn_decode_fused, dim3(nsp, HKV, rows.n), dim3(DA_THREADS), (pps > 1 ? 2 : 1) * DA_SMEM, s, qkvg,
                rows, L, At, nsp, pps, part, y);
#else
  return launch(k_attn_decode_fused, dim3(nsp, HKV, rows.n), dim3(DA_THREADS), (pps > 1 ? 2 : 1) * DA_SMEM, s, qkvg,
                rows, L, A, nsp, pps, part, y);
#endif
}

cudaError_t attn_init() {
  return cudaFuncSetAttribute(k_attn_decode_fused, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * DA_SMEM);
}

// ------------------------------------------------------------------------------------------ fixed scratch
// Fixed scratch for callers that cannot allocate device memory (lfm3_decode_step_noalloc): 4 MiB
// of split partials, one copy per GPU that loads the library, kept until the process exits.
// Host code never names the array directly: the symbol is a host-side stand-in, so its device
// address is looked up with the device current and passed to the kernels. The address is kept
// per CUDA context, so a context destroyed and made again (cudaDeviceReset) is looked up anew.
constexpr size_t ATTN_STATIC_FLOATS = (size_t(4) << 20) / sizeof(float);
static __device__ __align__(256) float g_attn_static[ATTN_STATIC_FLOATS];

cudaError_t attn_static_scratch(float** ptr, size_t* nfloats) {
  static std::mutex mu;
  static std::vector<std::pair<unsigned long long, float*>> cache;  // (context id, address)
  static PFN_cuCtxGetCurrent_v4000 get_ctx = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!get_ctx || !get_id) {
    cudaDriverEntryPointQueryResult q1, q2;
    void* f1 = nullptr;
    void* f2 = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess || !f1 || !f2)
      return cudaErrorNotSupported;
    get_ctx = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f1);
    get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f2);
  }
  // the current context's id (unique for the life of the process, unlike its handle)
  auto current_id = [&](unsigned long long* id) -> bool {
    CUcontext cx = nullptr;
    return get_ctx(&cx) == CUDA_SUCCESS && cx && get_id(cx, id) == CUDA_SUCCESS;
  };
  unsigned long long id = 0;
  if (current_id(&id))
    for (auto& c : cache)
      if (c.first == id) {
        *ptr = c.second;
        *nfloats = ATTN_STATIC_FLOATS;
        return cudaSuccess;
      }
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_attn_static);  // also makes the device's context current
  if (e != cudaSuccess) return e;
  if (!current_id(&id)) return cudaErrorInvalidDevice;
  cache.emplace_back(id, static_cast<float*>(p));
  *ptr = static_cast<float*>(p);
  *nfloats = ATTN_STATIC_FLOATS;
  return cudaSuccess;
}

}  // namespace lfm3
