// GQA attention of the LFM3 decoder (16 q heads over 4 kv heads of 128; coreai-model-zoo note
// "lfm3-1.7b-port", diff table rows 2 and 4, and "window_size, with no mask input").
//
// A key at position k is visible to a query at position p iff k <= p and, on sliding layers,
// p - k < 256. Scores are q.k / sqrt(128), softmax in fp32, and the per-head gate sigmoid(g_h)
// multiplies each head's output before o_proj (fused into the epilogues here).
//
// Decode: split-KV. Block (split, kv head, stream) stages its key range (up to 128 keys) of K and
// V in shared memory with asynchronous copies, scores it for the 4 query heads of the group and
// writes unnormalised (max, sum, o) partials; the merge kernel combines splits, applies the gate
// and writes bf16 o. Full layers read keys through the page table (64
// positions per page); sliding layers read the 256-slot ring (slot = position % 256).
//
// Prefill: flash attention on the tensor cores (m16n8k16), one block per (32 query rows, kv
// head): 8 warps = 4 heads x 2 row groups share every K/V tile staged in shared memory.
#include <mutex>

#include "kernels.cuh"

namespace lfm3 {

constexpr int DEC_SPLIT = DEC_KEYS_FULL;       // two 64-position pages
constexpr int DEC_SPLIT_RING = DEC_KEYS_RING;
constexpr int DEC_SMEM = 2 * DEC_SPLIT * HD * 2;  // K and V tiles, bf16

// 16-byte chunk c of key row r in a K tile: rotated by the row so that one key per thread reads
// distinct banks.
DEVI int krot(int r, int c) { return r * HD + ((c + r) & 15) * 8; }

__global__ void __launch_bounds__(128) k_attn_decode(const bf16* __restrict__ q, Rows rows, AttnLayer L, int splits,
                                                     float* __restrict__ part) {
  extern __shared__ __align__(16) unsigned char dsm[];
  bf16* ks = reinterpret_cast<bf16*>(dsm);
  bf16* vs = ks + DEC_SPLIT * HD;
  __shared__ float qs[GQA][HD];
  __shared__ float sc[GQA][DEC_SPLIT];
  __shared__ float ored[2][GQA][HD];
  __shared__ float ml[GQA][2];
  pdl_wait();
  pdl_launch_dependents();
  const int sp = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slot = rows.slot[b], pos = rows.pos[b];
  const int span = L.full ? DEC_SPLIT : DEC_SPLIT_RING;
  const int nkeys = L.full ? pos + 1 : min(pos + 1, WIN);  // ring: slots 0..nkeys-1 are live
  const int j0 = sp * span, j1 = min(nkeys, j0 + span), cnt = j1 - j0;
  float* out = part + (((size_t)b * HQ + kvh * GQA) * splits + sp) * (HD + 2);
  if (cnt <= 0) {  // empty split
    for (int e = tid; e < GQA * (HD + 2); e += blockDim.x) {
      const int h = e / (HD + 2), k = e % (HD + 2);
      out[(size_t)h * splits * (HD + 2) + k] = (k == HD) ? -INFINITY : 0.f;
    }
    return;
  }
  // stage the split's keys and values: cnt rows x 16 chunks of 16 B each, all in flight at once
  auto row_ptr = [&](const bf16* base, int j) -> const bf16* {
    if (L.full) {
      const int page = L.page_table[(size_t)slot * L.max_pages + j / PAGE];
      return base + (((size_t)page * HKV + kvh) * PAGE + j % PAGE) * HD;
    }
    return base + (((size_t)slot * HKV + kvh) * WIN + j) * HD;
  };
  for (int e = tid; e < cnt * 16; e += blockDim.x) {
    const int r = e >> 4, c = e & 15;
    const uint32_t kd = (uint32_t)__cvta_generic_to_shared(ks + krot(r, c));
    const uint32_t vd = (uint32_t)__cvta_generic_to_shared(vs + r * HD + c * 8);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(kd), "l"(row_ptr(L.k, j0 + r) + c * 8));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(vd), "l"(row_ptr(L.v, j0 + r) + c * 8));
  }
  asm volatile("cp.async.commit_group;");
  const float scale = rsqrtf((float)HD);
  for (int e = tid; e < GQA * HD; e += blockDim.x)
    qs[e / HD][e % HD] = bf2f(q[((size_t)b * HQ + kvh * GQA + e / HD) * HD + e % HD]) * scale;
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  // scores: one key per thread (span <= 128)
  if (tid < cnt) {
    float s[GQA] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int c = 0; c < 16; ++c) {
      const uint4 w = *reinterpret_cast<const uint4*>(ks + krot(tid, c));
      const float kv[8] = {bflo(w.x), bfhi(w.x), bflo(w.y), bfhi(w.y), bflo(w.z), bfhi(w.z), bflo(w.w), bfhi(w.w)};
#pragma unroll
      for (int h = 0; h < GQA; ++h)
#pragma unroll
        for (int e = 0; e < 8; ++e) s[h] += qs[h][c * 8 + e] * kv[e];
    }
#pragma unroll
    for (int h = 0; h < GQA; ++h) sc[h][tid] = s[h];
  }
  __syncthreads();
  {
    const int h = warp;
    float m = -INFINITY;
    for (int j = lane; j < cnt; j += 32) m = fmaxf(m, sc[h][j]);
    m = warp_max(m);
    float l = 0.f;
    for (int j = lane; j < cnt; j += 32) {
      const float p = __expf(sc[h][j] - m);
      sc[h][j] = p;
      l += p;
    }
    l = warp_sum(l);
    if (lane == 0) { ml[h][0] = m; ml[h][1] = l; }
  }
  __syncthreads();
  {
    const int par = tid >> 6, dp = (tid & 63) * 2;
    float o[GQA][2] = {};
#pragma unroll 4
    for (int j = par; j < cnt; j += 2) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(vs + j * HD + dp);
      const float v0 = bflo(w), v1 = bfhi(w);
#pragma unroll
      for (int h = 0; h < GQA; ++h) {
        const float p = sc[h][j];
        o[h][0] += p * v0;
        o[h][1] += p * v1;
      }
    }
#pragma unroll
    for (int h = 0; h < GQA; ++h) { ored[par][h][dp] = o[h][0]; ored[par][h][dp + 1] = o[h][1]; }
  }
  __syncthreads();
  for (int e = tid; e < GQA * HD; e += blockDim.x) {
    const int h = e / HD, d = e % HD;
    out[(size_t)h * splits * (HD + 2) + d] = ored[0][h][d] + ored[1][h][d];
  }
  if (tid < GQA) {
    out[(size_t)tid * splits * (HD + 2) + HD] = ml[tid][0];
    out[(size_t)tid * splits * (HD + 2) + HD + 1] = ml[tid][1];
  }
}

// Combine splits, divide, gate: y[b][h*128 + d] = bf16(sigmoid(g[b][h]) * o).
__global__ void __launch_bounds__(128) k_attn_merge(const float* __restrict__ part, int splits,
                                                    const float* __restrict__ gate, bf16* __restrict__ y) {
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x, h = blockIdx.y, d = threadIdx.x;
  const float* p = part + ((size_t)b * HQ + h) * splits * (HD + 2);
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, p[(size_t)s * (HD + 2) + HD]);
  float l = 0.f, o = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float ms = p[(size_t)s * (HD + 2) + HD];
    if (ms == -INFINITY) continue;
    const float f = __expf(ms - M);
    l += f * p[(size_t)s * (HD + 2) + HD + 1];
    o += f * p[(size_t)s * (HD + 2) + d];
  }
  const float gt = sigmoidf_(gate[b * HQ + h]);
  y[(size_t)b * HQ * HD + h * HD + d] = f2bf(gt * (o / l));
}

// Fixed scratch for callers that cannot allocate device memory (lfm3_decode_step_noalloc): 4 MiB
// of split-KV partials, one copy per GPU that loads the library, kept until the process exits.
// Host code never names the array directly: the symbol is a host-side stand-in, so its device
// address is looked up once per device (with that device current) and passed to the kernels.
constexpr size_t ATTN_STATIC_FLOATS = (size_t(4) << 20) / sizeof(float);
static __device__ __align__(256) float g_attn_static[ATTN_STATIC_FLOATS];

cudaError_t attn_static_scratch(float** ptr, size_t* nfloats) {
  static std::mutex mu;
  static float* addr[128] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attn_static);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<float*>(p);
  }
  *ptr = addr[dev];
  *nfloats = ATTN_STATIC_FLOATS;
  return cudaSuccess;
}

cudaError_t attn_decode(const bf16* q, Rows rows, AttnLayer L, int splits, float* part, const float* gate, bf16* y,
                        cudaStream_t s) {
  cudaError_t e = launch(k_attn_decode, dim3(splits, HKV, rows.n), dim3(128), DEC_SMEM, s, q, rows, L, splits, part);
  if (e != cudaSuccess) return e;
  return launch(k_attn_merge, dim3(rows.n, HQ), dim3(HD), 0, s, part, splits, gate, y);
}

// ------------------------------------------------------------------------------------------ decode, one kernel
// Decode attention of one layer in one launch, from the raw q|k|v|gate projection (fp32, one row
// per stream): block (split, kv head, stream) normalises and rotates its four query heads and
// the head's new key (RMS over the head, gain, rotary pairs (i, i + 64), bf16) and rounds the
// new value; it scores its key range with the new key and value standing in for the current
// position's cache row, which the block holding that position also writes. The cached rows are
// staged before the block waits for the projection kernel (they do not depend on it). The last
// block of a (stream, kv head) to finish - counted with an atomic - merges the splits, applies
// the sigmoid gate and writes the bf16 output, then resets the count for the next layer.
__global__ void __launch_bounds__(128) k_attn_decode_fused(const float* __restrict__ qkvg, Rows rows, AttnLayer L,
                                                           AttnDecodeArgs A, int splits, float* __restrict__ part,
                                                           bf16* __restrict__ y) {
  extern __shared__ __align__(16) unsigned char dsm[];
  bf16* ks = reinterpret_cast<bf16*>(dsm);
  bf16* vs = ks + DEC_SPLIT * HD;
  __shared__ float qs[GQA][HD];
  __shared__ float kn[HD], vn[HD];
  __shared__ float sc[GQA][DEC_SPLIT];
  __shared__ float ored[2][GQA][HD];
  __shared__ float ml[GQA][2];
  __shared__ float red[GQA + 1][4];
  __shared__ int last;
  const int sp = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slot = rows.slot[b], pos = rows.pos[b];
  const int span = L.full ? DEC_SPLIT : DEC_SPLIT_RING;
  const int nkeys = L.full ? pos + 1 : min(pos + 1, WIN);  // ring: slots 0..nkeys-1 are live
  const int cur = L.full ? pos : pos % WIN;                 // index of the current position's key
  const int j0 = sp * span, j1 = min(nkeys, j0 + span), cnt = j1 - j0;
  auto row_ptr = [&](const bf16* base, int j) -> const bf16* {
    if (L.full) {
      const int page = L.page_table[(size_t)slot * L.max_pages + j / PAGE];
      return base + (((size_t)page * HKV + kvh) * PAGE + j % PAGE) * HD;
    }
    return base + (((size_t)slot * HKV + kvh) * WIN + j) * HD;
  };
  // ---- stage the split's keys / values: whole 64-position blocks, each contiguous in the pool
  // (a page of one kv head) or the ring, one bulk copy per block for K and one for V. Rows past
  // the visible keys and the current position's stale row come along and are never used.
  __shared__ __align__(8) uint64_t kv_bar;
  const int nblk = cnt > 0 ? (cnt + 63) / 64 : 0;
  if (tid == 0) {
    mbar_init(su32(&kv_bar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (nblk) {
      mbar_expect_tx(su32(&kv_bar), (uint32_t)nblk * 2 * 64 * HD * 2);
      for (int i = 0; i < nblk; ++i) {
        bulk_g2s(su32(ks + i * 64 * HD), row_ptr(L.k, j0 + 64 * i), 64 * HD * 2, su32(&kv_bar));
        bulk_g2s(su32(vs + i * 64 * HD), row_ptr(L.v, j0 + 64 * i), 64 * HD * 2, su32(&kv_bar));
      }
    }
  }
  // gains and rotary coefficients of this thread's dimension d = tid are weights too
  const int d = tid, pd = d < 64 ? d + 64 : d - 64, ir = d & 63;
  const float gq = bf2f(A.q_norm[d]), gk = bf2f(A.k_norm[d]);
  const float cr = A.rope_cos[(size_t)pos * (HD / 2) + ir], sr = A.rope_sin[(size_t)pos * (HD / 2) + ir];
  pdl_wait();
  pdl_launch_dependents();
  // ---- queries and the new key / value: thread = dimension d of each of the 4 heads
  const float* raw = qkvg + (size_t)b * NQKVG;
  float qv[GQA], s2[GQA + 1];
#pragma unroll
  for (int hh = 0; hh < GQA; ++hh) {
    qv[hh] = raw[(kvh * GQA + hh) * HD + d];
    s2[hh] = warp_sum(qv[hh] * qv[hh]);
  }
  const float kv = raw[HQ * HD + kvh * HD + d];
  const float vv = raw[HQ * HD + HKV * HD + kvh * HD + d];
  s2[GQA] = warp_sum(kv * kv);
  if (lane == 0)
#pragma unroll
    for (int hh = 0; hh <= GQA; ++hh) red[hh][warp] = s2[hh];
  __syncthreads();
#pragma unroll
  for (int hh = 0; hh < GQA; ++hh) {
    const float inv = rsqrtf((red[hh][0] + red[hh][1] + red[hh][2] + red[hh][3]) * (1.0f / HD) + A.eps);
    qs[hh][d] = gq * (qv[hh] * inv);
  }
  kn[d] = gk * (kv * rsqrtf((red[GQA][0] + red[GQA][1] + red[GQA][2] + red[GQA][3]) * (1.0f / HD) + A.eps));
  vn[d] = round_bf(vv);
  __syncthreads();
  const float scale = rsqrtf((float)HD);
  float qr[GQA];
#pragma unroll
  for (int hh = 0; hh < GQA; ++hh) qr[hh] = d < 64 ? qs[hh][d] * cr - qs[hh][pd] * sr : qs[hh][d] * cr + qs[hh][pd] * sr;
  const float kr = d < 64 ? kn[d] * cr - kn[pd] * sr : kn[d] * cr + kn[pd] * sr;
  __syncthreads();
#pragma unroll
  for (int hh = 0; hh < GQA; ++hh) qs[hh][d] = round_bf(qr[hh]) * scale;
  kn[d] = round_bf(kr);
  const bool has_cur = cur >= j0 && cur < j1;
  if (has_cur) {  // the new key and value into the cache (bf16, as every later step reads them)
    bf16* kd = const_cast<bf16*>(row_ptr(L.k, cur));
    bf16* vd = const_cast<bf16*>(row_ptr(L.v, cur));
    kd[d] = f2bf(kn[d]);
    vd[d] = f2bf(vn[d]);
  }
  __syncthreads();  // also orders the barrier's initialisation before every thread's wait
  if (nblk && !mbar_wait(su32(&kv_bar), 0, A.err)) {
    // a copy that never lands: report through the status word, drop this block's partial
    asm volatile("" ::: "memory");
  }
  float* out = part + (((size_t)b * HQ + kvh * GQA) * splits + sp) * (HD + 2);
  if (cnt > 0) {
    // scores: one key per thread (span <= 128)
    if (tid < cnt) {
      float s[GQA] = {0.f, 0.f, 0.f, 0.f};
      if (j0 + tid == cur) {
        for (int c = 0; c < HD; ++c)
#pragma unroll
          for (int hh = 0; hh < GQA; ++hh) s[hh] += qs[hh][c] * kn[c];
      } else {
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
          // rows are 256 B apart: rotating the chunk order by the key spreads a warp's reads over all
          // banks (and the q chunks it needs over 8 broadcast groups)
          const int ch = (c + tid) & 15;
          const uint4 w = *reinterpret_cast<const uint4*>(ks + tid * HD + ch * 8);
          const float k8[8] = {bflo(w.x), bfhi(w.x), bflo(w.y), bfhi(w.y), bflo(w.z), bfhi(w.z), bflo(w.w), bfhi(w.w)};
#pragma unroll
          for (int hh = 0; hh < GQA; ++hh)
#pragma unroll
            for (int e = 0; e < 8; ++e) s[hh] += qs[hh][ch * 8 + e] * k8[e];
        }
      }
#pragma unroll
      for (int hh = 0; hh < GQA; ++hh) sc[hh][tid] = s[hh];
    }
    __syncthreads();
    {
      const int hh = warp;
      float mx = -INFINITY;
      for (int j = lane; j < cnt; j += 32) mx = fmaxf(mx, sc[hh][j]);
      mx = warp_max(mx);
      float l = 0.f;
      for (int j = lane; j < cnt; j += 32) {
        const float p = __expf(sc[hh][j] - mx);
        sc[hh][j] = p;
        l += p;
      }
      l = warp_sum(l);
      if (lane == 0) { ml[hh][0] = mx; ml[hh][1] = l; }
    }
    __syncthreads();
    {
      const int par = tid >> 6, dp = (tid & 63) * 2;
      float o[GQA][2] = {};
#pragma unroll 4
      for (int j = par; j < cnt; j += 2) {
        float v0, v1;
        if (j0 + j == cur) {
          v0 = vn[dp];
          v1 = vn[dp + 1];
        } else {
          const uint32_t w = *reinterpret_cast<const uint32_t*>(vs + j * HD + dp);
          v0 = bflo(w);
          v1 = bfhi(w);
        }
#pragma unroll
        for (int hh = 0; hh < GQA; ++hh) {
          const float p = sc[hh][j];
          o[hh][0] += p * v0;
          o[hh][1] += p * v1;
        }
      }
#pragma unroll
      for (int hh = 0; hh < GQA; ++hh) { ored[par][hh][dp] = o[hh][0]; ored[par][hh][dp + 1] = o[hh][1]; }
    }
    __syncthreads();
    for (int e = tid; e < GQA * HD; e += blockDim.x) {
      const int hh = e / HD, dd = e % HD;
      out[(size_t)hh * splits * (HD + 2) + dd] = ored[0][hh][dd] + ored[1][hh][dd];
    }
    if (tid < GQA) {
      out[(size_t)tid * splits * (HD + 2) + HD] = ml[tid][0];
      out[(size_t)tid * splits * (HD + 2) + HD + 1] = ml[tid][1];
    }
  } else {  // empty split
    for (int e = tid; e < GQA * (HD + 2); e += blockDim.x) {
      const int hh = e / (HD + 2), k = e % (HD + 2);
      out[(size_t)hh * splits * (HD + 2) + k] = (k == HD) ? -INFINITY : 0.f;
    }
  }
  // ---- the last block of (stream, kv head) merges the splits and applies the gates
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    unsigned* ctr = A.counters + b * HKV + kvh;
    last = atomicAdd(ctr, 1u) == (unsigned)(splits - 1);
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int hh = 0; hh < GQA; ++hh) {
    const float* pp = part + ((size_t)b * HQ + kvh * GQA + hh) * splits * (HD + 2);
    float M = -INFINITY, l = 0.f, o = 0.f;
    for (int s = 0; s < splits; ++s) {
      const float* q = pp + (size_t)s * (HD + 2);
      const float ms = __ldcg(q + HD), ls = __ldcg(q + HD + 1), os = __ldcg(q + d);
      if (ms == -INFINITY) continue;
      const float Mn = fmaxf(M, ms);
      const float fo = __expf(M - Mn), fs = __expf(ms - Mn);
      l = l * fo + ls * fs;
      o = o * fo + os * fs;
      M = Mn;
    }
    const float gt = sigmoidf_(raw[HQ * HD + 2 * HKV * HD + kvh * GQA + hh]);
    y[(size_t)b * HQ * HD + (kvh * GQA + hh) * HD + d] = f2bf(gt * (o / l));
  }
  if (tid == 0) A.counters[b * HKV + kvh] = 0u;
}

cudaError_t attn_decode_fused(const float* qkvg, Rows rows, AttnLayer L, const AttnDecodeArgs& A, int splits,
                              float* part, bf16* y, cudaStream_t s) {
  return launch(k_attn_decode_fused, dim3(splits, HKV, rows.n), dim3(128), DEC_SMEM, s, qkvg, rows, L, A, splits, part,
                y);
}

// ------------------------------------------------------------------------------------------ prefill
constexpr int PA_ROWS = 32;        // query rows per block
constexpr int PA_KT = 64;          // keys per tile
constexpr int PA_THREADS = 256;    // 8 warps
constexpr int PA_TILE_BYTES = PA_KT * HD * 2;   // 16 KB per K or V tile

DEVI uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// 16-byte chunk c (0..15) of row r in a [64][128] bf16 tile, XOR-swizzled against bank conflicts.
DEVI uint32_t tile_off(int r, int c) { return (uint32_t)(r * 256 + ((c ^ (r & 7)) << 4)); }

DEVI void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0));
}
DEVI void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
DEVI void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N)); }

DEVI void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
DEVI void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

struct PrefillArgs {
  const bf16* q;     // [n][HQ][HD]
  int n, p0, slot;
  AttnLayer L;
  const bf16* sk; const bf16* sv; int scratch_rows;
  const float* gate; // [n][HQ]
  bf16* y;           // [n][HQ*HD]
};

__global__ void __launch_bounds__(PA_THREADS) k_attn_prefill(const PrefillArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int kvh = blockIdx.y;
  const int h = kvh * GQA + (warp & 3);
  const int r0 = blockIdx.x * PA_ROWS + (warp >> 2) * 16;   // this warp's first row
  const int rb0 = blockIdx.x * PA_ROWS;                    // block's first row
  const int rb1 = min(a.n, rb0 + PA_ROWS) - 1;             // block's last row
  const bool full = a.L.full;
  // key index space: full -> positions; sliding -> scratch index i (position p0 - WIN + i)
  const int koff = full ? 0 : a.p0 - WIN;
  const int qpos_lo = a.p0 + rb0, qpos_hi = a.p0 + rb1;
  int klo = full ? 0 : max(0, qpos_lo - (WIN - 1)) - koff;
  const int khi = qpos_hi - koff;                          // last index needed (inclusive)
  const int kmax_valid = a.p0 + a.n - 1 - koff;            // last written key
  klo = (klo / PA_KT) * PA_KT;
  const int ntiles = (khi - klo) / PA_KT + 1;

  // Q fragments (16 rows x 128 dims): 8 k-steps x 4 regs
  uint32_t qf[8][4];
  {
    const int ra = r0 + g, rbb = r0 + g + 8;
    const bool va = ra < a.n, vb = rbb < a.n;
    const bf16* qa = a.q + ((size_t)(va ? ra : 0) * HQ + h) * HD;
    const bf16* qb = a.q + ((size_t)(vb ? rbb : 0) * HQ + h) * HD;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qf[ks][0] = va ? *reinterpret_cast<const uint32_t*>(qa + ks * 16 + 2 * t) : 0u;
      qf[ks][1] = vb ? *reinterpret_cast<const uint32_t*>(qb + ks * 16 + 2 * t) : 0u;
      qf[ks][2] = va ? *reinterpret_cast<const uint32_t*>(qa + ks * 16 + 8 + 2 * t) : 0u;
      qf[ks][3] = vb ? *reinterpret_cast<const uint32_t*>(qb + ks * 16 + 8 + 2 * t) : 0u;
    }
  }
  const float sl2 = rsqrtf((float)HD) * 1.4426950408889634f;  // scale * log2(e)
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  const int qp0 = a.p0 + r0 + g, qp1 = qp0 + 8;  // query positions of this lane's two rows

  auto issue_tile = [&](int it, int buf) {
    const int kt0 = klo + it * PA_KT;
    unsigned char* kb = smem + buf * 2 * PA_TILE_BYTES;
    unsigned char* vb = kb + PA_TILE_BYTES;
    const bf16 *ksrc, *vsrc;
    if (full) {
      const int page = a.L.page_table[(size_t)a.slot * a.L.max_pages + kt0 / PAGE];
      const size_t off = ((size_t)page * HKV + kvh) * PAGE * HD;
      ksrc = a.L.k + off;
      vsrc = a.L.v + off;
    } else {
      const size_t off = ((size_t)kvh * a.scratch_rows + kt0) * HD;
      ksrc = a.sk + off;
      vsrc = a.sv + off;
    }
    // 64 rows x 16 chunks = 1024 chunks per tensor; 4 per thread each
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int idx = tid + e * PA_THREADS, r = idx >> 4, c = idx & 15;
      const bool valid = kt0 + r <= kmax_valid;
      const size_t so = valid ? (size_t)r * HD + c * 8 : 0;
      cp_async16(smem_u32(kb) + tile_off(r, c), ksrc + so, valid);
      cp_async16(smem_u32(vb) + tile_off(r, c), vsrc + so, valid);
    }
    cp_async_commit();
  };

  issue_tile(0, 0);
  for (int it = 0; it < ntiles; ++it) {
    const int buf = it & 1;
    if (it + 1 < ntiles) {
      issue_tile(it + 1, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t kb = smem_u32(smem + buf * 2 * PA_TILE_BYTES);
    const uint32_t vb = kb + PA_TILE_BYTES;
    const int kt0 = klo + it * PA_KT;
    // S = Q K^T : 16 x 64
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int ks = 0; ks < 8; ks += 2) {
        const int m = lane >> 3;  // matrix: (ks, lo), (ks, hi), (ks+1, lo), (ks+1, hi)
        const int r = nt * 8 + (lane & 7);
        const int c = (ks + (m >> 1)) * 2 + (m & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + tile_off(r, c), b0, b1, b2, b3);
        mma_bf16_16816(s[nt], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b0, b1);
        mma_bf16_16816(s[nt], qf[ks + 1][0], qf[ks + 1][1], qf[ks + 1][2], qf[ks + 1][3], b2, b3);
      }
    }
    // mask + online softmax (rows g and g+8 of this warp)
    float mnew[2] = {mrow[0], mrow[1]};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int kp = kt0 + nt * 8 + 2 * t + (j & 1) + koff;   // key position
        const int qp = (j < 2) ? qp0 : qp1;
        bool ok = kp <= qp && kp >= 0;
        if (!full) ok = ok && (qp - kp < WIN);
        s[nt][j] = ok ? s[nt][j] * sl2 : -INFINITY;
        mnew[j >> 1] = fmaxf(mnew[j >> 1], s[nt][j]);
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mnew[i] = fmaxf(mnew[i], __shfl_xor_sync(0xffffffffu, mnew[i], 1));
      mnew[i] = fmaxf(mnew[i], __shfl_xor_sync(0xffffffffu, mnew[i], 2));
    }
    float alpha[2], mu[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mu[i] = mnew[i] == -INFINITY ? 0.f : mnew[i];
      alpha[i] = exp2f(mrow[i] - mu[i]);
      mrow[i] = mnew[i];
    }
    float lsum[2] = {0.f, 0.f};
    uint32_t pf[4][4];  // P as A fragments: 4 k-steps of 16 keys
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p0 = exp2f(s[nt][0] - mu[0]), p1 = exp2f(s[nt][1] - mu[0]);
      const float p2 = exp2f(s[nt][2] - mu[1]), p3 = exp2f(s[nt][3] - mu[1]);
      lsum[0] += p0 + p1;
      lsum[1] += p2 + p3;
      const int kk = nt >> 1;
      if ((nt & 1) == 0) {
        pf[kk][0] = pack_bf2(p0, p1);
        pf[kk][1] = pack_bf2(p2, p3);
      } else {
        pf[kk][2] = pack_bf2(p0, p1);
        pf[kk][3] = pack_bf2(p2, p3);
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      lsum[i] += __shfl_xor_sync(0xffffffffu, lsum[i], 1);
      lsum[i] += __shfl_xor_sync(0xffffffffu, lsum[i], 2);
      lrow[i] = lrow[i] * alpha[i] + lsum[i];
    }
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      o[dt][0] *= alpha[0]; o[dt][1] *= alpha[0];
      o[dt][2] *= alpha[1]; o[dt][3] *= alpha[1];
    }
    // O += P V : V tile [64 keys][128 dims], B fragments via transposed ldmatrix
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int dt = 0; dt < 16; dt += 2) {
        const int m = lane >> 3;  // (keys lo, dt), (keys hi, dt), (keys lo, dt+1), (keys hi, dt+1)
        const int r = kk * 16 + (m & 1) * 8 + (lane & 7);
        const int c = dt + (m >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + tile_off(r, c), b0, b1, b2, b3);
        mma_bf16_16816(o[dt], pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3], b0, b1);
        mma_bf16_16816(o[dt + 1], pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3], b2, b3);
      }
    }
    __syncthreads();
  }
  // epilogue: divide, gate, store bf16
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = r0 + g + 8 * i;
    if (r >= a.n) continue;
    const float gt = sigmoidf_(a.gate[r * HQ + h]) / lrow[i];
    bf16* dst = a.y + (size_t)r * HQ * HD + h * HD;
#pragma unroll
    for (int dt = 0; dt < 16; ++dt)
      *reinterpret_cast<uint32_t*>(dst + dt * 8 + 2 * t) = pack_bf2(o[dt][2 * i] * gt, o[dt][2 * i + 1] * gt);
  }
}

cudaError_t attn_prefill(const bf16* q, int n, int p0, int slot, AttnLayer L, const bf16* sk, const bf16* sv,
                         int scratch_rows, const float* gate, bf16* y, cudaStream_t s) {
  PrefillArgs a{q, n, p0, slot, L, sk, sv, scratch_rows, gate, y};
  const size_t sm = 4 * PA_TILE_BYTES;
  return launch(k_attn_prefill, dim3((n + PA_ROWS - 1) / PA_ROWS, HKV), dim3(PA_THREADS), sm, s, a);
}

cudaError_t attn_init() {
  cudaError_t e = cudaFuncSetAttribute(k_attn_decode, cudaFuncAttributeMaxDynamicSharedMemorySize, DEC_SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_attn_decode_fused, cudaFuncAttributeMaxDynamicSharedMemorySize, DEC_SMEM);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(k_attn_prefill, cudaFuncAttributeMaxDynamicSharedMemorySize, 4 * PA_TILE_BYTES);
}

}  // namespace lfm3
