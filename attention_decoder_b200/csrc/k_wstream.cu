// Decode-time projections, weight-streaming: y[b][n] = sum_k x[b][k] W[n][k] for up to 16 streams.
//
// Decode is bound by reading each weight once from HBM, so this kernel is a pipeline built around
// that stream. Persistent blocks (about two per SM) each own a K range (blockIdx.y) and walk a
// strided list of row tiles. One producer warp copies the tiles' weight rows into a padded ring of
// shared-memory stages with 1-D bulk asynchronous copies (cp.async.bulk + mbarrier transaction
// counts), starting before the block waits for the previous kernel - the weights do not depend on
// it - so each launch's first stages are already in flight when its inputs become ready. Eight
// consumer warps read 16-byte slices of the rows and feed them to the tensor cores as the 16-row A
// operand of m16n8k16 MMAs whose 8 columns are the streams (the activations are read with the same
// K permutation). Per-warp partial sums are reduced in shared memory per tile, then:
//   PARTIAL - fp32 partial sums of this K range (the consumer adds the ranges)
//   SWIGLU  - rows j of w1 and w3 in one tile: u = silu(w1 x) * (w3 x), bf16
//   CONV    - rows c of B, C and x of in_proj (three tiles), then the gated 7-tap conv over the
//             stream's carried columns and the state shift
//   HEAD    - tied-head logits and a running greedy argmax per stream
// Prologue: the activations come either as bf16 rows (LOAD) or from the fp32 residual stream
// (NORM): the block adds the previous projection's K-range partials through the post-norm
// (x' = x + g_post * RMS(sum parts)), normalises (bf16(g_next * RMS(x'))) and keeps its K range
// in shared memory; block (0, 0) writes x' to the other residual buffer (and the hidden dump), so
// no block ever reads a residual another block is rewriting.
// NVFP4 weights (E2M1 codes + E4M3 block scales) are expanded to exact bf16 values through a
// byte -> bf16x2 table in shared memory (one copy per bank, so lookups never conflict) and a bf16
// multiply by the block scale (exact: at most 6 significant bits); the fp32 tensor scale
// multiplies the finished sums.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "kernels.cuh"

// Ring depths (stages) and blocks per SM; compile-time, measured on B200.
#ifndef LFM3_WS_STAGES_BF16
#define LFM3_WS_STAGES_BF16 5
#endif
#ifndef LFM3_WS_STAGES_CONV
#define LFM3_WS_STAGES_CONV 5
#endif
#ifndef LFM3_WS_STAGES_FP4
#define LFM3_WS_STAGES_FP4 12
#endif
#ifndef LFM3_WS_BPS
#define LFM3_WS_BPS 2
#endif

namespace lfm3 {

constexpr int WS_CW = 8;                    // consumer warps
constexpr int WS_EPT = D / (WS_CW * 32);      // residual elements per consumer thread in the prologue
constexpr int WS_MAX_PARTS = 5;                // K-split partials the prologue adds at most
// Largest dynamic shared memory a launch asks for (in_proj + conv with 16 streams: ~192 KB).
constexpr int WS_SMEM_MAX = 200 * 1024;
constexpr int WS_THREADS = 32 * (WS_CW + 1);

template <int EPI>
struct WsRows { static constexpr int NRT = (EPI == GEMV_CONV) ? 3 : 1; };

template <int EPI, bool FP4>
struct WsGeom {
  static constexpr int NRT = WsRows<EPI>::NRT;
  static constexpr int RPT = 16 * NRT;                        // weight rows per tile
  static constexpr int BR = EPI == GEMV_SWIGLU ? 8 : 16;      // rows per copy request (w1 | w3 halves)
  static constexpr int NREQ = RPT / BR;                       // copy requests per stage
  static constexpr int KBLK = FP4 ? 128 : 32;                 // K per 64-byte block of a row
  // K per lane step: a bf16 step reads 16 B of a row per lane; an NVFP4 step reads 8 B (16 codes,
  // one E4M3 block), so that a stage has 8 steps and every consumer warp has one
  static constexpr int KSTEP = FP4 ? 64 : 32;
  static constexpr int KCH = FP4 ? 512 : (NRT == 3 ? 256 : 512);  // K per stage
  static constexpr int NKB = KCH / KBLK;                      // 64-byte blocks per row per stage
  static constexpr int REQB = 64 * BR * NKB;                  // bytes of one request: [block][row][64 B]
  static constexpr int ROWB = 64 * NKB;                       // weight bytes per row per stage
  static constexpr int SCB = FP4 ? KCH / 16 : 0;              // scale bytes per row per stage
  static constexpr int STAGES = FP4 ? LFM3_WS_STAGES_FP4 : (NRT == 3 ? LFM3_WS_STAGES_CONV : LFM3_WS_STAGES_BF16);
  static constexpr int STAGE_BYTES = RPT * ROWB + RPT * SCB;
  static constexpr int TX_BYTES = STAGE_BYTES;
  static constexpr int STEPS = KCH / KSTEP;                   // lane steps per stage
};

// Byte offset, inside a stage, of what lane chunk t reads from row r at step j: 16 bytes of the
// j-th 64-byte block (bf16), or 8 bytes of the (j / 2)-th block's half j % 2 (NVFP4).
template <class G, bool FP4>
DEVI int ws_woff(int r, int j, int t) {
  if constexpr (FP4)
    return (r / G::BR) * G::REQB + (j >> 1) * (G::BR * 64) + (r % G::BR) * 64 + (j & 1) * 32 + t * 8;
  else
    return (r / G::BR) * G::REQB + j * (G::BR * 64) + (r % G::BR) * 64 + t * 16;
}

// Row of tile `tile`, sub-tile rt, fragment row g (0..15); `which` selects w3 for SwiGLU.
template <int EPI>
DEVI int ws_row(int tile, int rt, int g, int& which) {
  which = 0;
  if constexpr (EPI == GEMV_SWIGLU) {
    which = g >= 8;
    return tile * 8 + (g & 7);
  } else if constexpr (EPI == GEMV_CONV) {
    return rt * D + tile * 16 + g;
  } else {
    return tile * 16 + g;
  }
}


// Weights are read once per step: their copies carry an evict-first L2 policy, so that the small
// data every kernel reads right after its dependency (residual, partials, gains, keys and values)
// keeps its place in L2.
#ifndef LFM3_WS_EVICT_FIRST
#define LFM3_WS_EVICT_FIRST 1
#endif
DEVI uint64_t ws_policy() {
  uint64_t p = 0;
#if LFM3_WS_EVICT_FIRST
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
#endif
  return p;
}
DEVI void ws_tma3(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar, uint64_t pol) {
#if LFM3_WS_EVICT_FIRST
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, %3, "
      "%4}], [%5], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar), "l"(pol)
      : "memory");
#else
  (void)pol;
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
#endif
}
DEVI void ws_tma2(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar, uint64_t pol) {
#if LFM3_WS_EVICT_FIRST
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
      "%3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(pol)
      : "memory");
#else
  (void)pol;
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
#endif
}

DEVI void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(WS_CW * 32) : "memory"); }

// Activations in shared memory: a 128-byte zero block (the MMA columns of absent streams read
// it), then one row per stream of the block's K range, 64-byte skewed against bank conflicts.
__host__ __device__ inline size_t ws_x_bytes(int rows, int Kc) { return 128 + (size_t)rows * (Kc + 32) * 2; }
// Stages start on a 1024-byte boundary after the activations.
__host__ __device__ inline size_t ws_stage_base(int rows, int Kc) { return (ws_x_bytes(rows, Kc) + 1023) / 1024 * 1024; }

// Consumer prologue of the weight-streaming kernels (consumer threads only): the activations of
// the block's K range into xs, either as given (LOAD) or through the sandwich-norm step (NORM), as
// bf16 - or, with X16, as f16 copies of the same bf16 values (exact for magnitudes in f16's
// normal range, which the normed activations and the SwiGLU products of this model stay in) for
// the NVFP4 kernel's f16 MMAs. Ends with the consumers synchronised.
template <bool X16>
DEVI void ws_prologue(const WsArgs& a, unsigned char* smem, bf16* xs, int XS, int Kc, int kcta, float* redn, unsigned long long* trb, int trid) {
  (void)XS; (void)Kc; (void)trb; (void)trid;
  const int ct = threadIdx.x, warp = ct >> 5, lane = ct & 31;
  // the norm gains are weights: requested before waiting for the previous kernel
  float gp[WS_EPT], gn[WS_EPT];
  if (a.pro == WS_PRO_NORM) {
    const int c0 = ct * WS_EPT;
    const uint4 z4 = make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int h = 0; h < WS_EPT / 8; ++h) {
      const uint4 pw = a.n_parts > 0 ? ldg16(a.g_post + c0 + 8 * h) : z4, nw = ldg16(a.g_next + c0 + 8 * h);
      const uint32_t pv[4] = {pw.x, pw.y, pw.z, pw.w}, nv[4] = {nw.x, nw.y, nw.z, nw.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        gp[8 * h + 2 * j] = bflo(pv[j]); gp[8 * h + 2 * j + 1] = bfhi(pv[j]);
        gn[8 * h + 2 * j] = bflo(nv[j]); gn[8 * h + 2 * j + 1] = bfhi(nv[j]);
      }
    }
  }
  pdl_wait();
  pdl_launch_dependents();
#ifdef LFM3_TRACE
  if (ct == 0) TRACE(trb, trid, 2);
#endif
  if (ct < 8) reinterpret_cast<uint4*>(smem)[ct] = make_uint4(0, 0, 0, 0);
  if (a.pro == WS_PRO_LOAD) {
    const int chunks = Kc / 8;
    for (int idx = ct; idx < a.rows * chunks; idx += WS_CW * 32) {
      const int b = idx / chunks, c = idx - b * chunks;
      uint4 v = ldg16(a.x + (size_t)b * a.K + kcta + c * 8);
      if constexpr (X16) v = make_uint4(bf2_to_h2(v.x), bf2_to_h2(v.y), bf2_to_h2(v.z), bf2_to_h2(v.w));
      *reinterpret_cast<uint4*>(xs + (size_t)b * XS + c * 8) = v;
    }
  } else {
    // residual + post-norm of the previous projection, then this projection's input norm. The
    // gains are requested first (HBM round trips), then each stream's residual and partials; one
    // reduction per stream gives both norms: with a = RMS^-1 of the partials' sum m and the post
    // gain g, x' = x + a g m and sum(x'^2) = sum(x^2) + 2a sum(g x m) + a^2 sum(g^2 m^2).
    const bool writer = blockIdx.x == 0 && blockIdx.y == 0;
    const int c0 = ct * WS_EPT;
    for (int b = 0; b < a.rows; ++b) {
      float x[WS_EPT], m[WS_EPT];
      // the residual and every partial of this thread's columns are requested together (one L2
      // round trip, not one per partial)
      const float4* xin = reinterpret_cast<const float4*>(a.x_in + (size_t)b * D + c0);
      float4 xv[WS_EPT / 4], pv[WS_MAX_PARTS][WS_EPT / 4];
#pragma unroll
      for (int q = 0; q < WS_EPT / 4; ++q) xv[q] = __ldcg(xin + q);
#pragma unroll
      for (int s = 0; s < WS_MAX_PARTS; ++s)
        if (s < a.n_parts) {
          const float4* p = reinterpret_cast<const float4*>(a.parts + s * a.part_stride + (size_t)b * D + c0);
#pragma unroll
          for (int q = 0; q < WS_EPT / 4; ++q) pv[s][q] = __ldcg(p + q);
        }
#pragma unroll
      for (int q = 0; q < WS_EPT / 4; ++q) {
        x[4 * q] = xv[q].x; x[4 * q + 1] = xv[q].y; x[4 * q + 2] = xv[q].z; x[4 * q + 3] = xv[q].w;
        m[4 * q] = m[4 * q + 1] = m[4 * q + 2] = m[4 * q + 3] = 0.f;
      }
#pragma unroll
      for (int s = 0; s < WS_MAX_PARTS; ++s)
        if (s < a.n_parts) {
#pragma unroll
          for (int q = 0; q < WS_EPT / 4; ++q) {
            m[4 * q] += pv[s][q].x; m[4 * q + 1] += pv[s][q].y; m[4 * q + 2] += pv[s][q].z; m[4 * q + 3] += pv[s][q].w;
          }
        }
      float q4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < WS_EPT; ++j) {
        const float gm = gp[j] * m[j];
        q4[0] += m[j] * m[j];
        q4[1] += x[j] * x[j];
        q4[2] += x[j] * gm;
        q4[3] += gm * gm;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) q4[c] = warp_sum(q4[c]);
      if (lane == 0) *reinterpret_cast<float4*>(redn + 4 * warp) = make_float4(q4[0], q4[1], q4[2], q4[3]);
      consumers_sync();
      float t[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int w = 0; w < WS_CW; ++w)
#pragma unroll
        for (int c = 0; c < 4; ++c) t[c] += redn[4 * w + c];
      const float al = a.n_parts > 0 ? rsqrtf(t[0] * (1.0f / D) + a.eps) : 0.f;
      const float inv = rsqrtf(fmaxf(t[1] + 2.f * al * t[2] + al * al * t[3], 0.f) * (1.0f / D) + a.eps);
#pragma unroll
      for (int j = 0; j < WS_EPT; ++j) x[j] += al * (gp[j] * m[j]);
      if (writer) {
        float* xo = a.x_out + (size_t)b * D + c0;
#pragma unroll
        for (int q = 0; q < WS_EPT / 4; ++q) reinterpret_cast<float4*>(xo)[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
        if (a.dump) {
          float* dd = a.dump + (size_t)b * D + c0;
#pragma unroll
          for (int q = 0; q < WS_EPT / 4; ++q)
            reinterpret_cast<float4*>(dd)[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
        }
      }
      // this thread's columns go to shared memory if they are in the block's K range
      if (c0 >= kcta && c0 < kcta + Kc) {
#pragma unroll
        for (int h = 0; h < WS_EPT / 8; ++h) {
          uint32_t w[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int e = 8 * h + 2 * j;
            w[j] = pack_bf2(gn[e] * (x[e] * inv), gn[e + 1] * (x[e + 1] * inv));
            if constexpr (X16) w[j] = bf2_to_h2(w[j]);
          }
          *reinterpret_cast<uint4*>(xs + (size_t)b * XS + (c0 - kcta) + 8 * h) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      consumers_sync();  // redn is reused by the next stream
    }
  }
  consumers_sync();

}

template <int EPI, int NT, bool FP4>
__global__ void __launch_bounds__(WS_THREADS, 2) k_wstream(const __grid_constant__ CUtensorMap tw,
                                                        const __grid_constant__ CUtensorMap tw3,
                                                        const __grid_constant__ CUtensorMap tsc,
                                                        const __grid_constant__ CUtensorMap tsc3, const WsArgs a) {
  static_assert(!FP4, "NVFP4 weights stream through k_wstream_fp4");
  using G = WsGeom<EPI, FP4>;
  constexpr int NRT = G::NRT;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int Kc = a.K / a.splits;
  const int XS = Kc + 32;  // activations row stride (elements): 64-byte skew against bank conflicts
  const bf16* xzero = reinterpret_cast<const bf16*>(smem);
  bf16* xs = reinterpret_cast<bf16*>(smem + 128);
  unsigned char* stages = smem + ws_stage_base(a.rows, Kc);
  const int NS = a.stages;  // ring depth chosen by the launcher
  float* red = reinterpret_cast<float*>(stages + (size_t)NS * G::STAGE_BYTES);
  float* res = red + WS_CW * NRT * NT * 128;
  uint64_t* bars = reinterpret_cast<uint64_t*>(res + NRT * 16 * NT * 8);
  __shared__ __align__(16) float redn[WS_CW * 4];
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kcta = blockIdx.y * Kc;
  const int nch = Kc / G::KCH;
  const int ntiles = (EPI == GEMV_SWIGLU) ? a.N / 8 : (EPI == GEMV_CONV ? D / 16 : a.N / 16);
  const uint32_t full0 = su32(bars), empty0 = su32(bars + NS);

#ifdef LFM3_TRACE
  unsigned long long* const trb = a.trace;
  const int trid = a.trace_id;
  if (tid == 0) {
    TRACE(trb, trid, 0);
    TRACE(trb, trid, 7);
  }
#endif
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, WS_CW);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == WS_CW) {
    // ------------------------------------------------------------ producer
    int it = 0;
    bool ok = true;
    const uint64_t pol = ws_policy();
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      for (int ch = 0; ch < nch && ok; ++ch, ++it) {
        const int s = it % NS;
        const uint32_t ph = (it / NS) & 1;
        if (lane == 0) ok = mbar_wait(empty0 + 8 * s, ph ^ 1, a.err);
        ok = __shfl_sync(0xffffffffu, ok, 0) && !*(volatile int*)&abort_flag;
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(full0 + 8 * s, G::TX_BYTES);
          unsigned char* st = stages + (size_t)s * G::STAGE_BYTES;
          const int k0 = kcta + ch * G::KCH;
#ifdef LFM3_TRACE
          if (it == 0) TRACE(trb, trid, 1);
#endif
#pragma unroll
          for (int q = 0; q < G::NREQ; ++q) {
            int which;
            const int row = ws_row<EPI>(tile, (q * G::BR) / 16, (q * G::BR) % 16, which);
            const CUtensorMap* m = which ? &tw3 : &tw;
            ws_tma3(su32(st + q * G::REQB), m, 0, row, k0 / G::KBLK, full0 + 8 * s, pol);
          }
        }
      }
    }
#ifdef LFM3_TRACE
    if (lane == 0) TRACE(trb, trid, 6);
#endif
    pdl_wait();
    pdl_launch_dependents();
    if (!ok) {
      // drain: copies already issued land before the block exits (bounded)
      for (int k = 0; k < NS && k < it; ++k) {
        const int i = it - 1 - k;
        if (lane == 0) mbar_wait(full0 + 8 * (i % NS), (i / NS) & 1, a.err);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers: prologue
#ifdef LFM3_TRACE
  ws_prologue<FP4>(a, smem, xs, XS, Kc, kcta, redn, trb, trid);
#else
  ws_prologue<FP4>(a, smem, xs, XS, Kc, kcta, redn, nullptr, 0);
#endif
  const int ct = tid;
  // -------------------------------------------------------------- consumers: main loop
#ifdef LFM3_TRACE
  if (ct == 0) TRACE(trb, trid, 3);
#endif
  const int g = lane >> 2, t = lane & 3;
  constexpr int LDR = NT * 8;
  int it = 0;
  bool ok = true;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    float acc[NRT][NT][4];
#pragma unroll
    for (int rt = 0; rt < NRT; ++rt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[rt][nt][j] = 0.f;
    for (int ch = 0; ch < nch; ++ch, ++it) {
      const int s = it % NS;
      const uint32_t ph = (it / NS) & 1;
      // after any bounded wait gives up, every warp keeps walking the same loop (so all of them
      // reach every consumer barrier) but waits for nothing and computes nothing
      if (ok && *(volatile int*)&abort_flag) ok = false;
      if (ok) {
        bool got = true;
        if (lane == 0) got = mbar_wait(full0 + 8 * s, ph, a.err);
#ifdef LFM3_TRACE
        if (it == 0 && ct == 0) TRACE(trb, trid, 4);
#endif
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          ok = false;
          abort_flag = 1;
        }
      }
      if (ok) {
        const unsigned char* st = stages + (size_t)s * G::STAGE_BYTES;
#pragma unroll
        for (int j = warp; j < G::STEPS; j += WS_CW) {
          const int kx = ch * G::KCH + j * G::KSTEP;  // K offset of this step in the block's range
#pragma unroll
          for (int rt = 0; rt < NRT; ++rt) {
            {
              const uint4 wa = *reinterpret_cast<const uint4*>(st + ws_woff<G, FP4>(rt * 16 + g, j, t));
              const uint4 wb = *reinterpret_cast<const uint4*>(st + ws_woff<G, FP4>(rt * 16 + g + 8, j, t));
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                const int sr = nt * 8 + g;
                const uint4 xv = *reinterpret_cast<const uint4*>(sr < a.rows ? xs + (size_t)sr * XS + kx + 8 * t : xzero);
                mma_bf16_16816(acc[rt][nt], wa.x, wb.x, wa.y, wb.y, xv.x, xv.y);
                mma_bf16_16816(acc[rt][nt], wa.z, wb.z, wa.w, wb.w, xv.z, xv.w);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * s);
    }

    // ---------------------------------------------------------- reduce the 4 warps, epilogue
#pragma unroll
    for (int rt = 0; rt < NRT; ++rt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        *reinterpret_cast<float4*>(red + ((((size_t)warp * NRT + rt) * NT + nt) * 32 + lane) * 4) =
            make_float4(acc[rt][nt][0], acc[rt][nt][1], acc[rt][nt][2], acc[rt][nt][3]);
    consumers_sync();
    for (int e = ct; e < NRT * NT * 128; e += WS_CW * 32) {
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < WS_CW; ++w) sum += red[(size_t)w * NRT * NT * 128 + e];
      const int j = e & 3, ln = (e >> 2) & 31, nt = (e >> 7) % NT, rt = (e >> 7) / NT;
      const int row = rt * 16 + (ln >> 2) + (j >= 2 ? 8 : 0);
      const int col = nt * 8 + 2 * (ln & 3) + (j & 1);
      res[row * LDR + col] = FP4 ? sum * a.tscale : sum;
    }
    consumers_sync();
    if (!ok) {
      consumers_sync();
      continue;
    }
    if constexpr (EPI == GEMV_PARTIAL) {
      for (int e = ct; e < 16 * a.rows; e += WS_CW * 32) {
        const int row = e & 15, b = e >> 4;
        a.part_out[((size_t)blockIdx.y * a.rows + b) * a.N + tile * 16 + row] = res[row * LDR + b];
      }
    } else if constexpr (EPI == GEMV_SWIGLU) {
      for (int e = ct; e < 8 * a.rows; e += WS_CW * 32) {
        const int j = e & 7, b = e >> 3;
        const float h1 = res[j * LDR + b], h3 = res[(j + 8) * LDR + b];
        a.out[(size_t)b * a.N + tile * 8 + j] = f2bf(siluf_(h1) * h3);
      }
    } else if constexpr (EPI == GEMV_CONV) {
      for (int e = ct; e < 16 * a.rows; e += WS_CW * 32) {
        const int cl = e & 15, b = e >> 4, c = tile * 16 + cl;
        const float Cv = res[(16 + cl) * LDR + b];
        bf16* stt = a.conv_state + (size_t)a.row_slot[b] * CST * D + c;
        const bf16* w = a.conv_w + (size_t)c * TAPS;
        if (a.win <= 1) {
          const float bx = round_bf(res[cl * LDR + b] * res[(32 + cl) * LDR + b]);
          float win[CST];
#pragma unroll
          for (int j = 0; j < CST; ++j) win[j] = bf2f(stt[(size_t)j * D]);
          float z = 0.f;
#pragma unroll
          for (int k = 0; k < CST; ++k) z += bf2f(w[k]) * win[k];
          z += bf2f(w[CST]) * bx;
          a.y[(size_t)b * D + c] = f2bf(Cv * z);
#pragma unroll
          for (int j = 0; j < CST - 1; ++j) stt[(size_t)j * D] = f2bf(win[j + 1]);
          stt[(size_t)(CST - 1) * D] = f2bf(bx);
        } else {
          // verify window: row wi of its stream sees [state | bx of the window's rows 0..wi]; the
          // state stays as it is and the state after this row goes to the snapshot
          const int wi = b % a.win, b0 = b - wi;
          float wnd[CST + MAX_WIN];
#pragma unroll
          for (int j = 0; j < CST; ++j) wnd[j] = bf2f(stt[(size_t)j * D]);
          for (int i = 0; i <= wi; ++i) wnd[CST + i] = round_bf(res[cl * LDR + b0 + i] * res[(32 + cl) * LDR + b0 + i]);
          float z = 0.f;
#pragma unroll
          for (int k = 0; k < TAPS; ++k) z += bf2f(w[k]) * wnd[wi + k];
          a.y[(size_t)b * D + c] = f2bf(Cv * z);
#pragma unroll
          for (int j = 0; j < CST; ++j) a.conv_snap[((size_t)b * CST + j) * D + c] = f2bf(wnd[wi + 1 + j]);
        }
      }
    } else if constexpr (EPI == GEMV_HEAD) {
      for (int b = warp; b < a.rows; b += WS_CW) {
        const float v = lane < 16 ? res[lane * LDR + b] : -INFINITY;
        const int n = tile * 16 + lane;
        if (lane < 16 && a.logits) a.logits[(size_t)b * a.N + n] = v;
        const float m = warp_max(v);
        const unsigned ballot = __ballot_sync(0xffffffffu, v == m && lane < 16);
        if (lane == 0) {
          const int idx = tile * 16 + (__ffs(ballot) - 1);
          uint32_t u = __float_as_uint(m);
          u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
          atomicMax(a.amax + b, ((unsigned long long)u << 32) | (0xffffffffu - (uint32_t)idx));
        }
      }
    }
    consumers_sync();
  }
#ifdef LFM3_TRACE
  if (ct == 0) TRACE(trb, trid, 5);
#endif
}

// ------------------------------------------------------------------------------------------ NVFP4
// NVFP4 weights (the FFN): a warp owns whole output rows, so partial sums never cross warps per
// tile. A unit is 64 weight rows - 64 rows of the matrix (PARTIAL), or 32 rows of w1 with the same
// 32 rows of w3 (SWIGLU) - over the block's K range. Warp w takes row tile w & 3 (16 rows: for
// SWIGLU rows g of w1 and of w3 sit in MMA rows g and g + 8 of one tile, so SiLU(w1 x) * (w3 x)
// needs nothing from other lanes) and K half w >> 2 of every stage; one reduction of the two K
// halves per unit. A stage is 256 codes of each row (64 rows x 128 B) and their 16 E4M3 scales
// per row; a lane step reads 8 B (16 codes, one scale) of rows g and g + 8, expands each code
// byte to an f16 pair with the hardware E2M1 conversion, multiplies by the block scale (E4M3 ->
// f16, also exact; so is the product: at most 5 significant bits, between 2^-10 and 2688) and
// issues two f16 m16n8k16 MMAs per 8 codes with the streams as the 8 columns. No code table in
// shared memory, so two blocks share an SM.
constexpr int Q4_UR = 64;                        // weight rows per unit
constexpr int Q4_KST = 256;                      // codes per row per stage
constexpr int Q4_CODE_B = Q4_UR * Q4_KST / 2;    // 8 KB
constexpr int Q4_SC_B = Q4_UR * Q4_KST / 16;     // 1 KB
constexpr int Q4_STAGE_B = Q4_CODE_B + Q4_SC_B;
constexpr int Q4_STAGES = 8;

__host__ __device__ inline size_t q4_stage_base(int rows, int Kc) { return ws_stage_base(rows, Kc); }

template <int EPI, int NT>
__global__ void __launch_bounds__(WS_THREADS, 2) k_wstream_fp4(const __grid_constant__ CUtensorMap tw,
                                                               const __grid_constant__ CUtensorMap tw3,
                                                               const __grid_constant__ CUtensorMap tsc,
                                                               const __grid_constant__ CUtensorMap tsc3, const WsArgs a) {
  constexpr bool SW = EPI == GEMV_SWIGLU;
  constexpr int RR = SW ? Q4_UR / 2 : Q4_UR;     // rows per region of a stage (w1 | w3, or all)
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int Kc = a.K / a.splits;
  const int XS = Kc + 32;
  const bf16* xzero = reinterpret_cast<const bf16*>(smem);
  bf16* xs = reinterpret_cast<bf16*>(smem + 128);
  unsigned char* stages = smem + q4_stage_base(a.rows, Kc);
  const int NS = a.stages;
  float* red = reinterpret_cast<float*>(stages + (size_t)NS * Q4_STAGE_B);  // [4 tiles][NT][32 lanes][4]
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 4 * NT * 32 * 4);
  __shared__ __align__(16) float redn[WS_CW * 4];
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kcta = blockIdx.y * Kc;
  const int nst = Kc / Q4_KST;
  const int nunits = a.N / (SW ? Q4_UR / 2 : Q4_UR);
  const uint32_t full0 = su32(bars), empty0 = su32(bars + NS);
#ifdef LFM3_TRACE
  unsigned long long* const trb = a.trace;
  const int trid = a.trace_id;
  if (tid == 0) {
    TRACE(trb, trid, 0);
    TRACE(trb, trid, 7);
  }
#endif
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, WS_CW);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == WS_CW) {
    // ------------------------------------------------------------ producer
    int it = 0;
    bool ok = true;
    const uint64_t pol = ws_policy();
    for (int unit = blockIdx.x; unit < nunits && ok; unit += gridDim.x) {
      for (int st = 0; st < nst && ok; ++st, ++it) {
        const int s = it % NS;
        const uint32_t ph = (it / NS) & 1;
        if (lane == 0) ok = mbar_wait(empty0 + 8 * s, ph ^ 1, a.err);
        ok = __shfl_sync(0xffffffffu, ok, 0) && !*(volatile int*)&abort_flag;
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(full0 + 8 * s, Q4_STAGE_B);
          unsigned char* sb = stages + (size_t)s * Q4_STAGE_B;
          const int k0 = kcta + st * Q4_KST;
#ifdef LFM3_TRACE
          if (it == 0) TRACE(trb, trid, 1);
#endif
          const int row0 = unit * RR;
          ws_tma3(su32(sb), &tw, 0, row0, k0 / 128, full0 + 8 * s, pol);
          ws_tma2(su32(sb + Q4_CODE_B), &tsc, k0 / 16, row0, full0 + 8 * s, pol);
          if constexpr (SW) {
            ws_tma3(su32(sb + Q4_CODE_B / 2), &tw3, 0, row0, k0 / 128, full0 + 8 * s, pol);
            ws_tma2(su32(sb + Q4_CODE_B + Q4_SC_B / 2), &tsc3, k0 / 16, row0, full0 + 8 * s, pol);
          }
        }
      }
    }
#ifdef LFM3_TRACE
    if (lane == 0) TRACE(trb, trid, 6);
#endif
    pdl_wait();
    pdl_launch_dependents();
    if (!ok) {
      for (int k = 0; k < NS && k < it; ++k) {
        const int i = it - 1 - k;
        if (lane == 0) mbar_wait(full0 + 8 * (i % NS), (i / NS) & 1, a.err);
      }
    }
    return;
  }

#ifdef LFM3_TRACE
  ws_prologue<true>(a, smem, xs, XS, Kc, kcta, redn, trb, trid);
  if (tid == 0) TRACE(trb, trid, 3);
#else
  ws_prologue<true>(a, smem, xs, XS, Kc, kcta, redn, nullptr, 0);
#endif

  // -------------------------------------------------------------- consumers: main loop
  const int g = lane >> 2, t = lane & 3;
  const int rt = warp & 3, kh = warp >> 2;
  // stage offsets of MMA rows g and g + 8 of this warp's tile (codes: [block][row][64 B])
  const int ra = SW ? 8 * rt + g : 16 * rt + g;
  const int rb = SW ? 8 * rt + g : 16 * rt + g + 8;
  const int ca = ra * 64 + t * 8, cb = (SW ? Q4_CODE_B / 2 : 0) + rb * 64 + t * 8;
  const int sa = Q4_CODE_B + ra * 16 + t, sbo = Q4_CODE_B + (SW ? Q4_SC_B / 2 : 0) + rb * 16 + t;
  int it = 0;
  bool ok = true;
  for (int unit = blockIdx.x; unit < nunits; unit += gridDim.x) {
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[nt][j] = 0.f;
    for (int st = 0; st < nst; ++st, ++it) {
      const int s = it % NS;
      const uint32_t ph = (it / NS) & 1;
      if (ok && *(volatile int*)&abort_flag) ok = false;
      if (ok) {
        bool got = true;
        if (lane == 0) got = mbar_wait(full0 + 8 * s, ph, a.err);
#ifdef LFM3_TRACE
        if (it == 0 && tid == 0) TRACE(trb, trid, 4);
#endif
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          ok = false;
          abort_flag = 1;
        }
      }
      if (ok) {
        const unsigned char* sb = stages + (size_t)s * Q4_STAGE_B;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int hs = 2 * kh + hh;                   // 64-code step of the stage
          const int off = (hs >> 1) * (RR * 64) + (hs & 1) * 32;
          const uint2 wa = *reinterpret_cast<const uint2*>(sb + ca + off);
          const uint2 wb = *reinterpret_cast<const uint2*>(sb + cb + off);
          const uint32_t sA = e4m3_to_h2(sb[sa + 4 * hs]), sB = e4m3_to_h2(sb[sbo + 4 * hs]);
          const int kx = st * Q4_KST + 64 * hs + 16 * t;  // K offset in the block's range
          const uint32_t wA[2] = {wa.x, wa.y}, wB[2] = {wb.x, wb.y};
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t a01, a23, a45, a67, b01, b23, b45, b67;
            e2m1x8_to_h2(wA[q], a01, a23, a45, a67);
            e2m1x8_to_h2(wB[q], b01, b23, b45, b67);
            a01 = hmul2_u(a01, sA); a23 = hmul2_u(a23, sA); a45 = hmul2_u(a45, sA); a67 = hmul2_u(a67, sA);
            b01 = hmul2_u(b01, sB); b23 = hmul2_u(b23, sB); b45 = hmul2_u(b45, sB); b67 = hmul2_u(b67, sB);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const int sr = nt * 8 + g;
              const uint4 xv = *reinterpret_cast<const uint4*>(sr < a.rows ? xs + (size_t)sr * XS + kx + 8 * q : xzero);
              mma_f16_16816(acc[nt], a01, b01, a23, b23, xv.x, xv.y);
              mma_f16_16816(acc[nt], a45, b45, a67, b67, xv.z, xv.w);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * s);
    }
    // ---------------------------------------------------------- the two K halves, then the rows
    if (kh == 1)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        *reinterpret_cast<float4*>(red + ((rt * NT + nt) * 32 + lane) * 4) =
            make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
    consumers_sync();
    if (kh == 0 && ok) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float4 o = *reinterpret_cast<const float4*>(red + ((rt * NT + nt) * 32 + lane) * 4);
        const float v0 = (acc[nt][0] + o.x) * a.tscale, v1 = (acc[nt][1] + o.y) * a.tscale;
        const float v2 = (acc[nt][2] + o.z) * a.tscale, v3 = (acc[nt][3] + o.w) * a.tscale;
        const int b0 = nt * 8 + 2 * t;  // streams of columns 2t, 2t + 1
        if constexpr (SW) {
          const int j = unit * (Q4_UR / 2) + 8 * rt + g;  // rows g (w1) and g + 8 (w3) of the tile
          if (b0 < a.rows) a.out[(size_t)b0 * a.N + j] = f2bf(siluf_(v0) * v2);
          if (b0 + 1 < a.rows) a.out[(size_t)(b0 + 1) * a.N + j] = f2bf(siluf_(v1) * v3);
        } else {
          const int r0 = unit * Q4_UR + 16 * rt + g;
          float* po = a.part_out + (size_t)blockIdx.y * a.rows * a.N;
          if (b0 < a.rows) {
            po[(size_t)b0 * a.N + r0] = v0;
            po[(size_t)b0 * a.N + r0 + 8] = v2;
          }
          if (b0 + 1 < a.rows) {
            po[(size_t)(b0 + 1) * a.N + r0] = v1;
            po[(size_t)(b0 + 1) * a.N + r0 + 8] = v3;
          }
        }
      }
    }
    consumers_sync();  // red is reused by the next unit
  }
#ifdef LFM3_TRACE
  if (tid == 0) TRACE(trb, trid, 5);
#endif
}

inline size_t q4_smem(int NT, int rows, int Kc, int stages) {  // no code table: expansion is by cvt
  return 1024 + q4_stage_base(rows, Kc) + (size_t)stages * Q4_STAGE_B + (size_t)4 * NT * 32 * 4 * 4 + 2 * stages * 8;
}

// ------------------------------------------------------------------------------------------ affine
// MLX affine weights (TensorFold issue #1491, "Checkpoint handling": groups of 64; w = s * q + b
// with bf16 s, b and q an unsigned `BITS`-bit code), on the NVFP4 kernel's structure: units of 64
// weight rows, warp = (row tile w & 3, K half w >> 2), a stage of 512 codes per row (8 groups).
// The dot product stays exact: a code enters the MMA as the bf16 value 128 + q (bits 0x4300 | q,
// exact), so a group of 64 gives P = sum((128 + q) x); with X = sum(x) over the group (from the
// bf16 activations), s * P + (b - 128 s) * X = sum((s q + b) x). 6- and 8-bit codes are split
// into a low nibble and a high part, each through its own MMAs (P = P_lo + 16 P_hi, and the
// offset becomes 128 * 17). Codes are copied as [block][row][bytes] with 64-byte blocks (96-byte
// for 6-bit codes, so that no lane's 16 codes straddle a block).
constexpr int AF_UR = 64;            // weight rows per unit
constexpr int AF_KST = 512;          // codes per row per stage (8 groups of 64)
__host__ __device__ constexpr int af_blkb(int bits) { return bits == 6 ? 96 : 64; }
__host__ __device__ constexpr int af_code_b(int bits) { return AF_UR * AF_KST * bits / 8; }
__host__ __device__ constexpr int af_stage_b(int bits) { return af_code_b(bits) + 2 * AF_UR * 16; }
__host__ __device__ constexpr int af_stages(int bits) { return bits == 4 ? 4 : 3; }

DEVI void ws_pair_bf16(uint32_t w, int sh, uint32_t& out) {
  out = ((w >> sh) & 0x000F000Fu) | 0x43004300u;  // bf16 pair (128 + nibble at sh, 128 + nibble at sh + 16)
}

template <int EPI, int NT, int BITS>
__global__ void __launch_bounds__(WS_THREADS, 2) k_wstream_aff(const __grid_constant__ CUtensorMap tw,
                                                               const __grid_constant__ CUtensorMap tw3,
                                                               const __grid_constant__ CUtensorMap ts,
                                                               const __grid_constant__ CUtensorMap ts3,
                                                               const __grid_constant__ CUtensorMap tb,
                                                               const __grid_constant__ CUtensorMap tb3, const WsArgs a) {
  constexpr bool SW = EPI == GEMV_SWIGLU;
  constexpr int RR = SW ? AF_UR / 2 : AF_UR;
  constexpr int BLKB = af_blkb(BITS);
  constexpr int CODE_B = af_code_b(BITS), STAGE_B = af_stage_b(BITS);
  constexpr int NBLK = AF_KST * BITS / 8 / BLKB;    // code blocks per row per stage
  constexpr float OFF = BITS == 4 ? 128.f : 128.f * 17.f;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int Kc = a.K / a.splits;
  const int XS = Kc + 32;
  const int NG = Kc / 64;                           // groups in the block's K range
  const bf16* xzero = reinterpret_cast<const bf16*>(smem);
  bf16* xs = reinterpret_cast<bf16*>(smem + 128);
  float* xsum = reinterpret_cast<float*>(smem + ws_x_bytes(a.rows, Kc));          // [rows][NG]
  unsigned char* stages = smem + (ws_x_bytes(a.rows, Kc) + (size_t)16 * NG * 4 + 1023) / 1024 * 1024;
  const int NS = a.stages;
  float* red = reinterpret_cast<float*>(stages + (size_t)NS * STAGE_B);
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 4 * NT * 32 * 4);
  __shared__ __align__(16) float redn[WS_CW * 4];
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kcta = blockIdx.y * Kc;
  const int nst = Kc / AF_KST;
  const int nunits = a.N / RR;
  const uint32_t full0 = su32(bars), empty0 = su32(bars + NS);
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, WS_CW);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == WS_CW) {
    // ------------------------------------------------------------ producer
    int it = 0;
    bool ok = true;
    const uint64_t pol = ws_policy();
    for (int unit = blockIdx.x; unit < nunits && ok; unit += gridDim.x) {
      for (int st = 0; st < nst && ok; ++st, ++it) {
        const int s = it % NS;
        const uint32_t ph = (it / NS) & 1;
        if (lane == 0) ok = mbar_wait(empty0 + 8 * s, ph ^ 1, a.err);
        ok = __shfl_sync(0xffffffffu, ok, 0) && !*(volatile int*)&abort_flag;
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(full0 + 8 * s, STAGE_B);
          unsigned char* sb = stages + (size_t)s * STAGE_B;
          const int k0 = kcta + st * AF_KST;
          const int row0 = unit * RR;
          const int z = k0 * BITS / 8 / BLKB;
          ws_tma3(su32(sb), &tw, 0, row0, z, full0 + 8 * s, pol);
          ws_tma2(su32(sb + CODE_B), &ts, k0 / 64, row0, full0 + 8 * s, pol);
          ws_tma2(su32(sb + CODE_B + AF_UR * 16), &tb, k0 / 64, row0, full0 + 8 * s, pol);
          if constexpr (SW) {
            ws_tma3(su32(sb + CODE_B / 2), &tw3, 0, row0, z, full0 + 8 * s, pol);
            ws_tma2(su32(sb + CODE_B + RR * 16), &ts3, k0 / 64, row0, full0 + 8 * s, pol);
            ws_tma2(su32(sb + CODE_B + AF_UR * 16 + RR * 16), &tb3, k0 / 64, row0, full0 + 8 * s, pol);
          }
        }
      }
    }
    pdl_wait();
    pdl_launch_dependents();
    if (!ok) {
      for (int k = 0; k < NS && k < it; ++k) {
        const int i = it - 1 - k;
        if (lane == 0) mbar_wait(full0 + 8 * (i % NS), (i / NS) & 1, a.err);
      }
    }
    return;
  }

  ws_prologue<false>(a, smem, xs, XS, Kc, kcta, redn, nullptr, 0);
  // sums of the bf16 activations over each group of 64 (the bias term and the 128 + q offset)
  for (int e = tid; e < a.rows * NG; e += WS_CW * 32) {
    const int b = e / NG, gi = e % NG;
    const bf16* xr = xs + (size_t)b * XS + 64 * gi;
    float sum = 0.f;
#pragma unroll 8
    for (int i = 0; i < 64; i += 2) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(xr + i);
      sum += bflo(w) + bfhi(w);
    }
    xsum[b * NG + gi] = sum;
  }
  consumers_sync();

  // -------------------------------------------------------------- consumers: main loop
  const int g = lane >> 2, t = lane & 3;
  const int rt = warp & 3, kh = warp >> 2;
  const int ra = SW ? 8 * rt + g : 16 * rt + g;            // region rows of MMA rows g and g + 8
  const int rb = SW ? 8 * rt + g : 16 * rt + g + 8;
  const int regb = SW ? CODE_B / 2 : 0;                    // w3's region
  const int sra = ra, srb = (SW ? RR : 0) + rb;            // rows of the scale / bias tables
  int it = 0;
  bool ok = true;
  for (int unit = blockIdx.x; unit < nunits; unit += gridDim.x) {
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[nt][j] = 0.f;
    for (int st = 0; st < nst; ++st, ++it) {
      const int s = it % NS;
      const uint32_t ph = (it / NS) & 1;
      if (ok && *(volatile int*)&abort_flag) ok = false;
      if (ok) {
        bool got = true;
        if (lane == 0) got = mbar_wait(full0 + 8 * s, ph, a.err);
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          ok = false;
          abort_flag = 1;
        }
      }
      if (ok) {
        const unsigned char* sb = stages + (size_t)s * STAGE_B;
        const bf16* scl = reinterpret_cast<const bf16*>(sb + CODE_B);
        const bf16* bia = reinterpret_cast<const bf16*>(sb + CODE_B + AF_UR * 16);
#pragma unroll 1
        for (int hh = 0; hh < 4; ++hh) {
          const int hs = 4 * kh + hh;                      // group of the stage
          const int o = (64 * hs + 16 * t) * BITS / 8;     // byte offset of this lane's 16 codes
          const int off = (o / BLKB) * (RR * BLKB) + (o % BLKB);
          const unsigned char* pa = sb + off + ra * BLKB;
          const unsigned char* pb = sb + regb + off + rb * BLKB;
          // this lane's 16 codes of rows a and b as 32-bit words (one code per byte for 6 and 8 bits)
          uint32_t wa[4], wb[4];
          if constexpr (BITS == 4) {
            const uint2 va = *reinterpret_cast<const uint2*>(pa), vb = *reinterpret_cast<const uint2*>(pb);
            wa[0] = va.x; wa[1] = va.y; wb[0] = vb.x; wb[1] = vb.y;
          } else if constexpr (BITS == 8) {
            const uint4 va = *reinterpret_cast<const uint4*>(pa), vb = *reinterpret_cast<const uint4*>(pb);
            wa[0] = va.x; wa[1] = va.y; wa[2] = va.z; wa[3] = va.w;
            wb[0] = vb.x; wb[1] = vb.y; wb[2] = vb.z; wb[3] = vb.w;
          } else {  // 6 bits: 12 bytes = 16 codes of a little-endian bit stream -> one byte each
            const uint32_t* qa = reinterpret_cast<const uint32_t*>(pa);
            const uint32_t* qb = reinterpret_cast<const uint32_t*>(pb);
            const uint32_t a3[4] = {qa[0], qa[1], qa[2], 0u}, b3[4] = {qb[0], qb[1], qb[2], 0u};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t xa = 0, xb = 0;
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int bo = 6 * (4 * j + i), wi = bo >> 5, sh = bo & 31;
                xa |= (__funnelshift_r(a3[wi], a3[wi + 1], sh) & 63u) << (8 * i);
                xb |= (__funnelshift_r(b3[wi], b3[wi + 1], sh) & 63u) << (8 * i);
              }
              wa[j] = xa; wb[j] = xb;
            }
          }
          float pl[NT][4], ph2[NT][4];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) pl[nt][j] = ph2[nt][j] = 0.f;
          const int kx = st * AF_KST + 64 * hs + 16 * t;   // K offset in the block's range
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const int sr = nt * 8 + g;
            const bf16* xr = sr < a.rows ? xs + (size_t)sr * XS + kx : nullptr;
            if constexpr (BITS == 4) {
              // word q holds codes 8q..8q+7; pairs (j, j + 4) come out of one mask
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                const uint4 xv = xr ? *reinterpret_cast<const uint4*>(xr + 8 * q) : *reinterpret_cast<const uint4*>(xzero);
                uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
                ws_pair_bf16(wa[q], 0, a0); ws_pair_bf16(wa[q], 4, a1); ws_pair_bf16(wa[q], 8, a2); ws_pair_bf16(wa[q], 12, a3);
                ws_pair_bf16(wb[q], 0, b0); ws_pair_bf16(wb[q], 4, b1); ws_pair_bf16(wb[q], 8, b2); ws_pair_bf16(wb[q], 12, b3);
                const uint32_t x04 = __byte_perm(xv.x, xv.z, 0x5410), x15 = __byte_perm(xv.x, xv.z, 0x7632);
                const uint32_t x26 = __byte_perm(xv.y, xv.w, 0x5410), x37 = __byte_perm(xv.y, xv.w, 0x7632);
                mma_bf16_16816(pl[nt], a0, b0, a1, b1, x04, x15);
                mma_bf16_16816(pl[nt], a2, b2, a3, b3, x26, x37);
              }
            } else {
              // word q holds codes 4q..4q+3, one per byte: low nibbles (c0, c2), (c1, c3) and high parts
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint2 xv = xr ? *reinterpret_cast<const uint2*>(xr + 4 * q) : *reinterpret_cast<const uint2*>(xzero);
                uint32_t la0, la1, lb0, lb1, ha0, ha1, hb0, hb1;
                ws_pair_bf16(wa[q], 0, la0); ws_pair_bf16(wa[q], 8, la1);
                ws_pair_bf16(wb[q], 0, lb0); ws_pair_bf16(wb[q], 8, lb1);
                ws_pair_bf16(wa[q], 4, ha0); ws_pair_bf16(wa[q], 12, ha1);
                ws_pair_bf16(wb[q], 4, hb0); ws_pair_bf16(wb[q], 12, hb1);
                const uint32_t x02 = __byte_perm(xv.x, xv.y, 0x5410), x13 = __byte_perm(xv.x, xv.y, 0x7632);
                mma_bf16_16816(pl[nt], la0, lb0, la1, lb1, x02, x13);
                mma_bf16_16816(ph2[nt], ha0, hb0, ha1, hb1, x02, x13);
              }
            }
          }
          // s * P + (b - OFF s) * X for rows a, b and this lane's two columns
          const int gk = (st * AF_KST) / 64 + hs;          // group in the block's K range
          const float sA = bf2f(scl[sra * 8 + hs]), sB = bf2f(scl[srb * 8 + hs]);
          const float bA = bf2f(bia[sra * 8 + hs]) - OFF * sA, bB = bf2f(bia[srb * 8 + hs]) - OFF * sB;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const int c0 = nt * 8 + 2 * t;
            const float X0 = c0 < a.rows ? xsum[c0 * NG + gk] : 0.f, X1 = c0 + 1 < a.rows ? xsum[(c0 + 1) * NG + gk] : 0.f;
            const float p0 = pl[nt][0] + 16.f * ph2[nt][0], p1 = pl[nt][1] + 16.f * ph2[nt][1];
            const float p2 = pl[nt][2] + 16.f * ph2[nt][2], p3 = pl[nt][3] + 16.f * ph2[nt][3];
            acc[nt][0] += sA * p0 + bA * X0;
            acc[nt][1] += sA * p1 + bA * X1;
            acc[nt][2] += sB * p2 + bB * X0;
            acc[nt][3] += sB * p3 + bB * X1;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * s);
    }
    if (kh == 1)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        *reinterpret_cast<float4*>(red + ((rt * NT + nt) * 32 + lane) * 4) =
            make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
    consumers_sync();
    if (kh == 0 && ok) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float4 o = *reinterpret_cast<const float4*>(red + ((rt * NT + nt) * 32 + lane) * 4);
        const float v0 = acc[nt][0] + o.x, v1 = acc[nt][1] + o.y, v2 = acc[nt][2] + o.z, v3 = acc[nt][3] + o.w;
        const int b0 = nt * 8 + 2 * t;
        if constexpr (SW) {
          const int j = unit * RR + 8 * rt + g;
          if (b0 < a.rows) a.out[(size_t)b0 * a.N + j] = f2bf(siluf_(v0) * v2);
          if (b0 + 1 < a.rows) a.out[(size_t)(b0 + 1) * a.N + j] = f2bf(siluf_(v1) * v3);
        } else {
          const int r0 = unit * AF_UR + 16 * rt + g;
          float* po = a.part_out + (size_t)blockIdx.y * a.rows * a.N;
          if (b0 < a.rows) {
            po[(size_t)b0 * a.N + r0] = v0;
            po[(size_t)b0 * a.N + r0 + 8] = v2;
          }
          if (b0 + 1 < a.rows) {
            po[(size_t)(b0 + 1) * a.N + r0] = v1;
            po[(size_t)(b0 + 1) * a.N + r0 + 8] = v3;
          }
        }
      }
    }
    consumers_sync();
  }
}

template <int BITS>
inline size_t af_smem(int NT, int rows, int Kc) {
  const size_t base = (ws_x_bytes(rows, Kc) + (size_t)16 * (Kc / 64) * 4 + 1023) / 1024 * 1024;
  return 1024 + base + (size_t)af_stages(BITS) * af_stage_b(BITS) + (size_t)4 * NT * 32 * 4 * 4 + 2 * af_stages(BITS) * 8;
}

// Expansion for the tensor-core GEMM: out[n][k] = bf16(s * q + b) (rounded once from fp32).
__global__ void __launch_bounds__(256) k_affine_to_bf16(const uint8_t* __restrict__ codes, const bf16* __restrict__ sc,
                                                        const bf16* __restrict__ bi, int bits, int N, int K,
                                                        bf16* __restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  const size_t total = (size_t)N * K / 8;
  const size_t rowb = (size_t)K * bits / 8;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const size_t n = i / (K / 8);
    const int k0 = (int)(i % (K / 8)) * 8;
    const uint8_t* rp = codes + n * rowb;
    const float s = bf2f(sc[n * (K / 64) + k0 / 64]), b = bf2f(bi[n * (K / 64) + k0 / 64]);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float v[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int k = k0 + 2 * j + e;
        const size_t bit = (size_t)k * bits;
        const uint32_t lo = rp[bit >> 3], hi = (bit >> 3) + 1 < rowb ? rp[(bit >> 3) + 1] : 0u;
        const uint32_t q = ((lo | (hi << 8)) >> (bit & 7)) & ((1u << bits) - 1u);
        v[e] = s * (float)q + b;
      }
      w[j] = pack_bf2(v[0], v[1]);
    }
    stg16(out + n * K + k0, make_uint4(w[0], w[1], w[2], w[3]));
  }
}

cudaError_t affine_to_bf16(const uint8_t* codes, const void* scales, const void* biases, int bits, int N, int K, bf16* out,
                           cudaStream_t s) {
  return launch(k_affine_to_bf16, dim3(4 * 148), dim3(256), 0, s, codes, reinterpret_cast<const bf16*>(scales),
                reinterpret_cast<const bf16*>(biases), bits, N, K, out);
}

template <int EPI, bool FP4>
size_t ws_smem(int NT, int rows, int Kc, int stages) {
  using G = WsGeom<EPI, FP4>;
  const size_t x = ws_stage_base(rows, Kc);
  return 1024 + x + (size_t)stages * G::STAGE_BYTES + (size_t)WS_CW * G::NRT * NT * 128 * 4 +
         (size_t)G::NRT * 16 * NT * 8 * 4 + 2 * stages * 8;
}

static int g_num_sms = 0;
constexpr int WS_BPS = LFM3_WS_BPS;  // blocks per SM, at most

// Blocks of `kern` that fit on one SM with `smem` bytes of dynamic shared memory (at most WS_BPS):
// the grid is one wave of them, so no block waits for a second wave.
template <typename K>
static int ws_fit(K kern, size_t smem) {
  struct Entry { const void* k; size_t smem; int n; };
  static Entry cache[64];
  static int used = 0;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].k == reinterpret_cast<const void*>(kern) && cache[i].smem == smem) return cache[i].n;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, WS_THREADS, smem) != cudaSuccess || n < 1) {
    (void)cudaGetLastError();
    n = 1;
  }
  n = std::min(n, WS_BPS);
  if (used < 64) cache[used++] = Entry{reinterpret_cast<const void*>(kern), smem, n};
  return n;
}

template <int EPI, bool FP4>
static cudaError_t launch_ws(const WsMaps& mp, const WsArgs& a, cudaStream_t s) {
  using G = WsGeom<EPI, FP4>;
  const int Kc = a.K / a.splits;
  if (Kc % G::KCH || a.K % a.splits) return cudaErrorInvalidValue;
  const int ntiles = (EPI == GEMV_SWIGLU) ? a.N / 8 : (EPI == GEMV_CONV ? D / 16 : a.N / 16);
  const int NT = a.rows <= 8 ? 1 : 2;
  WsArgs b = a;
  b.stages = G::STAGES;
#ifdef LFM3_TRACE
  b.trace = g_trace;
  b.trace_id = g_launches;
#endif
  const size_t smem = ws_smem<EPI, FP4>(NT, a.rows, Kc, b.stages);
  if (smem > (size_t)WS_SMEM_MAX) return cudaErrorInvalidValue;
  // blocks per K range: as many blocks as fit on the SMs at once (one wave), spread evenly
  // over the tiles
  auto kern = NT == 1 ? k_wstream<EPI, 1, FP4> : k_wstream<EPI, 2, FP4>;
  int gx = std::max(1, ws_fit(kern, smem) * g_num_sms / a.splits);
  gx = std::min(gx, ntiles);
  const int per = (ntiles + gx - 1) / gx;
  gx = (ntiles + per - 1) / per;
  dim3 grid(gx, a.splits);
  return launch(kern, grid, dim3(WS_THREADS), smem, s, mp.w, mp.w3, mp.s, mp.s3, b);
}

template <int EPI>
static cudaError_t launch_q4(const WsMaps& mp, const WsArgs& a, cudaStream_t s) {
  const int Kc = a.K / a.splits;
  if (Kc % Q4_KST || a.K % a.splits) return cudaErrorInvalidValue;
  const int nunits = a.N / (EPI == GEMV_SWIGLU ? Q4_UR / 2 : Q4_UR);
  const int NT = a.rows <= 8 ? 1 : 2;
  WsArgs b = a;
#ifdef LFM3_TRACE
  b.trace = g_trace;
  b.trace_id = g_launches;
#endif
  auto kern = NT == 1 ? k_wstream_fp4<EPI, 1> : k_wstream_fp4<EPI, 2>;
  // the deepest ring that still lets two blocks share an SM (wide batches hold more activations)
  b.stages = Q4_STAGES;
  while (b.stages > Q4_STAGES / 2 && ws_fit(kern, q4_smem(NT, a.rows, Kc, b.stages)) < 2) --b.stages;
  const size_t smem = q4_smem(NT, a.rows, Kc, b.stages);
  if (smem > (size_t)WS_SMEM_MAX) return cudaErrorInvalidValue;
  int gx = std::max(1, ws_fit(kern, smem) * g_num_sms / a.splits);
  gx = std::min(gx, nunits);
  const int per = (nunits + gx - 1) / gx;
  gx = (nunits + per - 1) / per;
  return launch(kern, dim3(gx, a.splits), dim3(WS_THREADS), smem, s, mp.w, mp.w3, mp.s, mp.s3, b);
}

template <int EPI, int BITS>
static cudaError_t launch_aff(const WsMaps& mp, const WsArgs& a, cudaStream_t s) {
  const int Kc = a.K / a.splits;
  if (Kc % AF_KST || a.K % a.splits) return cudaErrorInvalidValue;
  const int nunits = a.N / (EPI == GEMV_SWIGLU ? AF_UR / 2 : AF_UR);
  const int NT = a.rows <= 8 ? 1 : 2;
  WsArgs b = a;
  b.stages = af_stages(BITS);
  const size_t smem = af_smem<BITS>(NT, a.rows, Kc);
  if (smem > (size_t)WS_SMEM_MAX) return cudaErrorInvalidValue;
  auto kern = NT == 1 ? k_wstream_aff<EPI, 1, BITS> : k_wstream_aff<EPI, 2, BITS>;
  int gx = std::max(1, ws_fit(kern, smem) * g_num_sms / a.splits);
  gx = std::min(gx, nunits);
  const int per = (nunits + gx - 1) / gx;
  gx = (nunits + per - 1) / per;
  return launch(kern, dim3(gx, a.splits), dim3(WS_THREADS), smem, s, mp.w, mp.w3, mp.s, mp.s3, mp.b, mp.b3, b);
}

template <int EPI>
static cudaError_t launch_aff_bits(const WsMaps& mp, const WsArgs& a, cudaStream_t s) {
  switch (a.bits) {
    case 4: return launch_aff<EPI, 4>(mp, a, s);
    case 6: return launch_aff<EPI, 6>(mp, a, s);
    case 8: return launch_aff<EPI, 8>(mp, a, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t wstream(int epi, int format, const WsMaps& mp, const WsArgs& a, cudaStream_t s) {
  if (a.rows > 16 || a.rows < 1) return cudaErrorInvalidValue;
  if (a.pro == WS_PRO_NORM && (a.n_parts < 0 || a.n_parts > WS_MAX_PARTS)) return cudaErrorInvalidValue;
  if (format == WS_AFFINE) {
    if (epi == GEMV_PARTIAL) return launch_aff_bits<GEMV_PARTIAL>(mp, a, s);
    if (epi == GEMV_SWIGLU) return launch_aff_bits<GEMV_SWIGLU>(mp, a, s);
    return cudaErrorInvalidValue;
  }
  const bool nvfp4 = format == WS_NVFP4;
  switch (epi) {
    case GEMV_PARTIAL: return nvfp4 ? launch_q4<GEMV_PARTIAL>(mp, a, s) : launch_ws<GEMV_PARTIAL, false>(mp, a, s);
    case GEMV_SWIGLU: return nvfp4 ? launch_q4<GEMV_SWIGLU>(mp, a, s) : launch_ws<GEMV_SWIGLU, false>(mp, a, s);
    case GEMV_CONV: return launch_ws<GEMV_CONV, false>(mp, a, s);
    case GEMV_HEAD: return launch_ws<GEMV_HEAD, false>(mp, a, s);
  }
  return cudaErrorInvalidValue;
}

// Weight maps: a bf16 matrix [N][K] seen as {32 elements, N rows, K/32 blocks} (an NVFP4 code
// matrix [N][K/2] as {64 bytes, N rows, K/128 blocks}), so that one box {., br rows, stage K}
// lands as [block][row][64 B] - rows 64 B apart, which the lane pattern reads without bank
// conflicts; NVFP4 scales [N][K/16] as a plain 2-D box {K-chunk/16, br}.
static PFN_cuTensorMapEncodeTiled_v12000 p_enc_ws = nullptr;

static bool ws_encoder() {
  if (p_enc_ws) return true;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return false;
  p_enc_ws = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

bool make_ws_map(CUtensorMap* m, const void* w, int N, int K, int fp4, int br, int kch) {
  if (!ws_encoder()) return false;
  const int eb = fp4 ? 64 : 32;        // elements per 64-byte block (bytes of codes, or bf16)
  const int kpb = fp4 ? 128 : 32;      // K per block
  cuuint64_t dims[3] = {(cuuint64_t)eb, (cuuint64_t)N, (cuuint64_t)(K / kpb)};
  cuuint64_t strides[2] = {(cuuint64_t)(fp4 ? K / 2 : K * 2), 64};
  cuuint32_t box[3] = {(cuuint32_t)eb, (cuuint32_t)br, (cuuint32_t)(kch / kpb)};
  cuuint32_t es[3] = {1, 1, 1};
  return p_enc_ws(m, fp4 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(w), dims,
                  strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Affine codes [N][K * bits / 8] as {block, row, block index} with 64-byte blocks (96-byte for
// 6-bit codes); a box of `br` rows and one stage (512 codes) lands as [block][row][block bytes].
bool make_aff_map(CUtensorMap* m, const void* codes, int N, int K, int bits, int br) {
  if (!ws_encoder()) return false;
  const int blk = bits == 6 ? 96 : 64;
  const uint64_t rowb = (uint64_t)K * bits / 8;
  if (rowb % blk) return false;
  cuuint64_t dims[3] = {(cuuint64_t)blk, (cuuint64_t)N, (cuuint64_t)(rowb / blk)};
  cuuint64_t strides[2] = {(cuuint64_t)rowb, (cuuint64_t)blk};
  cuuint32_t box[3] = {(cuuint32_t)blk, (cuuint32_t)br, (cuuint32_t)(512 * bits / 8 / blk)};
  cuuint32_t es[3] = {1, 1, 1};
  return p_enc_ws(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(codes), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Affine scales or biases: bf16 [N][K / 64], a box of 8 groups (one stage) x `br` rows.
bool make_aff_sb_map(CUtensorMap* m, const void* sb, int N, int K, int br) {
  if (!ws_encoder()) return false;
  cuuint64_t dims[2] = {(cuuint64_t)(K / 64), (cuuint64_t)N};
  cuuint64_t strides[1] = {(cuuint64_t)(K / 64) * 2};
  cuuint32_t box[2] = {8, (cuuint32_t)br};
  cuuint32_t es[2] = {1, 1};
  return p_enc_ws(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(sb), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int aff_br(int epi) { return epi == GEMV_SWIGLU ? AF_UR / 2 : AF_UR; }

bool make_ws_scale_map(CUtensorMap* m, const void* sc, int N, int K, int br, int kch) {
  if (!ws_encoder()) return false;
  cuuint64_t dims[2] = {(cuuint64_t)(K / 16), (cuuint64_t)N};
  cuuint64_t strides[1] = {(cuuint64_t)(K / 16)};
  cuuint32_t box[2] = {(cuuint32_t)(kch / 16), (cuuint32_t)br};
  cuuint32_t es[2] = {1, 1};
  return p_enc_ws(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(sc), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int ws_kch(int epi, int fp4) { return fp4 ? Q4_KST : (epi == GEMV_CONV ? 256 : 512); }
int ws_br(int epi, int fp4) {
  if (fp4) return epi == GEMV_SWIGLU ? Q4_UR / 2 : Q4_UR;
  return epi == GEMV_SWIGLU ? 8 : 16;
}

template <int EPI, bool FP4>
static cudaError_t ws_attr() {
  const int mx = WS_SMEM_MAX;
  cudaError_t e = cudaFuncSetAttribute(k_wstream<EPI, 1, FP4>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(k_wstream<EPI, 2, FP4>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
}
template <int EPI, int BITS>
static cudaError_t aff_attr() {
  const int mx = WS_SMEM_MAX;
  cudaError_t e = cudaFuncSetAttribute(k_wstream_aff<EPI, 1, BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(k_wstream_aff<EPI, 2, BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
}
template <int EPI>
static cudaError_t q4_attr() {
  const int mx = WS_SMEM_MAX;
  cudaError_t e = cudaFuncSetAttribute(k_wstream_fp4<EPI, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(k_wstream_fp4<EPI, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
}

cudaError_t wstream_init() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = ws_attr<GEMV_PARTIAL, false>()) != cudaSuccess) return e;
  if ((e = q4_attr<GEMV_PARTIAL>()) != cudaSuccess) return e;
  if ((e = ws_attr<GEMV_SWIGLU, false>()) != cudaSuccess) return e;
  if ((e = q4_attr<GEMV_SWIGLU>()) != cudaSuccess) return e;
  if ((e = aff_attr<GEMV_PARTIAL, 4>()) != cudaSuccess) return e;
  if ((e = aff_attr<GEMV_PARTIAL, 6>()) != cudaSuccess) return e;
  if ((e = aff_attr<GEMV_PARTIAL, 8>()) != cudaSuccess) return e;
  if ((e = aff_attr<GEMV_SWIGLU, 4>()) != cudaSuccess) return e;
  if ((e = aff_attr<GEMV_SWIGLU, 6>()) != cudaSuccess) return e;
  if ((e = aff_attr<GEMV_SWIGLU, 8>()) != cudaSuccess) return e;
  if ((e = ws_attr<GEMV_CONV, false>()) != cudaSuccess) return e;
  return ws_attr<GEMV_HEAD, false>();
}

}  // namespace lfm3
