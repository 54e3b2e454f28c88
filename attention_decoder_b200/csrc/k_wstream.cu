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

// E2M1 code (bit 3 sign, bits 2..1 exponent with bias 1, bit 0 mantissa) -> bf16 bits, exact:
// 0, 0.5, 1, 1.5, 2, 3, 4, 6 and their negatives.
DEVI uint32_t e2m1_bf16_bits(uint32_t c) {
  const uint32_t e = (c >> 1) & 3u, m = c & 1u;
  const uint32_t mag = e == 0 ? (m ? 0x3F00u : 0u) : (((e + 126u) << 7) | (m << 6));
  return mag | ((c & 8u) << 12);
}

DEVI uint32_t ws_e4m3x2(uint32_t b) {
  const uint32_t s = (b & 0x80u) << 8;
  const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
  uint32_t bits = e == 0 ? (__float_as_uint((float)m * (1.0f / 512.0f)) >> 16) : (((e + 120u) << 7) | (m << 4));
  bits |= s;
  return bits | (bits << 16);
}

DEVI uint32_t ws_hmul2(uint32_t a, uint32_t b) {
  __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a), y = *reinterpret_cast<__nv_bfloat162*>(&b);
  __nv_bfloat162 r = __hmul2(x, y);
  return *reinterpret_cast<uint32_t*>(&r);
}

DEVI void ws_tma3(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
DEVI void ws_tma2(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

DEVI void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(WS_CW * 32) : "memory"); }

// Activations in shared memory: a 128-byte zero block (the MMA columns of absent streams read
// it), then one row per stream of the block's K range, 64-byte skewed against bank conflicts.
__host__ __device__ inline size_t ws_x_bytes(int rows, int Kc) { return 128 + (size_t)rows * (Kc + 32) * 2; }
// Stages start on a 1024-byte boundary after the activations (and the NVFP4 table).
__host__ __device__ inline size_t ws_stage_base(int rows, int Kc, bool fp4) {
  return (ws_x_bytes(rows, Kc) + (fp4 ? 256 * 32 * 4 : 0) + 1023) / 1024 * 1024;
}

template <int EPI, int NT, bool FP4>
__global__ void __launch_bounds__(WS_THREADS, 2) k_wstream(const __grid_constant__ CUtensorMap tw,
                                                        const __grid_constant__ CUtensorMap tw3,
                                                        const __grid_constant__ CUtensorMap tsc,
                                                        const __grid_constant__ CUtensorMap tsc3, const WsArgs a) {
  using G = WsGeom<EPI, FP4>;
  constexpr int NRT = G::NRT;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int Kc = a.K / a.splits;
  const int XS = Kc + 32;  // activations row stride (elements): 64-byte skew against bank conflicts
  const bf16* xzero = reinterpret_cast<const bf16*>(smem);
  bf16* xs = reinterpret_cast<bf16*>(smem + 128);
  // NVFP4: byte (two E2M1 codes) -> bf16x2, 256 entries x 32 copies (one per bank)
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + ws_x_bytes(a.rows, Kc));
  unsigned char* stages = smem + ws_stage_base(a.rows, Kc, FP4);
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
            ws_tma3(su32(st + q * G::REQB), m, 0, row, k0 / G::KBLK, full0 + 8 * s);
            if constexpr (FP4)
              ws_tma2(su32(st + G::RPT * G::ROWB + q * G::BR * G::SCB), which ? &tsc3 : &tsc, k0 / 16, row,
                      full0 + 8 * s);
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
  const int ct = tid;  // 0..127
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
  if constexpr (FP4) {
    for (int i = ct; i < 256 * 32; i += WS_CW * 32) {
      const uint32_t v = (uint32_t)i >> 5;
      lut[i] = e2m1_bf16_bits(v & 15u) | (e2m1_bf16_bits(v >> 4) << 16);
    }
  }
  if (a.pro == WS_PRO_LOAD) {
    const int chunks = Kc / 8;
    for (int idx = ct; idx < a.rows * chunks; idx += WS_CW * 32) {
      const int b = idx / chunks, c = idx - b * chunks;
      *reinterpret_cast<uint4*>(xs + (size_t)b * XS + c * 8) = ldg16(a.x + (size_t)b * a.K + kcta + c * 8);
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
      const float* xin = a.x_in + (size_t)b * D + c0;
#pragma unroll
      for (int q = 0; q < WS_EPT / 4; ++q) {
        const float4 v = reinterpret_cast<const float4*>(xin)[q];
        x[4 * q] = v.x; x[4 * q + 1] = v.y; x[4 * q + 2] = v.z; x[4 * q + 3] = v.w;
      }
#pragma unroll
      for (int j = 0; j < WS_EPT; ++j) m[j] = 0.f;
      for (int s = 0; s < a.n_parts; ++s) {
        const float* p = a.parts + s * a.part_stride + (size_t)b * D + c0;
#pragma unroll
        for (int q = 0; q < WS_EPT / 4; ++q) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(p) + q);
          m[4 * q] += v.x; m[4 * q + 1] += v.y; m[4 * q + 2] += v.z; m[4 * q + 3] += v.w;
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
          }
          *reinterpret_cast<uint4*>(xs + (size_t)b * XS + (c0 - kcta) + 8 * h) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      consumers_sync();  // redn is reused by the next stream
    }
  }
  consumers_sync();

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
            if constexpr (!FP4) {
              const uint4 wa = *reinterpret_cast<const uint4*>(st + ws_woff<G, FP4>(rt * 16 + g, j, t));
              const uint4 wb = *reinterpret_cast<const uint4*>(st + ws_woff<G, FP4>(rt * 16 + g + 8, j, t));
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                const int sr = nt * 8 + g;
                const uint4 xv = *reinterpret_cast<const uint4*>(sr < a.rows ? xs + (size_t)sr * XS + kx + 8 * t : xzero);
                mma_bf16_16816(acc[rt][nt], wa.x, wb.x, wa.y, wb.y, xv.x, xv.y);
                mma_bf16_16816(acc[rt][nt], wa.z, wb.z, wa.w, wb.w, xv.z, xv.w);
              }
            } else {
              // 16 codes of rows g and g + 8: one E4M3 block scale each
              const uint2 wa = *reinterpret_cast<const uint2*>(st + ws_woff<G, FP4>(rt * 16 + g, j, t));
              const uint2 wb = *reinterpret_cast<const uint2*>(st + ws_woff<G, FP4>(rt * 16 + g + 8, j, t));
              const unsigned char* sc = st + G::RPT * G::ROWB;  // scales: [row][SCB]
              const uint32_t sA = ws_e4m3x2(sc[(rt * 16 + g) * G::SCB + j * 4 + t]);
              const uint32_t sB = ws_e4m3x2(sc[(rt * 16 + g + 8) * G::SCB + j * 4 + t]);
              const uint32_t wA[2] = {wa.x, wa.y};
              const uint32_t wB[2] = {wb.x, wb.y};
              const uint32_t* tab = lut + lane;  // this lane's copy of the table
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                uint32_t a01 = tab[(wA[q] & 0xFFu) << 5], a23 = tab[((wA[q] >> 8) & 0xFFu) << 5];
                uint32_t a45 = tab[((wA[q] >> 16) & 0xFFu) << 5], a67 = tab[(wA[q] >> 24) << 5];
                uint32_t b01 = tab[(wB[q] & 0xFFu) << 5], b23 = tab[((wB[q] >> 8) & 0xFFu) << 5];
                uint32_t b45 = tab[((wB[q] >> 16) & 0xFFu) << 5], b67 = tab[(wB[q] >> 24) << 5];
                a01 = ws_hmul2(a01, sA); a23 = ws_hmul2(a23, sA); a45 = ws_hmul2(a45, sA); a67 = ws_hmul2(a67, sA);
                b01 = ws_hmul2(b01, sB); b23 = ws_hmul2(b23, sB); b45 = ws_hmul2(b45, sB); b67 = ws_hmul2(b67, sB);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                  const int sr = nt * 8 + g;
                  const uint4 xv = *reinterpret_cast<const uint4*>(sr < a.rows ? xs + (size_t)sr * XS + kx + 16 * t + 8 * q
                                                                               : xzero);
                  mma_bf16_16816(acc[rt][nt], a01, b01, a23, b23, xv.x, xv.y);
                  mma_bf16_16816(acc[rt][nt], a45, b45, a67, b67, xv.z, xv.w);
                }
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

template <int EPI, bool FP4>
size_t ws_smem(int NT, int rows, int Kc, int stages) {
  using G = WsGeom<EPI, FP4>;
  const size_t x = ws_stage_base(rows, Kc, FP4);
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

cudaError_t wstream(int epi, int nvfp4, const WsMaps& mp, const WsArgs& a, cudaStream_t s) {
  if (a.rows > 16 || a.rows < 1) return cudaErrorInvalidValue;
  switch (epi) {
    case GEMV_PARTIAL: return nvfp4 ? launch_ws<GEMV_PARTIAL, true>(mp, a, s) : launch_ws<GEMV_PARTIAL, false>(mp, a, s);
    case GEMV_SWIGLU: return nvfp4 ? launch_ws<GEMV_SWIGLU, true>(mp, a, s) : launch_ws<GEMV_SWIGLU, false>(mp, a, s);
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

int ws_kch(int epi, int fp4) { return fp4 ? 512 : (epi == GEMV_CONV ? 256 : 512); }
int ws_br(int epi) { return epi == GEMV_SWIGLU ? 8 : 16; }

template <int EPI, bool FP4>
static cudaError_t ws_attr() {
  const int mx = WS_SMEM_MAX;
  cudaError_t e = cudaFuncSetAttribute(k_wstream<EPI, 1, FP4>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(k_wstream<EPI, 2, FP4>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
}

cudaError_t wstream_init() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = ws_attr<GEMV_PARTIAL, false>()) != cudaSuccess) return e;
  if ((e = ws_attr<GEMV_PARTIAL, true>()) != cudaSuccess) return e;
  if ((e = ws_attr<GEMV_SWIGLU, false>()) != cudaSuccess) return e;
  if ((e = ws_attr<GEMV_SWIGLU, true>()) != cudaSuccess) return e;
  if ((e = ws_attr<GEMV_CONV, false>()) != cudaSuccess) return e;
  return ws_attr<GEMV_HEAD, false>();
}

}  // namespace lfm3
