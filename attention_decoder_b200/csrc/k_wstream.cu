// Decode-time projections, weight-streaming: y[b][n] = sum_k x[b][k] W[n][k] for up to 16 streams.
//
// Decode is bound by reading each weight once from HBM, so this kernel is a pipeline built around
// that stream. Persistent blocks (about two per SM) each own a K range (blockIdx.y) and walk a
// strided list of row tiles. One producer warp copies the tiles' weight rows into a padded ring of
// shared-memory stages with 1-D bulk asynchronous copies (cp.async.bulk + mbarrier transaction
// counts), starting before the block waits for the previous kernel - the weights do not depend on
// it - so each launch's first stages are already in flight when its inputs become ready. Four
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
// NVFP4 weights (E2M1 codes + E4M3 block scales) are expanded in registers to exact bf16 values;
// the fp32 tensor scale multiplies the finished sums.
#include "kernels.cuh"

namespace lfm3 {

constexpr int WS_CW = 4;                    // consumer warps
// Largest dynamic shared memory a launch asks for (in_proj + conv with 16 streams: ~192 KB).
constexpr int WS_SMEM_MAX = 200 * 1024;
constexpr int WS_THREADS = 32 * (WS_CW + 1);

template <int EPI>
struct WsRows { static constexpr int NRT = (EPI == GEMV_CONV) ? 3 : 1; };

template <int EPI, bool FP4>
struct WsGeom {
  static constexpr int NRT = WsRows<EPI>::NRT;
  static constexpr int RPT = 16 * NRT;                        // weight rows per tile
  static constexpr int KB = FP4 ? 128 : 32;                   // K per lane step
  static constexpr int KCH = FP4 ? 512 : (NRT == 3 ? 256 : 512);  // K per stage
  static constexpr int ROWB = FP4 ? KCH / 2 : KCH * 2;        // weight bytes per row per stage
  static constexpr int RS = ROWB + 64;                        // padded row stride in shared memory
  static constexpr int SCB = FP4 ? KCH / 16 : 0;              // scale bytes per row per stage
  static constexpr int STAGES = FP4 ? 8 : 4;
  static constexpr int STAGE_BYTES = RPT * RS + RPT * SCB;
  static constexpr int TX_BYTES = RPT * (ROWB + SCB);
  static constexpr int STEPS = KCH / KB;                      // lane steps per stage
  static constexpr int STEPB = 64;                            // bytes of a row per lane step
};

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

// E2M1 magnitude (3 bits) -> bf16 high and low bytes, as byte-permute tables (0 .. 6).
constexpr uint32_t WS_HI_LO = 0x3F3F3F00u, WS_HI_HI = 0x40404040u;
constexpr uint32_t WS_LO_LO = 0xC0800000u, WS_LO_HI = 0xC0804000u;

DEVI void ws_e2m1x4(uint32_t w, uint32_t& o01, uint32_t& o23) {
  const uint32_t sel = w & 0x7777u;
  const uint32_t hi = __byte_perm(WS_HI_LO, WS_HI_HI, sel);
  const uint32_t lo = __byte_perm(WS_LO_LO, WS_LO_HI, sel);
  o01 = __byte_perm(lo, hi, 0x5140);
  o23 = __byte_perm(lo, hi, 0x7362);
  const uint32_t s = w & 0x8888u;
  o01 |= ((s << 12) & 0x8000u) | ((s << 24) & 0x80000000u);
  o23 |= ((s << 4) & 0x8000u) | ((s << 16) & 0x80000000u);
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

DEVI void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(WS_CW * 32) : "memory"); }

template <int NT>
DEVI size_t ws_x_bytes(int Kc) { return (size_t)NT * 8 * (Kc + 32) * 2; }

template <int EPI, int NT, bool FP4>
__global__ void __launch_bounds__(WS_THREADS) k_wstream(const WsArgs a) {
  using G = WsGeom<EPI, FP4>;
  constexpr int NRT = G::NRT;
  extern __shared__ __align__(128) unsigned char smem[];
  const int Kc = a.K / a.splits;
  const int XS = Kc + 32;  // activations row stride (elements): 64-byte skew against bank conflicts
  bf16* xs = reinterpret_cast<bf16*>(smem);
  unsigned char* stages = smem + ws_x_bytes<NT>(Kc);
  float* red = reinterpret_cast<float*>(stages + (size_t)G::STAGES * G::STAGE_BYTES);
  float* res = red + WS_CW * NRT * NT * 128;
  uint64_t* bars = reinterpret_cast<uint64_t*>(res + NRT * 16 * NT * 8);
  __shared__ float redn[WS_CW];
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kcta = blockIdx.y * Kc;
  const int nch = Kc / G::KCH;
  const int ntiles = (EPI == GEMV_SWIGLU) ? a.N / 8 : (EPI == GEMV_CONV ? D / 16 : a.N / 16);
  const uint32_t full0 = su32(bars), empty0 = su32(bars + G::STAGES);

  if (tid == 0) {
    for (int s = 0; s < G::STAGES; ++s) {
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
        const int s = it % G::STAGES;
        const uint32_t ph = (it / G::STAGES) & 1;
        if (lane == 0) ok = mbar_wait(empty0 + 8 * s, ph ^ 1, a.err);
        ok = __shfl_sync(0xffffffffu, ok, 0) && !*(volatile int*)&abort_flag;
        if (!ok) break;
        if (lane == 0) mbar_expect_tx(full0 + 8 * s, G::TX_BYTES);
        __syncwarp();
        unsigned char* st = stages + (size_t)s * G::STAGE_BYTES;
        const int k0 = kcta + ch * G::KCH;
        for (int r = lane; r < G::RPT; r += 32) {
          int which;
          const int row = ws_row<EPI>(tile, r / 16, r % 16, which);
          if constexpr (FP4) {
            const uint8_t* cs = which ? a.codes3 : a.codes;
            const uint8_t* ss = which ? a.scales3 : a.scales;
            bulk_g2s(su32(st + r * G::RS), cs + (size_t)row * (a.K / 2) + k0 / 2, G::ROWB, full0 + 8 * s);
            bulk_g2s(su32(st + G::RPT * G::RS + r * G::SCB), ss + (size_t)row * (a.K / 16) + k0 / 16, G::SCB,
                     full0 + 8 * s);
          } else {
            const bf16* wm = which ? a.w3 : a.w;
            bulk_g2s(su32(st + r * G::RS), wm + (size_t)row * a.K + k0, G::ROWB, full0 + 8 * s);
          }
        }
      }
    }
    pdl_wait();
    pdl_launch_dependents();
    if (!ok) {
      // drain: copies already issued land before the block exits (bounded)
      for (int k = 0; k < G::STAGES && k < it; ++k) {
        const int i = it - 1 - k;
        if (lane == 0) mbar_wait(full0 + 8 * (i % G::STAGES), (i / G::STAGES) & 1, a.err);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers: prologue
  pdl_wait();
  pdl_launch_dependents();
  const int ct = tid;  // 0..127
  if (a.pro == WS_PRO_LOAD) {
    const int chunks = Kc / 8;
    for (int idx = ct; idx < NT * 8 * chunks; idx += WS_CW * 32) {
      const int b = idx / chunks, c = idx - b * chunks;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (b < a.rows) v = ldg16(a.x + (size_t)b * a.K + kcta + c * 8);
      *reinterpret_cast<uint4*>(xs + (size_t)b * XS + c * 8) = v;
    }
  } else {
    // residual + post-norm of the previous projection, then this projection's input norm
    const bool writer = blockIdx.x == 0 && blockIdx.y == 0;
    for (int b = 0; b < NT * 8; ++b) {
      if (b >= a.rows) {
        for (int c = ct; c < Kc / 8; c += WS_CW * 32)
          *reinterpret_cast<uint4*>(xs + (size_t)b * XS + c * 8) = make_uint4(0, 0, 0, 0);
        continue;
      }
      float x[16];
      const float* xin = a.x_in + (size_t)b * D + ct * 16;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 v = reinterpret_cast<const float4*>(xin)[q];
        x[4 * q] = v.x; x[4 * q + 1] = v.y; x[4 * q + 2] = v.z; x[4 * q + 3] = v.w;
      }
      if (a.n_parts > 0) {
        float m[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) m[j] = 0.f;
        for (int s = 0; s < a.n_parts; ++s) {
          const float* p = a.parts + s * a.part_stride + (size_t)b * D + ct * 16;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(p) + q);
            m[4 * q] += v.x; m[4 * q + 1] += v.y; m[4 * q + 2] += v.z; m[4 * q + 3] += v.w;
          }
        }
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) ss += m[j] * m[j];
        ss = warp_sum(ss);
        if (lane == 0) redn[warp] = ss;
        consumers_sync();
        ss = redn[0] + redn[1] + redn[2] + redn[3];
        consumers_sync();
        const float inv = rsqrtf(ss * (1.0f / D) + a.eps);
#pragma unroll
        for (int j = 0; j < 16; ++j) x[j] += bf2f(a.g_post[ct * 16 + j]) * (m[j] * inv);
      }
      if (writer) {
        float* xo = a.x_out + (size_t)b * D + ct * 16;
#pragma unroll
        for (int q = 0; q < 4; ++q) reinterpret_cast<float4*>(xo)[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
        if (a.dump) {
          float* dd = a.dump + (size_t)b * D + ct * 16;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            reinterpret_cast<float4*>(dd)[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
        }
      }
      float ss = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) ss += x[j] * x[j];
      ss = warp_sum(ss);
      if (lane == 0) redn[warp] = ss;
      consumers_sync();
      ss = redn[0] + redn[1] + redn[2] + redn[3];
      consumers_sync();
      const float inv = rsqrtf(ss * (1.0f / D) + a.eps);
      // this thread's 16 columns go to shared memory if they are in the block's K range
      const int c0 = ct * 16;
      if (c0 >= kcta && c0 < kcta + Kc) {
        uint32_t w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          w[j] = pack_bf2(bf2f(a.g_next[c0 + 2 * j]) * (x[2 * j] * inv), bf2f(a.g_next[c0 + 2 * j + 1]) * (x[2 * j + 1] * inv));
        uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)b * XS + (c0 - kcta));
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
  }
  consumers_sync();

  // -------------------------------------------------------------- consumers: main loop
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
      const int s = it % G::STAGES;
      const uint32_t ph = (it / G::STAGES) & 1;
      // after any bounded wait gives up, every warp keeps walking the same loop (so all of them
      // reach every consumer barrier) but waits for nothing and computes nothing
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
        const unsigned char* st = stages + (size_t)s * G::STAGE_BYTES;
#pragma unroll
        for (int j = warp; j < G::STEPS; j += WS_CW) {
          const int kx = ch * G::KCH + j * G::KB;  // K offset of this step in the block's range
#pragma unroll
          for (int rt = 0; rt < NRT; ++rt) {
            const uint4 wa = *reinterpret_cast<const uint4*>(st + (rt * 16 + g) * G::RS + j * G::STEPB + t * 16);
            const uint4 wb = *reinterpret_cast<const uint4*>(st + (rt * 16 + g + 8) * G::RS + j * G::STEPB + t * 16);
            if constexpr (!FP4) {
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                const uint4 xv = *reinterpret_cast<const uint4*>(xs + (size_t)(nt * 8 + g) * XS + kx + 8 * t);
                mma_bf16_16816(acc[rt][nt], wa.x, wb.x, wa.y, wb.y, xv.x, xv.y);
                mma_bf16_16816(acc[rt][nt], wa.z, wb.z, wa.w, wb.w, xv.z, xv.w);
              }
            } else {
              const unsigned char* sc = st + G::RPT * G::RS;
              const uint32_t sa = *reinterpret_cast<const uint16_t*>(sc + (rt * 16 + g) * G::SCB + j * 8 + 2 * t);
              const uint32_t sb = *reinterpret_cast<const uint16_t*>(sc + (rt * 16 + g + 8) * G::SCB + j * 8 + 2 * t);
              const uint32_t s0a = ws_e4m3x2(sa & 0xFF), s1a = ws_e4m3x2(sa >> 8);
              const uint32_t s0b = ws_e4m3x2(sb & 0xFF), s1b = ws_e4m3x2(sb >> 8);
              const uint32_t wA[4] = {wa.x, wa.y, wa.z, wa.w};
              const uint32_t wB[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                uint32_t a01, a23, a45, a67, b01, b23, b45, b67;
                ws_e2m1x4(wA[q], a01, a23);
                ws_e2m1x4(wA[q] >> 16, a45, a67);
                ws_e2m1x4(wB[q], b01, b23);
                ws_e2m1x4(wB[q] >> 16, b45, b67);
                const uint32_t sA = q < 2 ? s0a : s1a, sB = q < 2 ? s0b : s1b;
                a01 = ws_hmul2(a01, sA); a23 = ws_hmul2(a23, sA); a45 = ws_hmul2(a45, sA); a67 = ws_hmul2(a67, sA);
                b01 = ws_hmul2(b01, sB); b23 = ws_hmul2(b23, sB); b45 = ws_hmul2(b45, sB); b67 = ws_hmul2(b67, sB);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                  const uint4 xv = *reinterpret_cast<const uint4*>(xs + (size_t)(nt * 8 + g) * XS + kx + 32 * t + 8 * q);
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
        const float Bv = res[cl * LDR + b], Cv = res[(16 + cl) * LDR + b], Xv = res[(32 + cl) * LDR + b];
        const float bx = round_bf(Bv * Xv);
        bf16* stt = a.conv_state + (size_t)a.row_slot[b] * CST * D + c;
        float win[CST];
#pragma unroll
        for (int j = 0; j < CST; ++j) win[j] = bf2f(stt[(size_t)j * D]);
        const bf16* w = a.conv_w + (size_t)c * TAPS;
        float z = 0.f;
#pragma unroll
        for (int k = 0; k < CST; ++k) z += bf2f(w[k]) * win[k];
        z += bf2f(w[CST]) * bx;
        a.y[(size_t)b * D + c] = f2bf(Cv * z);
#pragma unroll
        for (int j = 0; j < CST - 1; ++j) stt[(size_t)j * D] = f2bf(win[j + 1]);
        stt[(size_t)(CST - 1) * D] = f2bf(bx);
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
}

template <int EPI, bool FP4>
size_t ws_smem(int NT, int Kc) {
  using G = WsGeom<EPI, FP4>;
  const size_t x = (size_t)NT * 8 * (Kc + 32) * 2;
  return x + (size_t)G::STAGES * G::STAGE_BYTES + (size_t)WS_CW * G::NRT * NT * 128 * 4 +
         (size_t)G::NRT * 16 * NT * 8 * 4 + 2 * G::STAGES * 8;
}

static int g_num_sms = 0;

template <int EPI, bool FP4>
static cudaError_t launch_ws(const WsArgs& a, cudaStream_t s) {
  using G = WsGeom<EPI, FP4>;
  const int Kc = a.K / a.splits;
  if (Kc % G::KCH || a.K % a.splits) return cudaErrorInvalidValue;
  const int ntiles = (EPI == GEMV_SWIGLU) ? a.N / 8 : (EPI == GEMV_CONV ? D / 16 : a.N / 16);
  const int NT = a.rows <= 8 ? 1 : 2;
  const size_t smem = ws_smem<EPI, FP4>(NT, Kc);
  if (smem > (size_t)WS_SMEM_MAX) return cudaErrorInvalidValue;
  // blocks per K range: about two per SM in all, spread evenly over the tiles
  const int per_sm = smem <= 110 * 1024 ? 2 : 1;
  int gx = std::max(1, per_sm * g_num_sms / a.splits);
  gx = std::min(gx, ntiles);
  const int per = (ntiles + gx - 1) / gx;
  gx = (ntiles + per - 1) / per;
  dim3 grid(gx, a.splits);
  if (NT == 1) return launch(k_wstream<EPI, 1, FP4>, grid, dim3(WS_THREADS), smem, s, a);
  return launch(k_wstream<EPI, 2, FP4>, grid, dim3(WS_THREADS), smem, s, a);
}

cudaError_t wstream(int epi, int nvfp4, const WsArgs& a, cudaStream_t s) {
  if (a.rows > 16 || a.rows < 1) return cudaErrorInvalidValue;
  switch (epi) {
    case GEMV_PARTIAL: return nvfp4 ? launch_ws<GEMV_PARTIAL, true>(a, s) : launch_ws<GEMV_PARTIAL, false>(a, s);
    case GEMV_SWIGLU: return nvfp4 ? launch_ws<GEMV_SWIGLU, true>(a, s) : launch_ws<GEMV_SWIGLU, false>(a, s);
    case GEMV_CONV: return launch_ws<GEMV_CONV, false>(a, s);
    case GEMV_HEAD: return launch_ws<GEMV_HEAD, false>(a, s);
  }
  return cudaErrorInvalidValue;
}

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
