// Decode-time projections: y[b][n] = sum_k x[b][k] W[n][k] for a handful of streams b.
//
// The weights are the only large operand, so the kernel is built to stream them from HBM once
// at full bandwidth: each lane issues 16-byte loads straight from global memory (no L1
// allocation) and feeds them to the tensor cores as the 16-row A operand of an m16n8k16 MMA
// whose 8 columns are the streams. Within each 32-wide K block a lane owns 8 consecutive
// weights of its row; the activations in shared memory are read with the same K permutation,
// so the products pair up correctly and every load is a full 16-byte vector. A block's 8 warps
// split its K range; partial sums are reduced in shared memory and handed to a fused epilogue:
//   PARTIAL - fp32 partial sums per K split (the consumer adds the splits)
//   SWIGLU  - rows j of w1 and w3 in one tile; u = silu(w1 x) * (w3 x)
//   CONV    - rows c of B, C and x of in_proj in three tiles; then the gated 7-tap conv of the
//             stream's state and the state shift (no separate conv launch)
//   HEAD    - tied head logits and a running greedy argmax per stream
// NVFP4 weights are expanded in registers from E2M1 codes and E4M3 block scales to exact bf16
// values; the fp32 tensor scale multiplies the finished dot products.
#include "kernels.cuh"

namespace lfm3 {

constexpr int GV_WARPS = 8;

// E2M1 magnitude (3 bits) -> bf16 bit patterns, split into high and low bytes, as byte-permute
// tables: 0, 0.5, 1, 1.5, 2, 3, 4, 6.
constexpr uint32_t E2M1_HI_LO = 0x3F3F3F00u, E2M1_HI_HI = 0x40404040u;
constexpr uint32_t E2M1_LO_LO = 0xC0800000u, E2M1_LO_HI = 0xC0804000u;

// Four E2M1 codes (the 16 low bits of w, code j in nibble j) -> two bf16x2 words (codes 0,1 and
// 2,3), exact.
DEVI void e2m1x4_to_bf16(uint32_t w, uint32_t& o01, uint32_t& o23) {
  const uint32_t sel = w & 0x7777u;
  const uint32_t hi = __byte_perm(E2M1_HI_LO, E2M1_HI_HI, sel);
  const uint32_t lo = __byte_perm(E2M1_LO_LO, E2M1_LO_HI, sel);
  o01 = __byte_perm(lo, hi, 0x5140);
  o23 = __byte_perm(lo, hi, 0x7362);
  const uint32_t s = w & 0x8888u;
  o01 |= ((s << 12) & 0x8000u) | ((s << 24) & 0x80000000u);
  o23 |= ((s << 4) & 0x8000u) | ((s << 16) & 0x80000000u);
}

// E4M3 byte -> bf16 (exact for the normal and subnormal range; NaN not expected).
DEVI uint32_t e4m3_to_bf16x2(uint32_t b) {
  const uint32_t s = (b & 0x80u) << 8;
  const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
  uint32_t bits;
  if (e == 0) {
    // subnormal: m/8 * 2^-6 = m * 2^-9
    const float f = (float)m * (1.0f / 512.0f);
    bits = __float_as_uint(f) >> 16;
  } else {
    bits = ((e + 120u) << 7) | (m << 4);
  }
  bits |= s;
  return bits | (bits << 16);
}

DEVI uint32_t hmul2_bf(uint32_t a, uint32_t b) {
  __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a), y = *reinterpret_cast<__nv_bfloat162*>(&b);
  __nv_bfloat162 r = __hmul2(x, y);
  return *reinterpret_cast<uint32_t*>(&r);
}

template <int EPI>
struct EpiRows { static constexpr int NRT = (EPI == GEMV_CONV) ? 3 : 1; };

// Row of tile rt, fragment row g (0..15) of block `blk`.
template <int EPI>
DEVI int tile_row(int blk, int rt, int g, int& which) {
  which = 0;
  if constexpr (EPI == GEMV_SWIGLU) {
    which = g >= 8;            // rows 0..7 from w1, 8..15 from w3
    return blk * 8 + (g & 7);
  } else if constexpr (EPI == GEMV_CONV) {
    return rt * D + blk * 16 + g;  // B | C | x blocks of in_proj
  } else {
    return blk * 16 + g;
  }
}

template <int EPI, int NT, bool FP4>
__global__ void __launch_bounds__(256) k_gemv(const GemvArgs a) {
  constexpr int NRT = EpiRows<EPI>::NRT;
  constexpr int KB = FP4 ? 128 : 32;         // K elements per lane-block step
  constexpr int U = FP4 ? 1 : (NRT == 1 ? 4 : 2);
  extern __shared__ __align__(16) unsigned char smem[];
  bf16* xs = reinterpret_cast<bf16*>(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  // This block covers K range [blockIdx.y * Kc, +Kc) in KB-wide steps; warp w takes steps
  // w, w + 8, w + 16, ... (so Kc only has to be a multiple of KB).
  const int Kc = a.K / a.splits, nsteps = Kc / KB;
  const int nmine = nsteps > warp ? (nsteps - warp + GV_WARPS - 1) / GV_WARPS : 0;
  const int XS = Kc + 8;                     // padded row stride (elements)
  const int kcta = blockIdx.y * Kc;

  // row pointers of this lane (rows g and g+8 of every tile), at this warp's first step
  const unsigned char* rp0[NRT];
  const unsigned char* rp1[NRT];
  const unsigned char* sp0[NRT];
  const unsigned char* sp1[NRT];
#pragma unroll
  for (int rt = 0; rt < NRT; ++rt) {
    int w0, w1;
    const int r0 = tile_row<EPI>(blockIdx.x, rt, g, w0), r1 = tile_row<EPI>(blockIdx.x, rt, g + 8, w1);
    const int k0 = kcta + warp * KB;
    if constexpr (FP4) {
      const uint8_t* c0 = (EPI == GEMV_SWIGLU && w0) ? a.codes3 : a.codes;
      const uint8_t* c1 = (EPI == GEMV_SWIGLU && w1) ? a.codes3 : a.codes;
      const uint8_t* s0 = (EPI == GEMV_SWIGLU && w0) ? a.scales3 : a.scales;
      const uint8_t* s1 = (EPI == GEMV_SWIGLU && w1) ? a.scales3 : a.scales;
      rp0[rt] = c0 + (size_t)r0 * (a.K / 2) + (k0 + 32 * t) / 2;
      rp1[rt] = c1 + (size_t)r1 * (a.K / 2) + (k0 + 32 * t) / 2;
      sp0[rt] = s0 + (size_t)r0 * (a.K / 16) + (k0 + 32 * t) / 16;
      sp1[rt] = s1 + (size_t)r1 * (a.K / 16) + (k0 + 32 * t) / 16;
    } else {
      const bf16* m0 = (EPI == GEMV_SWIGLU && w0) ? a.w3 : a.w;
      const bf16* m1 = (EPI == GEMV_SWIGLU && w1) ? a.w3 : a.w;
      rp0[rt] = reinterpret_cast<const unsigned char*>(m0 + (size_t)r0 * a.K + k0 + 8 * t);
      rp1[rt] = reinterpret_cast<const unsigned char*>(m1 + (size_t)r1 * a.K + k0 + 8 * t);
      sp0[rt] = sp1[rt] = nullptr;
    }
  }
  // bytes between this warp's consecutive steps along a row (steps are 8 apart)
  constexpr int STEP = GV_WARPS * (FP4 ? KB / 2 : KB * 2);
  constexpr int SSTEP = GV_WARPS * (KB / 16);

  float acc[NRT][NT][4];
#pragma unroll
  for (int rt = 0; rt < NRT; ++rt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[rt][nt][j] = 0.f;

  // first weight group is issued before waiting on the previous kernel (weights are constant)
  uint4 wa[U][NRT], wb[U][NRT];
  uint16_t sa[U][NRT], sb[U][NRT];
  auto load_group = [&](int i0) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (i0 + u < nmine) {
#pragma unroll
        for (int rt = 0; rt < NRT; ++rt) {
          wa[u][rt] = ldg_stream(rp0[rt] + (size_t)(i0 + u) * STEP);
          wb[u][rt] = ldg_stream(rp1[rt] + (size_t)(i0 + u) * STEP);
          if constexpr (FP4) {
            sa[u][rt] = *reinterpret_cast<const uint16_t*>(sp0[rt] + (size_t)(i0 + u) * SSTEP);
            sb[u][rt] = *reinterpret_cast<const uint16_t*>(sp1[rt] + (size_t)(i0 + u) * SSTEP);
          }
        }
      }
    }
  };
  load_group(0);

  pdl_wait();
  pdl_launch_dependents();

  // activations of this block's K range -> shared memory (streams past `rows` are zero)
  {
    const int chunks = Kc / 8;
    for (int idx = tid; idx < NT * 8 * chunks; idx += blockDim.x) {
      const int b = idx / chunks, c = idx - b * chunks;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (b < a.rows) v = ldg16(a.x + (size_t)b * a.K + kcta + c * 8);
      *reinterpret_cast<uint4*>(xs + (size_t)b * XS + c * 8) = v;
    }
  }
  __syncthreads();

  for (int i0 = 0; i0 < nmine; i0 += U) {
    uint4 ca[U][NRT], cb[U][NRT];
    uint16_t csa[U][NRT], csb[U][NRT];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int rt = 0; rt < NRT; ++rt) {
        ca[u][rt] = wa[u][rt]; cb[u][rt] = wb[u][rt];
        if constexpr (FP4) { csa[u][rt] = sa[u][rt]; csb[u][rt] = sb[u][rt]; }
      }
    if (i0 + U < nmine) load_group(i0 + U);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (i0 + u >= nmine) break;
      const int kx = (warp + (i0 + u) * GV_WARPS) * KB;   // offset of this step in the block's range
      if constexpr (!FP4) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint4 xv = *reinterpret_cast<const uint4*>(xs + (size_t)(nt * 8 + g) * XS + kx + 8 * t);
#pragma unroll
          for (int rt = 0; rt < NRT; ++rt) {
            mma_bf16_16816(acc[rt][nt], ca[u][rt].x, cb[u][rt].x, ca[u][rt].y, cb[u][rt].y, xv.x, xv.y);
            mma_bf16_16816(acc[rt][nt], ca[u][rt].z, cb[u][rt].z, ca[u][rt].w, cb[u][rt].w, xv.z, xv.w);
          }
        }
      } else {
        // 32 codes per row per lane: bytes 0..15, scale 0 for codes 0..15, scale 1 for 16..31
#pragma unroll
        for (int rt = 0; rt < NRT; ++rt) {
          const uint32_t s0a = e4m3_to_bf16x2(csa[u][rt] & 0xFF), s1a = e4m3_to_bf16x2(csa[u][rt] >> 8);
          const uint32_t s0b = e4m3_to_bf16x2(csb[u][rt] & 0xFF), s1b = e4m3_to_bf16x2(csb[u][rt] >> 8);
          const uint32_t wA[4] = {ca[u][rt].x, ca[u][rt].y, ca[u][rt].z, ca[u][rt].w};
          const uint32_t wB[4] = {cb[u][rt].x, cb[u][rt].y, cb[u][rt].z, cb[u][rt].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {     // word q holds codes 8q..8q+7
            uint32_t a01, a23, a45, a67, b01, b23, b45, b67;
            e2m1x4_to_bf16(wA[q], a01, a23);
            e2m1x4_to_bf16(wA[q] >> 16, a45, a67);
            e2m1x4_to_bf16(wB[q], b01, b23);
            e2m1x4_to_bf16(wB[q] >> 16, b45, b67);
            const uint32_t sA = q < 2 ? s0a : s1a, sB = q < 2 ? s0b : s1b;
            a01 = hmul2_bf(a01, sA); a23 = hmul2_bf(a23, sA); a45 = hmul2_bf(a45, sA); a67 = hmul2_bf(a67, sA);
            b01 = hmul2_bf(b01, sB); b23 = hmul2_bf(b23, sB); b45 = hmul2_bf(b45, sB); b67 = hmul2_bf(b67, sB);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              // codes 8q..8q+7 of this lane sit at K offset 32t + 8q .. +7 of the step
              const uint4 xv = *reinterpret_cast<const uint4*>(xs + (size_t)(nt * 8 + g) * XS + kx + 32 * t + 8 * q);
              mma_bf16_16816(acc[rt][nt], a01, b01, a23, b23, xv.x, xv.y);
              mma_bf16_16816(acc[rt][nt], a45, b45, a67, b67, xv.z, xv.w);
            }
          }
        }
      }
    }
  }

  // cross-warp reduction in shared memory: red[warp][rt][nt][lane][4]
  __syncthreads();
  float* red = reinterpret_cast<float*>(smem);
#pragma unroll
  for (int rt = 0; rt < NRT; ++rt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      *reinterpret_cast<float4*>(red + ((((size_t)warp * NRT + rt) * NT + nt) * 32 + lane) * 4) =
          make_float4(acc[rt][nt][0], acc[rt][nt][1], acc[rt][nt][2], acc[rt][nt][3]);
  __syncthreads();
  // res[row (NRT*16)][col (NT*8)]
  float* res = red + GV_WARPS * NRT * NT * 128;
  for (int e = tid; e < NRT * NT * 128; e += blockDim.x) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < GV_WARPS; ++w) s += red[(size_t)w * NRT * NT * 128 + e];
    const int j = e & 3, ln = (e >> 2) & 31, nt = (e >> 7) % NT, rt = (e >> 7) / NT;
    const int row = rt * 16 + (ln >> 2) + (j >= 2 ? 8 : 0);
    const int col = nt * 8 + 2 * (ln & 3) + (j & 1);
    res[row * (NT * 8) + col] = FP4 ? s * a.tscale : s;
  }
  __syncthreads();
  constexpr int LDR = NT * 8;

  if constexpr (EPI == GEMV_PARTIAL) {
    for (int e = tid; e < 16 * a.rows; e += blockDim.x) {
      const int row = e & 15, b = e >> 4;
      a.part[((size_t)blockIdx.y * a.rows + b) * a.N + blockIdx.x * 16 + row] = res[row * LDR + b];
    }
  } else if constexpr (EPI == GEMV_SWIGLU) {
    for (int e = tid; e < 8 * a.rows; e += blockDim.x) {
      const int j = e & 7, b = e >> 3;
      const float h1 = res[j * LDR + b], h3 = res[(j + 8) * LDR + b];
      a.out[(size_t)b * a.N + blockIdx.x * 8 + j] = f2bf(siluf_(h1) * h3);
    }
  } else if constexpr (EPI == GEMV_CONV) {
    for (int e = tid; e < 16 * a.rows; e += blockDim.x) {
      const int cl = e & 15, b = e >> 4, c = blockIdx.x * 16 + cl;
      const float Bv = res[cl * LDR + b];
      const float Cv = res[(16 + cl) * LDR + b];
      const float Xv = res[(32 + cl) * LDR + b];
      const float bx = round_bf(Bv * Xv);
      bf16* st = a.conv_state + (size_t)a.row_slot[b] * CST * D + c;
      float win[CST];
#pragma unroll
      for (int j = 0; j < CST; ++j) win[j] = bf2f(st[(size_t)j * D]);
      const bf16* w = a.conv_w + (size_t)c * TAPS;
      float z = 0.f;
#pragma unroll
      for (int k = 0; k < CST; ++k) z += bf2f(w[k]) * win[k];
      z += bf2f(w[CST]) * bx;
      a.y[(size_t)b * D + c] = f2bf(Cv * z);
#pragma unroll
      for (int j = 0; j < CST - 1; ++j) st[(size_t)j * D] = f2bf(win[j + 1]);
      st[(size_t)(CST - 1) * D] = f2bf(bx);
    }
  } else if constexpr (EPI == GEMV_HEAD) {
    for (int b = warp; b < a.rows; b += GV_WARPS) {
      float v = lane < 16 ? res[lane * LDR + b] : -INFINITY;
      const int n = blockIdx.x * 16 + lane;
      if (lane < 16 && a.part) a.part[(size_t)b * a.N + n] = v;
      // max, then the lowest row holding it
      float m = warp_max(v);
      unsigned ballot = __ballot_sync(0xffffffffu, v == m && lane < 16);
      if (lane == 0) {
        const int idx = blockIdx.x * 16 + (__ffs(ballot) - 1);
        uint32_t u = __float_as_uint(m);
        u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
        const unsigned long long key = ((unsigned long long)u << 32) | (0xffffffffu - (uint32_t)idx);
        atomicMax(a.amax + b, key);
      }
    }
  }
}

template <int EPI, bool FP4>
static cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t s) {
  constexpr int NRT = EpiRows<EPI>::NRT;
  const int Kc = a.K / a.splits;
  int gx;
  if (EPI == GEMV_SWIGLU) gx = a.N / 8;
  else if (EPI == GEMV_CONV) gx = D / 16;
  else gx = a.N / 16;
  dim3 grid(gx, a.splits);
  auto smem_for = [&](int nt) {
    size_t xb = (size_t)nt * 8 * (Kc + 8) * 2;
    size_t rb = (size_t)GV_WARPS * NRT * nt * 128 * 4 + (size_t)NRT * 16 * nt * 8 * 4;
    return xb > rb ? xb : rb;
  };
  if (a.rows <= 8) return launch(k_gemv<EPI, 1, FP4>, grid, dim3(256), smem_for(1), s, a);
  return launch(k_gemv<EPI, 2, FP4>, grid, dim3(256), smem_for(2), s, a);
}

// Largest dynamic shared memory any launch asks for: NT = 2, the whole K = 7680 range is never
// one block (w2 is split), so K = 2048 with 16 streams bounds it.
constexpr int GEMV_SMEM_MAX = 2 * 8 * (2048 + 8) * 2;

template <int EPI, bool FP4>
static cudaError_t set_attr() {
  cudaError_t e = cudaFuncSetAttribute(k_gemv<EPI, 1, FP4>, cudaFuncAttributeMaxDynamicSharedMemorySize, GEMV_SMEM_MAX);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(k_gemv<EPI, 2, FP4>, cudaFuncAttributeMaxDynamicSharedMemorySize, GEMV_SMEM_MAX);
}

cudaError_t gemv_init() {
  cudaError_t e;
  if ((e = set_attr<GEMV_PARTIAL, false>()) != cudaSuccess) return e;
  if ((e = set_attr<GEMV_PARTIAL, true>()) != cudaSuccess) return e;
  if ((e = set_attr<GEMV_SWIGLU, false>()) != cudaSuccess) return e;
  if ((e = set_attr<GEMV_SWIGLU, true>()) != cudaSuccess) return e;
  if ((e = set_attr<GEMV_CONV, false>()) != cudaSuccess) return e;
  return set_attr<GEMV_HEAD, false>();
}

cudaError_t gemv(int epi, int nvfp4, const GemvArgs& a, cudaStream_t s) {
  if (a.rows > 16) return cudaErrorInvalidValue;
  switch (epi) {
    case GEMV_PARTIAL: return nvfp4 ? launch_gemv<GEMV_PARTIAL, true>(a, s) : launch_gemv<GEMV_PARTIAL, false>(a, s);
    case GEMV_SWIGLU: return nvfp4 ? launch_gemv<GEMV_SWIGLU, true>(a, s) : launch_gemv<GEMV_SWIGLU, false>(a, s);
    case GEMV_CONV: return launch_gemv<GEMV_CONV, false>(a, s);
    case GEMV_HEAD: return launch_gemv<GEMV_HEAD, false>(a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace lfm3
