// Prefill projections on the 5th-generation tensor cores: C[M][N] = alpha * A[M][K] . W[N][K]^T
// with A the bf16 activations of a prompt chunk and W a bf16 weight, both K-major.
//
// Persistent blocks (one per SM, 6 warps) walk 128 x BN output tiles (BN = 128 or 256):
//   warp 0      TMA producer: 128x64 A box and BNx64 W box per stage (128-byte swizzle), into a
//               4- or 6-stage ring guarded by full/empty mbarriers;
//   warp 1      allocates 2 x BN TMEM columns (two accumulators); one elected lane issues
//               tcgen05.mma (kind::f16, M=128, N=BN, K=16 per instruction, fp32 accumulate in TMEM),
//               commits each stage back to the producer and each finished accumulator to the
//               epilogue, and moves on to the next tile in the other accumulator;
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 32 columns at a time (warp w reads TMEM lanes
//               32*(w%4) ..), apply the fused epilogue, store, release the accumulator.
// Epilogues: fp32 out, bf16 out, and SwiGLU (the tile's 256 columns are 128 rows of w1 and the
// same 128 rows of w3: u = silu(alpha a) * (alpha b), bf16).
// Every mbarrier wait is bounded; a wait that gives up sets the device error word and the
// block runs to completion without further MMAs so that TMEM is always released.
#include <cudaTypedefs.h>

#include <algorithm>

#include <cstdlib>

#include "kernels.cuh"

namespace lfm3 {

constexpr int GM_BM = 128, GM_BK = 64;

static PFN_cuTensorMapEncodeTiled_v12000 p_encode = nullptr;

bool tma_init() {
  if (p_encode) return true;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return false;
  p_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  if (!p_encode) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (cols * 2) % 16) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = p_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- PTX wrappers
DEVI void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
DEVI void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
DEVI void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// K-major operand tile in shared memory, 128-byte swizzle: rows of 128 B, 8-row atoms 1024 B
// apart (SBO), descriptor version 1, layout type 2 (SWIZZLE_128B).
DEVI uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

DEVI void umma_f16(uint32_t tmem_d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(
          tmem_d),
      "l"(ad), "l"(bd), "r"(idesc), "r"(accum));
}
DEVI void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

DEVI void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%"
      "19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

struct GemmArgs {
  int M, N, K, ld;
  void* out;
  float alpha;
  int* err;
};

template <int BN>
struct GemmGeom {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr uint32_t A_BYTES = GM_BM * GM_BK * 2;
  static constexpr uint32_t B_BYTES = BN * GM_BK * 2;
  static constexpr uint32_t STAGE = A_BYTES + B_BYTES;
};

// Persistent: block b takes tiles b, b + gridDim.x, ... (M tiles fastest, so consecutive blocks
// share a weight tile through L2). TMEM holds two BN-column accumulators: the MMA thread fills
// one while the epilogue warps drain the other (acc_full / acc_empty barriers).
template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1) k_gemm(const __grid_constant__ CUtensorMap ta,
                                                 const __grid_constant__ CUtensorMap tb,
                                                 const __grid_constant__ CUtensorMap tb3, const GemmArgs g) {
  using G = GemmGeom<BN>;
  constexpr int S = G::STAGES;
  constexpr int NOUT = EPI == GEMM_SWIGLU ? BN / 2 : BN;  // output columns per tile
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * G::STAGE);
  const uint32_t full0 = su32(bars), empty0 = su32(bars + S);
  const uint32_t accf0 = su32(bars + 2 * S), acce0 = su32(bars + 2 * S + 2);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (g.M + GM_BM - 1) / GM_BM, num_n = (g.N + NOUT - 1) / NOUT;
  const int ntiles = num_m * num_n;
  const int nk = g.K / GM_BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf0 + 8 * b, 1);
      mbar_init(acce0 + 8 * b, 4);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&ta)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tb)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                 "r"(2 * BN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int m0 = (tile % num_m) * GM_BM, n0 = (tile / num_m) * NOUT;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1, g.err)) {
            ok = false;
            break;
          }
          const uint32_t a_s = su32(smem + s * G::STAGE), b_s = a_s + G::A_BYTES;
          mbar_expect_tx(full0 + 8 * s, G::STAGE);
          tma_load_2d(a_s, &ta, kb * GM_BK, m0, full0 + 8 * s);
          if constexpr (EPI == GEMM_SWIGLU) {
            tma_load_2d(b_s, &tb, kb * GM_BK, n0, full0 + 8 * s);
            tma_load_2d(b_s + G::B_BYTES / 2, &tb3, kb * GM_BK, n0, full0 + 8 * s);
          } else {
            tma_load_2d(b_s, &tb, kb * GM_BK, n0, full0 + 8 * s);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                 ((uint32_t)(GM_BM >> 4) << 24);
      int it = 0, i = 0, after_fail = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
        const int buf = i & 1;
        if (ok && !mbar_wait(acce0 + 8 * buf, ((i >> 1) & 1) ^ 1, g.err)) ok = false;
        tc_fence_after();
        const uint32_t td = tmem + buf * BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          // after a failure keep draining (bounded) the stages the producer may still have in
          // flight - it runs at most S ahead - so no copy lands after the block exits
          if (!ok && ++after_fail > S) break;
          const bool got = mbar_wait(full0 + 8 * s, ph, g.err);
          ok = ok && got;
          tc_fence_after();
          if (ok) {
            const uint64_t ad = sw128_desc(su32(smem + s * G::STAGE));
            const uint64_t bd = sw128_desc(su32(smem + s * G::STAGE + G::A_BYTES));
#pragma unroll
            for (int k = 0; k < GM_BK / 16; ++k) umma_f16(td, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0);
          }
          umma_commit(empty0 + 8 * s);
        }
        umma_commit(accf0 + 8 * buf);
        if (after_fail > S) break;
      }
    }
  } else {
    const int quarter = warp & 3;
    int i = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++i) {
      const int buf = i & 1;
      const int m0 = (tile % num_m) * GM_BM, n0 = (tile / num_m) * NOUT;
      const int row = m0 + quarter * 32 + lane;
      ok = mbar_wait(accf0 + 8 * buf, (i >> 1) & 1, g.err);
      tc_fence_after();
      if (!ok) break;
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + buf * BN;
      if constexpr (EPI == GEMM_SWIGLU) {
        bf16* out = reinterpret_cast<bf16*>(g.out);
#pragma unroll 1
        for (int c = 0; c < BN / 64; ++c) {
          float va[32], vb[32];
          tmem_ld32(tbase + c * 32, va);
          tmem_ld32(tbase + BN / 2 + c * 32, vb);
          if (row < g.M) {
            uint4* dst = reinterpret_cast<uint4*>(out + (size_t)row * g.ld + n0 + c * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int j = q * 8 + e * 2;
                w[e] = pack_bf2(siluf_(g.alpha * va[j]) * (g.alpha * vb[j]),
                                siluf_(g.alpha * va[j + 1]) * (g.alpha * vb[j + 1]));
              }
              dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          float v[32];
          tmem_ld32(tbase + c * 32, v);
          const int col = n0 + c * 32;
          if (row < g.M && col < g.N) {
            if constexpr (EPI == GEMM_F32) {
              float* dst = reinterpret_cast<float*>(g.out) + (size_t)row * g.ld + col;
              if (col + 32 <= g.N) {
#pragma unroll
                for (int q = 0; q < 8; ++q)
                  reinterpret_cast<float4*>(dst)[q] = make_float4(g.alpha * v[4 * q], g.alpha * v[4 * q + 1],
                                                                  g.alpha * v[4 * q + 2], g.alpha * v[4 * q + 3]);
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (j < g.N - col) dst[j] = g.alpha * v[j];
              }
            } else {
              bf16* dst = reinterpret_cast<bf16*>(g.out) + (size_t)row * g.ld + col;
              if (col + 32 <= g.N) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  uint32_t w[4];
#pragma unroll
                  for (int e = 0; e < 4; ++e) w[e] = pack_bf2(g.alpha * v[q * 8 + 2 * e], g.alpha * v[q * 8 + 2 * e + 1]);
                  reinterpret_cast<uint4*>(dst)[q] = make_uint4(w[0], w[1], w[2], w[3]);
                }
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (j < g.N - col) dst[j] = f2bf(g.alpha * v[j]);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce0 + 8 * buf);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * BN));
}

template <int BN>
constexpr size_t gemm_smem() { return 1024 + GemmGeom<BN>::STAGES * (size_t)GemmGeom<BN>::STAGE + 256; }

static int g_gemm_sms = 0;

template <int BN, int EPI>
static cudaError_t launch_gemm(const GemmPlan& p, int M, int* err, cudaStream_t s) {
  constexpr size_t smem = gemm_smem<BN>();
  auto k = k_gemm<BN, EPI>;
  GemmArgs g{M, p.N, p.K, p.ld, p.out, p.alpha, err};
  const int ntile = EPI == GEMM_SWIGLU ? BN / 2 : BN;
  const int tiles = ((p.N + ntile - 1) / ntile) * ((M + GM_BM - 1) / GM_BM);
  dim3 grid(std::min(tiles, g_gemm_sms > 0 ? g_gemm_sms : 148));
  return launch(k, grid, dim3(192), smem, s, p.a, p.b, EPI == GEMM_SWIGLU ? p.b3 : p.b, g);
}

// Output widths from which a tile is 256 columns wide (fewer, more L2-efficient tiles) rather than
// 128 (more tiles to spread over the SMs); LFM3_GEMM_WIDE_MIN_N overrides.
static int g_gemm_wide_min = 2048;  // measured: 8k prefill 37.8 -> 34.6 ms against 4097

cudaError_t gemm_init() {
  if (const char* v = getenv("LFM3_GEMM_WIDE_MIN_N")) g_gemm_wide_min = atoi(v);
  cudaError_t e;
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&g_gemm_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(k_gemm<128, GEMM_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_smem<128>())))
    return e;
  if ((e = cudaFuncSetAttribute(k_gemm<256, GEMM_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_smem<256>())))
    return e;
  if ((e = cudaFuncSetAttribute(k_gemm<128, GEMM_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_smem<128>())))
    return e;
  if ((e = cudaFuncSetAttribute(k_gemm<256, GEMM_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_smem<256>())))
    return e;
  return cudaFuncSetAttribute(k_gemm<256, GEMM_SWIGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_smem<256>());
}

bool gemm_wide(int N) { return N >= g_gemm_wide_min; }

cudaError_t gemm(const GemmPlan& p, int M, int* err, cudaStream_t s) {
  if (p.K % GM_BK) return cudaErrorInvalidValue;
  switch (p.epi) {
    case GEMM_F32: return gemm_wide(p.N) ? launch_gemm<256, GEMM_F32>(p, M, err, s) : launch_gemm<128, GEMM_F32>(p, M, err, s);
    case GEMM_BF16: return gemm_wide(p.N) ? launch_gemm<256, GEMM_BF16>(p, M, err, s) : launch_gemm<128, GEMM_BF16>(p, M, err, s);
    case GEMM_SWIGLU: return launch_gemm<256, GEMM_SWIGLU>(p, M, err, s);
  }
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------- NVFP4 -> bf16 (prefill)
// w = e2m1(code) * e4m3(scale): exact in bf16; the tensor scale is the GEMM's alpha.
__global__ void __launch_bounds__(256) k_nvfp4_to_bf16(const uint8_t* __restrict__ codes,
                                                       const uint8_t* __restrict__ scales, long n8, int K,
                                                       bf16* __restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;  // group of 8 weights
  if (i >= n8) return;
  const uint32_t w = *reinterpret_cast<const uint32_t*>(codes + i * 4);
  const long e0 = i * 8;
  const long row = e0 / K, col = e0 % K;
  const uint8_t sb = scales[row * (K / 16) + col / 16];
  const uint32_t se = (sb >> 3) & 0xF, sm = sb & 7;
  float sc = se == 0 ? (float)sm * (1.0f / 512.0f) : __uint_as_float(((se + 120u) << 23) | (sm << 20));
  if (sb & 0x80) sc = -sc;
  // E2M1: exponent field e (bias 1), mantissa m; e == 0 is 0.5 * m
  auto e2m1 = [](uint32_t c) -> float {
    const uint32_t e = (c >> 1) & 3, m = c & 1;
    const float mag = e == 0 ? 0.5f * (float)m : __uint_as_float(((e + 126u) << 23) | (m << 22));
    return (c & 8) ? -mag : mag;
  };
  uint32_t o[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t c0 = (w >> (8 * j)) & 0xF, c1 = (w >> (8 * j + 4)) & 0xF;
    o[j] = pack_bf2(e2m1(c0) * sc, e2m1(c1) * sc);
  }
  reinterpret_cast<uint4*>(out)[i] = make_uint4(o[0], o[1], o[2], o[3]);
}

cudaError_t nvfp4_to_bf16(const uint8_t* codes, const uint8_t* scales, float tscale, int N, int K, bf16* out,
                          cudaStream_t s) {
  (void)tscale;
  const long n8 = (long)N * K / 8;
  return launch(k_nvfp4_to_bf16, dim3((unsigned)((n8 + 255) / 256)), dim3(256), 0, s, codes, scales, n8, K, out);
}

}  // namespace lfm3
