// Projections on the 5th-generation tensor cores: C[M][N] = alpha * A[M][K] . W[N][K]^T with A
// the bf16 activations of a prompt chunk (or of a decode batch over 16 rows) and W a bf16 weight,
// both K-major. k_gemm_q4 (further down) takes NVFP4 weights and expands them on the chip.
//
// Persistent blocks (one per SM, 6 warps) walk output tiles:
//   warp 0      TMA producer: A and W boxes of 64 K-columns per stage (128-byte swizzle) into a ring
//               guarded by full/empty mbarriers;
//   warp 1      allocates two accumulators in TMEM; one elected lane issues tcgen05.mma (kind::f16,
//               K=16 per instruction, fp32 accumulate), commits each stage back to the producer and
//               each finished accumulator to the epilogue, and moves on to the next tile in the
//               other accumulator;
//   warps 2..5  epilogue: tcgen05.ld of their 32 TMEM lanes (warp w reads lanes 32*(w%4) ..), the
//               fused epilogue, a 128-byte-swizzled staging tile in shared memory and a TMA tensor
//               store per 32 rows x 128 bytes; then the accumulator is released.
// k_gemm: one SM per 128 x BN tile (BN = 128 or 256). k_gemm2: a cluster of two SMs per 256 x 256
// tile (tcgen05 cta_group::2), each SM staging its 128 rows of A and half of the weight rows.
// Epilogues: fp32 out, bf16 out, SwiGLU (the tile's BN columns are BN/2 rows of w1 and the same
// rows of w3: u = silu(alpha a) * (alpha b), bf16), and the head (fp32 logits, optional, and each
// row's maximum and first index as a packed argmax key). A batch of at most 128 rows may split an
// fp32 output along K: split s writes its partial sums at out + s * M * ld with plain stores, and
// the consumer adds the splits in order.
// Every mbarrier wait is bounded; a wait that gives up sets the device error word, and the MMA
// thread drains (bounded) the stages still in flight so that TMEM is always released.
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

bool make_tmap_out(CUtensorMap* m, void* base, bool fp32, uint64_t rows, uint64_t cols, uint64_t ld) {
  if (!p_encode) return false;
  const uint64_t es = fp32 ? 4 : 2;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (ld * es) % 16 || cols > ld) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * es};
  cuuint32_t box[2] = {(cuuint32_t)(128 / es), 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = p_encode(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
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

// Two 64-column TMEM loads (this thread's lane) behind a single wait, in one statement so that no
// use of the registers can be scheduled before the wait.
DEVI void tmem_ld64x2(uint32_t ta, uint32_t tb, float* va, float* vb) {
  uint32_t r[128];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%128];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,"
      "%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,"
      "%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%129];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]),
        "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]),
        "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
        "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]),
        "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]),
        "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]),
        "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]),
        "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]),
        "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]),
        "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]),
        "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]),
        "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]),
        "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]),
        "=r"(r[126]), "=r"(r[127])
      : "r"(ta), "r"(tb));
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    va[i] = __uint_as_float(r[i]);
    vb[i] = __uint_as_float(r[64 + i]);
  }
}

// SiLU for the GEMM epilogue: the fast division (the argument of the exponential is capped so that
// the divisor stays finite; silu(x) for x < -80 is 0 at fp32 precision anyway).
DEVI float silu_fast(float x) { return __fdividef(x, 1.f + __expf(fminf(-x, 80.f))); }

struct GemmArgs {
  int M, N, K, ld;
  void* out;
  float alpha;
  int* err;
  int splits;                  // K splits (fp32 partial sums at out + s * M * ld)
  unsigned long long* amax;    // GEMM_HEAD
  int f16out;                  // GEMM_SWIGLU: the bf16-rounded products stored as f16
  int w_const;                 // the weights are not written by an earlier kernel of the stream
};

// Tile t of a launch: M tiles fastest (consecutive blocks share a weight tile through L2), then
// N tiles, then K splits; the split's 64-column K blocks are [kb0, kb1).
struct GemmTile { int m0, n0, s, kb0, kb1; };
DEVI GemmTile gemm_tile(int t, int num_m, int num_n, int bm, int nout, int nk, int splits) {
  GemmTile r;
  r.m0 = (t % num_m) * bm;
  const int q = t / num_m;
  r.n0 = (q % num_n) * nout;
  r.s = q / num_n;
  r.kb0 = r.s * nk / splits;
  r.kb1 = (r.s + 1) * nk / splits;
  return r;
}

template <int BN>
struct GemmGeom {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr uint32_t A_BYTES = GM_BM * GM_BK * 2;
  static constexpr uint32_t B_BYTES = BN * GM_BK * 2;
  static constexpr uint32_t STAGE = A_BYTES + B_BYTES;
};

DEVI void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(src)
               : "memory");
}
DEVI void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
DEVI void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
DEVI void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
DEVI void sts128(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

constexpr uint32_t GM_STG_WARP = 2 * 4096;  // per epilogue warp: two 32-row x 128-byte staging tiles
constexpr uint32_t GM_STG = 4 * GM_STG_WARP;

// Epilogue of one 128-row x BN-column accumulator, run by each of the 4 epilogue warps on its 32
// rows [wrow0, wrow0 + 32) (TMEM lanes of its quarter; tbase points at the quarter and the
// accumulator's first column). Per 128 output bytes of a row (32 fp32 or 64 bf16 columns) the
// warp stages its 32 rows in shared memory with the 128-byte swizzle and writes them with one TMA
// tensor store, so each row segment leaves the SM as whole lines; the two staging tiles alternate,
// and a tile is rewritten only once the store issued from it two steps earlier has read it. Rows
// past M (the last tile of a ragged chunk) take plain per-thread stores instead; column chunks past
// N are skipped, and a chunk that straddles N is clipped by the store.
template <int BN, int EPI>
DEVI void gemm_epilogue(uint32_t tbase, int wrow0, int n0, int split, const GemmArgs& g, const CUtensorMap* to,
                        uint32_t stg, int lane) {
  constexpr int NOUT = EPI == GEMM_SWIGLU ? BN / 2 : BN;
  constexpr int CPC = (EPI == GEMM_F32 || EPI == GEMM_HEAD) ? 32 : 64;  // output columns per 128-byte row segment
  const int row = wrow0 + lane;
  // K-split partial sums and head logits take plain stores (no output map covers them)
  const bool staged = wrow0 + 32 <= g.M && g.splits == 1 && EPI != GEMM_HEAD;
  float best = -INFINITY;  // GEMM_HEAD: this row's maximum over the tile and its first column
  int best_col = -1;
#pragma unroll 1
  for (int c = 0; c < NOUT / CPC; ++c) {
    const int col = n0 + c * CPC;
    uint32_t w[32];  // this row's 128 output bytes
    if constexpr (EPI == GEMM_HEAD) {
      float v[32];
      tmem_ld32(tbase + c * 32, v);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        w[j] = __float_as_uint(v[j]);
        if (col + j < g.N && v[j] > best) {  // strictly greater: the first column of a tie
          best = v[j];
          best_col = col + j;
        }
      }
      if (g.out == nullptr) continue;
    } else if constexpr (EPI == GEMM_F32) {
      float v[32];
      tmem_ld32(tbase + c * 32, v);
#pragma unroll
      for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(g.alpha * v[j]);
    } else if constexpr (EPI == GEMM_BF16) {
      float v[64];
      tmem_ld32(tbase + c * 64, v);
      tmem_ld32(tbase + c * 64 + 32, v + 32);
#pragma unroll
      for (int j = 0; j < 32; ++j) w[j] = pack_bf2(g.alpha * v[2 * j], g.alpha * v[2 * j + 1]);
    } else {  // w1 products in columns [0, BN/2), w3 products in [BN/2, BN)
      float va[64], vb[64];
      tmem_ld64x2(tbase + c * 64, tbase + BN / 2 + c * 64, va, vb);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        w[j] = pack_bf2(silu_fast(g.alpha * va[2 * j]) * (g.alpha * vb[2 * j]),
                        silu_fast(g.alpha * va[2 * j + 1]) * (g.alpha * vb[2 * j + 1]));
      if (g.f16out)
#pragma unroll
        for (int j = 0; j < 32; ++j) w[j] = bf2_to_h2(w[j]);
    }
    if (col >= g.N) continue;  // the same for the whole warp
    if (staged) {
      const uint32_t buf = stg + (uint32_t)(c & 1) * 4096;
      if (lane == 0) bulk_wait_read_1();
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 8; ++q)
        sts128(buf + lane * 128 + ((q ^ (lane & 7)) << 4), make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]));
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(to, buf, col, wrow0);
        bulk_commit();
      }
    } else if (row < g.M) {
      if constexpr (EPI == GEMM_F32 || EPI == GEMM_HEAD) {
        float* dst = reinterpret_cast<float*>(g.out) + ((size_t)split * g.M + row) * g.ld + col;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col + j < g.N) dst[j] = __uint_as_float(w[j]);
      } else {
        uint32_t* dst = reinterpret_cast<uint32_t*>(reinterpret_cast<bf16*>(g.out) + (size_t)row * g.ld + col);
#pragma unroll
        for (int j = 0; j < 32; ++j)  // output widths are even
          if (col + 2 * j < g.N) dst[j] = w[j];
      }
    }
  }
  if constexpr (EPI == GEMM_HEAD) {
    if (row < g.M && best_col >= 0) {
      uint32_t u = __float_as_uint(best);
      u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
      atomicMax(g.amax + row, ((unsigned long long)u << 32) | (0xffffffffu - (uint32_t)best_col));
    }
  }
}

// Persistent: block b takes tiles b, b + gridDim.x, ... (M tiles fastest, so consecutive blocks
// share a weight tile through L2). TMEM holds two BN-column accumulators: the MMA thread fills
// one while the epilogue warps drain the other (acc_full / acc_empty barriers).
template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1) k_gemm(const __grid_constant__ CUtensorMap ta,
                                                 const __grid_constant__ CUtensorMap tb,
                                                 const __grid_constant__ CUtensorMap tb3,
                                                 const __grid_constant__ CUtensorMap to, const GemmArgs g) {
  using G = GemmGeom<BN>;
  constexpr int S = G::STAGES;
  constexpr int NOUT = EPI == GEMM_SWIGLU ? BN / 2 : BN;  // output columns per tile
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t stg0 = su32(smem + S * G::STAGE);  // epilogue staging (GM_STG bytes)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * G::STAGE + GM_STG);
  const uint32_t full0 = su32(bars), empty0 = su32(bars + S);
  const uint32_t accf0 = su32(bars + 2 * S), acce0 = su32(bars + 2 * S + 2);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (g.M + GM_BM - 1) / GM_BM, num_n = (g.N + NOUT - 1) / NOUT;
  const int ntiles = num_m * num_n * g.splits;
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

  if (warp == 0) {
    if (lane == 0) {
      // the weight boxes of one stage (the activations come from the previous kernel)
      auto load_w = [&](uint32_t b_s, int kb, int n0, uint32_t bar) {
        if constexpr (EPI == GEMM_SWIGLU) {  // BN / 2 rows of w1, then the same rows of w3
          tma_load_2d(b_s, &tb, kb * GM_BK, n0, bar);
          tma_load_2d(b_s + G::B_BYTES / 2, &tb3, kb * GM_BK, n0, bar);
        } else {  // weight boxes are 128 rows: a 256-wide tile takes two
#pragma unroll
          for (int h = 0; h < BN / 128; ++h) tma_load_2d(b_s + h * (G::B_BYTES / (BN / 128)), &tb, kb * GM_BK, n0 + 128 * h, bar);
        }
      };
      // constant weights: the first tile's first stages are requested before the wait for the
      // previous kernel, so their latency overlaps its tail
      int pre = 0;
      if (g.w_const && (int)blockIdx.x < ntiles) {
        const GemmTile T = gemm_tile(blockIdx.x, num_m, num_n, GM_BM, NOUT, nk, g.splits);
        pre = min(S, T.kb1 - T.kb0);
        for (int j = 0; j < pre; ++j) {
          const uint32_t a_s = su32(smem + j * G::STAGE);
          mbar_expect_tx(full0 + 8 * j, G::STAGE);
          load_w(a_s + G::A_BYTES, T.kb0 + j, T.n0, full0 + 8 * j);
        }
      }
      pdl_wait();
      pdl_launch_dependents();
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const GemmTile T = gemm_tile(tile, num_m, num_n, GM_BM, NOUT, nk, g.splits);
        const int m0 = T.m0, n0 = T.n0;
        for (int kb = T.kb0; kb < T.kb1; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1, g.err)) {
            ok = false;
            break;
          }
          const uint32_t a_s = su32(smem + s * G::STAGE), b_s = a_s + G::A_BYTES;
          if (it >= pre) {
            mbar_expect_tx(full0 + 8 * s, G::STAGE);
            load_w(b_s, kb, n0, full0 + 8 * s);
          }
          tma_load_2d(a_s, &ta, kb * GM_BK, m0, full0 + 8 * s);
        }
      }
      if (!ok)  // stages whose weights went out before the wait still complete (bounded)
        for (int j = it; j < pre; ++j) mbar_wait(full0 + 8 * j, 0, g.err);
    } else {
      pdl_wait();
      pdl_launch_dependents();
    }
  } else if (warp == 1) {
    pdl_wait();
    pdl_launch_dependents();
    if (lane == 0) {
      constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                 ((uint32_t)(GM_BM >> 4) << 24);
      // The issue loop is latency-bound when it does more than wait, issue and commit: keep the
      // k-loop to exactly that (the stage barriers order the copies before the MMAs; the fence is
      // only needed where TMEM changes hands).
      const uint32_t smem0 = su32(smem);
      int it = 0, i = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++i) {
        const int buf = i & 1;
        const GemmTile T = gemm_tile(tile, num_m, num_n, GM_BM, NOUT, nk, g.splits);
        if (!mbar_wait(acce0 + 8 * buf, ((i >> 1) & 1) ^ 1, g.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t td = tmem + buf * BN;
        for (int kb = T.kb0; kb < T.kb1; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(full0 + 8 * s, (it / S) & 1, g.err)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem0 + s * G::STAGE;
          const uint64_t ad = sw128_desc(sa), bd = sw128_desc(sa + G::A_BYTES);
#pragma unroll
          for (int k = 0; k < GM_BK / 16; ++k) umma_f16(td, ad + 2 * k, bd + 2 * k, idesc, (kb != T.kb0 || k) ? 1u : 0u);
          umma_commit(empty0 + 8 * s);
        }
        if (ok) umma_commit(accf0 + 8 * buf);
      }
      if (!ok) {
        // a wait gave up: drain (bounded) the stages the producer may still have in flight - it
        // runs at most S ahead - so that no copy lands after the block exits
        for (int d = 0; d < S; ++d, ++it) {
          mbar_wait(full0 + 8 * (it % S), (it / S) & 1, g.err);
          umma_commit(empty0 + 8 * (it % S));
        }
      }
    }
  } else {
    pdl_wait();
    pdl_launch_dependents();
    const int quarter = warp & 3;
    int i = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++i) {
      const int buf = i & 1;
      const GemmTile T = gemm_tile(tile, num_m, num_n, GM_BM, NOUT, nk, g.splits);
      ok = mbar_wait(accf0 + 8 * buf, (i >> 1) & 1, g.err);
      tc_fence_after();
      if (!ok) break;
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + buf * BN;
      gemm_epilogue<BN, EPI>(tbase, T.m0 + quarter * 32, T.n0, T.s, g, &to, stg0 + quarter * GM_STG_WARP, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce0 + 8 * buf);
    }
    if (lane == 0) bulk_wait_all();  // the output is written before the block exits
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * BN));
}

// ---------------------------------------------------------------- 2-SM tiles (prefill, M > 128)
// A cluster of two CTAs on two SMs computes one 256 x BN tile with tcgen05.mma.cta_group::2
// (M = 256): CTA rank r holds rows [128 r, 128 r + 128) of the A tile and rows [BN/2 r, BN/2 r +
// BN/2) of the weight tile (SwiGLU: rank 0 the 128 rows of w1, rank 1 the same rows of w3), and
// its TMEM receives the accumulator of its own 128 rows over all BN columns. Each SM thus stages
// half of the weight tile that a 1-SM 128 x BN tile needs. Rank 0 issues every MMA; its full
// barrier counts the bytes of both CTAs' copies, and each commit arrives on the barrier at the
// same offset in both CTAs, so each producer and each epilogue waits on its own CTA's barriers.
// The epilogue warps of both CTAs hand an accumulator back through rank 0's acc_empty barrier.
DEVI uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
DEVI uint32_t peer_addr(uint32_t saddr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(saddr), "r"(rank));
  return d;
}
DEVI void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Copy into this CTA's shared memory, completing on a barrier that may sit in the peer CTA.
DEVI void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}
DEVI void umma_f16_pair(uint32_t tmem_d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(
          tmem_d),
      "l"(ad), "l"(bd), "r"(idesc), "r"(accum));
}
// Arrive (once the issued MMAs finish) on the barrier at offset `bar` in both CTAs of the pair.
DEVI void umma_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"((unsigned short)3)
      : "memory");
}
DEVI void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

template <int BN>
struct Gemm2Geom {
  static constexpr int STAGES = 6;
  static constexpr uint32_t A_BYTES = 128 * GM_BK * 2;       // this CTA's 128 rows of the A tile
  static constexpr uint32_t B_BYTES = (BN / 2) * GM_BK * 2;  // this CTA's half of the weight rows
  static constexpr uint32_t STAGE = A_BYTES + B_BYTES;
};

template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1) k_gemm2(const __grid_constant__ CUtensorMap ta,
                                                  const __grid_constant__ CUtensorMap tb,
                                                  const __grid_constant__ CUtensorMap tb3,
                                                 const __grid_constant__ CUtensorMap to, const GemmArgs g) {
  using G = Gemm2Geom<BN>;
  constexpr int S = G::STAGES;
  constexpr int NOUT = EPI == GEMM_SWIGLU ? BN / 2 : BN;
  static_assert(BN == 256, "each CTA copies one 128-row weight box per stage");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t stg0 = su32(smem + S * G::STAGE);  // epilogue staging (GM_STG bytes)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * G::STAGE + GM_STG);
  const uint32_t full0 = su32(bars), empty0 = su32(bars + S);
  const uint32_t accf0 = su32(bars + 2 * S), acce0 = su32(bars + 2 * S + 2);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int num_m = (g.M + 2 * GM_BM - 1) / (2 * GM_BM), num_n = (g.N + NOUT - 1) / NOUT;
  const int ntiles = num_m * num_n;
  const int nk = g.K / GM_BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf0 + 8 * b, 1);
      mbar_init(acce0 + 8 * b, 8);  // 4 epilogue warps in each CTA (only rank 0's is waited on)
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&ta)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tb)) : "memory");
  }
  if (warp == 1) {  // the same warp in both CTAs allocates the pair's columns
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                 "r"(2 * BN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised before any copy or commit reaches them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = pair; tile < ntiles && ok; tile += npairs) {
        const int m0 = (tile % num_m) * 2 * GM_BM + (int)rank * GM_BM, n0 = (tile / num_m) * NOUT;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1, g.err)) {
            ok = false;
            break;
          }
          const uint32_t a_s = su32(smem + s * G::STAGE), b_s = a_s + G::A_BYTES;
          const uint32_t bar = peer_addr(full0 + 8 * s, 0);
          if (rank == 0) mbar_expect_tx(full0 + 8 * s, 2 * G::STAGE);
          tma_load_2d_pair(a_s, &ta, kb * GM_BK, m0, bar);
          if constexpr (EPI == GEMM_SWIGLU) {
            tma_load_2d_pair(b_s, rank ? &tb3 : &tb, kb * GM_BK, n0, bar);
          } else {
            tma_load_2d_pair(b_s, &tb, kb * GM_BK, n0 + (int)rank * (BN / 2), bar);  // one 128-row box
          }
        }
      }
    }
  } else if (warp == 1) {
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                 ((uint32_t)((2 * GM_BM) >> 4) << 24);
      const uint32_t smem0 = su32(smem);
      int it = 0, i = 0;
      bool ok = true;
      for (int tile = pair; tile < ntiles && ok; tile += npairs, ++i) {
        const int buf = i & 1;
        if (!mbar_wait(acce0 + 8 * buf, ((i >> 1) & 1) ^ 1, g.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t td = tmem + buf * BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(full0 + 8 * s, (it / S) & 1, g.err)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem0 + s * G::STAGE;
          const uint64_t ad = sw128_desc(sa), bd = sw128_desc(sa + G::A_BYTES);
#pragma unroll
          for (int k = 0; k < GM_BK / 16; ++k) umma_f16_pair(td, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0);
          umma_commit_pair(empty0 + 8 * s);
        }
        if (ok) umma_commit_pair(accf0 + 8 * buf);
      }
      if (!ok) {  // drain (bounded) the stages both producers may still have in flight
        for (int d = 0; d < S; ++d, ++it) {
          mbar_wait(full0 + 8 * (it % S), (it / S) & 1, g.err);
          umma_commit_pair(empty0 + 8 * (it % S));
        }
      }
    }
  } else {
    const int quarter = warp & 3;
    int i = 0;
    bool ok = true;
    for (int tile = pair; tile < ntiles && ok; tile += npairs, ++i) {
      const int buf = i & 1;
      const int m0 = (tile % num_m) * 2 * GM_BM + (int)rank * GM_BM, n0 = (tile / num_m) * NOUT;
      ok = mbar_wait(accf0 + 8 * buf, (i >> 1) & 1, g.err);
      tc_fence_after();
      if (!ok) break;
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + buf * BN;
      gemm_epilogue<BN, EPI>(tbase, m0 + quarter * 32, n0, 0, g, &to, stg0 + quarter * GM_STG_WARP, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(peer_addr(acce0 + 8 * buf, 0));
    }
    if (lane == 0) bulk_wait_all();  // the output is written before the block exits
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();  // no MMA, copy or arrival of either CTA still targets the other
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * BN));
}

template <int BN>
constexpr size_t gemm_smem() { return 1024 + GemmGeom<BN>::STAGES * (size_t)GemmGeom<BN>::STAGE + GM_STG + 256; }

static int g_gemm_sms = 0;
static int g_gemm_pairs = 0;  // clusters of two that fit on the device at once (paired kernel)
// Paired (2-SM) tiles from this many rows on, for the FFN projections and the wide or deep ones
// (measured on 2048-row chunks: w13 92.0 -> 91.6 us, w2 48.8 -> 46.8, in_proj 42.5 -> 40.5; the
// 2048 x 2048 projections are 1.2 us faster on single-SM tiles).
static int g_gemm_pair_min_m = 129;

template <int BN, int EPI>
static cudaError_t launch_gemm(const GemmPlan& p, int M, int* err, cudaStream_t s) {
  constexpr size_t smem = gemm_smem<BN>();
  auto k = k_gemm<BN, EPI>;
  const int splits = EPI == GEMM_F32 ? std::max(1, p.splits) : 1;
  GemmArgs g{M, p.N, p.K, p.ld, p.out, p.alpha, err, splits, p.amax, 0, p.w_const};
  const int ntile = EPI == GEMM_SWIGLU ? BN / 2 : BN;
  const int tiles = ((p.N + ntile - 1) / ntile) * ((M + GM_BM - 1) / GM_BM) * splits;
  dim3 grid(std::min(tiles, g_gemm_sms > 0 ? g_gemm_sms : 148));
  // a 128-column SwiGLU tile takes w1 and w3 in boxes of 64 rows
  const CUtensorMap& b1 = (EPI == GEMM_SWIGLU && BN == 128) ? p.bh : p.b;
  const CUtensorMap& b3 = EPI == GEMM_SWIGLU ? (BN == 128 ? p.b3h : p.b3) : p.b;
  return launch(k, grid, dim3(192), smem, s, p.a, b1, b3, p.o, g);
}

template <int BN>
constexpr size_t gemm2_smem() { return 1024 + Gemm2Geom<BN>::STAGES * (size_t)Gemm2Geom<BN>::STAGE + GM_STG + 256; }

static cudaLaunchConfig_t pair_config(int pairs, size_t smem, cudaStream_t s, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cfg;
}

template <int EPI>
static cudaError_t launch_gemm2(const GemmPlan& p, int M, int* err, cudaStream_t s) {
  constexpr int BN = 256;
  constexpr int ntile = EPI == GEMM_SWIGLU ? BN / 2 : BN;
  GemmArgs g{M, p.N, p.K, p.ld, p.out, p.alpha, err, 1, nullptr, 0, 0};
  const int tiles = ((p.N + ntile - 1) / ntile) * ((M + 2 * GM_BM - 1) / (2 * GM_BM));
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = pair_config(std::min(tiles, g_gemm_pairs), gemm2_smem<BN>(), s, attr);
  ++g_launches;
  return cudaLaunchKernelEx(&cfg, k_gemm2<BN, EPI>, p.a, p.b, EPI == GEMM_SWIGLU ? p.b3 : p.b, p.o, g);
}

// ---------------------------------------------------------------- NVFP4 weights (128-column tiles)
// The weight operand is expanded on the chip: warp 0 streams each tile's E2M1 codes (128 rows x
// 64 K = 4 KB per K block) through a 16-deep ring, four expansion warps turn a block into the f16
// operand tile (code pairs by the hardware E2M1 conversion, times the block's E4M3 scale: both
// exact in f16, and so is their product) in the 128-byte-swizzled layout the MMA reads, and warp
// 10 streams the activations, which are f16 copies of the bf16 values. kind::f16 with f16
// operands, fp32 accumulation, the tensor scale as alpha. Warps 1 (MMA) and 2..5 (epilogue) work
// as in k_gemm. SwiGLU tiles are 64 rows of w1 over 64 rows of w3.
constexpr int Q4G_S = 3;                    // operand stages (activations + expanded weights)
constexpr int Q4G_RS = 16;                  // code stages
constexpr uint32_t Q4G_AB = 128 * GM_BK * 2;  // one operand stage: 128 rows x 64 K
constexpr uint32_t Q4G_RAW = 128 * GM_BK / 2; // codes of 128 rows x 64 K
constexpr int Q4G_THREADS = 11 * 32;
constexpr size_t q4g_smem() { return 1024 + 2 * Q4G_S * Q4G_AB + Q4G_RS * Q4G_RAW + GM_STG + 512; }

template <int EPI>
__global__ void __launch_bounds__(Q4G_THREADS, 1) k_gemm_q4(const __grid_constant__ CUtensorMap ta,
                                                            const __grid_constant__ CUtensorMap tq,
                                                            const __grid_constant__ CUtensorMap tq3,
                                                            const __grid_constant__ CUtensorMap to, const GemmArgs g,
                                                            const uint8_t* __restrict__ sc,
                                                            const uint8_t* __restrict__ sc3) {
  constexpr int BN = 128;
  constexpr bool SW = EPI == GEMM_SWIGLU;
  constexpr int NOUT = SW ? BN / 2 : BN;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ra = smem;                             // activations [S][128 rows][128 B]
  unsigned char* rb = smem + Q4G_S * Q4G_AB;            // expanded weights [S][128 rows][128 B]
  unsigned char* rc = smem + 2 * Q4G_S * Q4G_AB;        // codes [RS][128 rows][32 B]
  const uint32_t stg0 = su32(rc + Q4G_RS * Q4G_RAW);    // epilogue staging (GM_STG bytes)
  uint64_t* bars = reinterpret_cast<uint64_t*>(rc + Q4G_RS * Q4G_RAW + GM_STG);
  const uint32_t a_full = su32(bars), b_full = a_full + 8 * Q4G_S, ab_empty = b_full + 8 * Q4G_S;
  const uint32_t r_full = ab_empty + 8 * Q4G_S, r_empty = r_full + 8 * Q4G_RS;
  const uint32_t accf0 = r_empty + 8 * Q4G_RS, acce0 = accf0 + 16, fin = acce0 + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * Q4G_S + 2 * Q4G_RS + 5);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (g.M + GM_BM - 1) / GM_BM, num_n = (g.N + NOUT - 1) / NOUT;
  const int ntiles = num_m * num_n * g.splits;
  const int nk = g.K / GM_BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Q4G_S; ++s) {
      mbar_init(a_full + 8 * s, 1);
      mbar_init(b_full + 8 * s, 4);
      mbar_init(ab_empty + 8 * s, 1);
    }
    for (int r = 0; r < Q4G_RS; ++r) {
      mbar_init(r_full + 8 * r, 1);
      mbar_init(r_empty + 8 * r, 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf0 + 8 * b, 1);
      mbar_init(acce0 + 8 * b, 4);
    }
    mbar_init(fin, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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

  if (warp == 0) {
    // ------------------------------------------------ codes (constants: streamed before the wait)
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const GemmTile T = gemm_tile(tile, num_m, num_n, GM_BM, NOUT, nk, g.splits);
        for (int kb = T.kb0; kb < T.kb1; ++kb, ++it) {
          const int r = it % Q4G_RS;
          if (!mbar_wait(r_empty + 8 * r, ((it / Q4G_RS) & 1) ^ 1, g.err)) {
            ok = false;
            break;
          }
          const uint32_t dst = su32(rc + r * Q4G_RAW);
          mbar_expect_tx(r_full + 8 * r, Q4G_RAW);
          if constexpr (SW) {
            tma_load_2d(dst, &tq, kb * (GM_BK / 2), T.n0, r_full + 8 * r);
            tma_load_2d(dst + Q4G_RAW / 2, &tq3, kb * (GM_BK / 2), T.n0, r_full + 8 * r);
          } else {
            tma_load_2d(dst, &tq, kb * (GM_BK / 2), T.n0, r_full + 8 * r);
          }
        }
      }
      // every copy issued has landed before the block can exit (bounded)
      for (int d = 1; d <= Q4G_RS && d <= it; ++d) mbar_wait(r_full + 8 * ((it - d) % Q4G_RS), ((it - d) / Q4G_RS) & 1, g.err);
    }
    pdl_wait();
    pdl_launch_dependents();
  } else if (warp == 10) {
    // ------------------------------------------------ activations (written by the previous kernel)
    pdl_wait();
    pdl_launch_dependents();
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const GemmTile T = gemm_tile(tile, num_m, num_n, GM_BM, NOUT, nk, g.splits);
        for (int kb = T.kb0; kb < T.kb1; ++kb, ++it) {
          const int s = it % Q4G_S;
          if (!mbar_wait(ab_empty + 8 * s, ((it / Q4G_S) & 1) ^ 1, g.err)) {
            ok = false;
            break;
          }
          mbar_expect_tx(a_full + 8 * s, Q4G_AB);
          tma_load_2d(su32(ra + s * Q4G_AB), &ta, kb * GM_BK, T.m0, a_full + 8 * s);
        }
      }
      for (int d = 1; d <= Q4G_S && d <= it; ++d) mbar_wait(a_full + 8 * ((it - d) % Q4G_S), ((it - d) / Q4G_S) & 1, g.err);
    }
  } else if (warp >= 6) {
    // ------------------------------------------------ expansion: thread c = row c of the tile
    // (codes and scales are constants: the first scales are requested before the wait)
    bool waited = false;
    const int c = threadIdx.x - 6 * 32;
    const uint32_t rowoff = (uint32_t)(c >> 3) * 1024 + (uint32_t)(c & 7) * 128;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      const GemmTile T = gemm_tile(tile, num_m, num_n, GM_BM, NOUT, nk, g.splits);
      const int wrow = SW ? T.n0 + (c & 63) : T.n0 + c;  // weight row
      const uint8_t* srow = (SW && c >= 64 ? sc3 : sc) + (size_t)wrow * (g.K / 16);
      const bool valid = wrow < g.N;  // rows past N: codes are zero-filled, scales read as 0
      // scales of four K blocks (16 bytes) per load; the next group is requested one group ahead
      int grp = T.kb0 >> 2;
      uint4 scv = valid ? ldg16(srow + grp * 16) : make_uint4(0, 0, 0, 0);
      uint4 scn = (valid && (grp + 1) * 4 < nk) ? ldg16(srow + (grp + 1) * 16) : make_uint4(0, 0, 0, 0);
      if (!waited) {
        pdl_wait();
        pdl_launch_dependents();
        waited = true;
      }
      for (int kb = T.kb0; kb < T.kb1; ++kb, ++it) {
        if ((kb >> 2) != grp) {
          grp = kb >> 2;
          scv = scn;
          scn = (valid && (grp + 1) * 4 < nk) ? ldg16(srow + (grp + 1) * 16) : make_uint4(0, 0, 0, 0);
        }
        const int r = it % Q4G_RS, s = it % Q4G_S;
        if (!mbar_wait(r_full + 8 * r, (it / Q4G_RS) & 1, g.err) ||
            !mbar_wait(ab_empty + 8 * s, ((it / Q4G_S) & 1) ^ 1, g.err)) {
          ok = false;
          break;
        }
        const uint4* cp = reinterpret_cast<const uint4*>(rc + r * Q4G_RAW + c * 32);
        const uint4 w0 = cp[0], w1 = cp[1];
        const uint32_t cw[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        const int kq = kb & 3;  // scales of this K block's four 16-code groups
        const uint32_t sw4 = kq == 0 ? scv.x : kq == 1 ? scv.y : kq == 2 ? scv.z : scv.w;
        const uint32_t bs = su32(rb + s * Q4G_AB) + rowoff;
#pragma unroll
        for (int q = 0; q < 8; ++q) {  // 8 codes -> one 16-byte chunk of the row
          const uint32_t sc2 = e4m3_to_h2(sw4 >> (8 * (q >> 1)));
          uint32_t h0, h1, h2, h3;
          e2m1x8_to_h2(cw[q], h0, h1, h2, h3);
          sts128(bs + ((uint32_t)(q ^ (c & 7)) << 4),
                 make_uint4(hmul2_u(h0, sc2), hmul2_u(h1, sc2), hmul2_u(h2, sc2), hmul2_u(h3, sc2)));
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(b_full + 8 * s);
          mbar_arrive(r_empty + 8 * r);
        }
      }
    }
    if (!waited) {
      pdl_wait();
      pdl_launch_dependents();
    }
  } else if (warp == 1) {
    pdl_wait();
    pdl_launch_dependents();
    if (lane == 0) {
      constexpr uint32_t idesc = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(GM_BM >> 4) << 24);  // f16 x f16
      int it = 0, i = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++i) {
        const int buf = i & 1;
        const GemmTile T = gemm_tile(tile, num_m, num_n, GM_BM, NOUT, nk, g.splits);
        if (!mbar_wait(acce0 + 8 * buf, ((i >> 1) & 1) ^ 1, g.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t td = tmem + buf * BN;
        for (int kb = T.kb0; kb < T.kb1; ++kb, ++it) {
          const int s = it % Q4G_S;
          if (!mbar_wait(a_full + 8 * s, (it / Q4G_S) & 1, g.err) || !mbar_wait(b_full + 8 * s, (it / Q4G_S) & 1, g.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_desc(su32(ra + s * Q4G_AB)), bd = sw128_desc(su32(rb + s * Q4G_AB));
#pragma unroll
          for (int k = 0; k < GM_BK / 16; ++k) umma_f16(td, ad + 2 * k, bd + 2 * k, idesc, (kb != T.kb0 || k) ? 1u : 0u);
          umma_commit(ab_empty + 8 * s);
        }
        if (ok) umma_commit(accf0 + 8 * buf);
      }
      // nothing issued may still run when TMEM is released (bounded)
      umma_commit(fin);
      mbar_wait(fin, 0, g.err);
    }
  } else {
    pdl_wait();
    pdl_launch_dependents();
    const int quarter = warp & 3;
    int i = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++i) {
      const int buf = i & 1;
      const GemmTile T = gemm_tile(tile, num_m, num_n, GM_BM, NOUT, nk, g.splits);
      ok = mbar_wait(accf0 + 8 * buf, (i >> 1) & 1, g.err);
      tc_fence_after();
      if (!ok) break;
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + buf * BN;
      gemm_epilogue<BN, EPI>(tbase, T.m0 + quarter * 32, T.n0, T.s, g, &to, stg0 + quarter * GM_STG_WARP, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce0 + 8 * buf);
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * BN));
}

template <int EPI>
static cudaError_t launch_gemm_q4(const GemmPlan& p, int M, int* err, cudaStream_t s) {
  const int splits = EPI == GEMM_F32 ? std::max(1, p.splits) : 1;
  GemmArgs g{M, p.N, p.K, p.ld, p.out, p.alpha, err, splits, nullptr, EPI == GEMM_SWIGLU ? 1 : 0, 1};
  const int ntile = EPI == GEMM_SWIGLU ? 64 : 128;
  const int tiles = ((p.N + ntile - 1) / ntile) * ((M + GM_BM - 1) / GM_BM) * splits;
  dim3 grid(std::min(tiles, g_gemm_sms > 0 ? g_gemm_sms : 148));
  return launch(k_gemm_q4<EPI>, grid, dim3(Q4G_THREADS), q4g_smem(), s, p.a, p.q, EPI == GEMM_SWIGLU ? p.q3 : p.q,
                p.o, g, p.sc, EPI == GEMM_SWIGLU ? p.sc3 : p.sc);
}

bool make_tmap_codes(CUtensorMap* m, const void* codes, uint64_t rows, uint64_t K, uint32_t box_rows) {
  if (!p_encode) return false;
  const uint64_t cols = K / 2;  // bytes per row
  if ((reinterpret_cast<uintptr_t>(codes) & 15) || cols % 16) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {GM_BK / 2, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = p_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Output widths from which a tile is 256 columns wide (fewer, more L2-efficient tiles) rather than
// 128 (more tiles to spread over the SMs).
static int g_gemm_wide_min = 2048;  // measured: 8k prefill 37.8 -> 34.6 ms against 4097

cudaError_t gemm_init() {
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
  if ((e = cudaFuncSetAttribute(k_gemm<256, GEMM_SWIGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_smem<256>())))
    return e;
  if ((e = cudaFuncSetAttribute(k_gemm<128, GEMM_SWIGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_smem<128>())))
    return e;
  if ((e = cudaFuncSetAttribute(k_gemm<128, GEMM_HEAD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_smem<128>())))
    return e;
  if ((e = cudaFuncSetAttribute(k_gemm_q4<GEMM_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)q4g_smem())))
    return e;
  if ((e = cudaFuncSetAttribute(k_gemm_q4<GEMM_SWIGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)q4g_smem())))
    return e;
  if ((e = cudaFuncSetAttribute(k_gemm2<256, GEMM_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm2_smem<256>())))
    return e;
  if ((e = cudaFuncSetAttribute(k_gemm2<256, GEMM_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm2_smem<256>())))
    return e;
  if ((e = cudaFuncSetAttribute(k_gemm2<256, GEMM_SWIGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm2_smem<256>())))
    return e;
  // every paired launch is persistent over the clusters that fit at once (one CTA per SM); where
  // no pair can be resident (or the query is refused) the single-SM tiles do all the work
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = pair_config(g_gemm_sms / 2, gemm2_smem<256>(), 0, attr);
  if (cudaOccupancyMaxActiveClusters(&g_gemm_pairs, k_gemm2<256, GEMM_F32>, &cfg) != cudaSuccess || g_gemm_pairs < 1) {
    (void)cudaGetLastError();
    g_gemm_pairs = 0;
    g_gemm_pair_min_m = 1 << 30;
  }
  return cudaSuccess;
}

bool gemm_wide(int N) { return N >= g_gemm_wide_min; }

cudaError_t gemm(const GemmPlan& p, int M, int* err, cudaStream_t s) {
  if (p.K % GM_BK) return cudaErrorInvalidValue;
  if (p.splits > 1 && (p.epi != GEMM_F32 || M > GM_BM || p.splits > p.K / GM_BK)) return cudaErrorInvalidValue;
  if (p.epi == GEMM_HEAD) return p.amax ? launch_gemm<128, GEMM_HEAD>(p, M, err, s) : cudaErrorInvalidValue;
  if (p.q4) {
    if (p.K % 256) return cudaErrorInvalidValue;  // scales are read 16 bytes (4 K blocks) at a time
    if (p.epi == GEMM_F32) return launch_gemm_q4<GEMM_F32>(p, M, err, s);
    if (p.epi == GEMM_SWIGLU) return launch_gemm_q4<GEMM_SWIGLU>(p, M, err, s);
    return cudaErrorInvalidValue;
  }
  if (M <= GM_BM) {
    // one row tile (a batch of decode rows): 128-column weight tiles, so that more of them stream
    // at once; fp32 outputs may also be split along K
    switch (p.epi) {
      case GEMM_F32: return launch_gemm<128, GEMM_F32>(p, M, err, s);
      case GEMM_BF16: return launch_gemm<128, GEMM_BF16>(p, M, err, s);
      case GEMM_SWIGLU: return launch_gemm<128, GEMM_SWIGLU>(p, M, err, s);
    }
    return cudaErrorInvalidValue;
  }
  if (M >= g_gemm_pair_min_m && (p.epi == GEMM_SWIGLU || p.N >= 4096 || p.K >= 4096)) {
    switch (p.epi) {
      case GEMM_F32: return launch_gemm2<GEMM_F32>(p, M, err, s);
      case GEMM_BF16: return launch_gemm2<GEMM_BF16>(p, M, err, s);
      case GEMM_SWIGLU: return launch_gemm2<GEMM_SWIGLU>(p, M, err, s);
    }
    return cudaErrorInvalidValue;
  }
  switch (p.epi) {
    case GEMM_F32: return gemm_wide(p.N) ? launch_gemm<256, GEMM_F32>(p, M, err, s) : launch_gemm<128, GEMM_F32>(p, M, err, s);
    case GEMM_BF16: return gemm_wide(p.N) ? launch_gemm<256, GEMM_BF16>(p, M, err, s) : launch_gemm<128, GEMM_BF16>(p, M, err, s);
    case GEMM_SWIGLU: return launch_gemm<256, GEMM_SWIGLU>(p, M, err, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace lfm3
