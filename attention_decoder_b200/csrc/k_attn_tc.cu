// Prefill attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Block = 32 query rows of one chunk x the 4 query heads that share one kv head: the MMA's M = 128
// rows are (row r, head j) with m = 4 r + j. Keys come in tiles of 128 (two 64-position pages of
// a full layer, or 128 consecutive rows of a sliding layer's chunk scratch), K and V by TMA into a
// two-stage ring. Per tile:
//   warp 1 (one lane):  S = Q K^T      (tcgen05.mma kind::f16, 128 x 128 x 128, fp32 in TMEM; two S
//                       buffers, so the next tile's scores are computed during this tile's softmax)
//   warps 2..9:         two warps per TMEM lane quarter, so each thread owns one row (TMEM lane)
//                       and half of its keys: read S, mask (causal, the 256-key window on sliding
//                       layers, written keys only), online softmax in fp32 (exp2 with the
//                       1/sqrt(128) scale folded in; the pair shares the row maximum), write P as bf16
//                       into a 128-byte-swizzled shared tile, rescale its half of the O row in TMEM
//                       when the running maximum grows, zero the V rows of unwritten keys
//   warp 1:             O += P V       (V read as an MN-major operand: dims contiguous)
// After the last tile the pair adds its two partial softmax sums; each thread divides its half row, multiplies by the head gate
// sigmoid(g) (coreai-model-zoo "lfm3-1.7b-port", diff table row 4) and stores bf16.
// Every mbarrier wait is bounded (the device error word is set when one gives up).
#include <cudaTypedefs.h>

#include "kernels.cuh"

namespace lfm3 {

constexpr int AT_ROWS = 32;                 // query positions per block
constexpr int AT_M = AT_ROWS * GQA;         // 128 MMA rows
constexpr int AT_KT = 128;                  // keys per tile
constexpr uint32_t AT_Q_BYTES = AT_M * HD * 2;      // 32 KB
constexpr uint32_t AT_KV_BYTES = AT_KT * HD * 2;    // 32 KB per K or V tile
constexpr uint32_t AT_P_BYTES = AT_M * AT_KT * 2;   // 32 KB
constexpr int AT_THREADS = 320;  // loader, MMA issuer, 8 softmax / epilogue warps

DEVI void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
DEVI void tma_load_2d_at(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
DEVI void at_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
DEVI void at_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 128-byte-swizzled operand tile, K-major: rows of 128 B, 8-row atoms 1024 B apart.
DEVI uint64_t at_desc_k(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// 128-byte-swizzled operand tile, MN-major: 64 contiguous N elements per 128-B row, rows along K
// 128 B apart in 1024-B atoms of 8; the next 64 N elements start `lbo` bytes later.
DEVI uint64_t at_desc_mn(uint32_t saddr, uint32_t lbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
DEVI void at_mma(uint32_t tmem_d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(
          tmem_d),
      "l"(ad), "l"(bd), "r"(idesc), "r"(accum));
}
DEVI void at_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
DEVI void at_ld32(uint32_t taddr, float* v) {
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
DEVI void at_ld64(uint32_t taddr, float* v) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]),
        "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]),
        "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
        "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]),
        "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}
DEVI void at_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 2^x with the hardware approximation (relative error about 2^-22; denormal results flush to 0).
DEVI float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Byte offset of 16-byte chunk c (0..7) of row r in a 128-byte-swizzled block of 128-B rows.
DEVI uint32_t sw_off(int r, int c) { return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)); }

__global__ void __launch_bounds__(AT_THREADS, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
              const __grid_constant__ CUtensorMap tv, const AttnTcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* qs = smem;                                   // [2 dim blocks][128 rows][128 B]
  unsigned char* ks = qs + AT_Q_BYTES;                        // 2 stages x [2][128 keys][128 B]
  unsigned char* vs = ks + 2 * AT_KV_BYTES;                   // 2 stages x [2][128 keys][128 B]
  unsigned char* ps = vs + 2 * AT_KV_BYTES;                   // [2 key blocks][128 rows][128 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(ps + AT_P_BYTES);
  const uint32_t q_full = su32(bars), kv_full0 = su32(bars + 1), kv_empty0 = su32(bars + 3);
  // S is double-buffered in TMEM (columns 0..127 and 128..255, one full barrier each) so the next
  // tile's Q K^T runs while the softmax works on this one; O lives in columns 256..383
  const uint32_t s_full0 = su32(bars + 5), p_full = su32(bars + 6), o_done = su32(bars + 7);
  const uint32_t s_full1 = su32(bars + 9);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the last query rows see the most keys: they are dispatched first, so the blocks left for the
  // final wave are the short ones (causal full layers)
  const int kvh = blockIdx.y;
  const int rb0 = (gridDim.x - 1 - blockIdx.x) * AT_ROWS;
  const int rb1 = min(a.n, rb0 + AT_ROWS) - 1;
  const bool full = a.full;
  const int koff = full ? 0 : a.p0 - WIN;                   // key index -> position
  const int qpos_lo = a.p0 + rb0, qpos_hi = a.p0 + rb1;
  int klo = full ? 0 : max(0, qpos_lo - (WIN - 1)) - koff;
  const int khi = qpos_hi - koff;
  const int kmax_valid = a.p0 + a.n - 1 - koff;
  klo = (klo / AT_KT) * AT_KT;
  const int ntiles = (khi - klo) / AT_KT + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(kv_full0 + 8 * s, 1);
      mbar_init(kv_empty0 + 8 * s, 1);
    }
    mbar_init(s_full0, 1);
    mbar_init(s_full1, 1);
    mbar_init(p_full, 8);
    mbar_init(o_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)), "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  at_fence_before();
  __syncthreads();
  at_fence_after();
  const uint32_t tmem = *tmem_slot;  // S: columns 0..127 / 128..255 by tile parity, O: 256..383
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    // ---------------------------------------------------------------- loader
    if (lane == 0) {
      mbar_expect_tx(q_full, AT_Q_BYTES);
      for (int db = 0; db < 2; ++db)  // rows (r, head) of this kv head, 64 dims at a time
        tma_load_3d(su32(qs + db * (AT_Q_BYTES / 2)), &tq, db * 64, kvh * GQA, a.row0 + rb0, q_full);
      bool ok = true;
      for (int j = 0; j < ntiles && ok; ++j) {
        const int st = j & 1;
        if (!mbar_wait(kv_empty0 + 8 * st, ((j >> 1) & 1) ^ 1, a.err)) {
          ok = false;
          break;
        }
        const int kt0 = klo + j * AT_KT;
        // pages (or scratch halves) holding keys we may read: [kt0, kt0 + 128) clipped to khi
        const int halves = (kt0 + 64 <= khi) ? 2 : 1;
        mbar_expect_tx(kv_full0 + 8 * st, (uint32_t)halves * 2 * 2 * 8192);
        unsigned char* kd = ks + st * AT_KV_BYTES;
        unsigned char* vd = vs + st * AT_KV_BYTES;
        for (int hf = 0; hf < halves; ++hf) {
          int y;
          if (full) {
            const int page = a.page_table[(size_t)a.slot * a.max_pages + (kt0 + 64 * hf) / PAGE];
            y = (page * HKV + kvh) * PAGE;
          } else {
            y = kvh * a.scratch_rows + kt0 + 64 * hf;
          }
          for (int db = 0; db < 2; ++db) {
            const uint32_t off = db * (AT_KV_BYTES / 2) + hf * 8192;
            tma_load_2d_at(su32(kd + off), &tk, db * 64, y, kv_full0 + 8 * st);
            tma_load_2d_at(su32(vd + off), &tv, db * 64, y, kv_full0 + 8 * st);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(AT_KT >> 3) << 17) |
                                   ((uint32_t)(AT_M >> 4) << 24);
      constexpr uint32_t idesc_o = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(HD >> 3) << 17) |
                                   ((uint32_t)(AT_M >> 4) << 24);
      bool ok = mbar_wait(q_full, 0, a.err);
      const uint32_t qb = su32(qs);
      auto issue_s = [&](int j) -> bool {  // S(j) = Q K(j)^T into S buffer j & 1
        const int st = j & 1;
        if (!mbar_wait(kv_full0 + 8 * st, (j >> 1) & 1, a.err)) return false;
        at_fence_after();
        const uint32_t kb = su32(ks + st * AT_KV_BYTES);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t off = (k >> 2) * (AT_Q_BYTES / 2) + (k & 3) * 32;
          const uint32_t koff_b = (k >> 2) * (AT_KV_BYTES / 2) + (k & 3) * 32;
          at_mma(tmem + (uint32_t)st * 128, at_desc_k(qb + off), at_desc_k(kb + koff_b), idesc_s, k != 0);
        }
        at_commit(st ? s_full1 : s_full0);
        return true;
      };
      if (ok && ntiles > 0) ok = issue_s(0);
      for (int j = 0; j < ntiles && ok; ++j) {
        const int st = j & 1;
        // the next tile's scores go into the other S buffer, whose last reader (the softmax of
        // tile j - 1) finished before its P was handed over below
        if (j + 1 < ntiles && !issue_s(j + 1)) break;
        if (!mbar_wait(p_full, j & 1, a.err)) break;
        at_fence_after();
        const uint32_t pb = su32(ps), vb = su32(vs + st * AT_KV_BYTES);
#pragma unroll
        for (int k = 0; k < AT_KT / 16; ++k) {
          const uint32_t poff = (k >> 2) * (AT_P_BYTES / 2) + (k & 3) * 32;   // P: K-major (keys)
          const uint32_t voff = k * 2048;                                      // V: 16 keys = 2 atoms
          at_mma(tmem + 256, at_desc_k(pb + poff), at_desc_mn(vb + voff, AT_KV_BYTES / 2), idesc_o,
                 (j | k) != 0);
        }
        at_commit(o_done);
        at_commit(kv_empty0 + 8 * st);
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax / epilogue
    // Two warps per TMEM lane quarter: `half` 0 takes keys 0..63 of each tile and dims 0..63 of O,
    // half 1 keys 64..127 and dims 64..127. The pair shares its rows' maxima and sums through
    // shared memory at a 64-thread named barrier, where it also agrees on giving up after a wait
    // that timed out, so both warps always reach the same barriers.
    const int quarter = warp & 3, half = (warp - 2) >> 2;
    const int m = quarter * 32 + lane;                     // this thread's row
    const int r = rb0 + (m >> 2), h = kvh * GQA + (m & 3);
    const int qp = a.p0 + r;                               // query position
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sl2 = rsqrtf((float)HD) * 1.4426950408889634f;
    float* pair_f = reinterpret_cast<float*>(bars + 16);   // [2 halves][128 rows]
    int* pair_ok = reinterpret_cast<int*>(pair_f + 256);   // [2 halves][4 quarters]
    auto pair_sync = [&]() { asm volatile("bar.sync %0, 64;" ::"r"(3 + quarter) : "memory"); };
    // Visible keys of this row, as key indices: [vis_lo, vis_hi] (causal, written keys, and on
    // sliding layers the 256-position window). A half tile all of whose keys are visible to every
    // row of the block takes the unmasked path (all but the diagonal and window-edge tiles).
    const int vis_hi = min(qp, kmax_valid + koff) - koff;
    const int vis_lo = (full ? 0 : max(0, qp - (WIN - 1))) - koff;
    const int dense_hi = min(qpos_lo, kmax_valid + koff) - koff;
    const int dense_lo = (full ? 0 : max(0, qpos_hi - (WIN - 1))) - koff;
    float mrun = -INFINITY, lrun = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
      const int kt0 = klo + j * AT_KT;
      bool got = mbar_wait((j & 1) ? s_full1 : s_full0, (j >> 1) & 1, a.err);
      at_fence_after();
      const uint32_t srow = trow + (uint32_t)(j & 1) * 128 + half * 64;  // this tile's S, my keys
      const int kh0 = kt0 + half * 64;
      const bool dense = kh0 >= dense_lo && kh0 + 63 <= dense_hi;  // the same for the whole block
      const int ilo = vis_lo - kh0, ihi = vis_hi - kh0;            // visible i in [ilo, ihi]
      // pass 1: maximum of the raw scores over my visible keys (the scale is positive); the 64
      // scores stay in registers for pass 2
      float tmax = -INFINITY;
      float v[64];
      if (got) {
        at_ld64(srow, v);
        if (dense) {
#pragma unroll
          for (int i = 0; i < 64; ++i) tmax = fmaxf(tmax, v[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (i >= ilo && i <= ihi) tmax = fmaxf(tmax, v[i]);
        }
        tmax *= sl2;
      }
      // the previous P.V must be finished before P is overwritten and O is rescaled
      if (got && j > 0) got = mbar_wait(o_done, (j - 1) & 1, a.err);
      pair_f[half * 128 + m] = tmax;
      if (lane == 0) pair_ok[half * 4 + quarter] = got;
      pair_sync();
      ok = pair_ok[quarter] && pair_ok[4 + quarter];
      tmax = fmaxf(pair_f[m], pair_f[128 + m]);
      pair_sync();  // pair_f is rewritten below
      if (!ok) break;
      at_fence_after();
      // The running maximum moves only when a score exceeds it by more than 8 (in log2 units):
      // probabilities stay below 2^8, O and the sum keep one common reference, and most tiles
      // skip the O rescale. The final division by the sum is unchanged.
      const float mnew = tmax > mrun + 8.f ? tmax : mrun;
      const float mu = mnew == -INFINITY ? 0.f : mnew;
      const float alpha = exp2f(mrun - mu);
      // tcgen05.ld/st are warp-wide: rescale when any row of the warp needs it (others use 1)
      if (__any_sync(0xffffffffu, j > 0 && alpha < 1.f)) {
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          float o[32];
          at_ld32(trow + 256 + half * 64 + c * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          at_st32(trow + 256 + half * 64 + c * 32, o);
        }
      }
      // pass 2: probabilities of my keys -> bf16 P (row m, key block `half`, 128-byte swizzle)
      float lsum = 0.f;
      unsigned char* pb = ps + half * (AT_P_BYTES / 2);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float pp[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            pp[e] = ex2_approx(fmaf(v[c * 32 + i + e], sl2, -mu));
            if (!dense && (c * 32 + i + e < ilo || c * 32 + i + e > ihi)) pp[e] = 0.f;
            lsum += pp[e];
          }
          pk[i >> 1] = pack_bf2(pp[0], pp[1]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(pb + sw_off(m, c * 4 + q)) = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
      lrun = lrun * alpha + lsum;  // my keys' share; the halves add up at the end
      mrun = mnew;
      // V rows of keys never written (past the chunk) or not loaded (the tile's second page lies
      // past every query of the block): zero them so 0 * V cannot bring in stale values
      const int loaded = (kt0 + 64 <= khi) ? AT_KT : 64;
      if (half == 0 && (kt0 + AT_KT - 1 > kmax_valid || loaded < AT_KT)) {
        const int st = j & 1;
        unsigned char* vd = vs + st * AT_KV_BYTES;
        const int key = m;  // one key row per thread
        if (kt0 + key > kmax_valid || key >= loaded) {
#pragma unroll
          for (int db = 0; db < 2; ++db)
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(vd + db * (AT_KV_BYTES / 2) + sw_off(key, c)) = make_uint4(0, 0, 0, 0);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      at_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // the row's softmax sum is the two halves' sums (both kept with the same running maximum)
    pair_f[half * 128 + m] = lrun;
    bool fin = ok && mbar_wait(o_done, (ntiles - 1) & 1, a.err);
    if (lane == 0) pair_ok[half * 4 + quarter] = fin;
    pair_sync();
    fin = pair_ok[quarter] && pair_ok[4 + quarter];
    const float ltot = pair_f[m] + pair_f[128 + m];
    if (fin) {
      at_fence_after();
      // every lane reads TMEM (warp-wide loads); rows past the chunk do not store
      const bool live = r <= rb1;
      const float gt = live ? sigmoidf_(a.gate[(size_t)r * HQ + h]) / ltot : 0.f;
      bf16* dst = a.y + (size_t)(live ? r : 0) * HQ * HD + h * HD + half * 64;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float o[32];
        at_ld32(trow + 256 + half * 64 + c * 32, o);
        if (live) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            d4[q] = make_uint4(pack_bf2(o[8 * q] * gt, o[8 * q + 1] * gt), pack_bf2(o[8 * q + 2] * gt, o[8 * q + 3] * gt),
                               pack_bf2(o[8 * q + 4] * gt, o[8 * q + 5] * gt), pack_bf2(o[8 * q + 6] * gt, o[8 * q + 7] * gt));
        }
      }
    }
  }
  at_fence_before();
  __syncthreads();
  at_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
}

constexpr size_t AT_SMEM = 1024 + AT_Q_BYTES + 4 * AT_KV_BYTES + AT_P_BYTES + 256 + 256 * 4 + 64;  // + pair scratch

cudaError_t attn_tc_init() {
  return cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)AT_SMEM);
}

cudaError_t attn_prefill_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnTcArgs& a,
                            cudaStream_t s) {
  return launch(k_attn_tc, dim3((a.n + AT_ROWS - 1) / AT_ROWS, HKV), dim3(AT_THREADS), AT_SMEM, s, tq, tk, tv, a);
}

// 3-D map over q [rows][16 heads][128 dims] (box 64 dims x 4 heads x 32 rows) and 2-D maps over
// K/V stores viewed as [rows][128 dims] (box 64 dims x `box_rows` rows), all 128-byte swizzled.
static PFN_cuTensorMapEncodeTiled_v12000 p_enc_at = nullptr;

static bool at_encoder() {
  if (p_enc_at) return true;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return false;
  p_enc_at = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

bool make_tmap_q(CUtensorMap* m, const void* q, uint64_t rows) {
  if (!at_encoder()) return false;
  cuuint64_t dims[3] = {HD, HQ, rows};
  cuuint64_t strides[2] = {HD * 2, HQ * HD * 2};
  cuuint32_t box[3] = {64, GQA, AT_ROWS};
  cuuint32_t es[3] = {1, 1, 1};
  return p_enc_at(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_kv(CUtensorMap* m, const void* base, uint64_t rows) {
  if (!at_encoder()) return false;
  cuuint64_t dims[2] = {HD, rows};
  cuuint64_t strides[1] = {HD * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t es[2] = {1, 1};
  return p_enc_at(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace lfm3
