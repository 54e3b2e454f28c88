// One decode token step of up to four streams as a single persistent launch.
//
// Batch-1 decode reads every weight of the model once per token, so its speed is the HBM stream
// rate minus whatever stalls that stream. Launching one kernel per projection stalls it at every
// launch boundary; this kernel instead keeps one block per SM resident for the whole step and
// separates the step's dependent phases with grid-wide barriers. The weights (and the cached
// keys and values, which do not depend on the step either) are fetched by one producer thread
// per block, with TMA tensor copies into a ring of 32 KB shared-memory slots, in exactly the
// order the block will consume them - across phase boundaries, so while the consumers wait at a
// barrier the next phase's bytes are already landing.
//
// Phases per layer (LFM3 hybrid decoder: a pre-norm / post-norm sandwich around each operator
// and the SwiGLU FFN):
//   conv layer       CONV (in_proj + gated short conv + state shift), OUT (out_proj), W13, W2
//   attention layer  QKVG (q|k|v|gate projection), ATTN, OUT (o_proj), W13, W2
// then HEAD (tied logits + greedy argmax) and the step's bookkeeping. A phase is a list of work
// units dealt round-robin to the blocks, the deal rotating from phase to phase so that every
// block streams about the same number of bytes per step.
//
// GEMV phases: a unit is a 16-row tile (in_proj: the B, C and x rows of 16 channels) over a K
// range; eight consumer warps split each 32 KB stage along K and feed the tensor cores
// (m16n8k16, the weight tile as A, the streams as the 8 columns of B), then reduce across warps.
// Phases that need the residual stream start with the sandwich step done redundantly by every
// block: x' = x + g_post * RMS(previous output), activations = bf16(g_next * RMS(x')); block 0
// writes x' to the other residual buffer.
// ATTN: a unit is (stream, kv head, key split of 128 positions - 64 ring slots on sliding
// layers). It normalises and rotates its four query heads itself; the unit holding the current
// position also builds the new key and value, uses them in place of the cached row and writes
// them to the cache. Partial softmax results go to scratch and the last unit of a (stream, kv
// head) to finish - counted with an atomic - merges them, applies the sigmoid head gate and
// writes the attention output.
//
// Every wait is bounded (mbarrier phases, grid barriers): a wait that gives up sets the error
// word, every other wait sees it and returns, and the blocks drain their copies in flight and
// exit; the host reads the word through lfm3_check_device_errors.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>

#include "kernels.cuh"

namespace lfm3 {

// Code executed once per phase or unit is kept out of line: the step runs ~100 phases, and code
// that is inlined at every call site does not stay in the instruction cache between them.
#define MK_COLD __device__ __noinline__

constexpr int MK_CW = 8;                       // consumer warps
constexpr int MK_CT = 32 * MK_CW;              // consumer threads
constexpr int MK_THREADS = MK_CT + 32;         // + one producer warp
constexpr int MK_SLOT = 32 * 1024;             // ring slot bytes
constexpr int MK_SMEM_MAX = 225 * 1024;        // dynamic shared memory of one block (+ static)
constexpr int MK_XS = F + 32;                  // activation row stride in shared memory (elements)
constexpr int MK_SCR_FLOATS = 3584;            // warp-reduction / attention scratch (14 KB)
constexpr int MK_LUT_BYTES = 256 * 32 * 4;     // NVFP4 byte -> bf16x2 table, one copy per bank
constexpr uint64_t MK_WAIT_NS = 500ull * 1000 * 1000;  // give up on any single wait after 0.5 s


enum MkKind { MK_CONV = 0, MK_QKVG, MK_ATTN, MK_OUT, MK_W13, MK_W2, MK_HEAD };

// Stage geometry of a GEMV phase: NRT 16-row tiles, copied as NREQ requests of BR rows, each row
// NKB 64-byte blocks of KB elements (bf16: 32; NVFP4: 128 codes), plus SCB scale bytes per row.
template <int NRT_, int BR_, int NREQ_, int KB_, int NKB_, bool FP4_, int SCB_>
struct MkG {
  static constexpr int NRT = NRT_, BR = BR_, NREQ = NREQ_, KB = KB_, NKB = NKB_, SCB = SCB_;
  static constexpr bool FP4 = FP4_;
  static constexpr int KCH = KB * NKB;            // K per stage
  static constexpr int RPT = 16 * NRT;            // rows per stage
  static constexpr int REQB = 64 * BR * NKB;      // bytes of one request
  static constexpr int ROWB = 64 * NKB;
  static constexpr int BYTES = RPT * ROWB + RPT * SCB;
  static constexpr int CH = (NRT >= 3 && !FP4_) ? 1 : 4;  // accumulator chains (3 row tiles are 3 already)
  static_assert(BYTES <= MK_SLOT, "stage larger than a slot");
};
using G_CONV = MkG<3, 16, 3, 32, 8, false, 0>;     // B|C|x rows of 16 channels x 256 K
using G_ROWS = MkG<1, 16, 1, 32, 32, false, 0>;    // 16 rows x 1024 K (qkvg, out_proj, o_proj, head)
using G_W13 = MkG<1, 8, 2, 32, 32, false, 0>;      // 8 rows of w1 + the same 8 rows of w3 x 1024 K
using G_W2 = MkG<1, 16, 1, 32, 30, false, 0>;      // 16 rows x 960 K
using G_W13F = MkG<1, 8, 2, 128, 16, true, 128>;   // NVFP4 w1|w3: 8 + 8 rows x 2048 K
using G_W2F = MkG<1, 16, 1, 128, 20, true, 160>;   // NVFP4 w2: 16 rows x 2560 K

// K splits (partial sums the next phase adds): q|k|v|gate and out/o_proj in halves (one stage
// each), bf16 w2 in quarters (two stages of 960), NVFP4 w2 in thirds (one stage of 2560).
constexpr int MK_KS_QO = 2;
constexpr int MK_KS_W2 = 4;
constexpr int MK_KS_W2F = 3;

// Stage byte offset of lane chunk t of row r at block j.
template <class G>
DEVI int mk_woff(int r, int j, int t) {
  return (r / G::BR) * G::REQB + j * (G::BR * 64) + (r % G::BR) * 64 + t * 16;
}

// ------------------------------------------------------------------------------ small helpers
DEVI uint64_t mk_now() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
DEVI unsigned mk_ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
DEVI int mk_err(const int* err) { return *reinterpret_cast<const volatile int*>(err); }

// Bounded mbarrier phase wait that also returns early once any block has flagged an error.
MK_COLD bool mk_bar_wait(uint32_t bar, uint32_t parity, int* err) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    if (mbar_try(bar, parity)) return true;
    if ((i & 255) == 255) {
      if (mk_err(err)) return false;
      const uint64_t t = mk_now();
      if (t0 == 0) t0 = t;
      else if (t - t0 > MK_WAIT_NS) {
        atomicCAS(err, 0, 11);
        return false;
      }
    }
  }
}

// Grid barrier: arrive (after the block's consumers have synchronised) and wait for `target`.
DEVI void mk_arrive(unsigned* cnt) {
  __threadfence();
  atomicAdd(cnt, 1u);
}
MK_COLD bool mk_grid_wait(const unsigned* cnt, unsigned target, int* err) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    if ((int)(mk_ld_acquire(cnt) - target) >= 0) return true;
    if (mk_err(err)) return false;
    if ((i & 63) == 63) {
      const uint64_t t = mk_now();
      if (t0 == 0) t0 = t;
      else if (t - t0 > MK_WAIT_NS) {
        atomicCAS(err, 0, 12);
        return false;
      }
    }
  }
}

DEVI void mk_sync() { asm volatile("bar.sync 1, %0;" ::"n"(MK_CT) : "memory"); }

DEVI void mk_tma3(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
DEVI void mk_tma2(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

DEVI float4 ldcg4(const float* p) { return __ldcg(reinterpret_cast<const float4*>(p)); }
DEVI uint4 ldcg16(const void* p) { return __ldcg(reinterpret_cast<const uint4*>(p)); }

// E2M1 code -> exact bf16 bits (0, 0.5, 1, 1.5, 2, 3, 4, 6 and negatives).
DEVI uint32_t mk_e2m1(uint32_t c) {
  const uint32_t e = (c >> 1) & 3u, m = c & 1u;
  const uint32_t mag = e == 0 ? (m ? 0x3F00u : 0u) : (((e + 126u) << 7) | (m << 6));
  return mag | ((c & 8u) << 12);
}
// E4M3 scale byte -> bf16 bits, twice (exact: at most 4 significant bits).
DEVI uint32_t mk_e4m3x2(uint32_t b) {
  const uint32_t s = (b & 0x80u) << 8;
  const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
  uint32_t bits = e == 0 ? (__float_as_uint((float)m * (1.0f / 512.0f)) >> 16) : (((e + 120u) << 7) | (m << 4));
  bits |= s;
  return bits | (bits << 16);
}
DEVI uint32_t mk_hmul2(uint32_t a, uint32_t b) {
  __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a), y = *reinterpret_cast<__nv_bfloat162*>(&b);
  __nv_bfloat162 r = __hmul2(x, y);
  return *reinterpret_cast<uint32_t*>(&r);
}

// ------------------------------------------------------------------------------ schedule
struct MkCtx {
  int nb;
  int pos[MK_MAX_NB], slot[MK_MAX_NB];
};

// Key splits of stream b on a layer: 128 positions (full) or 64 ring slots (sliding) each.
DEVI int mk_nsplit(const MkCtx& c, int b, bool full) {
  const int nkeys = full ? c.pos[b] + 1 : min(c.pos[b] + 1, WIN);
  return full ? (nkeys + 127) / 128 : (nkeys + 63) / 64;
}

struct MkAttnUnit {
  int b, h, sp, nsplit, cnt, nst;
};
DEVI MkAttnUnit mk_attn_unit(const MkCtx& c, bool full, int u) {
  MkAttnUnit r{};
  for (int b = 0; b < c.nb; ++b) {
    const int ns = mk_nsplit(c, b, full);
    if (u < 4 * ns) {
      r.b = b;
      r.h = u / ns;
      r.sp = u % ns;
      r.nsplit = ns;
      const int nkeys = full ? c.pos[b] + 1 : min(c.pos[b] + 1, WIN);
      const int span = full ? 128 : 64;
      r.cnt = min(span, nkeys - r.sp * span);
      r.nst = (r.cnt + 63) / 64;
      return r;
    }
    u -= 4 * ns;
  }
  return r;
}

DEVI int mk_kind(int type, int sub) {
  if (type == 0) {
    const int k[4] = {MK_CONV, MK_OUT, MK_W13, MK_W2};
    return k[sub];
  }
  const int k[5] = {MK_QKVG, MK_ATTN, MK_OUT, MK_W13, MK_W2};
  return k[sub];
}

DEVI int mk_units(const MkModel& m, const MkCtx& c, int kind, bool full) {
  switch (kind) {
    case MK_CONV: return D / 16;
    case MK_QKVG: return NQKVG / 16 * MK_KS_QO;
    case MK_OUT: return D / 16 * MK_KS_QO;
    case MK_W13: return F / 8;
    case MK_W2: return (D / 16) * (m.fp4 ? MK_KS_W2F : MK_KS_W2);
    case MK_HEAD: return m.vocab / 16;
    default: {
      int n = 0;
      for (int b = 0; b < c.nb; ++b) n += 4 * mk_nsplit(c, b, full);
      return n;
    }
  }
}

// Stages of one GEMV unit.
DEVI int mk_gemv_stages(const MkModel& m, int kind) {
  switch (kind) {
    case MK_CONV: return D / G_CONV::KCH;
    case MK_W13: return m.fp4 ? 1 : D / G_W13::KCH;
    case MK_W2: return m.fp4 ? F / G_W2F::KCH / MK_KS_W2F : F / G_W2::KCH / MK_KS_W2;
    case MK_QKVG:
    case MK_OUT: return D / G_ROWS::KCH / MK_KS_QO;
    default: return D / G_ROWS::KCH;  // head: K = 2048
  }
}

// Units dealt per round: one per consumer warp, except the conv in_proj, whose units (a third of
// the rows of 16 channels over all of K, with the conv as epilogue) every warp works on together.
DEVI int mk_round(int kind) { return kind == MK_CONV ? 1 : MK_CW; }

DEVI int mk_ksplit(const MkModel& m, int kind) {
  if (kind == MK_QKVG || kind == MK_OUT) return MK_KS_QO;
  if (kind == MK_W2) return m.fp4 ? MK_KS_W2F : MK_KS_W2;
  return 1;
}

// ------------------------------------------------------------------------------ producer
// Weight-map slots per layer: 0 in_proj | qkvg, 1 out_proj | o_proj, 2 w1, 3 w3, 4 w2,
// 5..7 NVFP4 scales of w1, w3, w2; the head's map follows the last layer.
// L2 prefetches of the same boxes the loads fetch (no shared memory, no barrier).
DEVI void mk_pf3(const CUtensorMap* map, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z)
               : "memory");
}
DEVI void mk_pf2(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}
// One box: a load into shared memory (completing on bar) or, with PF, an L2 prefetch.
template <bool PF>
DEVI void mk_box3(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
  if constexpr (PF) mk_pf3(map, x, y, z);
  else mk_tma3(dst, map, x, y, z, bar);
}
template <bool PF>
DEVI void mk_box2(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  if constexpr (PF) mk_pf2(map, x, y);
  else mk_tma2(dst, map, x, y, bar);
}

// The boxes of GEMV stage s of a unit (tile, K split ks): loaded into the slot at dst, arming
// bar with the stage's bytes, or (PF) prefetched into L2.
template <bool PF>
DEVI void mk_copy_gemv(const MkModel& m, int kind, const CUtensorMap* lm, int tile, int ks, int s, int nst,
                       uint32_t dst, uint32_t bar) {
  auto arm = [&](int bytes) {
    if constexpr (!PF) mbar_expect_tx(bar, bytes);
  };
  switch (kind) {
    case MK_CONV: {
      arm(G_CONV::BYTES);
      const int kb = s * G_CONV::NKB;
#pragma unroll
      for (int q = 0; q < 3; ++q) mk_box3<PF>(dst + q * G_CONV::REQB, lm + 0, 0, q * D + tile * 16, kb, bar);
      break;
    }
    case MK_QKVG:
    case MK_OUT:
    case MK_HEAD: {
      arm(G_ROWS::BYTES);
      mk_box3<PF>(dst, lm + (kind == MK_OUT ? 1 : 0), 0, tile * 16, (ks * nst + s) * G_ROWS::NKB, bar);
      break;
    }
    case MK_W13: {
      if (m.fp4) {
        arm(G_W13F::BYTES);
        mk_box3<PF>(dst, lm + 2, 0, tile * 8, 0, bar);
        mk_box3<PF>(dst + G_W13F::REQB, lm + 3, 0, tile * 8, 0, bar);
        const uint32_t sc = dst + G_W13F::RPT * G_W13F::ROWB;
        mk_box2<PF>(sc, lm + 5, 0, tile * 8, bar);
        mk_box2<PF>(sc + 8 * G_W13F::SCB, lm + 6, 0, tile * 8, bar);
      } else {
        arm(G_W13::BYTES);
        mk_box3<PF>(dst, lm + 2, 0, tile * 8, s * G_W13::NKB, bar);
        mk_box3<PF>(dst + G_W13::REQB, lm + 3, 0, tile * 8, s * G_W13::NKB, bar);
      }
      break;
    }
    case MK_W2: {
      if (m.fp4) {
        arm(G_W2F::BYTES);
        const int k0 = (ks * nst + s) * G_W2F::KCH;
        mk_box3<PF>(dst, lm + 4, 0, tile * 16, k0 / G_W2F::KB, bar);
        mk_box2<PF>(dst + G_W2F::RPT * G_W2F::ROWB, lm + 7, k0 / 16, tile * 16, bar);
      } else {
        arm(G_W2::BYTES);
        mk_box3<PF>(dst, lm + 4, 0, tile * 16, (ks * nst + s) * G_W2::NKB, bar);
      }
      break;
    }
  }
}

// ------------------------------------------------------------------------------ consumer pieces
// One K block (64 bytes of each of the stage's rows) against the activations, into chain ch.
template <class G, int CH>
DEVI void mk_mma_block(const unsigned char* st, int j, const bf16* xrow, const bf16* xzero, int kx,
                       const uint32_t* lut, float (&acc)[G::NRT][G::CH][4], int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int rt = 0; rt < G::NRT; ++rt) {
    const uint4 wa = *reinterpret_cast<const uint4*>(st + mk_woff<G>(rt * 16 + g, j, t));
    const uint4 wb = *reinterpret_cast<const uint4*>(st + mk_woff<G>(rt * 16 + g + 8, j, t));
    if constexpr (!G::FP4) {
      const uint4 xv = *reinterpret_cast<const uint4*>(xrow ? xrow + kx + 8 * t : xzero);
      mma_bf16_16816(acc[rt][CH], wa.x, wb.x, wa.y, wb.y, xv.x, xv.y);
      mma_bf16_16816(acc[rt][CH], wa.z, wb.z, wa.w, wb.w, xv.z, xv.w);
    } else {
      const unsigned char* sc = st + G::RPT * G::ROWB;
      const uint32_t sa = *reinterpret_cast<const uint16_t*>(sc + (rt * 16 + g) * G::SCB + j * 8 + 2 * t);
      const uint32_t sb = *reinterpret_cast<const uint16_t*>(sc + (rt * 16 + g + 8) * G::SCB + j * 8 + 2 * t);
      const uint32_t s0a = mk_e4m3x2(sa & 0xFF), s1a = mk_e4m3x2(sa >> 8);
      const uint32_t s0b = mk_e4m3x2(sb & 0xFF), s1b = mk_e4m3x2(sb >> 8);
      const uint32_t wA[4] = {wa.x, wa.y, wa.z, wa.w};
      const uint32_t wB[4] = {wb.x, wb.y, wb.z, wb.w};
      const uint32_t* tab = lut + lane;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t a01 = tab[(wA[q] & 0xFFu) << 5], a23 = tab[((wA[q] >> 8) & 0xFFu) << 5];
        uint32_t a45 = tab[((wA[q] >> 16) & 0xFFu) << 5], a67 = tab[(wA[q] >> 24) << 5];
        uint32_t b01 = tab[(wB[q] & 0xFFu) << 5], b23 = tab[((wB[q] >> 8) & 0xFFu) << 5];
        uint32_t b45 = tab[((wB[q] >> 16) & 0xFFu) << 5], b67 = tab[(wB[q] >> 24) << 5];
        const uint32_t sA = q < 2 ? s0a : s1a, sB = q < 2 ? s0b : s1b;
        a01 = mk_hmul2(a01, sA); a23 = mk_hmul2(a23, sA); a45 = mk_hmul2(a45, sA); a67 = mk_hmul2(a67, sA);
        b01 = mk_hmul2(b01, sB); b23 = mk_hmul2(b23, sB); b45 = mk_hmul2(b45, sB); b67 = mk_hmul2(b67, sB);
        const uint4 xv = *reinterpret_cast<const uint4*>(xrow ? xrow + kx + 32 * t + 8 * q : xzero);
        mma_bf16_16816(acc[rt][q], a01, b01, a23, b23, xv.x, xv.y);  // NVFP4: one chain per word
        mma_bf16_16816(acc[rt][q], a45, b45, a67, b67, xv.z, xv.w);
      }
    }
  }
}

// A whole stage by one warp: its K blocks round-robin over the accumulator chains.
template <class G>
DEVI void mk_mma_stage(const unsigned char* st, const bf16* xs, const bf16* xzero, int nb, int kbase,
                       const uint32_t* lut, float (&acc)[G::NRT][G::CH][4], int lane) {
  const int g = lane >> 2;
  const bf16* xrow = g < nb ? xs + (size_t)g * MK_XS : nullptr;
  if constexpr (G::FP4) {  // the 4 words of a block already feed 4 chains
#pragma unroll 1
    for (int j = 0; j < G::NKB; ++j) mk_mma_block<G, 0>(st, j, xrow, xzero, kbase + j * G::KB, lut, acc, lane);
    return;
  } else if constexpr (G::CH == 1) {  // three row tiles already give three chains
#pragma unroll 2
    for (int j = 0; j < G::NKB; ++j) mk_mma_block<G, 0>(st, j, xrow, xzero, kbase + j * G::KB, lut, acc, lane);
    return;
  }
#pragma unroll 1
  for (int j = 0; j < G::NKB; j += 4) {
    const int kx = kbase + j * G::KB;
    mk_mma_block<G, 0>(st, j, xrow, xzero, kx, lut, acc, lane);
    if (j + 1 < G::NKB) mk_mma_block<G, 1 % G::CH>(st, j + 1, xrow, xzero, kx + G::KB, lut, acc, lane);
    if (j + 2 < G::NKB) mk_mma_block<G, 2 % G::CH>(st, j + 2, xrow, xzero, kx + 2 * G::KB, lut, acc, lane);
    if (j + 3 < G::NKB) mk_mma_block<G, 3 % G::CH>(st, j + 3, xrow, xzero, kx + 3 * G::KB, lut, acc, lane);
  }
}

struct MkRing {
  unsigned char* slots;
  uint32_t full0, empty0;
  int nslot;
  uint32_t it;                  // first stream position of the next phase
  unsigned long long* wait_ns;  // profiling: warp 0's time spent waiting for stages (null: off)
  const volatile uint32_t* issued;  // stream positions the producer has issued so far
};

// Bounded wait until the producer has issued stream position pos. Warps take their stages out of
// stream order, so a warp may reach position pos before pos - nslot (the slot's previous
// occupant) has even been issued; a parity wait on the slot's barrier then would match an older
// phase. Once pos is issued, the slot's barrier is in pos's phase.
MK_COLD bool mk_wait_issued(const volatile uint32_t* issued, uint32_t pos, int* err) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    if ((int)(*issued - pos) > 0) return true;
    if ((i & 255) == 255) {
      if (mk_err(err)) return false;
      const uint64_t t = mk_now();
      if (t0 == 0) t0 = t;
      else if (t - t0 > MK_WAIT_NS) {
        atomicCAS(err, 0, 13);
        return false;
      }
    }
  }
}

// Wait (lane 0) for the stage at stream position pos; its address, or null once the block gave up.
DEVI const unsigned char* mk_take(const MkRing& R, uint32_t pos, int lane, int* err, int* abort_flag) {
  const int s = pos % R.nslot;
  bool ok = !*reinterpret_cast<volatile int*>(abort_flag);
  if (ok && lane == 0) {
    const uint64_t t0 = R.wait_ns && threadIdx.x == 0 ? mk_now() : 0;
    ok = mk_wait_issued(R.issued, pos, err) && mk_bar_wait(R.full0 + 8 * s, (pos / R.nslot) & 1, err);
    if (t0) *R.wait_ns += mk_now() - t0;
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (!ok) {
    *reinterpret_cast<volatile int*>(abort_flag) = 1;
    return nullptr;
  }
  return R.slots + (size_t)s * MK_SLOT;
}
// Hand the slot of stream position pos back to the producer (one arrival per stage).
DEVI void mk_release(const MkRing& R, uint32_t pos, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(R.empty0 + 8 * (pos % R.nslot));
}

// One GEMV unit by one warp: stages at positions pos0, pos0 + stride, ...; finished sums (chains
// added) in out; false once the block gave up.
template <class G>
DEVI bool mk_warp_unit(const MkRing& R, uint32_t pos0, int stride, int nst, int kfirst, const bf16* xs,
                       const bf16* xzero, int nb, const uint32_t* lut, float (&out)[G::NRT][4], int* err,
                       int* abort_flag, int lane) {
  float acc[G::NRT][G::CH][4];
#pragma unroll
  for (int rt = 0; rt < G::NRT; ++rt)
#pragma unroll
    for (int c = 0; c < G::CH; ++c)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[rt][c][j] = 0.f;
  bool ok = true;
  for (int s = 0; s < nst; ++s) {
    const uint32_t pos = pos0 + (uint32_t)(s * stride);
    const unsigned char* st = mk_take(R, pos, lane, err, abort_flag);
    if (!st) {
      ok = false;
      break;
    }
    mk_mma_stage<G>(st, xs, xzero, nb, kfirst + s * G::KCH, lut, acc, lane);
    mk_release(R, pos, lane);
  }
#pragma unroll
  for (int rt = 0; rt < G::NRT; ++rt)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if constexpr (G::CH == 4)
        out[rt][j] = (acc[rt][0][j] + acc[rt][1][j]) + (acc[rt][2][j] + acc[rt][3][j]);
      else
        out[rt][j] = acc[rt][0][j];
    }
  return ok;
}

// Sandwich step into shared memory: x' = x_in + g_post * RMS(sum of n_parts partials) (no parts:
// x' = x_in; x_in null: the embedding rows), block 0 writes x' to x_out and dump; if g_next, the
// block's activations become bf16(g_next * RMS(x')).
struct MkNorm {
  const float* x_in;
  const bf16* emb;        // x_in == null: embedding table (tokens) or input vectors
  const int32_t* tokens;
  const float* parts;
  int n_parts;
  const bf16* g_post;
  const bf16* g_next;
  float* x_out;
  float* dump;
  unsigned long long* stamp;  // profiling: [0] loads in and first sum, [1] done (null: off)
};
DEVI void mk_unpack8(uint4 w, float* v) {
  v[0] = bflo(w.x); v[1] = bfhi(w.x); v[2] = bflo(w.y); v[3] = bfhi(w.y);
  v[4] = bflo(w.z); v[5] = bfhi(w.z); v[6] = bflo(w.w); v[7] = bfhi(w.w);
}

// The gains are requested before anything else (an HBM or L2 round trip each), then each
// stream's residual row and partial sums; one block reduction per stream gives both norms: with
// a = RMS^-1 of the partials' sum m and the post gain g, x' = x + a g m, so
// sum(x'^2) = sum(x^2) + 2a sum(g x m) + a^2 sum(g^2 m^2).
MK_COLD void mk_norm(const MkNorm& p, int nb, float eps, bool writer, bf16* xs, float* red, int ct) {
  const int warp = ct >> 5, lane = ct & 31;
  const int i0 = ct * 8;  // 256 threads x 8 = d_model
  float gp[8], gn[8];
  const uint4 z4 = make_uint4(0, 0, 0, 0);
  const uint4 gpw = p.n_parts > 0 ? ldg16(p.g_post + i0) : z4;
  const uint4 gnw = p.g_next ? ldg16(p.g_next + i0) : z4;
  for (int b = 0; b < nb; ++b) {
    float x[8], mv[8];
    if (p.x_in) {
      const float4 a = ldcg4(p.x_in + (size_t)b * D + i0), c = ldcg4(p.x_in + (size_t)b * D + i0 + 4);
      x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = c.x; x[5] = c.y; x[6] = c.z; x[7] = c.w;
    } else {
      const bf16* src = p.tokens ? p.emb + (size_t)p.tokens[b] * D : p.emb + (size_t)b * D;
      mk_unpack8(ldg16(src + i0), x);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) mv[j] = 0.f;
    for (int s = 0; s < p.n_parts; ++s) {
      const float* q = p.parts + ((size_t)s * nb + b) * D + i0;
      const float4 a = ldcg4(q), c = ldcg4(q + 4);
      mv[0] += a.x; mv[1] += a.y; mv[2] += a.z; mv[3] += a.w; mv[4] += c.x; mv[5] += c.y; mv[6] += c.z; mv[7] += c.w;
    }
    if (b == 0) {
      mk_unpack8(gpw, gp);
      mk_unpack8(gnw, gn);
    }
    float q[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float gm = gp[j] * mv[j];
      q[0] += mv[j] * mv[j];
      q[1] += x[j] * x[j];
      q[2] += x[j] * gm;
      q[3] += gm * gm;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) q[c] = warp_sum(q[c]);
    if (lane == 0) *reinterpret_cast<float4*>(red + warp * 4) = make_float4(q[0], q[1], q[2], q[3]);
    if (b == 0 && p.stamp && ct == 0) p.stamp[0] = mk_now();
    mk_sync();
    float t[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int w = 0; w < MK_CW; ++w)
#pragma unroll
      for (int c = 0; c < 4; ++c) t[c] += red[w * 4 + c];
    const float a = p.n_parts > 0 ? rsqrtf(t[0] * (1.0f / D) + eps) : 0.f;
    const float inv = rsqrtf(fmaxf(t[1] + 2.f * a * t[2] + a * a * t[3], 0.f) * (1.0f / D) + eps);
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] += a * (gp[j] * mv[j]);
    if (writer) {
      const float4 lo = make_float4(x[0], x[1], x[2], x[3]), hi = make_float4(x[4], x[5], x[6], x[7]);
      if (p.x_out) {
        float4* o = reinterpret_cast<float4*>(p.x_out + (size_t)b * D + i0);
        o[0] = lo;
        o[1] = hi;
      }
      if (p.dump) {
        float4* o = reinterpret_cast<float4*>(p.dump + (size_t)b * D + i0);
        o[0] = lo;
        o[1] = hi;
      }
    }
    if (p.g_next) {
      uint32_t w4[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) w4[j] = pack_bf2(gn[2 * j] * (x[2 * j] * inv), gn[2 * j + 1] * (x[2 * j + 1] * inv));
      *reinterpret_cast<uint4*>(xs + (size_t)b * MK_XS + i0) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
    mk_sync();  // the reduction slots are reused by the next stream; the activations are complete
  }
  if (p.stamp && ct == 0) p.stamp[1] = mk_now();
}

// Warm L2 with a small constant vector a coming phase reads (the gains of a sandwich step).
DEVI void mk_prefetch_l2(const void* p, int bytes, int ct) {
  if (p && ct >= 0 && ct * 128 < bytes) asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(p) + ct * 128));
}

// bf16 activations [nb][K] (written earlier in this launch) -> shared memory.
MK_COLD void mk_load_x(const bf16* src, int K, int nb, bf16* xs, int ct) {
  const int chunks = K / 8;
  for (int idx = ct; idx < nb * chunks; idx += MK_CT) {
    const int b = idx / chunks, c = idx - b * chunks;
    *reinterpret_cast<uint4*>(xs + (size_t)b * MK_XS + c * 8) = ldcg16(src + (size_t)b * K + c * 8);
  }
  mk_sync();
}

// ------------------------------------------------------------------------------ attention unit
// K / V tile of 64 rows x 128 dims as two 64-column halves of 8 KB, 128-byte swizzled.
DEVI int mk_kv_off(int r, int d) {
  return (d >> 6) * 8192 + r * 128 + ((((d & 63) >> 3) ^ (r & 7)) << 4) + (d & 7) * 2;
}

MK_COLD bool mk_attn_unit(const MkModel& m, const MkStep& S, const MkCtx& C, const MkLayer& L, const MkAttnUnit& U,
                       MkRing& R, float* scr, int* abort_flag, int ct) {
  const int warp = ct >> 5, lane = ct & 31;
  const bool full = L.type == 1;
  const int b = U.b, h = U.h, pos = C.pos[b], slot = C.slot[b];
  const int span = full ? 128 : 64;
  const int j0 = U.sp * span;
  const int cur = full ? pos : pos % WIN;
  const bool has_cur = cur >= j0 && cur < j0 + U.cnt;
  float* qs = scr;            // [4][128] rotated, rounded, pre-scaled queries
  float* kn = qs + 512;       // [128] new key (rounded), [128] new value
  float* vn = kn + 128;
  float* sc = vn + 128;       // [4][128] scores, then probabilities
  float* ored = sc + 512;     // [4 key groups][4 heads][128]
  float* wr = ored + 2048;    // [8 warps][2] reduction scratch
  float* hm = wr + 16;        // [4 heads][2]: max, sum
  const float* qkv = m.part3 + (size_t)b * NQKVG;  // K halves at qkv and qkv + half
  const size_t half = (size_t)C.nb * NQKVG;
  auto qkv_at = [&](int i) { return __ldcg(qkv + i) + __ldcg(qkv + half + i); };
  const float* cs = m.rope_cos[full ? 0 : 1] + (size_t)pos * (HD / 2);
  const float* sn = m.rope_sin[full ? 0 : 1] + (size_t)pos * (HD / 2);
  // ---- every global input of the unit is requested up front (each is an L2 round trip)
  const int hh = ct >> 6, d0 = (ct & 63) * 2;
  const bool kthr = has_cur && ct < 64, vthr = has_cur && ct >= 64 && ct < 128;
  const int qi = (4 * h + hh) * HD + d0;
  const float q0 = qkv_at(qi), q1 = qkv_at(qi + 1);
  const float gq0 = bf2f(L.q_norm[d0]), gq1 = bf2f(L.q_norm[d0 + 1]);
  float k0 = 0.f, k1 = 0.f, gk0 = 0.f, gk1 = 0.f, v0n = 0.f, v1n = 0.f;
  if (kthr) {
    const int ki = HQ * HD + h * HD + d0;
    k0 = qkv_at(ki);
    k1 = qkv_at(ki + 1);
    gk0 = bf2f(L.k_norm[d0]);
    gk1 = bf2f(L.k_norm[d0 + 1]);
  } else if (vthr) {
    const int vi = HQ * HD + HKV * HD + h * HD + (ct - 64) * 2;
    v0n = qkv_at(vi);
    v1n = qkv_at(vi + 1);
  }
  const float gate_logit = qkv_at(HQ * HD + 2 * HKV * HD + 4 * h + hh);
  const int i0 = d0 & 63;  // this thread's dims d0, d0 + 1 rotate with pair coefficients i0, i0 + 1
  const float cs0 = cs[i0], cs1 = cs[i0 + 1], sn0 = sn[i0], sn1 = sn[i0 + 1];
  // ---- q and k RMS norms (a head spans two warps; the key lives in warps 0-1)
  {
    const float sq = warp_sum(q0 * q0 + q1 * q1);
    const float sk = warp_sum(k0 * k0 + k1 * k1);
    if (lane == 0) {
      wr[warp] = sq;
      wr[8 + warp] = sk;
    }
    mk_sync();
    const float inv = rsqrtf((wr[2 * hh] + wr[2 * hh + 1]) * (1.0f / HD) + m.eps);
    qs[hh * HD + d0] = gq0 * (q0 * inv);
    qs[hh * HD + d0 + 1] = gq1 * (q1 * inv);
    if (kthr) {
      const float ik = rsqrtf((wr[8] + wr[9]) * (1.0f / HD) + m.eps);
      kn[d0] = gk0 * (k0 * ik);
      kn[d0 + 1] = gk1 * (k1 * ik);
    } else if (vthr) {
      vn[(ct - 64) * 2] = round_bf(v0n);
      vn[(ct - 64) * 2 + 1] = round_bf(v1n);
    }
  }
  mk_sync();
  // ---- rotary embedding on pairs (i, i + 64), then bf16 rounding (queries pre-scaled)
  {
    const float scale = rsqrtf((float)HD);
    float r[2], rk[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int d = d0 + e;
      const float c = e ? cs1 : cs0, sgn = e ? sn1 : sn0;
      const float* v = qs + hh * HD;
      r[e] = d < 64 ? v[d] * c - v[d + 64] * sgn : v[d] * c + v[d - 64] * sgn;
      if (kthr) rk[e] = d < 64 ? kn[d] * c - kn[d + 64] * sgn : kn[d] * c + kn[d - 64] * sgn;
    }
    mk_sync();
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      qs[hh * HD + d0 + e] = round_bf(r[e]) * scale;
      if (kthr) kn[d0 + e] = round_bf(rk[e]);
    }
  }
  mk_sync();
  // ---- the split's key / value tiles
  const unsigned char* tiles[2] = {nullptr, nullptr};
  for (int i = 0; i < U.nst; ++i) tiles[i] = mk_take(R, R.it + i, lane, m.err, abort_flag);
  mk_sync();  // a warp whose wait gave up has raised the flag by now: the decision below is uniform
  if (!*reinterpret_cast<volatile int*>(abort_flag)) {
    // scores: thread (head hh, key jj of each 64-key tile)
    const int jj = ct & 63;
    float s[2] = {-INFINITY, -INFINITY};
    for (int i = 0; i < U.nst; ++i) {
      const int j = 64 * i + jj;
      if (j >= U.cnt) continue;
      float a = 0.f;
      const float* q = qs + hh * HD;
      if (j0 + j == cur) {
#pragma unroll 8
        for (int d = 0; d < HD; ++d) a += q[d] * kn[d];
      } else {
        const unsigned char* kt = tiles[i];
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(kt + mk_kv_off(jj, c * 8));
          const float* qc = q + c * 8;
          a += qc[0] * bflo(w.x) + qc[1] * bfhi(w.x) + qc[2] * bflo(w.y) + qc[3] * bfhi(w.y) + qc[4] * bflo(w.z) +
               qc[5] * bfhi(w.z) + qc[6] * bflo(w.w) + qc[7] * bfhi(w.w);
        }
      }
      s[i] = a;
    }
    float mx = warp_max(fmaxf(s[0], s[1]));
    if (lane == 0) wr[warp] = mx;
    mk_sync();
    mx = fmaxf(wr[2 * hh], wr[2 * hh + 1]);
    float l = 0.f;
    for (int i = 0; i < 2; ++i) {
      const float p = s[i] == -INFINITY ? 0.f : __expf(s[i] - mx);
      sc[hh * 128 + 64 * i + jj] = p;
      l += p;
    }
    l = warp_sum(l);
    if (lane == 0) wr[8 + warp] = l;
    mk_sync();
    if ((ct & 63) == 0) {
      hm[2 * hh] = mx;
      hm[2 * hh + 1] = wr[8 + 2 * hh] + wr[8 + 2 * hh + 1];
    }
    // P V: thread (key group kg = ct / 64, dims dp, dp + 1) over keys kg, kg + 4, ...
    const int kg = ct >> 6, dp = (ct & 63) * 2;
    float o[4][2] = {};
    for (int j = kg; j < U.cnt; j += 4) {
      float v0, v1;
      if (j0 + j == cur) {
        v0 = vn[dp];
        v1 = vn[dp + 1];
      } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(tiles[j >> 6] + 16384 + mk_kv_off(j & 63, dp));
        v0 = bflo(w);
        v1 = bfhi(w);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float p = sc[q * 128 + j];
        o[q][0] += p * v0;
        o[q][1] += p * v1;
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      ored[(kg * 4 + q) * HD + dp] = o[q][0];
      ored[(kg * 4 + q) * HD + dp + 1] = o[q][1];
    }
  }
  mk_sync();  // every warp is done with the tiles
  if (warp == 0)
    for (int i = 0; i < U.nst; ++i) mk_release(R, R.it + i, lane);
  R.it += U.nst;
  if (*reinterpret_cast<volatile int*>(abort_flag)) return false;
  // ---- this split's partial result, and the new key / value into the cache
  {
    const int stride = S.attn_splits;
    float* out = S.attn_part + (((size_t)b * HQ + 4 * h + hh) * stride + U.sp) * (HD + 2);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int d = d0 + e;
      out[d] = ored[(0 * 4 + hh) * HD + d] + ored[(1 * 4 + hh) * HD + d] + ored[(2 * 4 + hh) * HD + d] +
               ored[(3 * 4 + hh) * HD + d];
    }
    if ((ct & 63) == 0) {
      out[HD] = hm[2 * hh];
      out[HD + 1] = hm[2 * hh + 1];
    }
    if (has_cur && ct < 128) {
      bf16* kb;
      bf16* vb;
      if (full) {
        const int page = S.page_table[(size_t)slot * m.max_pages + pos / PAGE];
        const size_t off = ((((size_t)L.kidx * m.n_pages + page) * HKV + h) * PAGE + pos % PAGE) * HD;
        kb = S.kv_k + off;
        vb = S.kv_v + off;
      } else {
        const size_t off = ((((size_t)L.kidx * m.max_streams + slot) * HKV + h) * WIN + pos % WIN) * HD;
        kb = S.ring_k + off;
        vb = S.ring_v + off;
      }
      const int d = ct < 64 ? d0 : (ct - 64) * 2;
      if (ct < 64) {
        *reinterpret_cast<uint32_t*>(kb + d) = pack_bf2(kn[d], kn[d + 1]);
      } else {
        *reinterpret_cast<uint32_t*>(vb + d) = pack_bf2(vn[d], vn[d + 1]);
      }
    }
  }
  // ---- the last split of (stream, kv head) to finish merges, gates and writes the output
  __shared__ int last_flag;
  mk_sync();
  if (ct == 0) {
    __threadfence();
    const unsigned old = atomicAdd(m.sync + 16 + b * HKV + h, 1u);
    last_flag = old == (unsigned)(U.nsplit - 1);
  }
  mk_sync();
  if (last_flag) {
    __threadfence();
    const int stride = S.attn_splits;
    const float* base = S.attn_part + ((size_t)b * HQ + 4 * h + hh) * stride * (HD + 2);
    // one pass with a running maximum: each split's loads are independent of the previous sums
    float M = -INFINITY, l = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll 4
    for (int s = 0; s < U.nsplit; ++s) {
      const float* p = base + (size_t)s * (HD + 2);
      const float ms = __ldcg(p + HD), ls = __ldcg(p + HD + 1), a0 = __ldcg(p + d0), a1 = __ldcg(p + d0 + 1);
      if (ms == -INFINITY) continue;
      const float Mn = fmaxf(M, ms);
      const float fo = __expf(M - Mn), fs = __expf(ms - Mn);
      l = l * fo + ls * fs;
      o0 = o0 * fo + a0 * fs;
      o1 = o1 * fo + a1 * fs;
      M = Mn;
    }
    const float gt = sigmoidf_(gate_logit);
    *reinterpret_cast<uint32_t*>(m.y + (size_t)b * D + (4 * h + hh) * HD + d0) = pack_bf2(gt * (o0 / l), gt * (o1 / l));
    if (ct == 0) atomicExch(m.sync + 16 + b * HKV + h, 0u);
  }
  return true;
}

// ------------------------------------------------------------------------------ conv in_proj unit
// The B, C and x rows of 16 channels over all of K (8 stages of 256): warp w accumulates stages
// w, w + 8, ..., the partial sums meet in shared memory, then the gated conv over the carried
// columns and the state shift. Every consumer warp calls this (block-level synchronisation).
MK_COLD bool mk_conv_unit(const MkModel& m, const MkStep& S, const MkCtx& C, const MkLayer& L, int tile, int nst,
                       const MkRing& R, uint32_t base, const bf16* xs, const bf16* xzero, int nb, float* red, int lane,
                       int warp, int ct, int* abort_flag) {
  float o[3][4] = {};
  bool ok = true;
  for (int s = warp; s < nst && ok; s += MK_CW) {
    float p[3][4];
    ok = mk_warp_unit<G_CONV>(R, base + s, 0, 1, s * G_CONV::KCH, xs, xzero, nb, nullptr, p, m.err, abort_flag, lane);
#pragma unroll
    for (int rt = 0; rt < 3; ++rt)
#pragma unroll
      for (int j = 0; j < 4; ++j) o[rt][j] += p[rt][j];
  }
#pragma unroll
  for (int rt = 0; rt < 3; ++rt)
    *reinterpret_cast<float4*>(red + ((warp * 3 + rt) * 32 + lane) * 4) = make_float4(o[rt][0], o[rt][1], o[rt][2], o[rt][3]);
  mk_sync();
  float* res = red + MK_CW * 3 * 128;  // [48 rows][8 columns]
  for (int e = ct; e < 3 * 128; e += MK_CT) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < MK_CW; ++w) sum += red[w * 3 * 128 + e];
    const int j = e & 3, ln = (e >> 2) & 31, rt = e >> 7;
    res[(rt * 16 + (ln >> 2) + (j >= 2 ? 8 : 0)) * 8 + 2 * (ln & 3) + (j & 1)] = sum;
  }
  mk_sync();
  if (!*reinterpret_cast<volatile int*>(abort_flag)) {
    bf16* state = S.conv_state + (size_t)L.kidx * m.max_streams * CST * D;
    for (int e = ct; e < 16 * nb; e += MK_CT) {
      const int cl = e & 15, b = e >> 4, c = tile * 16 + cl;
      const float bx = round_bf(res[cl * 8 + b] * res[(32 + cl) * 8 + b]);
      bf16* stt = state + (size_t)C.slot[b] * CST * D + c;
      float win[CST];
#pragma unroll
      for (int q = 0; q < CST; ++q) win[q] = bf2f(stt[(size_t)q * D]);
      const bf16* w = L.conv_w + (size_t)c * TAPS;
      float z = 0.f;
#pragma unroll
      for (int q = 0; q < CST; ++q) z += bf2f(w[q]) * win[q];
      z += bf2f(w[CST]) * bx;
      m.y[(size_t)b * D + c] = f2bf(res[(16 + cl) * 8 + b] * z);
#pragma unroll
      for (int q = 0; q < CST - 1; ++q) stt[(size_t)q * D] = f2bf(win[q + 1]);
      stt[(size_t)(CST - 1) * D] = f2bf(bx);
    }
  }
  mk_sync();  // the reduction buffers are free again
  return !*reinterpret_cast<volatile int*>(abort_flag);
}

// ------------------------------------------------------------------------------ GEMV units
// One unit of a GEMV phase by one warp, with its epilogue. Lane (g, t) ends holding rows g and
// g + 8 of each 16-row tile for streams 2t and 2t + 1.
template <bool FP4>
MK_COLD bool mk_gemv_unit(const MkModel& m, const MkStep& S, const MkCtx& C, const MkLayer& L, int kind, int tile,
                       int ks, int nst, const MkRing& R, uint32_t pos0, int stride, const bf16* xs, const bf16* xzero,
                       int nb, const uint32_t* lut, int* abort_flag, int lane) {
  const int g = lane >> 2, t = lane & 3;
  switch (kind) {
    case MK_CONV: {
      float o[3][4];
      if (!mk_warp_unit<G_CONV>(R, pos0, stride, nst, 0, xs, xzero, nb, lut, o, m.err, abort_flag, lane)) return false;
      bf16* state = S.conv_state + (size_t)L.kidx * m.max_streams * CST * D;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int b = 2 * t + (j & 1);
        if (b >= nb) continue;
        const int c = tile * 16 + g + (j >= 2 ? 8 : 0);
        const float bx = round_bf(o[0][j] * o[2][j]);
        bf16* stt = state + (size_t)C.slot[b] * CST * D + c;
        float win[CST];
#pragma unroll
        for (int q = 0; q < CST; ++q) win[q] = bf2f(stt[(size_t)q * D]);
        const bf16* w = L.conv_w + (size_t)c * TAPS;
        float z = 0.f;
#pragma unroll
        for (int q = 0; q < CST; ++q) z += bf2f(w[q]) * win[q];
        z += bf2f(w[CST]) * bx;
        m.y[(size_t)b * D + c] = f2bf(o[1][j] * z);
#pragma unroll
        for (int q = 0; q < CST - 1; ++q) stt[(size_t)q * D] = f2bf(win[q + 1]);
        stt[(size_t)(CST - 1) * D] = f2bf(bx);
      }
      return true;
    }
    case MK_QKVG:
    case MK_OUT: {
      float o[1][4];
      const int k0 = ks * nst * G_ROWS::KCH;
      if (!mk_warp_unit<G_ROWS>(R, pos0, stride, nst, k0, xs, xzero, nb, lut, o, m.err, abort_flag, lane)) return false;
      float* out = kind == MK_QKVG ? m.part3 : m.part;
      const int N = kind == MK_QKVG ? NQKVG : D;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int b = 2 * t + (j & 1);
        if (b < nb) out[((size_t)ks * nb + b) * N + tile * 16 + g + (j >= 2 ? 8 : 0)] = o[0][j];
      }
      return true;
    }
    case MK_W13: {
      float o[1][4];
      float sc = 1.f;
      if constexpr (FP4) {
        if (!mk_warp_unit<G_W13F>(R, pos0, stride, nst, 0, xs, xzero, nb, lut, o, m.err, abort_flag, lane)) return false;
        sc = L.w13_scale;
      } else if (!mk_warp_unit<G_W13>(R, pos0, stride, nst, 0, xs, xzero, nb, lut, o, m.err, abort_flag, lane)) {
        return false;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {  // rows g: w1 row, g + 8: the same row of w3
        const int b = 2 * t + j;
        if (b < nb) m.u[(size_t)b * F + tile * 8 + g] = f2bf(siluf_(o[0][j] * sc) * (o[0][j + 2] * sc));
      }
      return true;
    }
    case MK_W2: {
      float o[1][4];
      float sc = 1.f;
      if constexpr (FP4) {
        if (!mk_warp_unit<G_W2F>(R, pos0, stride, nst, ks * nst * G_W2F::KCH, xs, xzero, nb, lut, o, m.err, abort_flag,
                                 lane))
          return false;
        sc = L.w2_scale;
      } else if (!mk_warp_unit<G_W2>(R, pos0, stride, nst, ks * nst * G_W2::KCH, xs, xzero, nb, lut, o, m.err,
                                     abort_flag, lane)) {
        return false;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int b = 2 * t + (j & 1);
        if (b < nb) m.part2[((size_t)ks * nb + b) * D + tile * 16 + g + (j >= 2 ? 8 : 0)] = o[0][j] * sc;
      }
      return true;
    }
    default: {  // MK_HEAD: logits and the running greedy argmax (ties: the lowest id)
      float o[1][4];
      if (!mk_warp_unit<G_ROWS>(R, pos0, stride, nst, 0, xs, xzero, nb, lut, o, m.err, abort_flag, lane)) return false;
#pragma unroll
      for (int jb = 0; jb < 2; ++jb) {
        const int b = 2 * t + jb;
        const float v0 = o[0][jb], v1 = o[0][jb + 2];  // rows g, g + 8
        if (b < nb && S.logits) {
          S.logits[(size_t)b * m.vocab + tile * 16 + g] = v0;
          S.logits[(size_t)b * m.vocab + tile * 16 + g + 8] = v1;
        }
        float best = v0;
        int idx = g;
        if (v1 > v0) {
          best = v1;
          idx = g + 8;
        }
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {  // across g, same t
          const float ob = __shfl_xor_sync(0xffffffffu, best, off);
          const int oi = __shfl_xor_sync(0xffffffffu, idx, off);
          if (ob > best || (ob == best && oi < idx)) {
            best = ob;
            idx = oi;
          }
        }
        if (g == 0 && b < nb) {
          uint32_t key = __float_as_uint(best);
          key = (key & 0x80000000u) ? ~key : (key | 0x80000000u);
          atomicMax(m.amax + b, ((unsigned long long)key << 32) | (0xffffffffu - (uint32_t)(tile * 16 + idx)));
        }
      }
      return true;
    }
  }
}

// ------------------------------------------------------------------------------ producer cursor
// A position in the block's stream of stages: phase (layer l, step sub; l == n_layers is the
// head) and stage k of the block's stages in that phase, in the order the consumers take them.
// The producer walks two: one issuing the loads into the ring, one running ahead of it issuing
// the same boxes as L2 prefetches, so HBM keeps streaming while the consumers sit at a barrier.
struct MkCursor {
  int l, sub, kind, rot, first, n, nst, ks, units, total, k, phase;
  int r0, nr, s, i;   // GEMV: round, its units, stage, unit within the round
  int j, ai;          // attention: the block's unit j, its stage ai
  MkAttnUnit U;
  bool full, done;
};

MK_COLD void mk_cursor_setup(MkCursor& c, const MkModel& m, const MkCtx& C, int cta, int G, bool do_head) {
  for (;;) {
    if (c.l > m.n_layers || (c.l == m.n_layers && !do_head)) {
      c.done = true;
      return;
    }
    const int type = c.l < m.n_layers ? m.layers[c.l].type : 0;
    c.kind = c.l < m.n_layers ? mk_kind(type, c.sub) : MK_HEAD;
    c.full = type == 1;
    c.units = mk_units(m, C, c.kind, c.full);
    c.first = (cta - c.rot % G + G) % G;
    c.n = c.units > c.first ? (c.units - c.first + G - 1) / G : 0;
    c.k = 0;
    c.r0 = c.s = c.i = c.j = c.ai = 0;
    c.nr = min(mk_round(c.kind), c.n);
    if (c.kind == MK_ATTN) {
      c.total = 0;
      for (int j = 0; j < c.n; ++j) c.total += mk_attn_unit(C, c.full, c.first + j * G).nst;
      if (c.n > 0) c.U = mk_attn_unit(C, c.full, c.first);
    } else {
      c.nst = mk_gemv_stages(m, c.kind);
      c.ks = mk_ksplit(m, c.kind);
      c.total = c.n * c.nst;
    }
    if (c.total > 0) return;
    // the block has nothing to fetch in this phase: on to the next
    c.rot = (c.rot + c.units) % G;
    ++c.phase;
    if (c.l < m.n_layers && ++c.sub < (type == 0 ? 4 : 5)) continue;
    c.sub = 0;
    ++c.l;
  }
}

MK_COLD void mk_cursor_init(MkCursor& c, const MkModel& m, const MkCtx& C, int cta, int G, bool do_head) {
  c = MkCursor{};
  mk_cursor_setup(c, m, C, cta, G, do_head);
}

MK_COLD void mk_cursor_next(MkCursor& c, const MkModel& m, const MkCtx& C, int cta, int G, bool do_head) {
  if (++c.k < c.total) {
    if (c.kind == MK_ATTN) {
      if (++c.ai == c.U.nst) {
        c.ai = 0;
        ++c.j;
        c.U = mk_attn_unit(C, c.full, c.first + c.j * G);
      }
    } else if (++c.i == c.nr) {  // rounds are stage-major: all units' stage s, then stage s + 1
      c.i = 0;
      if (++c.s == c.nst) {
        c.s = 0;
        c.r0 += mk_round(c.kind);
        c.nr = min(mk_round(c.kind), c.n - c.r0);
      }
    }
    return;
  }
  c.rot = (c.rot + c.units) % G;
  ++c.phase;
  if (c.l < m.n_layers && ++c.sub < (m.layers[c.l].type == 0 ? 4 : 5)) {
    mk_cursor_setup(c, m, C, cta, G, do_head);
    return;
  }
  c.sub = 0;
  ++c.l;
  mk_cursor_setup(c, m, C, cta, G, do_head);
}

// The boxes of the cursor's stage: loads into the slot at dst (arming bar), or L2 prefetches.
template <bool PF>
MK_COLD void mk_copy_stage(const MkCursor& c, const MkModel& m, const MkStep& S, const MkCtx& C, int G,
                        const CUtensorMap* tkk, const CUtensorMap* tkv, const CUtensorMap* trk, const CUtensorMap* trv,
                        uint32_t dst, uint32_t bar) {
  const CUtensorMap* lm = m.maps + (size_t)c.l * MK_MAPS;
  if (c.kind != MK_ATTN) {
    const int u = c.first + (c.r0 + c.i) * G;
    int tile = u, ks = 0;  // constant divisors: the K splits are 1..4
    switch (c.ks) {
      case 2: tile = u >> 1; ks = u & 1; break;
      case 3: tile = u / 3; ks = u - 3 * tile; break;
      case 4: tile = u >> 2; ks = u & 3; break;
      default: break;
    }
    mk_copy_gemv<PF>(m, c.kind, lm, tile, ks, c.s, c.nst, dst, bar);
    return;
  }
  // attention: the block's units in order, each its key / value tiles of 64 positions
  const int k = c.ai;
  const MkAttnUnit& U = c.U;
  const MkLayer& L = m.layers[c.l];
  int row;
  const CUtensorMap* mk;
  const CUtensorMap* mv;
  if (c.full) {
    const int page = S.page_table[(size_t)C.slot[U.b] * m.max_pages + (U.sp * 128 + 64 * k) / PAGE];
    row = (((L.kidx * m.n_pages + page) * HKV) + U.h) * PAGE;
    mk = tkk;
    mv = tkv;
  } else {
    row = (((L.kidx * m.max_streams + C.slot[U.b]) * HKV) + U.h) * WIN + U.sp * 64;
    mk = trk;
    mv = trv;
  }
  if constexpr (!PF) mbar_expect_tx(bar, 4 * 8192);
  mk_box2<PF>(dst, mk, 0, row, bar);
  mk_box2<PF>(dst + 8192, mk, 64, row, bar);
  mk_box2<PF>(dst + 16384, mv, 0, row, bar);
  mk_box2<PF>(dst + 24576, mv, 64, row, bar);
}

// ------------------------------------------------------------------------------ the kernel
template <bool FP4>
__global__ void __launch_bounds__(MK_THREADS, 1) k_decode_mk(const __grid_constant__ CUtensorMap tkk,
                                                             const __grid_constant__ CUtensorMap tkv,
                                                             const __grid_constant__ CUtensorMap trk,
                                                             const __grid_constant__ CUtensorMap trv,
                                                             const MkModel m, const MkStep S) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nslot = m.nslot;
  unsigned char* slots = smem;
  bf16* xzero = reinterpret_cast<bf16*>(smem + (size_t)nslot * MK_SLOT);
  bf16* xs = xzero + 64;
  uint32_t* lut = reinterpret_cast<uint32_t*>(reinterpret_cast<unsigned char*>(xs) + (size_t)S.nb * MK_XS * 2);
  float* scr = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(lut) + (m.fp4 ? MK_LUT_BYTES : 0));
  uint64_t* bars = reinterpret_cast<uint64_t*>(scr + MK_SCR_FLOATS);
  __shared__ MkCtx C;
  __shared__ int abort_flag;
  __shared__ uint32_t issued;  // stream positions issued by the producer

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const uint32_t full0 = su32(bars), empty0 = su32(bars + nslot);
  if (tid == 0) {
    for (int s = 0; s < nslot; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    abort_flag = 0;
    issued = 0;
    C.nb = S.nb;
    for (int b = 0; b < S.nb; ++b) {
      C.slot[b] = S.slots[b];
      C.pos[b] = S.seq_len[C.slot[b]];
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  const bool do_head = m.has_head && (S.logits || S.argmax_out);

  if (warp == MK_CW) {
    // ========================================================== producer (one thread)
    if (lane != 0) return;
    // loads into the ring; L2 prefetches up to m.pf stages ahead of them (kept in shared memory:
    // this thread's registers are squeezed by the consumer paths' allocation, and spilled state
    // would round-trip to L2 on every stage)
    __shared__ MkCursor ld, pf;
    mk_cursor_init(ld, m, C, cta, G, do_head);
    mk_cursor_init(pf, m, C, cta, G, do_head);
    uint32_t it = 0, pit = 0;
    int slot = 0;
    uint32_t par = 1;  // parity of the slot's previous release (the first pass finds them free)
    unsigned long long* ptrace = m.trace ? m.trace + (size_t)cta * MK_TRACE_PHASES * MK_TRACE_WORDS : nullptr;
    int traced_phase = -1;
    while (!ld.done) {
      while (!pf.done && (int)(pit - it) < m.pf) {
        mk_copy_stage<true>(pf, m, S, C, G, &tkk, &tkv, &trk, &trv, 0u, 0u);
        mk_cursor_next(pf, m, C, cta, G, do_head);
        ++pit;
      }
      if (!mk_bar_wait(empty0 + 8 * slot, par, m.err)) break;
      if (*reinterpret_cast<volatile int*>(&abort_flag)) break;
      mk_copy_stage<false>(ld, m, S, C, G, &tkk, &tkv, &trk, &trv, su32(slots + (size_t)slot * MK_SLOT),
                           full0 + 8 * slot);
      ++it;
      *reinterpret_cast<volatile uint32_t*>(&issued) = it;  // after the slot's barrier is armed
      if (++slot == nslot) {
        slot = 0;
        par ^= 1u;
      }
      if (ptrace && ld.phase < MK_TRACE_PHASES) {
        const unsigned long long now = mk_now();
        unsigned long long* r = ptrace + MK_TRACE_WORDS * ld.phase;
        if (traced_phase != ld.phase) {  // first copy of the phase
          r[5] = now;
          traced_phase = ld.phase;
        }
        r[3] = now;  // last copy so far
      }
      mk_cursor_next(ld, m, C, cta, G, do_head);
    }
    // copies already issued land before the block exits (immediate unless the consumers gave up)
    for (int k = 0; k < nslot && k < (int)it; ++k) {
      const uint32_t i = it - 1 - k;
      mk_bar_wait(full0 + 8 * (i % nslot), (i / nslot) & 1, m.err);
    }
    return;
  }

  // ============================================================ consumers
  const int ct = tid;
  const int nb = C.nb;
  if (ct < 32) reinterpret_cast<uint32_t*>(xzero)[ct] = 0u;
  if (FP4)
    for (int i = ct; i < 256 * 32; i += MK_CT) {
      const uint32_t v = (uint32_t)i >> 5;
      lut[i] = mk_e2m1(v & 15u) | (mk_e2m1(v >> 4) << 16);
    }
  if (cta == 0 && ct < nb) m.amax[ct] = 0ull;
  MkRing R{slots, full0, empty0, nslot, 0, nullptr, &issued};
  float* red = scr;
  const bool writer = cta == 0;
  float* cur = m.x_res;
  float* nxt = m.x_res2;
  unsigned phase = 0;
  int rot = 0;
  bool ok = true;
  bool wok = true;  // this warp's units went through (the block decides at the phase barrier)
  const float* pend = nullptr;  // partial sums still to be added into the residual
  int pend_n = 0;
  const bf16* pend_g = nullptr;

  unsigned long long* trace = m.trace ? m.trace + (size_t)cta * MK_TRACE_PHASES * MK_TRACE_WORDS : nullptr;
  __shared__ unsigned long long wait_ns;
  if (trace && ct == 0) {
    trace[0] = mk_now();
    wait_ns = 0;
    R.wait_ns = &wait_ns;
  }
  auto barrier = [&]() -> bool {  // end of a phase: all blocks' outputs are visible after it
    mk_sync();
    if (ct == 0) {
      if (trace && phase < MK_TRACE_PHASES) {
        trace[MK_TRACE_WORDS * phase + 1] = mk_now();
        trace[MK_TRACE_WORDS * phase + 2] = wait_ns;
        wait_ns = 0;
      }
      mk_arrive(m.sync);
      if (!mk_grid_wait(m.sync, (phase + 1) * (unsigned)G, m.err)) abort_flag = 1;
    }
    ++phase;
    if (trace && ct == 0 && phase < MK_TRACE_PHASES) trace[MK_TRACE_WORDS * phase] = mk_now();
    mk_sync();
    return !*reinterpret_cast<volatile int*>(&abort_flag);
  };

  for (int l = 0; l < m.n_layers && ok; ++l) {
    const MkLayer& L = m.layers[l];
    const int nsub = L.type == 0 ? 4 : 5;
    for (int sub = 0; sub < nsub && ok; ++sub) {
      const int kind = mk_kind(L.type, sub);
      const bool full = L.type == 1;
      const int units = mk_units(m, C, kind, full);
      const int first = (cta - rot % G + G) % G;
      // ---- prologue
      if (kind == MK_CONV || kind == MK_QKVG || kind == MK_W13) {
        MkNorm p{};
        if (sub == 0 && l == 0) {
          p.x_in = nullptr;
          p.emb = S.tokens ? m.embed : S.embeds;
          p.tokens = S.tokens;
          p.dump = S.hidden;
        } else {
          p.x_in = cur;
          p.parts = pend;
          p.n_parts = pend_n;
          p.g_post = pend_g;
          p.dump = (sub == 0 && S.hidden) ? S.hidden + (size_t)l * nb * D : nullptr;
        }
        p.g_next = kind == MK_W13 ? L.ffn_norm : L.op_norm;
        p.x_out = nxt;
        p.stamp = (trace && phase < MK_TRACE_PHASES) ? trace + MK_TRACE_WORDS * phase + 6 : nullptr;
        mk_norm(p, nb, m.eps, writer, xs, red, ct);
        { float* t_ = cur; cur = nxt; nxt = t_; }
      } else if (kind == MK_OUT) {
        mk_load_x(m.y, D, nb, xs, ct);
      } else if (kind == MK_W2) {
        mk_load_x(m.u, F, nb, xs, ct);
      }
      if (trace && ct == 0 && phase < MK_TRACE_PHASES) trace[MK_TRACE_WORDS * phase + 4] = mk_now();
      // ---- warm L2 with the small constant vectors the coming phases read
      if (kind == MK_CONV || kind == MK_QKVG) {
        mk_prefetch_l2(L.post_op_norm, D * 2, ct);
        mk_prefetch_l2(L.ffn_norm, D * 2, ct - 32);
        if (kind == MK_QKVG) {
          const int k = L.type == 1 ? 0 : 1;
          mk_prefetch_l2(L.q_norm, HD * 2, ct - 64);
          mk_prefetch_l2(L.k_norm, HD * 2, ct - 66);
          for (int b = 0; b < nb; ++b) {
            mk_prefetch_l2(m.rope_cos[k] + (size_t)C.pos[b] * (HD / 2), HD * 2, ct - 68 - 4 * b);
            mk_prefetch_l2(m.rope_sin[k] + (size_t)C.pos[b] * (HD / 2), HD * 2, ct - 84 - 4 * b);
          }
        }
      } else if (kind == MK_W13) {
        mk_prefetch_l2(L.post_ffn_norm, D * 2, ct);
        mk_prefetch_l2(l + 1 < m.n_layers ? m.layers[l + 1].op_norm : m.final_norm, D * 2, ct - 32);
      }
      // ---- units
      if (kind == MK_ATTN) {
        for (int u = first; u < units && ok; u += G) {
          const MkAttnUnit U = mk_attn_unit(C, full, u);
          ok = mk_attn_unit(m, S, C, L, U, R, scr, &abort_flag, ct);
        }
      } else {
        // the block's units, dealt to the consumer warps in rounds (the producer's order)
        const int nst = mk_gemv_stages(m, kind);
        const int ks_n = mk_ksplit(m, kind);
        const int n = units > first ? (units - first + G - 1) / G : 0;
        uint32_t base = R.it;
        if (kind == MK_CONV) {
          // all warps on each unit: warp w takes stages w, w + MK_CW, ...; sums meet in shared memory
          for (int r0 = 0; r0 < n; ++r0) {
            wok = mk_conv_unit(m, S, C, L, first + r0 * G, nst, R, base, xs, xzero, nb, red, lane, warp, ct,
                               &abort_flag) && wok;  // every warp takes part (block-level syncs inside)
            base += (uint32_t)nst;
          }
          R.it = base;
          wok = wok && !*reinterpret_cast<volatile int*>(&abort_flag);
        }
        for (int r0 = 0; kind != MK_CONV && r0 < n; r0 += MK_CW) {
          const int nr = min(MK_CW, n - r0);
          if (warp < nr && wok) {
            const int u = first + (r0 + warp) * G;
            const int tile = u / ks_n, ks = u % ks_n;
            wok = mk_gemv_unit<FP4>(m, S, C, L, kind, tile, ks, nst, R, base + warp, nr, xs, xzero, nb, lut, &abort_flag,
                               lane);
          }
          base += (uint32_t)(nst * nr);
        }
        if (kind != MK_CONV) R.it = base;
      }
      rot = (rot + units) % G;
      if (ok) ok = barrier();
      // what the next sandwich step adds into the residual
      if (kind == MK_OUT) {
        pend = m.part;
        pend_n = MK_KS_QO;
        pend_g = L.post_op_norm;
      } else if (kind == MK_W2) {
        pend = m.part2;
        pend_n = m.fp4 ? MK_KS_W2F : MK_KS_W2;
        pend_g = L.post_ffn_norm;
      }
    }
  }
  if (ok && do_head) {
    MkNorm p{};
    p.x_in = cur;
    p.parts = pend;
    p.n_parts = pend_n;
    p.g_post = pend_g;
    p.g_next = m.final_norm;
    p.x_out = nxt;
    p.dump = S.hidden ? S.hidden + (size_t)m.n_layers * nb * D : nullptr;
    mk_norm(p, nb, m.eps, writer, xs, red, ct);
    { float* t_ = cur; cur = nxt; nxt = t_; }
    const int units = m.vocab / 16;
    const int first = (cta - rot % G + G) % G;
    const int nst = mk_gemv_stages(m, MK_HEAD);
    const int n = units > first ? (units - first + G - 1) / G : 0;
    uint32_t base = R.it;
    for (int r0 = 0; r0 < n; r0 += MK_CW) {
      const int nr = min(MK_CW, n - r0);
      if (warp < nr && wok)
        wok = mk_gemv_unit<FP4>(m, S, C, m.layers[0], MK_HEAD, first + (r0 + warp) * G, 0, nst, R, base + warp, nr, xs,
                           xzero, nb, lut, &abort_flag, lane);
      base += (uint32_t)(nst * nr);
    }
    R.it = base;
    if (ok) ok = barrier();
  } else if (ok && S.hidden) {
    // no head: the final residual (after the last FFN's sandwich step) is the last hidden dump
    MkNorm p{};
    p.x_in = cur;
    p.parts = pend;
    p.n_parts = pend_n;
    p.g_post = pend_g;
    p.dump = S.hidden + (size_t)m.n_layers * nb * D;
    mk_norm(p, nb, m.eps, writer, xs, red, ct);
  }
  if (!ok) return;
  // ---- bookkeeping of the step (block 0, after every block passed the last barrier)
  if (ct == 0) {
    // the last block through resets the barrier counter for the next launch
    __threadfence();
    const unsigned done = atomicAdd(m.sync + 1, 1u);
    if (done == (unsigned)G - 1) {
      atomicExch(m.sync, 0u);
      atomicExch(m.sync + 1, 0u);
    }
  }
  if (cta == 0 && ct < nb) {
    if (do_head && S.argmax_out) {
      const unsigned long long k = __ldcg(m.amax + ct);
      S.argmax_out[ct] = (int32_t)(0xffffffffu - (uint32_t)(k & 0xffffffffull));
    }
    S.seq_len[C.slot[ct]] += 1;
  }
}

// ------------------------------------------------------------------------------ host side
static int g_mk_sms = 0;

size_t mk_smem_bytes(int nb, int fp4, int nslot) {
  return 1024 + (size_t)nslot * MK_SLOT + 128 + (size_t)nb * MK_XS * 2 + (fp4 ? MK_LUT_BYTES : 0) +
         MK_SCR_FLOATS * 4 + 2 * (size_t)nslot * 8;
}

int mk_slots(int nb, int fp4) {
  int n = 8;
  while (n > 2 && mk_smem_bytes(nb, fp4, n) > (size_t)MK_SMEM_MAX) --n;
  return n;
}

cudaError_t mk_init() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&g_mk_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_decode_mk<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, MK_SMEM_MAX);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(k_decode_mk<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, MK_SMEM_MAX);
}

int mk_grid() { return g_mk_sms; }

cudaError_t decode_mk(const CUtensorMap* kv_maps, const MkModel& m, const MkStep& s, cudaStream_t st) {
  if (s.nb < 1 || s.nb > MK_MAX_NB) return cudaErrorInvalidValue;
  MkModel mm = m;
  if (g_mk_sms > MK_TRACE_BLOCKS) mm.trace = nullptr;
  mm.nslot = mk_slots(s.nb, m.fp4);
  if (mm.nslot < 3) return cudaErrorInvalidValue;
  const size_t smem = mk_smem_bytes(s.nb, m.fp4, mm.nslot);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(g_mk_sms);
  cfg.blockDim = dim3(MK_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  ++g_launches;
  if (m.fp4) return cudaLaunchKernelEx(&cfg, k_decode_mk<true>, kv_maps[0], kv_maps[1], kv_maps[2], kv_maps[3], mm, s);
  return cudaLaunchKernelEx(&cfg, k_decode_mk<false>, kv_maps[0], kv_maps[1], kv_maps[2], kv_maps[3], mm, s);
}

}  // namespace lfm3
