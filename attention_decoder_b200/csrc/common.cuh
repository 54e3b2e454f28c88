// Device helpers shared by the LFM3 kernels (sm_100a only).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#define DEVI __device__ __forceinline__

typedef __nv_bfloat16 bf16;

// ---------------------------------------------------------------- numeric conversions
DEVI float bf2f(bf16 x) { return __bfloat162float(x); }
DEVI bf16 f2bf(float x) { return __float2bfloat16_rn(x); }
DEVI float bflo(uint32_t w) { return __uint_as_float(w << 16); }
DEVI float bfhi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
DEVI uint32_t pack_bf2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
DEVI float round_bf(float x) { return bf2f(f2bf(x)); }

// ---------------------------------------------------------------- reductions
DEVI float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
DEVI float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
// Sum over a block of NW warps; `red` holds NW floats. Every thread gets the total.
template <int NW>
DEVI float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < NW; ++i) t += red[i];
  return t;
}

// ---------------------------------------------------------------- memory
// Streaming 16-byte load that skips L1 (weights are read once per step).
DEVI uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
DEVI uint4 ldg16(const void* p) { return *reinterpret_cast<const uint4*>(p); }
DEVI void stg16(void* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }

// ---------------------------------------------------------------- programmatic dependent launch
// Kernels are launched with programmatic stream serialisation: each one may start while its
// predecessor drains. pdl_wait() blocks until the predecessor grid has completed and its writes
// are visible; every block calls it before touching data a previous kernel produced (and before
// exiting), so completion stays transitive along the stream.
DEVI void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
DEVI void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// ---------------------------------------------------------------- tensor-core fragment (legacy warp MMA)
// D[16x8] += A[16x16] (row) * B[16x8] (col), bf16 inputs, fp32 accumulate.
DEVI void mma_bf16_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same with f16 operands.
DEVI void mma_f16_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16x2 -> f16x2 of the same two values (exact within f16's range).
DEVI uint32_t bf2_to_h2(uint32_t w) {
  __half2 h = __floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  return *reinterpret_cast<uint32_t*>(&h);
}
// Four bytes of E2M1 code pairs (element 2j in the low nibble of byte j) -> four f16x2, exact.
DEVI void e2m1x8_to_h2(uint32_t w, uint32_t& c01, uint32_t& c23, uint32_t& c45, uint32_t& c67) {
  asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n cvt.rn.f16x2.e2m1x2 %0, b0;\n"
      " cvt.rn.f16x2.e2m1x2 %1, b1;\n cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(c01), "=r"(c23), "=r"(c45), "=r"(c67)
      : "r"(w));
}
// An E4M3 byte -> f16x2 holding its value twice, exact.
DEVI uint32_t e4m3_to_h2(uint32_t b) {
  uint32_t r;
  const uint32_t two = (b & 0xFFu) * 0x0101u;
  asm("{\n .reg .b16 h;\n cvt.u16.u32 h, %1;\n cvt.rn.f16x2.e4m3x2 %0, h;\n}" : "=r"(r) : "r"(two));
  return r;
}
DEVI uint32_t hmul2_u(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

DEVI float sigmoidf_(float x) { return 1.f / (1.f + __expf(-x)); }
DEVI float siluf_(float x) { return x / (1.f + __expf(-x)); }

// ---------------------------------------------------------------- mbarriers and bulk copies
constexpr uint32_t WAIT_LIMIT = 1u << 22;  // try_wait rounds before a wait gives up

DEVI uint32_t su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
DEVI void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
DEVI void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
DEVI void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
DEVI bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait: returns false (and sets *err) if the phase did not complete in time.
DEVI bool mbar_wait(uint32_t bar, uint32_t parity, int* err) {
  for (uint32_t i = 0; i < WAIT_LIMIT; ++i)
    if (mbar_try(bar, parity)) return true;
  atomicExch(err, 1);
  return false;
}
// One contiguous global -> shared copy (16-byte aligned, size a multiple of 16) that completes
// `bytes` of the barrier's transaction count.
DEVI void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// ---------------------------------------------------------------- optional launch timeline
// Built only with -DLFM3_TRACE (a diagnostic build): blocks stamp the global timer (ns) into a
// caller-provided buffer [launch][block][8]; the product build has none of this.
#ifdef LFM3_TRACE
constexpr int TRACE_BLOCKS = 512;
DEVI void trace_at(unsigned long long* buf, int id, int slot) {
  if (!buf || id < 0 || id >= 256) return;
  const unsigned blk = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
  if (blk >= TRACE_BLOCKS) return;
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  if (slot == 7) {
    unsigned sm;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
    t = sm;
  }
  buf[((size_t)id * TRACE_BLOCKS + blk) * 8 + slot] = t;
}
#define TRACE(buf, id, slot) trace_at(buf, id, slot)
#else
#define TRACE(buf, id, slot) ((void)0)
#endif

