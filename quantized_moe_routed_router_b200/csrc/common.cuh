// Device helpers for the sm_100a kernels: mbarriers, 1-D bulk (TMA) copies,
// tensor-core MMA, packed format conversions, programmatic dependent launch.
// Hand-written inline PTX; no library kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define TSM_DEV __device__ __forceinline__

namespace tsm {

// ----------------------------------------------------------------------------- error word bits
enum : unsigned {
  ERR_TIMEOUT_WFULL = 1u << 0,   // consumer gave up waiting for a weight stage
  ERR_TIMEOUT_WEMPTY = 1u << 1,  // producer gave up waiting for a free weight stage
  ERR_TIMEOUT_XFULL = 1u << 2,   // consumer gave up waiting for an activation window
  ERR_TIMEOUT_XEMPTY = 1u << 3,  // producer gave up waiting for a free activation window
  ERR_BAD_INDEX = 1u << 4,       // an expert / token index read from the route list was out of range
  ERR_BAD_META = 1u << 5,        // route metadata inconsistent with the launch
  ERR_TIMEOUT_GRID = 1u << 6,    // a CTA gave up waiting at the grid-wide barrier
  ERR_TIMEOUT_ACTS = 1u << 7,    // a down producer gave up waiting for an expert's acts
  ERR_TIMEOUT_XSTAGE = 1u << 8,  // the routing gave up waiting for the bulk copy of x
  ERR_TIMEOUT_XH = 1u << 9,      // a producer gave up waiting for the shared FP16 x
  ERR_TIMEOUT_ROUTE = 1u << 10,  // a CTA gave up waiting for the published router logits
  ERR_BAD_ROUTER_INPUT = 1u << 11,  // a router bias or per-expert scale read by the route kernel was not finite
  ERR_TIMEOUT_TABLES = 1u << 12,    // a decode launch gave up waiting for its precomputed range tables
};

// A bounded wait gives up after this many nanoseconds of %globaltimer.
constexpr unsigned long long WAIT_LIMIT_NS = 2000000000ull;  // 2 s

TSM_DEV unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

TSM_DEV uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// ----------------------------------------------------------------------------- mbarrier
TSM_DEV void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

TSM_DEV void fence_barrier_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

TSM_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar))
               : "memory");
}

TSM_DEV void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

TSM_DEV bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits until the phase with `parity` of `bar` has completed.  Gives up after
// WAIT_LIMIT_NS (or at once when *dead is set by another thread of the CTA),
// records `errbit` in the device error word and marks the CTA dead, so every
// later wait of the CTA returns at once and the kernel runs to its end.
TSM_DEV bool mbar_wait(uint64_t* bar, unsigned parity, volatile int* dead, unsigned* err, unsigned errbit) {
  if (mbar_try_wait(bar, parity)) return true;
  unsigned long long t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*dead) return false;
    if (globaltimer() - t0 > WAIT_LIMIT_NS) {
      *dead = 1;
      atomicOr(err, errbit);
      return false;
    }
  }
}

// ----------------------------------------------------------------------------- bulk copies (TMA, 1-D, no multicast)
TSM_DEV uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// global -> shared copy of `bytes` (multiple of 16, both addresses 16-byte
// aligned) completing on `bar` as transaction bytes.
TSM_DEV void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

TSM_DEV void bulk_g2s_hint(void* dst, const void* src, unsigned bytes, uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(pol)
      : "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) writes to the same bytes.
TSM_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Orders generic-proxy global memory accesses (made visible to this thread)
// before later async-proxy (bulk copy) reads of the same global memory.
TSM_DEV void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// ----------------------------------------------------------------------------- PDL
TSM_DEV void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
TSM_DEV void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ----------------------------------------------------------------------------- named barrier among the consumer warps
TSM_DEV void bar_sync(int id, int nthreads) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory"); }

// ----------------------------------------------------------------------------- loads that bypass L1 (data written by other CTAs)
TSM_DEV float ld_cg(const float* p) {
  float v;
  asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}
TSM_DEV float2 ld_cg2(const float* p) {
  float2 v;
  asm volatile("ld.global.cg.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(p));
  return v;
}
TSM_DEV unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
// Adds v at gpu scope with release semantics (this thread's earlier writes, and
// those ordered before them by a CTA barrier, are visible before the add); no
// value comes back, so the thread does not wait for the round trip.
TSM_DEV void red_release_add_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
TSM_DEV void red_release_add_u32(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Atomic add at gpu scope with acquire-release semantics: earlier writes are
// published with it, and writes published by the adds it reads are visible after.
TSM_DEV unsigned atom_acq_rel_add_u32(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
TSM_DEV unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// ----------------------------------------------------------------------------- tensor core MMA (m16n8k16, f16 x f16 -> f32)
// A fragment (4 regs of f16x2): {row g, k 2c..2c+1}, {row g+8, k 2c..}, {row g, k 2c+8..}, {row g+8, k 2c+8..}
// B fragment (2 regs): {k 2c..2c+1, col g}, {k 2c+8.., col g};  C/D: {row g, col 2c..2c+1}, {row g+8, col 2c..}
// with g = lane / 4, c = lane % 4.
// D = A * B (accumulator input zero).
TSM_DEV void mma_f16_zc(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

// D += A * B.
TSM_DEV void mma_f16_acc(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ----------------------------------------------------------------------------- packed conversions
// Four bytes, each holding two E2M1 codes (low nibble = first element), to
// four f16x2 registers (first element in the low half), exactly.
TSM_DEV void e2m1x8_to_f16x8(uint32_t w, uint32_t (&out)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
      : "r"(w));
}

// Two bytes holding biased int8 values u = q + 128 (bytes sel0, sel1 of w) to
// an f16x2 of q, exactly: the bytes become the low mantissa bits of 1024 + u
// (f16 exponent 10 gives unit spacing), then 1152 = 1024 + 128 is subtracted.
template <int SEL>
TSM_DEV uint32_t u8x2_to_f16x2(uint32_t w) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(w), "r"(0x64646464u), "r"(SEL));
  __half2 h = *reinterpret_cast<__half2*>(&r);
  const __half2 off = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
  h = __hsub2(h, off);
  return *reinterpret_cast<uint32_t*>(&h);
}

// INT4-affine codes: a word of eight nibbles (layout in repack.cuh) to the
// four f16x2 A registers by masks alone.  Nibbles 0/4 masked into the
// mantissas of 0x6400 (1024) give 1024 + q, nibbles 1/5 give 1024 + 16 q, and
// the word shifted right by 8 gives nibbles 2/6 and 3/7 the same way.  The
// registers of tile row g (0 and 2) hold 1024 + q, those of row g + 8 (1 and
// 3) hold 1024 + 16 q, both exact; the consumer removes the 1024 and the 16
// per row with the block's column sums (see mma_chunk).
TSM_DEV void i4x8_to_f16x8_biased(uint32_t w, uint32_t (&out)[4]) {
  const uint32_t w8 = w >> 8;
  out[0] = (w & 0x000F000Fu) | 0x64006400u;
  out[1] = (w & 0x00F000F0u) | 0x64006400u;
  out[2] = (w8 & 0x000F000Fu) | 0x64006400u;
  out[3] = (w8 & 0x00F000F0u) | 0x64006400u;
}

// E8M0 byte `k` of w as an FP32 power of two (2^(e-127)); e = 0 maps to 0.0
// (2^-127 is below FP32's normal range; such blocks contribute < 1e-37 per weight).
template <int K>
TSM_DEV float e8m0_byte_to_f32(uint32_t w) {
  uint32_t bits = (K == 3) ? (w >> 1) : (w << (23 - 8 * K));
  return __uint_as_float(bits & 0x7F800000u);
}

}  // namespace tsm
