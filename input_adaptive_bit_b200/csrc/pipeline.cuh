// pipeline.cuh -- device helpers of the decode kernels (decode.cu, batch.cu):
// cp.async and 1-D bulk copies, mbarrier waits with a bound, the m16n8k16 MMA.
#pragma once

#include "grinqh_internal.cuh"

namespace grinqh {
namespace pipe {

constexpr int kWaitTries = 1 << 16;     // bounded mbarrier waits: tries ...
constexpr uint32_t kSuspendNs = 20000;  // ... of at most 20 us each (about 1.3 s in all)

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes));
}
// 16-byte copy global -> shared through L2 only, with an L2 cache policy.
__device__ __forceinline__ void cp_async16_hint(void *dst, const void *src, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)),
               "l"(src), "l"(policy));
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(dst)), "l"(src));
}
// The mbarrier counts one arrival of this thread once all of its earlier cp.async
// copies have landed (its expected count includes that arrival).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;\n" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// Waits for the phase of `parity` to complete, each try suspending the thread
// for at most kSuspendNs (it resumes as soon as the phase completes); gives up
// after kWaitTries tries, records error 5 and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *error) {
  const uint32_t a = smem_u32(bar);
  for (int i = 0; i < kWaitTries; ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(a), "r"(parity), "r"(kSuspendNs)
        : "memory");
    if (done) return true;
  }
  atomicCAS(error, 0, kDevErrPipeTimeout);
  return false;
}

// 1-D bulk copy global -> shared on the TMA engine, completing `bytes` on `bar`.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;\n" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// D += A B, m16n8k16, fp16 operands, fp32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Relaxed (non-cached, coherent at GPU scope) loads and stores of words that
// another CTA of the grid reads or writes while this one runs.
__device__ __forceinline__ uint4 ld_relaxed_v4(const uint32_t *p) {
  uint4 v;
  asm volatile("ld.relaxed.gpu.global.v4.u32 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_v4(uint32_t *p, uint4 v) {
  asm volatile("st.relaxed.gpu.global.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_relaxed_u32(uint32_t *p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}
// A partial sum as a word that is never zero, so that zero can mean "not written
// yet": +0.0 is stored as -0.0 (the same number); every other float already has a
// non-zero bit pattern.
__device__ __forceinline__ uint32_t tag_word(float v) {
  const uint32_t u = __float_as_uint(v);
  return u != 0u ? u : 0x80000000u;
}
__device__ __forceinline__ unsigned long long ld_acquire64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];\n" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Barrier of the first n threads of the CTA only (named barrier 1).
template <int N>
__device__ __forceinline__ void sync_first() { asm volatile("bar.sync 1, %0;\n" ::"n"(N)); }

__device__ __forceinline__ float4 f4add(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

// 2^e as a float, for |e| well inside the normal range.
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

// Bit position of output t's 2-bit field inside its fp16 half after the
// extraction below: t' = t mod 8; t' <= 4 stays at 2t', t' >= 5 is shifted
// down by 6 (so it stays inside the 10 mantissa bits).
__host__ __device__ constexpr int field_pos(int t) {
  return (t & 7) <= 4 ? 2 * (t & 7) : 2 * (t & 7) - 6;
}

}  // namespace pipe
}  // namespace grinqh
