// Shared device helpers for the MoE layer kernels (sm_100a).
//
// Inline-PTX wrappers for mbarriers, 1-D bulk copies (cp.async.bulk), the
// legacy warp-level tensor-core MMA used by the decode path, fp4 -> fp16
// conversion, and the bounded waits every kernel uses instead of unbounded
// spins.  A wait that runs out records MOE_ERR_TIMEOUT in the library's device
// status word and returns false; it never traps.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Sticky device status word (first error wins).  Defined in moe_api.cu.
extern __device__ int g_status;

__device__ __forceinline__ void set_status(int code) { atomicCAS(&g_status, 0, code); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Limit for any single device-side wait.  Every legitimate wait in these
// kernels ends within microseconds; two seconds only guards against a bug.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.
__device__ __forceinline__ bool mbar_wait_limit(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) {
      set_status(MOE_ERR_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  return mbar_wait_limit(bar, parity, kWaitLimitNs);
}

// -------------------------------------------------------------- bulk copy
// L2 policy for streamed-once weights.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 1-D bulk copy global -> this CTA's shared memory, completing `bytes` on `bar`.
// dst/src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
      "%4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// ------------------------------------------------------------ smem loads
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds8(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

// ------------------------------------------------------------------- MMA
// D = A(16x16, row) * B(16x8, col) + C, fp32 accumulate.
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------ format conversion
// Four packed E2M1 pairs (one 32-bit word = 8 codes) -> four f16x2 words.
// Output i holds the codes of byte i: low nibble in the low half.
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t w, uint32_t& o0, uint32_t& o1, uint32_t& o2,
                                                uint32_t& o3) {
  asm("{\n .reg .b8 q0, q1, q2, q3;\n mov.b32 {q0, q1, q2, q3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, q0;\n cvt.rn.f16x2.e2m1x2 %1, q1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, q2;\n cvt.rn.f16x2.e2m1x2 %3, q3;\n}\n"
      : "=r"(o0), "=r"(o1), "=r"(o2), "=r"(o3)
      : "r"(w));
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// Two E8M0 scales (low byte, high byte of a 16-bit value) -> two fp32 values
// 2^(v-127), exact (v = 0 gives 2^-127, v = 255 NaN), via the hardware
// conversion to bf16x2 (same exponent range as fp32) and a shift.
__device__ __forceinline__ void e8m0x2_to_f32x2(uint32_t pair16, float& lo, float& hi) {
  uint32_t b2;
  asm("{\n .reg .b16 t;\n cvt.u16.u32 t, %1;\n cvt.rn.bf16x2.ue8m0x2 %0, t;\n}\n" : "=r"(b2) : "r"(pair16));
  lo = __uint_as_float(b2 << 16);
  hi = __uint_as_float(b2 & 0xffff0000u);
}

// (d0, d1) += (a0, a1) * s with one packed fp32x2 FMA (each lane rounds once,
// exactly like two fmaf).
__device__ __forceinline__ void ffma2_scalar(float& d0, float& d1, float a0, float a1, float s) {
  asm("{\n .reg .b64 rd, ra, rs;\n mov.b64 ra, {%2, %3};\n mov.b64 rs, {%4, %4};\n mov.b64 rd, {%0, %1};\n"
      " fma.rn.f32x2 rd, ra, rs, rd;\n mov.b64 {%0, %1}, rd;\n}\n"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1), "f"(s));
}

// D = A * B (accumulator starts at zero).
__device__ __forceinline__ void mma_f16_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  const float z = 0.f;
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(z));
}

// E8M0 byte -> fp32 2^(v-127) (v = 255 -> NaN).
__device__ __forceinline__ float e8m0_to_f32(uint32_t v) {
  if (v == 0u) return __int_as_float(0x00400000);  // 2^-127 (subnormal)
  if (v == 255u) return __int_as_float(0x7fc00000);
  return __int_as_float(static_cast<int>(v << 23));
}

// Two E4M3 (FN) bytes (low byte, high byte of a 16-bit value) -> f16x2 with
// the low byte's value in the low half (exact: every E4M3 value is an fp16
// value), by the hardware conversion.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t pair16) {
  uint32_t r;
  asm("{\n .reg .b16 t;\n cvt.u16.u32 t, %1;\n cvt.rn.f16x2.e4m3x2 %0, t;\n}\n" : "=r"(r) : "r"(pair16));
  return r;
}

// 8 INT4 codes (two's complement q in [-8, 7], one 32-bit word) -> four f16x2
// words holding offset integers, one AND-XOR each: the even nibbles become
// 1024 + (q + 8) and the odd nibbles 1024 + 16 (q + 8) (exact in fp16, whose
// spacing at 1024 is 1).  Pairing: o0 = (n0, n4), o1 = (n1, n5), o2 = (n2, n6),
// o3 = (n3, n7), nI being nibble I counting from bit 0.  The caller divides
// the activations that meet odd nibbles by 16 and removes the constant part,
// 1032 x (even) and 1152 x' (odd, x' = x / 16), per scale group.
__device__ __forceinline__ void int4x8_to_f16x8_offset(uint32_t w, uint32_t& o0, uint32_t& o1, uint32_t& o2,
                                                       uint32_t& o3) {
  const uint32_t w8 = w >> 8;
  o0 = (w & 0x000f000fu) ^ 0x64086408u;
  o1 = (w & 0x00f000f0u) ^ 0x64806480u;
  o2 = (w8 & 0x000f000fu) ^ 0x64086408u;
  o3 = (w8 & 0x00f000f0u) ^ 0x64806480u;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __int_as_float(static_cast<int>(b << 16)); }

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace moe

namespace moe {
// Programmatic dependent launch: every kernel of the library waits for the
// previous kernel in its stream (griddepcontrol.wait) before its first global
// memory access, then lets the next kernel start launching.  Launched without
// the PDL attribute, both instructions are no-ops.
__device__ __forceinline__ void pdl_wait_and_trigger() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
}  // namespace moe
