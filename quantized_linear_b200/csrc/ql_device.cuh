// Device helpers shared by the libqlinear kernels (not part of the ABI): bf16 and fp16
// conversions, programmatic-dependent-launch hooks, and packed fp32 pairs.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace qld {

__device__ __forceinline__ float bf16_to_f32(uint32_t h16) { return __uint_as_float(h16 << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
  uint16_t h;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(f));
  return h;
}

__device__ __forceinline__ float f16_to_f32(uint16_t h) {
  float f;
  asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"(h));
  return f;
}

// Programmatic dependent launch: wait until the preceding grid in the stream has completed and
// its writes are visible (a no-op when the kernel was launched without overlap), and allow the
// next grid to be scheduled (it still waits for this one to complete before touching its data).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// acc + a * b with bf16 a, b and fp32 accumulate; the product is exact in fp32.
__device__ __forceinline__ float fma_bf16(uint16_t a, uint16_t b, float acc) {
  asm("fma.rn.f32.bf16 %0, %1, %2, %0;" : "+f"(acc) : "h"(a), "h"(b));
  return acc;
}

// silu(g) * u = g / (1 + e^-g) * u in fp32: the library expf and IEEE division (for g < -88 the
// exponential overflows to +inf and the gate is -0, its limit).
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdiv_rn(g, 1.0f + expf(-g)) * u; }

// Packed fp32 pairs, the operands of fma.rn.f32x2 (two fp32 FMAs in one instruction, each
// rounded as a scalar fma.rn.f32 would be).
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ uint64_t f2u(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ void f2split(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

}  // namespace qld
