// tq_common.cuh -- device helpers shared by the libtq kernels (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ != 1000)
#error "libtq is written for sm_100a (B200) only"
#endif

namespace tq {

// ---- SplitMix64 (Steele, Lea & Flood 2014; Vigna's public reference) ------
// The k-th output (k = 0, 1, ...) of a generator whose state starts at s is
// mix64(s + (k+1) * gamma).  The RHT diagonal d[k] is -1 when its top bit is set.
__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

__device__ __forceinline__ bool rht_sign_negative(uint64_t seed, uint32_t k) {
  return (mix64(seed + (uint64_t)(k + 1) * 0x9E3779B97F4A7C15ULL) >> 63) != 0;
}

// ---- warp-level MMA (m16n8k16, fp16 inputs, fp32 accumulate) --------------
// Fragment ownership, with g = lane / 4 and q = lane % 4:
//   a[0]: A(g,   2q..2q+1)   a[1]: A(g+8, 2q..2q+1)
//   a[2]: A(g,   2q+8..+9)   a[3]: A(g+8, 2q+8..+9)
//   b[0]: B(2q..2q+1, g)     b[1]: B(2q+8..+9, g)
//   c[0..1]: C(g, 2q..2q+1)  c[2..3]: C(g+8, 2q..2q+1)
__device__ __forceinline__ void mma_16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ uint32_t f2_to_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float2 h2_to_f2(uint32_t v) {
  return __half22float2(*reinterpret_cast<const __half2*>(&v));
}

__device__ __forceinline__ uint16_t f_to_bf16_bits(float v) {
  __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t*>(&b);
}

__device__ __forceinline__ float bf16_bits_to_f(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// ---- loads ------------------------------------------------------------------
// Streaming 16-byte load of read-once data (the code bytes): no L1 allocation.
__device__ __forceinline__ uint4 ldg_stream_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint16_t ldg_u16(const uint16_t* p) { return __ldg(p); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- programmatic dependent launch -------------------------------------------
// Wait until the preceding kernel in the stream has completed and its writes
// are visible; a no-op when the launch carries no programmatic dependency.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
// Allow the next kernel in the stream to be scheduled (it still waits in pdl_wait).
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

}  // namespace tq
