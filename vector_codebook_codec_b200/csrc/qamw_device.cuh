// qamw_device.cuh -- device helpers shared by the libqamw kernels (sm_100a only).
//
// Nothing here is shared with the CPU oracle; the sign-mask generator below is
// an independent implementation of SplitMix64 from its published definition
// (Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
// OOPSLA 2014).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "qamw.h"

namespace qamw {

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libqamw targets sm_100a (B200) only"
#endif

// ----------------------------------------------------------------------------
// SplitMix64 sign mask: d_j = -1 iff bit 63 of output number j+1 is set.
// ----------------------------------------------------------------------------
__host__ __device__ __forceinline__ uint64_t splitmix64_output(uint64_t seed, uint64_t n) {
  uint64_t z = seed + n * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ bool mask_is_negative(uint64_t seed, int64_t col) {
  return (splitmix64_output(seed, (uint64_t)col + 1ull) >> 63) != 0ull;
}

// ----------------------------------------------------------------------------
// Packed fp32x2 arithmetic (sm_100 FADD2 / FMUL2 / FFMA2 through the CUDA
// intrinsics), round-to-nearest-even. Each lane of the pair is an independent
// IEEE fp32 operation, identical to __fadd_rn / __fsub_rn / __fmul_rn / __fmaf_rn.
// ----------------------------------------------------------------------------
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  return __fadd2_rn(a, make_float2(-b.x, -b.y));
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Squared distance in the direct-difference form, (x0-c0)^2 + (x1-c1)^2 with
// the second square fused: fma(dy, dy, dx*dx). The scalar and the packed
// versions round identically.
__device__ __forceinline__ float dist2_scalar(float x0, float x1, float c0, float c1) {
  const float dx = __fsub_rn(x0, c0);
  const float dy = __fsub_rn(x1, c1);
  return __fmaf_rn(dy, dy, __fmul_rn(dx, dx));
}

// ----------------------------------------------------------------------------
// Element loads.
// ----------------------------------------------------------------------------
__device__ __forceinline__ double bf16_bits_to_double(uint32_t bits16) {
  return (double)__uint_as_float(bits16 << 16);
}

// ----------------------------------------------------------------------------
// cp.async (global -> shared, asynchronous, per thread) for prefetching.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void cp_async8(void *smem, const void *gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void *smem, const void *gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void status_or(int32_t *status, uint32_t bits) {
  if (status != nullptr && bits != 0u) atomicOr(reinterpret_cast<unsigned int *>(status), bits);
}

}  // namespace qamw
