// Shared device helpers for the Gated DeltaNet kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

// Device error word, one per device per translation unit that includes this
// header. Bit 0: a bounded wait ran out; bit 1: an index check of the
// GDN_DEBUG build failed (g_error_line then holds the first failing check's
// source line). Read and cleared by the host.
__device__ unsigned int g_error_word;
__device__ unsigned int g_error_line;

enum : unsigned int { kErrTimeout = 1u, kErrCheck = 2u };

__device__ __forceinline__ void flag_error(unsigned int bits) {
  atomicOr(&g_error_word, bits);
}

// Index checks of the GDN_DEBUG build: GDN_CHECK(cond) is `true` in the normal
// build (no code) and, with GDN_DEBUG defined, evaluates cond and on failure
// records kErrCheck and the line in the error word and returns false, so that
// the caller skips the access and stops its loop -- it never traps.
__device__ __forceinline__ bool debug_check(bool ok, unsigned int line) {
  if (!ok) {
    atomicCAS(&g_error_line, 0u, line);
    flag_error(kErrCheck);
  }
  return ok;
}
#ifdef GDN_DEBUG
#define GDN_CHECK(cond) (::gdn::debug_check((cond), __LINE__))
#else
#define GDN_CHECK(cond) true
#endif

// L2-normalisation epsilon (added inside the square root), as in the oracle.
constexpr float kNormEps = 1e-6f;

// ---- loads of 4 consecutive elements as fp32 --------------------------------
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  uint2 raw = *reinterpret_cast<const uint2*>(p);
  __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162*>(&raw.x);
  __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162*>(&raw.y);
  float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float4 load4(const __half* p) {
  uint2 raw = *reinterpret_cast<const uint2*>(p);
  __half2 lo = *reinterpret_cast<__half2*>(&raw.x);
  __half2 hi = *reinterpret_cast<__half2*>(&raw.y);
  float2 a = __half22float2(lo), b = __half22float2(hi);
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float4 load4(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}

__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }
__device__ __forceinline__ float to_f32(float x) { return x; }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
template <> __device__ __forceinline__ __half from_f32<__half>(float x) {
  return __float2half_rn(x);
}

// Streaming (evict-first) 16-byte global accesses for data touched once.
__device__ __forceinline__ float4 ld_stream(const float4* p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(float4* p, float4 v) { __stcs(p, v); }

template <int kWidth>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int off = kWidth / 2; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

}  // namespace gdn
