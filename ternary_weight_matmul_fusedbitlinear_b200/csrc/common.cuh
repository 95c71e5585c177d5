// Shared device helpers of the mmf CUDA library (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mmf.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library is written for sm_100a (B200) only"
#endif

namespace mmf {

using bf16 = __nv_bfloat16;

// ---------------------------------------------------------------- activations in either dtype

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

// round an fp32 value to what the storage type keeps (identity for fp32)
template <typename T> __device__ __forceinline__ float round_to(float v) { return to_f32(from_f32<T>(v)); }

// load 8 consecutive activations (16-byte aligned for bf16, 32-byte for fp32)
__device__ __forceinline__ void load8(const bf16* p, float out[8]) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float out[8]) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}
__device__ __forceinline__ void store8(bf16* p, const float v[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store8(float* p, const float v[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

// Four int32 codes -> four saturated int8 bytes in memory order c0..c3.
__device__ __forceinline__ uint32_t pack4_sat(int c0, int c1, int c2, int c3) {
  uint32_t hi, w;
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, 0;" : "=r"(hi) : "r"(c3), "r"(c2));
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(w) : "r"(c1), "r"(c0), "r"(hi));
  return w;
}

// ---------------------------------------------------------------- gates
// sigmoid(z) = 1 / (1 + e^-z); e^-z overflows to +inf for very negative z and
// the reciprocal then gives exactly 0, which is the limit.
__device__ __forceinline__ float sigmoidf_(float z) { return __frcp_rn(1.0f + __expf(-z)); }
__device__ __forceinline__ float siluf_(float z) { return z * sigmoidf_(z); }

// ---------------------------------------------------------------- decode epilogue steps
// Written once so that every decode kernel rounds them the same way.
// Rescale of an int32 accumulator: acc * gamma / s, each a correctly rounded fp32 operation.
__device__ __forceinline__ float rescale_acc(int acc, float gamma, float s) {
  return __fdiv_rn(__fmul_rn((float)acc, gamma), s);
}
// One MLGRU step of one channel from its f, c, g pre-activations: h becomes
// f h + (1 - f) c (f = sigmoid, c = SiLU); returns the gated output g h.
__device__ __forceinline__ float mlgru_step(float pf, float pc, float pg, float& h) {
  const float f = sigmoidf_(pf), c = siluf_(pc), g = sigmoidf_(pg);
  h = __fmaf_rn(f, h, __fmul_rn(1.0f - f, c));
  return g * h;
}

// ---------------------------------------------------------------- programmatic dependent launch
// A kernel launched with programmatic stream serialization may start before
// its predecessor in the stream has finished. pdl_wait() blocks until every
// predecessor grid has completed and its memory is visible: call it before the
// first read of a predecessor's output and before the first global write.
// pdl_trigger() lets the next kernel in the stream start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- misc
__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace mmf
