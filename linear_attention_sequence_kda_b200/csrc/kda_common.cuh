// Shared device helpers for the KDA kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

constexpr int D = KDA_HEAD_DIM;   // d_k = d_v = 128
constexpr float LOG_DECAY_FLOOR = -5.0f;
constexpr float NORM_EPS = 1e-6f;
constexpr float LOG2E = 1.4426950408889634f;

// Device status word (one per device per process): kernels that give up on a
// bounded wait write a nonzero kda_status here; kda_check_async_status reads it.
__device__ int g_status;

__device__ __forceinline__ void set_status(int code) { atomicCAS(&g_status, 0, code); }

// The CUDA error behind the last KDA_ERR_CUDA returned on this host thread
// (kda_last_cuda_error); every host-side CUDA call is checked through cuda_ok.
inline thread_local int t_last_cuda_error = 0;
inline bool cuda_ok(cudaError_t e) {
  if (e == cudaSuccess) return true;
  t_last_cuda_error = (int)e;
  return false;
}

// ---- element loads/stores in either dtype, converted to/from fp32 ----------
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// 4 consecutive elements -> float4 (pointer 8/16-byte aligned).
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}

__device__ __forceinline__ float silu(float y) { return y / (1.0f + __expf(-y)); }

// Causal width-4 conv tap sum: w.x = w0*x_{t-3} + w1*x_{t-2} + w2*x_{t-1} + w3*x_t
__device__ __forceinline__ float conv4(float4 w, float xm3, float xm2, float xm1, float x0) {
  return fmaf(w.w, x0, fmaf(w.z, xm1, fmaf(w.y, xm2, w.x * xm3)));
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Packed fp32 pairs (sm_100 f32x2 forms): two lanes per instruction, each
// lane rounded exactly as the scalar fmaf / multiply would round it.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n.reg .b64 a, b, c, d;\nmov.b64 a, {%2, %3};\nmov.b64 b, {%4, %5};\nmov.b64 c, {%6, %7};\n"
      "fma.rn.f32x2 d, a, b, c;\nmov.b64 {%0, %1}, d;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n.reg .b64 a, b, d;\nmov.b64 a, {%2, %3};\nmov.b64 b, {%4, %5};\n"
      "mul.rn.f32x2 d, a, b;\nmov.b64 {%0, %1}, d;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n.reg .b64 a, b, d;\nmov.b64 a, {%2, %3};\nmov.b64 b, {%4, %5};\n"
      "add.rn.f32x2 d, a, b;\nmov.b64 {%0, %1}, d;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 lo2(float4 v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(float4 v) { return make_float2(v.z, v.w); }
__device__ __forceinline__ float4 cat2(float2 a, float2 b) { return make_float4(a.x, a.y, b.x, b.y); }
__device__ __forceinline__ float2 dup2(float x) { return make_float2(x, x); }

// Streaming (evict-first) 16-byte global load/store for data touched once.
__device__ __forceinline__ float4 ld_stream(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ void st_stream(float* p, float4 v) { __stcs(reinterpret_cast<float4*>(p), v); }

// State storage: fp32, or bf16 (rounded to nearest, ties to even, when
// stored).  Arithmetic on the state is always fp32; a bf16 state element reads
// back as the fp32 value it was rounded to.  Four consecutive elements per
// call, streaming (the states are touched once per step).
__device__ __forceinline__ float4 ld_state4(const float* p) { return ld_stream(p); }
__device__ __forceinline__ float4 ld_state4(const __nv_bfloat16* p) {
  const uint2 u = __ldcs(reinterpret_cast<const uint2*>(p));  // element 2j in the low half of word j
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xFFFF0000u));
}
__device__ __forceinline__ void st_state4(float* p, float4 v) { st_stream(p, v); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);  // .x (low half) = lo
  return *reinterpret_cast<const uint32_t*>(&b);
}
__device__ __forceinline__ void st_state4(__nv_bfloat16* p, float4 v) {
  __stcs(reinterpret_cast<uint2*>(p), make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w)));
}
// Four consecutive state elements from shared memory (a prefetched state).
__device__ __forceinline__ float4 ld_state4_shared(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 ld_state4_shared(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xFFFF0000u));
}
// The value an element has after a store and a load in storage type Ts.
template <typename Ts> __device__ __forceinline__ float4 as_stored4(float4 v);
template <> __device__ __forceinline__ float4 as_stored4<float>(float4 v) { return v; }
template <> __device__ __forceinline__ float4 as_stored4<__nv_bfloat16>(float4 v) {
  const uint32_t a = pack_bf16x2(v.x, v.y), b = pack_bf16x2(v.z, v.w);  // one convert per pair
  return make_float4(__uint_as_float(a << 16), __uint_as_float(a & 0xFFFF0000u), __uint_as_float(b << 16),
                     __uint_as_float(b & 0xFFFF0000u));
}

}  // namespace kda
