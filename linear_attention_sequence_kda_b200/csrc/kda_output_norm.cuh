// The output epilogue on its own: the gated RMS normalisation of rows of the
// mixer output that were produced outside the chunked prefill (decode and
// multi-token decode outputs, the fp32 recurrent path).  Page "GLM-5.3-Flash
// Internals -- a measured profile", section "Findings": the mixer output goes
// through o_norm, gated by the g_b_proj output, before o_proj; read as
//     y = o / sqrt(mean_v o^2 + eps) * w * sigmoid(z)
// over each head's 128 value channels.  The chunked prefill applies the same
// epilogue inside its output store (kda_chunk_scan.cuh).
//
// One warp per (row, head): each lane holds 4 consecutive channels, so a row
// is one coalesced 512-byte (fp32) or 256-byte (bf16) read; the sum of squares
// is a warp butterfly.  HBM-bound: 2 x 128 x esize + 256 bytes per row-head.
#pragma once
#include "kda_common.cuh"

namespace kda {

constexpr int NORM_THREADS = 256;

template <typename Tin>
__global__ void __launch_bounds__(NORM_THREADS)
output_norm_kernel(const Tin* o, const __nv_bfloat16* __restrict__ z, const float* __restrict__ w,
                   float eps, __nv_bfloat16* y, int64_t row_heads) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (NORM_THREADS / 32);
  const float4 wv = *reinterpret_cast<const float4*>(w + 4 * lane);
  for (int64_t r = (int64_t)blockIdx.x * (NORM_THREADS / 32) + (threadIdx.x >> 5); r < row_heads; r += warps) {
    const int64_t base = r * D + 4 * lane;
    float x[4];
    if constexpr (sizeof(Tin) == 4) {
      const float4 t = *reinterpret_cast<const float4*>(o + base);
      x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    } else {
      const uint2 t = *reinterpret_cast<const uint2*>(o + base);
      const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&t.x);
      const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&t.y);
      x[0] = __low2float(a); x[1] = __high2float(a); x[2] = __low2float(b); x[3] = __high2float(b);
    }
    const uint2 zr = *reinterpret_cast<const uint2*>(z + base);
    const __nv_bfloat162 z01 = *reinterpret_cast<const __nv_bfloat162*>(&zr.x);
    const __nv_bfloat162 z23 = *reinterpret_cast<const __nv_bfloat162*>(&zr.y);
    const float zz[4] = {__low2float(z01), __high2float(z01), __low2float(z23), __high2float(z23)};
    float s = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
    const float rs = rsqrtf(s * (1.f / D) + eps);
    const float ww[4] = {wv.x, wv.y, wv.z, wv.w};
    float out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) out[j] = x[j] * rs * ww[j] * (1.f / (1.f + __expf(-zz[j])));
    const __nv_bfloat162 y01 = __floats2bfloat162_rn(out[0], out[1]);
    const __nv_bfloat162 y23 = __floats2bfloat162_rn(out[2], out[3]);
    uint2 yr;
    yr.x = *reinterpret_cast<const uint32_t*>(&y01);
    yr.y = *reinterpret_cast<const uint32_t*>(&y23);
    *reinterpret_cast<uint2*>(y + base) = yr;
  }
}

}  // namespace kda
