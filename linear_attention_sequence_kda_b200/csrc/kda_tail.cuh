// Conv tail: the last 3 raw q/k/v tokens of concat(init_conv, segment), the
// conv history a following prefill or decode step continues from (the conv
// state the page "GLM-5.3-Flash im Detail", section "Sequenz-Mixing: 34
// KDA-Schichten mit festem Zustand", notes is kept beside the recurrent state).
// One thread per (segment, tensor, channel) reads all three values before it
// writes any, so the tail may overwrite init_conv in place.
#pragma once
#include "kda_common.cuh"

namespace kda {

template <typename Tin>
__global__ void __launch_bounds__(256)
conv_tail_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                 const Tin* init_conv, const int32_t* __restrict__ cu, int N, int H, Tin* tail) {
  const int64_t HD = (int64_t)H * D;
  const int64_t total = (int64_t)N * 3 * HD;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = idx % HD;
    const int64_t rest = idx / HD;
    const int x = (int)(rest % 3);
    const int64_t n = rest / 3;
    const Tin* src = x == 0 ? q : (x == 1 ? k : v);
    const int64_t s0 = cu[n], T = cu[n + 1] - s0;
    Tin vals[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int64_t pos = T - 3 + j;  // position in the segment; < 0 -> history slot 3 + pos
      if (pos >= 0)
        vals[j] = src[(s0 + pos) * HD + c];
      else
        vals[j] = init_conv ? init_conv[((n * 3 + x) * 3 + (3 + pos)) * HD + c] : from_f<Tin>(0.f);
    }
#pragma unroll
    for (int j = 0; j < 3; ++j) tail[((n * 3 + x) * 3 + j) * HD + c] = vals[j];
  }
}

}  // namespace kda
