// Chunked bf16 prefill entry (interim: evaluated by the recurrent kernel).
#pragma once
#include "kda_common.cuh"
#include "kda_recurrent.cuh"

namespace kda {

inline size_t chunked_workspace_bytes(int /*N*/, int /*H*/) { return 0; }

inline kda_status launch_chunked(const void* q, const void* k, const void* v, const void* g,
                                 const void* beta, const float* conv_w, const float* init_state,
                                 const void* init_conv, const int32_t* cu_dev,
                                 const int32_t* /*cu_host*/, int N, int H, kda_conv_act act,
                                 void* o, float* final_state, void* /*workspace*/,
                                 cudaStream_t stream) {
  using T = __nv_bfloat16;
  dim3 grid(H, N);
  if (act == KDA_CONV_SILU)
    recurrent_prefill_kernel<T, KDA_CONV_SILU><<<grid, 128, 0, stream>>>(
        (const T*)q, (const T*)k, (const T*)v, (const T*)g, (const T*)beta, conv_w, init_state,
        (const T*)init_conv, cu_dev, H, (T*)o, final_state);
  else
    recurrent_prefill_kernel<T, KDA_CONV_NONE><<<grid, 128, 0, stream>>>(
        (const T*)q, (const T*)k, (const T*)v, (const T*)g, (const T*)beta, conv_w, init_state,
        (const T*)init_conv, cu_dev, H, (T*)o, final_state);
  return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace kda
