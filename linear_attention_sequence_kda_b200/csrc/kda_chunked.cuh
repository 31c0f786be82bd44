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
                                 kda_dtype o_dt, void* o, float* final_state,
                                 void* /*workspace*/, size_t /*workspace_bytes*/, int /*max_len*/,
                                 cudaStream_t stream) {
  using T = __nv_bfloat16;
  dim3 grid(H, N);
  const bool silu = act == KDA_CONV_SILU;
#define KDA_REC(TO, A)                                                                          \
  recurrent_prefill_kernel<T, TO, A><<<grid, 128, 0, stream>>>(                                  \
      (const T*)q, (const T*)k, (const T*)v, (const T*)g, (const T*)beta, conv_w, init_state,   \
      (const T*)init_conv, cu_dev, H, (TO*)o, final_state)
  if (o_dt == KDA_F32) {
    if (silu) KDA_REC(float, KDA_CONV_SILU); else KDA_REC(float, KDA_CONV_NONE);
  } else {
    if (silu) KDA_REC(T, KDA_CONV_SILU); else KDA_REC(T, KDA_CONV_NONE);
  }
#undef KDA_REC
  return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace kda
