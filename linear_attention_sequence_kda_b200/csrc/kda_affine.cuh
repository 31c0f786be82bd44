// Affine composition of per-head states, the exchange step of a sequence
// split into contiguous segments (context parallelism).
//
// Page "GLM-5.3-Flash im Detail", section "Sequenz-Mixing: 34 KDA-Schichten mit
// festem Zustand": a state is handed from chunk to chunk.  For a whole segment
// the hand-over is linear in the state it starts from: every chunk maps
// S -> (Diag(gamma) - Kbar^T W) S + Kbar^T T V, so a segment maps
//     S_out = A S_in + B,
// A (128 x 128 over key channels) the product of the chunks' transitions and B
// the segment's final state from a zero start.  A is the final state of the
// same segment run from S_in = I with v = 0 (each value column a probe), B the
// final state from S_in = 0.  Given every earlier segment's (A, B), a rank
// composes the state its own segment starts from.
//
// state_affine_kernel: one 256-thread block per (sequence, head) pair,
// S_out = A S_in + B in fp32 (S_in / S_out in the state storage type).  A and
// S_in are staged in shared memory; thread (ty, tx) computes an 8 x 8 tile of
// S_out (rows 8 ty.., columns 8 tx..) with a k-ascending fp32 sum.
#pragma once
#include "kda_common.cuh"

namespace kda {

constexpr uint32_t AFFINE_SMEM = 2 * D * D * sizeof(float);

template <typename Ts>
__global__ void __launch_bounds__(256)
state_affine_kernel(const float* __restrict__ A, const Ts* __restrict__ S_in, const float* __restrict__ B,
                    Ts* __restrict__ S_out) {
  extern __shared__ __align__(16) float sm_affine[];
  float* sA = sm_affine;          // [128][128] row-major
  float* sS = sm_affine + D * D;  // [128][128] row-major
  const int64_t base = (int64_t)blockIdx.x * D * D;
  const int tid = threadIdx.x;
  for (int e = tid; e < D * D / 4; e += 256) {
    reinterpret_cast<float4*>(sA)[e] = reinterpret_cast<const float4*>(A + base)[e];
    const Ts* sp = S_in + base + 4 * e;
    reinterpret_cast<float4*>(sS)[e] = make_float4(to_f(sp[0]), to_f(sp[1]), to_f(sp[2]), to_f(sp[3]));
  }
  __syncthreads();
  const int ty = tid >> 4, tx = tid & 15;  // rows 8 ty .. 8 ty + 7, columns 8 tx .. 8 tx + 7
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int k = 0; k < D; ++k) {
    float a[8], b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = sA[(8 * ty + i) * D + k];
    const float4 b0 = *reinterpret_cast<const float4*>(sS + k * D + 8 * tx);
    const float4 b1 = *reinterpret_cast<const float4*>(sS + k * D + 8 * tx + 4);
    b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w; b[4] = b1.x; b[5] = b1.y; b[6] = b1.z; b[7] = b1.w;
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t row = base + (int64_t)(8 * ty + i) * D + 8 * tx;
#pragma unroll
    for (int j = 0; j < 8; ++j) S_out[row + j] = from_f<Ts>(acc[i][j] + B[row + j]);
  }
}

}  // namespace kda
