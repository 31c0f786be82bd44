// Token-by-token fp32 KDA prefill (exact path; the fp32 inputs route here).
//
// One thread block per (segment, head); thread v owns column v of the
// 128 x 128 state S (row = key channel) in registers for the whole segment.
// Tokens are processed in blocks of TB: a prologue computes, per token, the
// conv outputs, the L2 norms and the decays into shared memory; the recurrence
// then applies, per token (page "GLM-5.3-Flash im Detail", section
// "Sequenz-Mixing: 34 KDA-Schichten mit festem Zustand"):
//     r = (Diag(alpha) S)^T k,  u = beta (v - r),
//     o = (Diag(alpha) S)^T q + u (k . q),   S <- Diag(alpha) S + k u^T
// which is S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T and
// o_t = S_t^T q_t evaluated with a single pass over S.
#pragma once
#include "kda_common.cuh"

namespace kda {

constexpr int REC_TB = 16;  // tokens per prologue block

template <typename Tin, typename Tout, int ACT, typename Ts>
__global__ void __launch_bounds__(128)
recurrent_prefill_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                         const Tin* __restrict__ v, const Tin* __restrict__ g,
                         const Tin* __restrict__ beta, const float* __restrict__ conv_w,
                         const Ts* init_state, const Tin* __restrict__ init_conv,
                         const int32_t* __restrict__ cu, int H, Tout* __restrict__ o,
                         Ts* final_state) {
  __shared__ __align__(16) float sh_kh[REC_TB][D];    // k_hat
  __shared__ __align__(16) float sh_ka[REC_TB][D];    // alpha * k_hat
  __shared__ __align__(16) float sh_qa[REC_TB][D];    // alpha * q_hat
  __shared__ __align__(16) float sh_al[REC_TB][D];    // alpha
  __shared__ __align__(16) float sh_v[REC_TB][D];     // conv(v)
  __shared__ float sh_beta[REC_TB], sh_kq[REC_TB], sh_rq[REC_TB], sh_rk[REC_TB];

  const int h = blockIdx.x, n = blockIdx.y, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t s0 = cu[n], s1 = cu[n + 1];
  const int64_t HD = (int64_t)H * D;
  const int64_t ch = (int64_t)h * D + tid;  // this thread's channel within [H*D]

  // conv taps and the 3-token history for channel `tid` of q, k, v
  const float4 wq = load4(conv_w + (0 * HD + ch) * 4);
  const float4 wk = load4(conv_w + (1 * HD + ch) * 4);
  const float4 wv = load4(conv_w + (2 * HD + ch) * 4);
  float hq[3] = {0.f, 0.f, 0.f}, hk[3] = {0.f, 0.f, 0.f}, hv[3] = {0.f, 0.f, 0.f};
  if (init_conv) {
    const Tin* c = init_conv + (int64_t)n * 9 * HD + ch;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      hq[j] = to_f(c[(0 * 3 + j) * HD]);
      hk[j] = to_f(c[(1 * 3 + j) * HD]);
      hv[j] = to_f(c[(2 * 3 + j) * HD]);
    }
  }

  // state column tid
  float S[D];
  Ts* Sg = final_state + ((int64_t)n * H + h) * D * D + tid;
  if (init_state) {
    const Ts* Si = init_state + ((int64_t)n * H + h) * D * D + tid;
#pragma unroll
    for (int i = 0; i < D; ++i) S[i] = to_f(Si[(int64_t)i * D]);
  } else {
#pragma unroll
    for (int i = 0; i < D; ++i) S[i] = 0.f;
  }

  for (int64_t tb = s0; tb < s1; tb += REC_TB) {
    const int nt = (int)((s1 - tb) < REC_TB ? (s1 - tb) : REC_TB);
    // ---- prologue 1: conv, decay, beta (thread = channel) ----
    for (int t = 0; t < nt; ++t) {
      const int64_t row = (tb + t) * HD + ch;
      const float xq = to_f(q[row]), xk = to_f(k[row]), xv = to_f(v[row]);
      float yq = conv4(wq, hq[0], hq[1], hq[2], xq);
      float yk = conv4(wk, hk[0], hk[1], hk[2], xk);
      float yv = conv4(wv, hv[0], hv[1], hv[2], xv);
      if (ACT == KDA_CONV_SILU) { yq = silu(yq); yk = silu(yk); yv = silu(yv); }
      hq[0] = hq[1]; hq[1] = hq[2]; hq[2] = xq;
      hk[0] = hk[1]; hk[1] = hk[2]; hk[2] = xk;
      hv[0] = hv[1]; hv[1] = hv[2]; hv[2] = xv;
      sh_qa[t][tid] = yq;
      sh_kh[t][tid] = yk;
      sh_v[t][tid] = yv;
      sh_al[t][tid] = expf(fmaxf(to_f(g[row]), LOG_DECAY_FLOOR));
      if (tid == 0) sh_beta[t] = to_f(beta[(tb + t) * H + h]);
    }
    __syncthreads();
    // ---- prologue 2: norms (warp per token) ----
    for (int t = warp; t < nt; t += 4) {
      const float4 a = *reinterpret_cast<const float4*>(&sh_qa[t][lane * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&sh_kh[t][lane * 4]);
      float nq = a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
      float nk = b.x * b.x + b.y * b.y + b.z * b.z + b.w * b.w;
      float qk = a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
      nq = warp_sum(nq); nk = warp_sum(nk); qk = warp_sum(qk);
      if (lane == 0) {
        const float rq = 1.0f / sqrtf(nq + NORM_EPS), rk = 1.0f / sqrtf(nk + NORM_EPS);
        sh_rq[t] = rq; sh_rk[t] = rk; sh_kq[t] = qk * rq * rk;
      }
    }
    __syncthreads();
    // ---- prologue 3: scaled vectors (thread = channel, own column only) ----
    for (int t = 0; t < nt; ++t) {
      const float a = sh_al[t][tid];
      const float kh = sh_kh[t][tid] * sh_rk[t];
      const float qh = sh_qa[t][tid] * sh_rq[t];
      sh_kh[t][tid] = kh;
      sh_ka[t][tid] = a * kh;
      sh_qa[t][tid] = a * qh;
    }
    __syncthreads();
    // ---- recurrence (thread = value column) ----
    for (int t = 0; t < nt; ++t) {
      float r0 = 0.f, r1 = 0.f, y0 = 0.f, y1 = 0.f;
#pragma unroll
      for (int i = 0; i < D; i += 4) {
        const float4 ka = *reinterpret_cast<const float4*>(&sh_ka[t][i]);
        const float4 qa = *reinterpret_cast<const float4*>(&sh_qa[t][i]);
        r0 = fmaf(S[i], ka.x, r0); r1 = fmaf(S[i + 1], ka.y, r1);
        r0 = fmaf(S[i + 2], ka.z, r0); r1 = fmaf(S[i + 3], ka.w, r1);
        y0 = fmaf(S[i], qa.x, y0); y1 = fmaf(S[i + 1], qa.y, y1);
        y0 = fmaf(S[i + 2], qa.z, y0); y1 = fmaf(S[i + 3], qa.w, y1);
      }
      const float u = sh_beta[t] * (sh_v[t][tid] - (r0 + r1));
      const float out = (y0 + y1) + u * sh_kq[t];
#pragma unroll
      for (int i = 0; i < D; i += 4) {
        const float4 al = *reinterpret_cast<const float4*>(&sh_al[t][i]);
        const float4 kh = *reinterpret_cast<const float4*>(&sh_kh[t][i]);
        S[i] = fmaf(al.x, S[i], kh.x * u);
        S[i + 1] = fmaf(al.y, S[i + 1], kh.y * u);
        S[i + 2] = fmaf(al.z, S[i + 2], kh.z * u);
        S[i + 3] = fmaf(al.w, S[i + 3], kh.w * u);
      }
      o[(tb + t) * HD + ch] = from_f<Tout>(out);
    }
    __syncthreads();  // before the next prologue overwrites shared memory
  }
#pragma unroll
  for (int i = 0; i < D; ++i) Sg[(int64_t)i * D] = from_f<Ts>(S[i]);
}

}  // namespace kda
