// Multi-token decode for speculative (multi-token-prediction) serving: verify
// R draft rows against a state without changing it, then commit the accepted
// prefix.
//
// Page "GLM-5.3-Flash im Detail", section "Sequenz-Mixing: 34 KDA-Schichten mit
// festem Zustand": decoding is one recurrent state update per token.  Page
// "GLM-5.3-Flash Internals — a measured profile" serves with multi-token
// prediction (k = 5 drafts, so 6 rows per verify step) and reports an
// acceptance of about four tokens: a verify step must be able to keep any
// prefix of its rows.  Both kernels follow the single-token step of
// kda_decode.cuh row by row (same arithmetic, same order), so committing n
// rows leaves exactly the state and conv cache of n single-token steps.
//
// decode_verify_kernel: one 256-thread block per (sequence, head).  The state
// is read once into registers (warp w rows [16w, 16w+16), lane l columns
// [4l, 4l+4)) and updated there row by row; it is not written back.  Per row t
// it writes o_t and the row's update (k_hat_t, u_t, alpha_t) to `deltas`.
// decode_commit_kernel: per (sequence, head), S <- Diag(alpha_t) S + k_hat_t u_t^T
// for the first n_accept rows (one read and one write of S), and the conv
// cache becomes the last three raw tokens of [cache, accepted rows].
#pragma once
#include "kda_common.cuh"

namespace kda {

constexpr int MAX_VERIFY_ROWS = KDA_MAX_VERIFY_ROWS;

template <typename Tin, typename Tout, int ACT>
__global__ void __launch_bounds__(256, 2)
decode_verify_kernel(const float* __restrict__ state, const Tin* __restrict__ cache,
                     const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                     const Tin* __restrict__ g, const Tin* __restrict__ beta, const float* __restrict__ conv_w,
                     int R, int H, Tout* __restrict__ o, float* __restrict__ deltas) {
  __shared__ __align__(16) float sh_kh[D], sh_ka[D], sh_qa[D], sh_al[D], sh_v[D], sh_u[D];
  __shared__ __align__(16) float sh_r[8][D], sh_y[8][D];
  __shared__ float sh_red[4][3];

  const int h = blockIdx.x, n = blockIdx.y, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t HD = (int64_t)H * D;
  const float* S = state + ((int64_t)n * H + h) * D * D;
  float4 s[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) s[i] = ld_stream(S + (warp * 16 + i) * D + lane * 4);

  // conv taps and history of this thread's channel: threads 0..127 q and k,
  // threads 128..255 v (history = the cache, then the rows of this call)
  const int c = tid & (D - 1);
  const int64_t ch = (int64_t)h * D + c;
  const Tin* cb = cache + (int64_t)n * 9 * HD + ch;  // [3 x][3 t] stride HD
  float4 w0, w1;
  float h0[3], h1[3];
  if (tid < D) {
    w0 = load4(conv_w + (0 * HD + ch) * 4);
    w1 = load4(conv_w + (1 * HD + ch) * 4);
    for (int j = 0; j < 3; ++j) { h0[j] = to_f(cb[j * HD]); h1[j] = to_f(cb[(3 + j) * HD]); }
  } else {
    w0 = load4(conv_w + (2 * HD + ch) * 4);
    w1 = w0;
    for (int j = 0; j < 3; ++j) { h0[j] = to_f(cb[(6 + j) * HD]); h1[j] = 0.f; }
  }
  float* dl = deltas + ((int64_t)n * H + h) * R * 3 * D;  // [R][3][D]

  for (int t = 0; t < R; ++t) {
    const int64_t tok = (((int64_t)n * R + t) * H + h) * D + c;  // [N, R, H, D]
    float yq = 0.f, yk = 0.f;
    if (tid < D) {
      const float xq = to_f(q[tok]), xk = to_f(k[tok]);
      yq = conv4(w0, h0[0], h0[1], h0[2], xq);
      yk = conv4(w1, h1[0], h1[1], h1[2], xk);
      if (ACT == KDA_CONV_SILU) { yq = silu(yq); yk = silu(yk); }
      h0[0] = h0[1]; h0[1] = h0[2]; h0[2] = xq;
      h1[0] = h1[1]; h1[1] = h1[2]; h1[2] = xk;
      float nq = warp_sum(yq * yq), nk = warp_sum(yk * yk), qk = warp_sum(yq * yk);
      if (lane == 0) { sh_red[warp][0] = nq; sh_red[warp][1] = nk; sh_red[warp][2] = qk; }
    } else {
      const float xv = to_f(v[tok]);
      float yv = conv4(w0, h0[0], h0[1], h0[2], xv);
      if (ACT == KDA_CONV_SILU) yv = silu(yv);
      h0[0] = h0[1]; h0[1] = h0[2]; h0[2] = xv;
      sh_v[c] = yv;
      sh_al[c] = __expf(fmaxf(to_f(g[tok]), LOG_DECAY_FLOOR));
    }
    __syncthreads();
    const float nq = sh_red[0][0] + sh_red[1][0] + sh_red[2][0] + sh_red[3][0];
    const float nk = sh_red[0][1] + sh_red[1][1] + sh_red[2][1] + sh_red[3][1];
    const float qk = sh_red[0][2] + sh_red[1][2] + sh_red[2][2] + sh_red[3][2];
    const float rq = rsqrtf(nq + NORM_EPS), rk = rsqrtf(nk + NORM_EPS);
    const float kq = qk * rq * rk;
    if (tid < D) {
      const float a = sh_al[c];
      const float kh = yk * rk;
      sh_kh[c] = kh;
      sh_ka[c] = a * kh;
      sh_qa[c] = a * yq * rq;
    }
    __syncthreads();
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f), y = r;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float ka = sh_ka[warp * 16 + i], qa = sh_qa[warp * 16 + i];
      r.x = fmaf(s[i].x, ka, r.x); r.y = fmaf(s[i].y, ka, r.y);
      r.z = fmaf(s[i].z, ka, r.z); r.w = fmaf(s[i].w, ka, r.w);
      y.x = fmaf(s[i].x, qa, y.x); y.y = fmaf(s[i].y, qa, y.y);
      y.z = fmaf(s[i].z, qa, y.z); y.w = fmaf(s[i].w, qa, y.w);
    }
    *reinterpret_cast<float4*>(&sh_r[warp][lane * 4]) = r;
    *reinterpret_cast<float4*>(&sh_y[warp][lane * 4]) = y;
    __syncthreads();
    if (tid < D) {
      float rr = 0.f, yy = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) { rr += sh_r[w][tid]; yy += sh_y[w][tid]; }
      const float b = to_f(beta[((int64_t)n * R + t) * H + h]);
      const float u = b * (sh_v[tid] - rr);
      sh_u[tid] = u;
      o[tok] = from_f<Tout>(yy + u * kq);
      dl[(t * 3 + 0) * D + tid] = sh_kh[tid];
      dl[(t * 3 + 1) * D + tid] = u;
      dl[(t * 3 + 2) * D + tid] = sh_al[tid];
    }
    __syncthreads();
    // S <- Diag(a) S + k u^T in registers (the same expression as the single step)
    const float4 u4 = *reinterpret_cast<const float4*>(&sh_u[lane * 4]);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int row = warp * 16 + i;
      const float a = sh_al[row], kh = sh_kh[row];
      s[i].x = fmaf(a, s[i].x, kh * u4.x);
      s[i].y = fmaf(a, s[i].y, kh * u4.y);
      s[i].z = fmaf(a, s[i].z, kh * u4.z);
      s[i].w = fmaf(a, s[i].w, kh * u4.w);
    }
    __syncthreads();  // shared rows are rewritten by the next row's prologue
  }
}

template <typename Tin>
__global__ void __launch_bounds__(256, 2)
decode_commit_kernel(float* __restrict__ state, Tin* __restrict__ cache, const Tin* __restrict__ q,
                     const Tin* __restrict__ k, const Tin* __restrict__ v, const float* __restrict__ deltas,
                     const int32_t* __restrict__ n_accept, int R, int H) {
  __shared__ __align__(16) float sh_kh[MAX_VERIFY_ROWS][D], sh_u[MAX_VERIFY_ROWS][D], sh_al[MAX_VERIFY_ROWS][D];
  const int h = blockIdx.x, n = blockIdx.y, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t HD = (int64_t)H * D;
  int na = n_accept[n];
  if (na < 0 || na > R) {  // out of range: record it and keep what can be kept
    if (tid == 0 && h == 0) set_status(KDA_ERR_INVALID_ARG);
    na = na < 0 ? 0 : R;
  }
  if (na == 0) return;  // nothing accepted: state and cache stay as they are
  float* S = state + ((int64_t)n * H + h) * D * D;
  float4 s[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) s[i] = ld_stream(S + (warp * 16 + i) * D + lane * 4);
  const float* dl = deltas + ((int64_t)n * H + h) * R * 3 * D;
  for (int e = tid; e < na * D; e += 256) {
    const int t = e / D, cc = e % D;
    sh_kh[t][cc] = dl[(t * 3 + 0) * D + cc];
    sh_u[t][cc] = dl[(t * 3 + 1) * D + cc];
    sh_al[t][cc] = dl[(t * 3 + 2) * D + cc];
  }
  // conv cache: the last three raw tokens of [cache (3 rows), accepted rows];
  // all three are read before any is written (the cache is updated in place)
  for (int e = tid; e < 3 * D; e += 256) {
    const int x = e / D, cc = e % D;  // tensor (q, k, v), channel
    const int64_t ch = (int64_t)h * D + cc;
    Tin* cb = cache + ((int64_t)n * 9 + 3 * x) * HD + ch;
    const Tin* src = x == 0 ? q : (x == 1 ? k : v);
    Tin nv[3];
    for (int j = 0; j < 3; ++j) {
      const int idx = na + j;  // position in [cache rows 0..2, accepted rows]
      nv[j] = idx < 3 ? cb[idx * HD] : src[(((int64_t)n * R + (idx - 3)) * H + h) * D + cc];
    }
    for (int j = 0; j < 3; ++j) cb[j * HD] = nv[j];
  }
  __syncthreads();
  for (int t = 0; t < na; ++t) {
    const float4 u4 = *reinterpret_cast<const float4*>(&sh_u[t][lane * 4]);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int row = warp * 16 + i;
      const float a = sh_al[t][row], kh = sh_kh[t][row];
      s[i].x = fmaf(a, s[i].x, kh * u4.x);
      s[i].y = fmaf(a, s[i].y, kh * u4.y);
      s[i].z = fmaf(a, s[i].z, kh * u4.z);
      s[i].w = fmaf(a, s[i].w, kh * u4.w);
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) st_stream(S + (warp * 16 + i) * D + lane * 4, s[i]);
}

}  // namespace kda
