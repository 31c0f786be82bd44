// Single-token KDA decode, in place, bound by streaming the fp32 states.
//
// Page "GLM-5.3-Flash im Detail", section "Sequenz-Mixing: 34 KDA-Schichten mit
// festem Zustand": decoding one token is one recurrent update of the per-head
// state.  Per (sequence, head), with S the 128 x 128 state (row = key channel):
//     y = conv4(cache, x) for q, k, v;  q, k L2-normalised;  a = exp(max(g,-5))
//     r = S^T (a * k),  u = beta (v - r),  o = S^T (a * q) + u (k . q)
//     S <- Diag(a) S + k u^T,  cache <- shift(cache, x)
// so S is read once and written once (single pass).
//
// Block = 256 threads = 8 warps, persistent (two per SM) over the (sequence,
// head) items.  Warp w owns rows [16w, 16w+16); lane l owns columns
// [4l, 4l+4): 16 float4 registers per thread.  While a block computes one item
// a single bulk copy brings the next item's state (64 KiB, or 32 KiB in bf16)
// into shared memory, so the state stream from HBM does not wait on the
// prologue, the reductions or the barriers; reductions over rows are finished
// through shared memory; the updated rows are written with streaming stores.
#pragma once
#include "kda_common.cuh"
#include "kda_tc.cuh"

namespace kda {

// A warp's 16 state rows, lane l holding columns [4l, 4l+4) of each: s[i] is
// row i.  The two helpers below are the whole state arithmetic of a decode
// step, shared by the single-token and the multi-token kernels so that both
// round identically.  Packed f32x2 instructions do two columns at a time; each
// column is rounded as its scalar fmaf would round it.
//
// r = sum_i x_i s_i and y = sum_i z_i s_i over the 16 rows, i ascending
// (x, z: this warp's 16 entries, shared memory, 16-byte aligned).
__device__ __forceinline__ void rows_dot2(const float4 (&s)[16], const float* x, const float* z, float4& r,
                                          float4& y) {
  float2 r0 = make_float2(0.f, 0.f), r1 = r0, y0 = r0, y1 = r0;
#pragma unroll
  for (int i4 = 0; i4 < 4; ++i4) {
    const float4 x4 = *reinterpret_cast<const float4*>(x + 4 * i4);
    const float4 z4 = *reinterpret_cast<const float4*>(z + 4 * i4);
    const float xs[4] = {x4.x, x4.y, x4.z, x4.w}, zs[4] = {z4.x, z4.y, z4.z, z4.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 si = s[4 * i4 + j];
      r0 = fma2(lo2(si), dup2(xs[j]), r0); r1 = fma2(hi2(si), dup2(xs[j]), r1);
      y0 = fma2(lo2(si), dup2(zs[j]), y0); y1 = fma2(hi2(si), dup2(zs[j]), y1);
    }
  }
  r = cat2(r0, r1);
  y = cat2(y0, y1);
}

// s_i <- a_i s_i + kh_i u (the delta-rule row update Diag(a) S + k u^T; a, kh:
// this warp's 16 entries in shared memory, u4: this lane's 4 columns of u).
__device__ __forceinline__ void rows_update(float4 (&s)[16], const float* a, const float* kh, float4 u4) {
  const float2 u0 = lo2(u4), u1 = hi2(u4);
#pragma unroll
  for (int i4 = 0; i4 < 4; ++i4) {
    const float4 a4 = *reinterpret_cast<const float4*>(a + 4 * i4);
    const float4 k4 = *reinterpret_cast<const float4*>(kh + 4 * i4);
    const float as[4] = {a4.x, a4.y, a4.z, a4.w}, ks[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float4& si = s[4 * i4 + j];
      si = cat2(fma2(dup2(as[j]), lo2(si), mul2(dup2(ks[j]), u0)),
                fma2(dup2(as[j]), hi2(si), mul2(dup2(ks[j]), u1)));
    }
  }
}

// Bytes of dynamic shared memory the persistent decode kernels need (the
// prefetched state).
template <typename Ts> __host__ __device__ constexpr uint32_t decode_smem_bytes() { return (uint32_t)(D * D * sizeof(Ts)); }

// State prefetch of the persistent decode kernels (256 threads, items visited
// as blockIdx.x, + gridDim.x, ...): while a block computes one (sequence, head)
// item, one bulk copy brings the next item's state into the dynamic shared
// memory buffer.  init() is called once by all threads before the item loop
// (it contains a barrier); take() by all threads at the top of each item.
template <typename Ts>
struct StatePrefetch {
  Ts* buf;
  const Ts* state;
  uint64_t* bar;
  int items;
  uint32_t par;

  __device__ __forceinline__ void issue(int item) {  // one thread
    tc::fence_async_smem();  // the buffer's previous contents were read by every thread
    tc::bar_expect_tx(bar, decode_smem_bytes<Ts>());
    tc::bulk_g2s(buf, state + (int64_t)item * D * D, decode_smem_bytes<Ts>(), bar);
  }
  __device__ __forceinline__ void init(const Ts* st, int n_items) {
    extern __shared__ __align__(128) uint8_t dsm[];
    __shared__ uint64_t bar_state;
    buf = reinterpret_cast<Ts*>(dsm);
    state = st;
    bar = &bar_state;
    items = n_items;
    par = 0;
    if (threadIdx.x == 0) {
      tc::bar_init(bar, 1);
      tc::bar_init_fence();
      if ((int)blockIdx.x < items) issue(blockIdx.x);
    }
    __syncthreads();
  }
  // This item's state into registers (warp w rows [16w, 16w+16), lane l
  // columns [4l, 4l+4)), then the next item's copy is issued.  Returns false
  // for the whole block if the copy did not land in time (recorded as
  // KDA_ERR_TIMEOUT; the copy in flight is awaited once more before the block
  // gives up, so nothing lands in shared memory after it exits).
  __device__ __forceinline__ bool take(int item, float4 (&s)[16]) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (!__syncthreads_and(tc::bar_wait(bar, par))) {
      if (threadIdx.x == 0) tc::bar_wait(bar, par);
      return false;
    }
    par ^= 1;
#pragma unroll
    for (int i = 0; i < 16; ++i) s[i] = ld_state4_shared(buf + (warp * 16 + i) * D + lane * 4);
    __syncthreads();
    if (threadIdx.x == 0 && item + (int)gridDim.x < items) issue(item + gridDim.x);
    return true;
  }
};

template <typename Tin, typename Tout, int ACT, typename Ts>
__global__ void __launch_bounds__(256, 2)
decode_kernel(Ts* __restrict__ state, Tin* __restrict__ cache, const Tin* __restrict__ q,
              const Tin* __restrict__ k, const Tin* __restrict__ v, const Tin* __restrict__ g,
              const Tin* __restrict__ beta, const float* __restrict__ conv_w, int N, int H,
              Tout* __restrict__ o) {
  __shared__ __align__(16) float sh_kh[D], sh_ka[D], sh_qa[D], sh_al[D], sh_v[D], sh_u[D];
  __shared__ __align__(16) float sh_r[8][D], sh_y[8][D];
  __shared__ float sh_red[4][3];
  StatePrefetch<Ts> pf;
  pf.init(state, N * H);  // item = n * H + h: consecutive items are adjacent states

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t HD = (int64_t)H * D;
  for (int item = blockIdx.x; item < pf.items; item += gridDim.x) {
    const int n = item / H, h = item % H;
    Ts* S = state + (int64_t)item * D * D;

    // 1. this item's state, prefetched into shared memory, into registers;
    //    then the buffer takes the next item's state
    float4 s[16];
    if (!pf.take(item, s)) return;

    // 2. prologue: threads 0..127 -> q and k of channel c; 128..255 -> v and g
    const int c = tid & (D - 1);
    const int64_t ch = (int64_t)h * D + c;
    const int64_t tok = (int64_t)n * HD + ch;   // [N, H, D] index
    Tin* cb = cache + (int64_t)n * 9 * HD + ch; // [3 x][3 t] stride HD
    float yq = 0.f, yk = 0.f;
    if (tid < D) {
      const float4 wq = load4(conv_w + (0 * HD + ch) * 4);
      const float4 wk = load4(conv_w + (1 * HD + ch) * 4);
      const float q0 = to_f(cb[0 * HD]), q1 = to_f(cb[1 * HD]), q2 = to_f(cb[2 * HD]);
      const float k0 = to_f(cb[3 * HD]), k1 = to_f(cb[4 * HD]), k2 = to_f(cb[5 * HD]);
      const Tin xq = q[tok], xk = k[tok];
      yq = conv4(wq, q0, q1, q2, to_f(xq));
      yk = conv4(wk, k0, k1, k2, to_f(xk));
      if (ACT == KDA_CONV_SILU) { yq = silu(yq); yk = silu(yk); }
      // shift the cache (all reads of this channel's history are done above)
      cb[0 * HD] = cb[1 * HD]; cb[1 * HD] = cb[2 * HD]; cb[2 * HD] = xq;
      cb[3 * HD] = cb[4 * HD]; cb[4 * HD] = cb[5 * HD]; cb[5 * HD] = xk;
      float nq = warp_sum(yq * yq), nk = warp_sum(yk * yk), qk = warp_sum(yq * yk);
      if (lane == 0) { sh_red[warp][0] = nq; sh_red[warp][1] = nk; sh_red[warp][2] = qk; }
    } else {
      const float4 wv = load4(conv_w + (2 * HD + ch) * 4);
      const float v0 = to_f(cb[6 * HD]), v1 = to_f(cb[7 * HD]), v2 = to_f(cb[8 * HD]);
      const Tin xv = v[tok];
      float yv = conv4(wv, v0, v1, v2, to_f(xv));
      if (ACT == KDA_CONV_SILU) yv = silu(yv);
      cb[6 * HD] = cb[7 * HD]; cb[7 * HD] = cb[8 * HD]; cb[8 * HD] = xv;
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

    // 3. partial reductions over this warp's 16 rows, 4 columns per lane
    float4 r, y;
    rows_dot2(s, &sh_ka[warp * 16], &sh_qa[warp * 16], r, y);
    *reinterpret_cast<float4*>(&sh_r[warp][lane * 4]) = r;
    *reinterpret_cast<float4*>(&sh_y[warp][lane * 4]) = y;
    __syncthreads();
    if (tid < D) {
      float rr = 0.f, yy = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) { rr += sh_r[w][tid]; yy += sh_y[w][tid]; }
      const float b = to_f(beta[(int64_t)n * H + h]);
      const float u = b * (sh_v[tid] - rr);
      sh_u[tid] = u;
      o[tok] = from_f<Tout>(yy + u * kq);
    }
    __syncthreads();

    // 4. S <- Diag(a) S + k u^T, written once.  The shared vectors are
    //    rewritten by the next item only after its first barrier, which every
    //    thread reaches after this update.
    rows_update(s, &sh_al[warp * 16], &sh_kh[warp * 16], *reinterpret_cast<const float4*>(&sh_u[lane * 4]));
#pragma unroll
    for (int i = 0; i < 16; ++i) st_state4(S + (warp * 16 + i) * D + lane * 4, s[i]);
  }
}

}  // namespace kda
