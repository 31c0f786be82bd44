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
// is read once into registers (the StateLane layout of kda_decode.cuh: each
// warp owns 16 value columns) and updated there row by row without block
// barriers; it is not written back.  Per row t
// it writes o_t and the row's update (k_hat_t, u_t, alpha_t) to `deltas`.
// decode_commit_kernel: per (sequence, head), S <- Diag(alpha_t) S + k_hat_t u_t^T
// for the first n_accept rows (one read and one write of S), and the conv
// cache becomes the last three raw tokens of [cache, accepted rows].
#pragma once
#include <type_traits>

#include "kda_common.cuh"
#include "kda_decode.cuh"

namespace kda {

constexpr int MAX_VERIFY_ROWS = KDA_MAX_VERIFY_ROWS;

// COMMIT = false: kda_decode_verify.  COMMIT = true: kda_decode_commit_verify,
// which first keeps the first n_accept rows of the previous step (its raw rows
// pq/pk/pv, PR of them per sequence, and its deltas) exactly as
// decode_commit_kernel would, stores the state and the conv cache, and then
// verifies the new rows from them: one pass over the state per step.
template <typename Tin, typename Tout, int ACT, typename Ts, bool COMMIT>
__global__ void __launch_bounds__(256, 2)
decode_verify_kernel(Ts* __restrict__ state, Tin* __restrict__ cache,
                     const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                     const Tin* __restrict__ g, const Tin* __restrict__ beta, const float* __restrict__ conv_w,
                     int R, int H, Tout* __restrict__ o, float* __restrict__ deltas,
                     const Tin* __restrict__ pq, const Tin* __restrict__ pk, const Tin* __restrict__ pv,
                     const float* __restrict__ pdeltas, const int32_t* __restrict__ pn_accept, int PR) {
  // per row: k_hat, alpha * k_hat, alpha * q_hat, alpha, conv(v); the row
  // prologues do not depend on the state, so all rows are prepared first
  // row vectors padded (rpad), the value column vectors plain
  __shared__ __align__(16) float sh_kh[MAX_VERIFY_ROWS][ROWV], sh_ka[MAX_VERIFY_ROWS][ROWV],
      sh_qa[MAX_VERIFY_ROWS][ROWV], sh_al[MAX_VERIFY_ROWS][ROWV], sh_v[MAX_VERIFY_ROWS][D];
  __shared__ float sh_red[MAX_VERIFY_ROWS][4][3], sh_kq[MAX_VERIFY_ROWS], sh_beta[MAX_VERIFY_ROWS];
  // the previous step's deltas, [row][k_hat, u, alpha] (commit only): k_hat and
  // alpha padded row vectors, u a column vector
  __shared__ __align__(16) float sh_prev[COMMIT ? 3 * MAX_VERIFY_ROWS : 1][ROWV];
  // one block per (sequence, head): the rows' compute dominates, and two
  // resident blocks per SM overlap one block's state load with the other's rows
  const int h = blockIdx.x, n = blockIdx.y, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const StateLane L = state_lane();
  const int64_t HD = (int64_t)H * D;
  Ts* S = state + ((int64_t)n * H + h) * D * D;
  float4 s[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) s[i] = ld_state4(S + state_off(L, i));
  int na = 0;  // rows of the previous step kept
  if (COMMIT) {
    na = pn_accept[n];
    if (na < 0 || na > PR) {  // out of range: record it and keep what can be kept
      if (tid == 0 && h == 0) set_status(KDA_ERR_INVALID_ARG);
      na = na < 0 ? 0 : PR;
    }
    const float* pdl = pdeltas + ((int64_t)n * H + h) * PR * 3 * D;
    for (int e = tid; e < na * 3 * D; e += 256) {
      const int row = e / D, cc = e % D;  // row = 3 t + part
      sh_prev[row][row % 3 == 1 ? cc : rpad(cc)] = pdl[e];
    }
  }

  // 1. prologues of all rows: threads 0..127 q and k of channel c, threads
  //    128..255 v and the gate (conv history = the cache, advanced by the
  //    kept rows of the previous step, then earlier rows)
  const int c = tid & (D - 1);
  const int64_t ch = (int64_t)h * D + c;
  float* dl = deltas + ((int64_t)n * H + h) * R * 3 * D;  // [R][3 (k_hat, u, alpha)][D]
  Tin* cb = cache + (int64_t)n * 9 * HD + ch;  // [3 x][3 t] stride HD
  // conv history of tensor x for channel c: the last three raw tokens of
  // [cache, kept rows of the previous step], written back as the committed
  // cache (this thread alone reads and writes these three entries)
  auto history = [&](int x, const Tin* prev, float (&hh)[3]) {
    Tin nv[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int idx = na + j;  // position in [cache rows 0..2, kept rows]
      nv[j] = idx < 3 ? cb[(3 * x + idx) * HD] : prev[(((int64_t)n * PR + (idx - 3)) * H + h) * D + c];
    }
    if (COMMIT && na > 0) {
#pragma unroll
      for (int j = 0; j < 3; ++j) cb[(3 * x + j) * HD] = nv[j];
    }
#pragma unroll
    for (int j = 0; j < 3; ++j) hh[j] = to_f(nv[j]);
  };
  float yq[MAX_VERIFY_ROWS], yk[MAX_VERIFY_ROWS];
  // raw inputs of all rows are loaded before any is used, so that their
  // global-memory latencies overlap instead of adding up row by row
  if (tid < D) {
    float xqs[MAX_VERIFY_ROWS], xks[MAX_VERIFY_ROWS];
#pragma unroll
    for (int t = 0; t < MAX_VERIFY_ROWS; ++t) {
      const int64_t tok = (((int64_t)n * R + t) * H + h) * D + c;  // [N, R, H, D]
      xqs[t] = t < R ? to_f(q[tok]) : 0.f;
      xks[t] = t < R ? to_f(k[tok]) : 0.f;
    }
    const float4 wq = load4(conv_w + (0 * HD + ch) * 4), wk = load4(conv_w + (1 * HD + ch) * 4);
    float hq[3], hk[3];
    history(0, pq, hq);
    history(1, pk, hk);
#pragma unroll
    for (int t = 0; t < MAX_VERIFY_ROWS; ++t) {
      if (t < R) {
        const float xq = xqs[t], xk = xks[t];
        float a = conv4(wq, hq[0], hq[1], hq[2], xq);
        float b = conv4(wk, hk[0], hk[1], hk[2], xk);
        if (ACT == KDA_CONV_SILU) { a = silu(a); b = silu(b); }
        hq[0] = hq[1]; hq[1] = hq[2]; hq[2] = xq;
        hk[0] = hk[1]; hk[1] = hk[2]; hk[2] = xk;
        yq[t] = a; yk[t] = b;
        const float nq = warp_sum(a * a), nk = warp_sum(b * b), qk = warp_sum(a * b);
        if (lane == 0) { sh_red[t][warp][0] = nq; sh_red[t][warp][1] = nk; sh_red[t][warp][2] = qk; }
      }
    }
  } else {
    float xvs[MAX_VERIFY_ROWS], xgs[MAX_VERIFY_ROWS];
#pragma unroll
    for (int t = 0; t < MAX_VERIFY_ROWS; ++t) {
      const int64_t tok = (((int64_t)n * R + t) * H + h) * D + c;
      xvs[t] = t < R ? to_f(v[tok]) : 0.f;
      xgs[t] = t < R ? to_f(g[tok]) : 0.f;
    }
    if (c < R) sh_beta[c] = to_f(beta[((int64_t)n * R + c) * H + h]);
    const float4 wv = load4(conv_w + (2 * HD + ch) * 4);
    float hv[3];
    history(2, pv, hv);
#pragma unroll
    for (int t = 0; t < MAX_VERIFY_ROWS; ++t) {
      if (t < R) {
        const float xv = xvs[t];
        float yv = conv4(wv, hv[0], hv[1], hv[2], xv);
        if (ACT == KDA_CONV_SILU) yv = silu(yv);
        hv[0] = hv[1]; hv[1] = hv[2]; hv[2] = xv;
        sh_v[t][c] = yv;
        sh_al[t][rpad(c)] = __expf(fmaxf(xgs[t], LOG_DECAY_FLOOR));
      }
    }
  }
  __syncthreads();
  if (tid < D) {
#pragma unroll
    for (int t = 0; t < MAX_VERIFY_ROWS; ++t) {
      if (t < R) {
        const float nq = sh_red[t][0][0] + sh_red[t][1][0] + sh_red[t][2][0] + sh_red[t][3][0];
        const float nk = sh_red[t][0][1] + sh_red[t][1][1] + sh_red[t][2][1] + sh_red[t][3][1];
        const float qk = sh_red[t][0][2] + sh_red[t][1][2] + sh_red[t][2][2] + sh_red[t][3][2];
        const float rq = rsqrtf(nq + NORM_EPS), rk = rsqrtf(nk + NORM_EPS);
        const float a = sh_al[t][rpad(c)];
        const float kh = yk[t] * rk;
        sh_kh[t][rpad(c)] = kh;
        sh_ka[t][rpad(c)] = a * kh;
        sh_qa[t][rpad(c)] = a * yq[t] * rq;
        if (c == 0) sh_kq[t] = qk * rq * rk;
        dl[(t * 3 + 0) * D + c] = kh;  // the parts of the row's update that do
        dl[(t * 3 + 2) * D + c] = a;   // not depend on the state
      }
    }
  }
  __syncthreads();

  // the kept rows of the previous step, as decode_commit_kernel applies them;
  // the committed state is stored, and verification starts from its stored
  // value (the commit's deltas reached shared memory before the barriers above)
  if (COMMIT && na > 0) {
    for (int t = 0; t < na; ++t) {
      rows_update(s, sh_prev[3 * t + 2], sh_prev[3 * t], L.rg,
                  *reinterpret_cast<const float4*>(&sh_prev[3 * t + 1][L.c0]));
      if (t + 1 < na) {
#pragma unroll
        for (int i = 0; i < 16; ++i) s[i] = as_stored4<Ts>(s[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      st_state4(S + state_off(L, i), s[i]);
      s[i] = as_stored4<Ts>(s[i]);
    }
  }

  // 2. the rows in turn against the state held in registers.  Each warp owns
  //    16 value columns, so the column sums, u, o and the update of a row need
  //    no block barrier: the row vectors were all written before the barrier
  //    above, and each warp only touches its own columns afterwards.
  for (int t = 0; t < R; ++t) {
    const ColStep cs = col_step(s, sh_ka[t], sh_qa[t], L.rg, sh_beta[t], &sh_v[t][L.c0], sh_kq[t]);
    if (L.rg & 1) store1(o + (((int64_t)n * R + t) * H + h) * D + L.c0 + cs.oc, cs.o);
    if (L.rg == 0) *reinterpret_cast<float4*>(dl + (t * 3 + 1) * D + L.c0) = cs.u;
    if (t + 1 < R) {
      rows_update(s, sh_al[t], sh_kh[t], L.rg, cs.u);
      // the next row starts from the state as a single step would have stored it
#pragma unroll
      for (int i = 0; i < 16; ++i) s[i] = as_stored4<Ts>(s[i]);
    }
  }
}

// The prefetch of decode_commit_kernel: the next item's state (StateImage) and
// its R rows of deltas ([R][3][D] fp32, one bulk copy) arrive on one mbarrier,
// the deltas into one of two slots, so that neither waits for global memory
// while an item is committed.  All R rows are copied, whatever the item keeps.
template <typename Ts>
struct CommitPrefetch {
  static constexpr uint32_t kState = StateImage<Ts>::kBytes;
  __host__ __device__ static constexpr uint32_t slot_bytes(int R) { return (uint32_t)R * 3 * D * sizeof(float); }
  __host__ __device__ static constexpr uint32_t bytes(int R) { return kState + 2 * slot_bytes(R); }

  uint8_t* base;
  const Ts* state;
  const float* deltas;
  uint64_t* bar;
  int items, R;
  uint32_t par, slot;

  __device__ __forceinline__ const float* rows(uint32_t sl) const {
    return reinterpret_cast<const float*>(base + kState + sl * slot_bytes(R));
  }
  __device__ __forceinline__ void issue(int item, uint32_t sl) {  // one thread
    tc::fence_async_smem();  // the buffers' previous contents were read by every thread
    tc::bar_expect_tx(bar, StateImage<Ts>::kCopied + slot_bytes(R));
    StateImage<Ts>::copy(base, state + (int64_t)item * D * D, bar);
    tc::bulk_g2s(base + kState + sl * slot_bytes(R), deltas + (int64_t)item * R * 3 * D, slot_bytes(R), bar);
  }
  __device__ __forceinline__ void init(const Ts* st, const float* dl, int n_items, int R_) {
    extern __shared__ __align__(128) uint8_t dsm[];
    __shared__ uint64_t bar_cp;
    base = dsm;
    state = st;
    deltas = dl;
    bar = &bar_cp;
    items = n_items;
    R = R_;
    par = 0;
    slot = 0;
    if (threadIdx.x == 0) {
      tc::bar_init(bar, 1);
      tc::bar_init_fence();
      if ((int)blockIdx.x < items) issue(blockIdx.x, 0);
    }
    __syncthreads();
  }
  // This item's state into registers; *cur = the slot holding its deltas; then
  // the next item's copies are issued into the other slot.  Bounded as
  // DecodePrefetch::take.
  __device__ __forceinline__ bool take(int item, float4 (&s)[16], uint32_t* cur) {
    const StateLane L = state_lane();
    if (!__syncthreads_and(tc::bar_wait(bar, par))) {
      if (threadIdx.x == 0) tc::bar_wait(bar, par);
      return false;
    }
    par ^= 1;
#pragma unroll
    for (int i = 0; i < 16; ++i) s[i] = StateImage<Ts>::load(base, L, i);
    *cur = slot;
    slot ^= 1;
    __syncthreads();
    if (threadIdx.x == 0 && item + (int)gridDim.x < items) issue(item + gridDim.x, slot);
    return true;
  }
};

template <typename Tin, typename Ts>
__global__ void __launch_bounds__(256, 2)
decode_commit_kernel(Ts* __restrict__ state, Tin* __restrict__ cache, const Tin* __restrict__ q,
                     const Tin* __restrict__ k, const Tin* __restrict__ v, const float* __restrict__ deltas,
                     const int32_t* __restrict__ n_accept, int N, int R, int H) {
  // row vectors k_hat, alpha padded (rpad); u a column vector
  __shared__ __align__(16) float sh_kh[MAX_VERIFY_ROWS][ROWV], sh_u[MAX_VERIFY_ROWS][D],
      sh_al[MAX_VERIFY_ROWS][ROWV];
  // new conv-cache rows [3][3 x 128] (each thread its own channel pairs)
  __shared__ __align__(16) uint8_t sh_cc_raw[3 * 3 * D * sizeof(Tin)];
  auto sh_cc = reinterpret_cast<Tin(*)[3 * D]>(sh_cc_raw);
  CommitPrefetch<Ts> pf;
  pf.init(state, deltas, N * H, R);
  const int tid = threadIdx.x;
  const StateLane L = state_lane();
  const int64_t HD = (int64_t)H * D;
  // n_accept of the item being committed, loaded one item ahead
  int na_next = (int)blockIdx.x < pf.items ? n_accept[blockIdx.x / H] : 0;

  // persistent loop over the (sequence, head) items
  for (int item = blockIdx.x; item < pf.items; item += gridDim.x) {
  const int n = item / H, h = item % H;
  Ts* S = state + (int64_t)item * D * D;
  float4 s[16];
  uint32_t sl;
  if (!pf.take(item, s, &sl)) return;
  int na = na_next;
  na_next = item + (int)gridDim.x < pf.items ? n_accept[(item + gridDim.x) / H] : 0;
  if (na < 0 || na > R) {  // out of range: record it and keep what can be kept
    if (tid == 0 && h == 0) set_status(KDA_ERR_INVALID_ARG);
    na = na < 0 ? 0 : R;
  }
  if (na == 0) continue;  // nothing accepted: state and cache stay as they are
  // conv cache: the last three raw tokens of [cache (3 rows), accepted rows].
  // Thread tid < 192 takes the channel pair (x, cc .. cc + 1) of the 3 x 128
  // (tensor, channel) columns: its three values are copied asynchronously into
  // its own shared slots now and stored back after the state update, so the
  // loads' latency is hidden and no registers are held across the update.
  const bool cache_thread = tid < 3 * D / 2;
  const int cx = tid / (D / 2), ccp = 2 * (tid % (D / 2));
  if (cache_thread) {
    const Tin* cb = cache + ((int64_t)n * 9 + 3 * cx) * HD + (int64_t)h * D + ccp;
    const Tin* src = cx == 0 ? q : (cx == 1 ? k : v);
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int idx = na + j;  // position in [cache rows 0..2, accepted rows]
      const Tin* from = idx < 3 ? cb + idx * HD : src + (((int64_t)n * R + (idx - 3)) * H + h) * D + ccp;
      tc::async_copy<2 * sizeof(Tin)>(&sh_cc[j][cx * D + ccp], from);
    }
    tc::async_commit();
  }
  // the kept rows' deltas from the prefetched slot into the padded row vectors
  const float* dl = pf.rows(sl);
  for (int e = tid; e < na * D; e += 256) {
    const int t = e / D, cc = e % D;
    sh_kh[t][rpad(cc)] = dl[(t * 3 + 0) * D + cc];
    sh_u[t][cc] = dl[(t * 3 + 1) * D + cc];
    sh_al[t][rpad(cc)] = dl[(t * 3 + 2) * D + cc];
  }
  __syncthreads();
  for (int t = 0; t < na; ++t) {
    rows_update(s, sh_al[t], sh_kh[t], L.rg, *reinterpret_cast<const float4*>(&sh_u[t][L.c0]));
    if (t + 1 < na) {  // every kept row stores its state (the last one below)
#pragma unroll
      for (int i = 0; i < 16; ++i) s[i] = as_stored4<Ts>(s[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) st_state4(S + state_off(L, i), s[i]);
  if (cache_thread) {  // the thread's own copies: no barrier needed
    tc::async_wait_all();
    Tin* cb = cache + ((int64_t)(item / H) * 9 + 3 * cx) * HD + (int64_t)(item % H) * D + ccp;
    using Pair = typename std::conditional<sizeof(Tin) == 2, uint32_t, uint2>::type;
#pragma unroll
    for (int j = 0; j < 3; ++j)
      *reinterpret_cast<Pair*>(cb + j * HD) = *reinterpret_cast<const Pair*>(&sh_cc[j][cx * D + ccp]);
  }
  }  // item loop
}

}  // namespace kda
