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
// head) items.  Warp w owns value columns [16w, 16w+16) of the state (layout
// below): the column sums r and y finish inside the warp, so after the
// prologue a row of the recurrence needs no block barrier.  While a block
// computes one item a single bulk copy brings the next item's state (64 KiB,
// or 32 KiB in bf16) into shared memory, so the state stream from HBM does not
// wait on the prologue or the reductions; the updated rows are written with
// streaming stores.
#pragma once
#include "kda_common.cuh"
#include "kda_tc.cuh"

namespace kda {

// Register layout of one (sequence, head) state in the decode kernels (256
// threads): warp w owns value columns [16w, 16w+16); lane l holds the four
// columns c0 = 16w + 4 (l & 3) .. c0 + 3 of the sixteen rows 16 rg + i,
// rg = l >> 2, i = 0..15, as s[i].  A warp load of one i touches 8 rows x 64
// contiguous bytes.
struct StateLane {
  int rg;  // row group: rows 16 rg .. 16 rg + 15
  int c0;  // first of the lane's four value columns
};
__device__ __forceinline__ StateLane state_lane() {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  return {l >> 2, 16 * w + 4 * (l & 3)};
}
__device__ __forceinline__ int state_off(StateLane L, int i) { return (16 * L.rg + i) * D + L.c0; }

// Per-row vectors (indexed by key channel = state row) live in shared memory
// with 4 floats of padding after every 16 rows: row r at rpad(r).  The 8 row
// groups of a warp then read their 16-byte vectors from 8 distinct bank quads.
constexpr int ROWV = D + 4 * (D / 16);
__device__ __forceinline__ int rpad(int r) { return r + 4 * (r >> 4); }

// The helpers below are the whole state arithmetic of a decode step, shared
// by the single-token and the multi-token kernels so that all of them round
// identically.  Packed f32x2 instructions do two columns at a time; each
// column is rounded as its scalar fmaf would round it.
//
// The column step of a row: the column sums r = sum_row x_row s_row and
// y = sum_row z_row s_row over all 128 rows (x, z: padded row vectors), then
// u = beta (v - r) and o = y + u kq.  Each lane sums its 16 rows (ascending);
// the 8 row groups of a column quad then combine by recursive halving over
// lanes xor 4, 8, 16: at each stage a lane adds its partner's value of the
// half it keeps, so every sum is formed from the same pairs in the same order
// as a full butterfly would form it, with 7 shuffles instead of 24.  This
// leaves each of the quad's 8 sums (r and y of its 4 columns) in one lane: the
// lane of row group rg holds sum number 4 (rg & 1) + 2 ((rg >> 1) & 1) +
// (rg >> 2), an r for even rg and a y for odd rg.  u is formed where r is and
// gathered into every lane of the quad; o is formed where y is.
struct ColStep {
  float4 u;  // u of the lane's 4 columns (every lane)
  float o;   // o of column c0 + oc (lanes of odd row groups)
  int oc;
};
__device__ __forceinline__ ColStep col_step(const float4 (&s)[16], const float* x, const float* z, int rg,
                                            float beta, const float* vcols, float kq) {
  float2 r0 = make_float2(0.f, 0.f), r1 = r0, y0 = r0, y1 = r0;
#pragma unroll
  for (int i4 = 0; i4 < 4; ++i4) {
    const float4 x4 = *reinterpret_cast<const float4*>(x + 20 * rg + 4 * i4);  // rows 16 rg + 4 i4 ..
    const float4 z4 = *reinterpret_cast<const float4*>(z + 20 * rg + 4 * i4);
    const float xs[4] = {x4.x, x4.y, x4.z, x4.w}, zs[4] = {z4.x, z4.y, z4.z, z4.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 si = s[4 * i4 + j];
      r0 = fma2(lo2(si), dup2(xs[j]), r0); r1 = fma2(hi2(si), dup2(xs[j]), r1);
      y0 = fma2(lo2(si), dup2(zs[j]), y0); y1 = fma2(hi2(si), dup2(zs[j]), y1);
    }
  }
  float v[8] = {r0.x, r0.y, r1.x, r1.y, y0.x, y0.y, y1.x, y1.y};
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int st = 0; st < 3; ++st) {
    const int m = 4 << st, n = 4 >> st;  // partner lane xor m; values kept after this stage
    const bool up = (lane & m) != 0;     // keeps the upper half
#pragma unroll
    for (int i = 0; i < n; ++i) {
      const float send = up ? v[i] : v[i + n];
      const float keep = up ? v[i + n] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
    }
  }
  const int idx = 4 * (rg & 1) + 2 * ((rg >> 1) & 1) + (rg >> 2);  // the sum this lane holds
  const float um = beta * (vcols[idx & 3] - v[0]);                 // meaningful for even rg
  // u of column c0 + j sits in the lane of row group 0, 4, 2, 6 for j = 0 .. 3
  const int q = lane & 3;
  ColStep cs;
  cs.u = make_float4(__shfl_sync(0xffffffffu, um, q), __shfl_sync(0xffffffffu, um, q + 16),
                     __shfl_sync(0xffffffffu, um, q + 8), __shfl_sync(0xffffffffu, um, q + 24));
  cs.oc = idx & 3;
  const float uo = cs.oc == 0 ? cs.u.x : (cs.oc == 1 ? cs.u.y : (cs.oc == 2 ? cs.u.z : cs.u.w));
  cs.o = v[0] + uo * kq;
  return cs;
}

// s_row <- a_row s_row + kh_row u (the delta-rule update Diag(a) S + k u^T;
// a, kh: padded row vectors; u4: the lane's 4 columns of u).
__device__ __forceinline__ void rows_update(float4 (&s)[16], const float* a, const float* kh, int rg, float4 u4) {
  const float2 u0 = lo2(u4), u1 = hi2(u4);
#pragma unroll
  for (int i4 = 0; i4 < 4; ++i4) {
    const float4 a4 = *reinterpret_cast<const float4*>(a + 20 * rg + 4 * i4);
    const float4 k4 = *reinterpret_cast<const float4*>(kh + 20 * rg + 4 * i4);
    const float as[4] = {a4.x, a4.y, a4.z, a4.w}, ks[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float4& si = s[4 * i4 + j];
      si = cat2(fma2(dup2(as[j]), lo2(si), mul2(dup2(ks[j]), u0)),
                fma2(dup2(as[j]), hi2(si), mul2(dup2(ks[j]), u1)));
    }
  }
}

// one output element
template <typename T> __device__ __forceinline__ void store1(T* p, float v) { *p = from_f<T>(v); }

// Shared-memory image of a prefetched state: its 8 row groups (16 rows each,
// StateLane::rg) as separate pieces.  One load instruction of a warp reads the
// same 4 columns of 8 rows 16 apart; with a 256-byte row pitch (bf16) those
// rows all start on the same bank, so a bf16 state's pieces are placed 32
// bytes further apart than their size, which spreads the 8 rows over all 32
// banks.  An fp32 state is kept as one unpadded piece.
template <typename Ts>
struct StateImage {
  static constexpr uint32_t kGroup = 16 * D * sizeof(Ts);  // bytes of one row group
  static constexpr uint32_t kPitch = kGroup + (sizeof(Ts) == 2 ? 32 : 0);
  static constexpr uint32_t kBytes = 8 * kPitch;           // shared memory taken
  static constexpr uint32_t kCopied = 8 * kGroup;          // bytes a copy transfers
  // one thread: the state at `src` into the image at `dst` (16-byte aligned),
  // completing on `bar`
  static __device__ __forceinline__ void copy(uint8_t* dst, const Ts* src, uint64_t* bar) {
    if constexpr (kPitch == kGroup) {
      tc::bulk_g2s(dst, src, kCopied, bar);
    } else {
#pragma unroll
      for (int r = 0; r < 8; ++r) tc::bulk_g2s(dst + r * kPitch, src + r * 16 * D, kGroup, bar);
    }
  }
  // row 16 rg + i, columns c0 .. c0 + 3 of the lane
  static __device__ __forceinline__ float4 load(const uint8_t* img, StateLane L, int i) {
    return ld_state4_shared(reinterpret_cast<const Ts*>(img + L.rg * kPitch) + i * D + L.c0);
  }
};

// The prefetch of decode_kernel.  With a bf16 state (INPUTS = true) the inputs
// of the next item's prologue (the q, k, v, g rows, the nine conv-cache rows,
// the three tap rows) arrive by bulk copies on the same mbarrier as its state,
// into one of two input slots (the prologue reads its slot after the next
// item's copies were issued): with half the state bytes the prologue's global
// loads would otherwise be exposed.  With an fp32 state the state stream
// alone keeps HBM busy and the prologue reads global memory.
template <typename Tin, typename Ts, bool INPUTS>
struct DecodePrefetch {
  static constexpr uint32_t kState = StateImage<Ts>::kBytes;  // the state image, then the input slots
  static constexpr uint32_t kRow = D * sizeof(Tin);
  static constexpr uint32_t kTaps = D * 4 * sizeof(float);   // one tensor's taps
  static constexpr uint32_t kSlot = INPUTS ? (13 * kRow + 3 * kTaps + 127) & ~127u : 0;
  __host__ __device__ static constexpr uint32_t bytes() { return kState + 2 * kSlot; }

  uint8_t* base;
  const Ts* state;
  const Tin *q, *k, *v, *g, *cache;
  const float* conv_w;
  uint64_t* bar;
  int items, H;
  uint32_t par, slot;

  // slot layout: rows 0..3 = q, k, v, g; rows 4 + 3 x + t = cache tensor x,
  // time t; then the taps of q, k, v ([D][4] each)
  __device__ __forceinline__ const Tin* row(uint32_t sl, int r) const {
    return reinterpret_cast<const Tin*>(base + kState + sl * kSlot + r * kRow);
  }
  __device__ __forceinline__ const float* taps(uint32_t sl, int x) const {
    return reinterpret_cast<const float*>(base + kState + sl * kSlot + 13 * kRow + x * kTaps);
  }
  __device__ __forceinline__ void issue(int item, uint32_t sl) {  // one thread
    const int64_t n = item / H, h = item % H, HD = (int64_t)H * D;
    uint8_t* dst = base + kState + sl * kSlot;
    tc::fence_async_smem();  // the buffers' previous contents were read by every thread
    constexpr uint32_t kCopied = StateImage<Ts>::kCopied;
    tc::bar_expect_tx(bar, INPUTS ? kCopied + 13 * kRow + 3 * kTaps : kCopied);
    StateImage<Ts>::copy(base, state + (int64_t)item * D * D, bar);
    if (!INPUTS) return;
    const Tin* in[4] = {q, k, v, g};
#pragma unroll
    for (int r = 0; r < 4; ++r) tc::bulk_g2s(dst + r * kRow, in[r] + n * HD + h * D, kRow, bar);
#pragma unroll
    for (int r = 0; r < 9; ++r) tc::bulk_g2s(dst + (4 + r) * kRow, cache + (n * 9 + r) * HD + h * D, kRow, bar);
#pragma unroll
    for (int x = 0; x < 3; ++x)
      tc::bulk_g2s(dst + 13 * kRow + x * kTaps, conv_w + (x * HD + h * D) * 4, kTaps, bar);
  }
  __device__ __forceinline__ void init(const Ts* st, const Tin* q_, const Tin* k_, const Tin* v_, const Tin* g_,
                                       const Tin* cache_, const float* w_, int n_items, int H_) {
    extern __shared__ __align__(128) uint8_t dsm[];
    __shared__ uint64_t bar_pf;
    base = dsm;
    state = st; q = q_; k = k_; v = v_; g = g_; cache = cache_; conv_w = w_;
    bar = &bar_pf;
    items = n_items;
    H = H_;
    par = 0;
    slot = 0;
    if (threadIdx.x == 0) {
      tc::bar_init(bar, 1);
      tc::bar_init_fence();
      if ((int)blockIdx.x < items) issue(blockIdx.x, 0);
    }
    __syncthreads();
  }
  // Called by all threads at the top of each item (init() once before the
  // item loop; both contain a barrier).  This item's state into registers
  // (the StateLane layout); *cur = the slot holding its inputs; then the next
  // item's copies are issued into the other slot.  Returns false for the
  // whole block if the copies did not land in time (recorded as
  // KDA_ERR_TIMEOUT; the copies in flight are awaited once more before the
  // block gives up, so nothing lands in shared memory after it exits).
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

template <typename Tin, typename Tout, int ACT, typename Ts>
__global__ void __launch_bounds__(256, 2)
decode_kernel(Ts* __restrict__ state, Tin* __restrict__ cache, const Tin* __restrict__ q,
              const Tin* __restrict__ k, const Tin* __restrict__ v, const Tin* __restrict__ g,
              const Tin* __restrict__ beta, const float* __restrict__ conv_w, int N, int H,
              Tout* __restrict__ o) {
  // row vectors (padded, see rpad) and the value column vector
  __shared__ __align__(16) float sh_kh[ROWV], sh_ka[ROWV], sh_qa[ROWV], sh_al[ROWV], sh_v[D];
  __shared__ float sh_red[4][3];
  constexpr bool kInputs = sizeof(Ts) == 2;
  DecodePrefetch<Tin, Ts, kInputs> pf;
  pf.init(state, q, k, v, g, cache, conv_w, N * H, H);  // item = n * H + h: consecutive items are adjacent

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const StateLane L = state_lane();
  const int64_t HD = (int64_t)H * D;
  // beta of the item being computed, loaded one item ahead
  float b_cur = kInputs && (int)blockIdx.x < pf.items ? to_f(beta[blockIdx.x]) : 0.f;
  for (int item = blockIdx.x; item < pf.items; item += gridDim.x) {
    const int n = item / H, h = item % H;
    Ts* S = state + (int64_t)item * D * D;

    // 1. this item's state and inputs, prefetched into shared memory; the
    //    state into registers, then the buffers take the next item's
    float4 s[16];
    uint32_t sl;
    if (!pf.take(item, s, &sl)) return;
    float b_next = 0.f;
    if constexpr (kInputs) b_next = item + (int)gridDim.x < pf.items ? to_f(beta[item + gridDim.x]) : 0.f;

    // 2. prologue: threads 0..127 -> q and k of channel c; 128..255 -> v and g.
    //    With a bf16 state the inputs come from the prefetched slot; with an
    //    fp32 state straight from global memory (loads issued together)
    const int c = tid & (D - 1);
    const int64_t ch = (int64_t)h * D + c;
    Tin* cb = cache + (int64_t)n * 9 * HD + ch; // [3 x][3 t] stride HD
    float yq = 0.f, yk = 0.f;
    if constexpr (kInputs) {
      // input r (0..3: q, k, v, g of the token; 4 + 3 x + t: cache tensor x,
      // time t) and the taps of tensor x, for channel c
      auto input = [&](int r) -> Tin { return pf.row(sl, r)[c]; };
      auto taps = [&](int x) -> float4 { return *reinterpret_cast<const float4*>(pf.taps(sl, x) + 4 * c); };
      if (tid < D) {
        const float4 wq = taps(0), wk = taps(1);
        const Tin hq0 = input(4), hq1 = input(5), hq2 = input(6);
        const Tin hk0 = input(7), hk1 = input(8), hk2 = input(9);
        const Tin xq = input(0), xk = input(1);
        yq = conv4(wq, to_f(hq0), to_f(hq1), to_f(hq2), to_f(xq));
        yk = conv4(wk, to_f(hk0), to_f(hk1), to_f(hk2), to_f(xk));
        if (ACT == KDA_CONV_SILU) { yq = silu(yq); yk = silu(yk); }
        // the shifted cache (its old contents were read from the prefetched copy)
        cb[0 * HD] = hq1; cb[1 * HD] = hq2; cb[2 * HD] = xq;
        cb[3 * HD] = hk1; cb[4 * HD] = hk2; cb[5 * HD] = xk;
        float nq = warp_sum(yq * yq), nk = warp_sum(yk * yk), qk = warp_sum(yq * yk);
        if (lane == 0) { sh_red[warp][0] = nq; sh_red[warp][1] = nk; sh_red[warp][2] = qk; }
      } else {
        const float4 wv = taps(2);
        const Tin hv0 = input(10), hv1 = input(11), hv2 = input(12);
        const Tin xv = input(2);
        float yv = conv4(wv, to_f(hv0), to_f(hv1), to_f(hv2), to_f(xv));
        if (ACT == KDA_CONV_SILU) yv = silu(yv);
        cb[6 * HD] = hv1; cb[7 * HD] = hv2; cb[8 * HD] = xv;
        sh_v[c] = yv;
        sh_al[rpad(c)] = __expf(fmaxf(to_f(input(3)), LOG_DECAY_FLOOR));
      }
    } else {
      const int64_t tok = (int64_t)n * HD + ch;  // [N, H, D] index
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
        sh_al[rpad(c)] = __expf(fmaxf(to_f(g[tok]), LOG_DECAY_FLOOR));
      }
    }
    __syncthreads();
    const float nq = sh_red[0][0] + sh_red[1][0] + sh_red[2][0] + sh_red[3][0];
    const float nk = sh_red[0][1] + sh_red[1][1] + sh_red[2][1] + sh_red[3][1];
    const float qk = sh_red[0][2] + sh_red[1][2] + sh_red[2][2] + sh_red[3][2];
    const float rq = rsqrtf(nq + NORM_EPS), rk = rsqrtf(nk + NORM_EPS);
    const float kq = qk * rq * rk;
    if (tid < D) {
      const float a = sh_al[rpad(c)];
      const float kh = yk * rk;
      sh_kh[rpad(c)] = kh;
      sh_ka[rpad(c)] = a * kh;
      sh_qa[rpad(c)] = a * yq * rq;
    }
    __syncthreads();

    // 3. column sums r = S^T (a k), y = S^T (a q) within each warp; u and o for
    //    the lane's 4 columns (lanes of row group 0 write o)
    const float b = kInputs ? b_cur : to_f(beta[(int64_t)n * H + h]);
    const ColStep cs = col_step(s, sh_ka, sh_qa, L.rg, b, &sh_v[L.c0], kq);
    if (L.rg & 1) store1(o + (int64_t)n * HD + (int64_t)h * D + L.c0 + cs.oc, cs.o);
    b_cur = b_next;

    // 4. S <- Diag(a) S + k u^T, written once.  The shared vectors are
    //    rewritten by the next item only after its first barrier, which every
    //    thread reaches after this update.
    rows_update(s, sh_al, sh_kh, L.rg, cs.u);
#pragma unroll
    for (int i = 0; i < 16; ++i) st_state4(S + state_off(L, i), s[i]);
  }
}

}  // namespace kda
