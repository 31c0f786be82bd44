// Chunk preparation (the state-independent half of the chunked KDA prefill).
//
// Page "GLM-5.3-Flash im Detail", section "Sequenz-Mixing: 34 KDA-Schichten mit
// festem Zustand": prefill evaluates the tokens of a chunk in parallel and hands
// a state from chunk to chunk.  Expanding S_t = Diag(alpha_t) S_{t-1} + k_t u_t^T,
// u_t = beta_t (v_t - (Diag(alpha_t) S_{t-1})^T k_t) over a chunk of C = 64
// tokens with Gamma_i = sum_{s<=i} g'_s (per key channel, g' = max(g, -5)):
//     M_ij = sum_c k_ic k_jc e^{Gamma_ic - Gamma_jc}  (i > j),  P_ij likewise with q_i (j <= i)
//     T    = (I + diag(beta) M)^-1 diag(beta),   W = T (e^Gamma * K)
//     U    = T V - W S,   O = (e^Gamma * Q) S + P U,
//     S   <- diag(e^{Gamma_C}) S + (e^{Gamma_C - Gamma} * K)^T U.
// Everything that does not involve S is computed here, for every chunk of every
// (segment, head) in parallel, and stored as a record of operand tiles already
// in the shared-memory layout the scan kernel's tensor-core instructions read.
//
// Record (REC_BYTES, 1024-aligned), all tiles fp32 values rounded to tf32,
// K-major 128-byte swizzled (kda_tc.cuh):
//   B1  [64 t][192]: columns 0..63 = T strictly below the diagonal, 64..191 = -W
//   QT  [64 t][128]: e^{Gamma_t} * q_hat_t
//   PS  [64 t][ 64]: P strictly below the diagonal
//   KB  [128 k][64]: (e^{Gamma_C - Gamma_t} * k_hat_t)^T
//   SC  fp32 beta[64], P_tt[64] (exact q_hat_t . k_hat_t), e^{Gamma_C}[128]
// The diagonal terms beta_t v_t (of T V) and P_tt u_t (of P U) are applied in
// fp32 by the scan kernel; they carry the largest single-token contributions.
//
// Gram blocks without overflow: tokens are grouped in 16-row blocks with
// midpoint m_J = 16J + 8.  For i in block I and j <= i,
//   e^{G_i - G_j} = [e^{G_i - G_{m_I}}] * [e^{G_{m_I} - G_{m_J}}] * [e^{G_{m_J} - G_j}]
// where the outer factors stay within e^{+-40} (|g'| <= 5, <= 8 steps) and the
// middle one is <= 1, so every operand is finite in fp32/tf32.  The tensor core
// computes, per block row I, D_I[j][i'] = sum_c A_I[j][c] B_I[i'][c] with
// A_I[j] = k_j e^{G_{m_I} - G_j} (j in blocks <= I, 0 elsewhere) and
// B_I = [k_i; q_i] e^{G_i - G_{m_I}} for the 16 i of block I.
//
// Block of 512 threads; thread (c, b) owns key/query channel c of token block
// b (rows 16b..16b+15), so each block's midpoint factors stay in one thread.
// The B operands of all four block rows are one tile written once (KQX); the
// A operands are built per 32-channel slab into two alternating buffers while
// the previous slab's MMAs run.
#pragma once
#include "kda_common.cuh"
#include "kda_tc.cuh"

namespace kda {

constexpr int CH = 64;  // chunk length
constexpr uint32_t REC_B1 = 0;           // 6 slabs x (64 rows x 128 B)
constexpr uint32_t REC_QT = 49152;       // 4 slabs x 8 KB
constexpr uint32_t REC_PS = 81920;       // 2 slabs x 8 KB
constexpr uint32_t REC_KB = 98304;       // 2 slabs x (128 rows x 128 B)
constexpr uint32_t REC_SC = 131072;      // 256 floats
constexpr uint32_t REC_BYTES = 132096;
constexpr uint32_t REC_TILES_A = REC_PS;              // B1 + QT: consumed by the first MMA group
constexpr uint32_t REC_TILES_B = REC_BYTES - REC_PS;  // PS + KB + SC: second MMA group + scalars

// shared memory plan (bytes from a 1024-aligned base); regions are reused
// phase by phase
constexpr int PREP_THREADS = 512;
constexpr uint32_t P_RAW = 0;        // step 0-1: raw q, k, g tiles (3 x RAW_BYTES)
                                     // step 5: Gram A operands, 2 buffers x 32 KB
                                     // step 7: solve temporaries; step 8: T tile (16 KB) + K~^T tile (32 KB)
constexpr uint32_t P_KQX = 65536;    // steps 1-3: conv(q), conv(k) row-major fp32 (2 x 32 KB)
                                     // steps 3-8: KQX tile [128 rows x 128] (rows 32I..32I+15: k e^{G-G_m(I)},
                                     //            rows 32I+16..32I+31: q e^{G-G_m(I)} of block I)
constexpr uint32_t P_G = 131072;     // steps 1-3: Gamma row-major; steps 3-5: KE = k e^{G_m - G} row-major
                                     // steps 6-8: diag(beta) M strict -> X (16 KB), P strict (16 KB)
constexpr uint32_t P_MISC = 163840;  // scalars (12 KB)
constexpr uint32_t PREP_SMEM = 176128 + 1024;

// misc region (floats)
constexpr int MS_BETA = 0, MS_RQ = 64, MS_RK = 128, MS_PD = 192, MS_GMID = 256 /*4x128*/,
              MS_GC = 768 /*128*/, MS_Z = 896 /*6x128*/, MS_EGM = 1664 /*4x128*/, MS_CARRY = 2176 /*4x128*/;
// ends at 2688 floats (10752 B) < 12 KB

__device__ __forceinline__ int zidx(int I, int J) { return (I * (I - 1)) / 2 + J; }  // J < I

// raw input tiles: 3 halo rows + 64 chunk rows of one head (128 bf16 = 256 B)
constexpr int RAW_ROWS = CH + 3;
constexpr uint32_t RAW_BYTES = RAW_ROWS * D * 2;  // 17152

template <int ACT>
__global__ void __launch_bounds__(PREP_THREADS, 1)
chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_g, const __nv_bfloat16* __restrict__ beta,
                  const float* __restrict__ conv_w, const __nv_bfloat16* __restrict__ init_conv,
                  const int32_t* __restrict__ cu, const int2* __restrict__ chunk_tab, int H,
                  int n_items, uint8_t* __restrict__ records) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  float* Yq = (float*)(sm + P_KQX);
  float* Yk = (float*)(sm + P_KQX + 32768);
  uint8_t* kqx = sm + P_KQX;
  float* Gm = (float*)(sm + P_G);  // Gamma, then KE
  float* Ms = (float*)(sm + P_G);
  float* Ps = (float*)(sm + P_G + 16384);
  float* ms = (float*)(sm + P_MISC);
  __shared__ uint64_t bar_ld, bar_g[2], bar_w;
  __shared__ uint32_t tmem_base;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ch = tid & 127, blk = tid >> 7;  // channel, 16-row token block
  const int64_t HD = (int64_t)H * D;
  const __nv_bfloat16* rq_t = reinterpret_cast<const __nv_bfloat16*>(sm + P_RAW);
  const __nv_bfloat16* rk_t = reinterpret_cast<const __nv_bfloat16*>(sm + P_RAW + RAW_BYTES);
  const __nv_bfloat16* rg_t = reinterpret_cast<const __nv_bfloat16*>(sm + P_RAW + 2 * RAW_BYTES);
  // raw q, k, g tiles of work item `it` (rows t0-3 .. t0+63; outside the tensor
  // reads as zero) into the raw region
  auto load_raw = [&](int it) {
    const int2 c = chunk_tab[it / H];
    const int hh = it % H;
    const int y = (int)(cu[c.x] + (int64_t)CH * c.y - 3);
    tc::bar_expect_tx(&bar_ld, 3 * RAW_BYTES);
    tc::tma_load_2d(sm + P_RAW, &tm_q, hh * D, y, &bar_ld);
    tc::tma_load_2d(sm + P_RAW + RAW_BYTES, &tm_k, hh * D, y, &bar_ld);
    tc::tma_load_2d(sm + P_RAW + 2 * RAW_BYTES, &tm_g, hh * D, y, &bar_ld);
  };

  // ---- 0. once per block: TMEM, barriers, first item's tiles ----------------
  if (warp == 0) tc::tmem_alloc(&tmem_base, 256);
  if (tid == 0) {
    tc::bar_init(&bar_ld, 1); tc::bar_init(&bar_g[0], 1); tc::bar_init(&bar_g[1], 1);
    tc::bar_init(&bar_w, 1);
    tc::bar_init_fence();
    if ((int)blockIdx.x < n_items) load_raw(blockIdx.x);
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tm = tmem_base;
  uint32_t par = 0;  // phase parity of the per-item barriers (bar_ld, bar_w)

  // persistent loop over (chunk, head) work items, chunk-major
  for (int item = blockIdx.x; item < n_items; item += gridDim.x, par ^= 1) {
  const int cid = item / H, h = item % H;
  const int2 nc = chunk_tab[cid];
  const int n = nc.x;
  const int64_t seg0 = cu[n], seg1 = cu[n + 1];
  const int64_t t0 = seg0 + (int64_t)CH * nc.y;
  const int L = (int)((seg1 - t0) < CH ? (seg1 - t0) : CH);
  const int64_t chan = (int64_t)h * D + ch;
  uint8_t* rec = records + ((int64_t)cid * H + h) * REC_BYTES;
  if (tid < CH) ms[MS_BETA + tid] = tid < L ? to_f(beta[(t0 + tid) * H + h]) : 0.f;
  const float4 wq = load4(conv_w + (0 * HD + chan) * 4);
  const float4 wk = load4(conv_w + (1 * HD + chan) * 4);
  tc::bar_wait(&bar_ld, par);

  // ---- 1. causal conv of q, k and block-local cumsum of the clamped gate ----
  const int r0 = 16 * blk;
  {
    float hq[3], hk[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int64_t p = t0 + r0 - 3 + j;  // token of tile row r0 + j
      float a = to_f(rq_t[(r0 + j) * D + ch]), b = to_f(rk_t[(r0 + j) * D + ch]);
      if (p < seg0) {  // before the segment: conv history (or zeros)
        a = b = 0.f;
        if (init_conv) {
          const int slot = (int)(3 + (p - seg0));
          a = to_f(init_conv[((int64_t)n * 9 + 0 * 3 + slot) * HD + chan]);
          b = to_f(init_conv[((int64_t)n * 9 + 1 * 3 + slot) * HD + chan]);
        }
      }
      hq[j] = a; hk[j] = b;
    }
    float cum = 0.f;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const int t = r0 + r;
      const float xq = to_f(rq_t[(t + 3) * D + ch]), xk = to_f(rk_t[(t + 3) * D + ch]);
      float yq = conv4(wq, hq[0], hq[1], hq[2], xq);
      float yk = conv4(wk, hk[0], hk[1], hk[2], xk);
      if (ACT == KDA_CONV_SILU) { yq = silu(yq); yk = silu(yk); }
      hq[0] = hq[1]; hq[1] = hq[2]; hq[2] = xq;
      hk[0] = hk[1]; hk[1] = hk[2]; hk[2] = xk;
      const bool valid = t < L;
      cum += valid ? fmaxf(to_f(rg_t[(t + 3) * D + ch]), LOG_DECAY_FLOOR) : 0.f;
      Yq[t * D + ch] = valid ? yq : 0.f;
      Yk[t * D + ch] = valid ? yk : 0.f;
      Gm[t * D + ch] = cum;
    }
    ms[MS_CARRY + blk * D + ch] = cum;  // this block's total
  }
  __syncthreads();

  // ---- 2. L2 norms (warp per 4 rows) -----------------------------------------
#pragma unroll
  for (int t = warp * 4; t < warp * 4 + 4; ++t) {
    const float4 a = *reinterpret_cast<const float4*>(&Yq[t * D + lane * 4]);
    const float4 b = *reinterpret_cast<const float4*>(&Yk[t * D + lane * 4]);
    float nq = a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
    float nk = b.x * b.x + b.y * b.y + b.z * b.z + b.w * b.w;
    float qk = a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
    nq = warp_sum(nq); nk = warp_sum(nk); qk = warp_sum(qk);
    if (lane == 0) {
      const float rq = 1.0f / sqrtf(nq + NORM_EPS), rk = 1.0f / sqrtf(nk + NORM_EPS);
      ms[MS_RQ + t] = rq; ms[MS_RK + t] = rk; ms[MS_PD + t] = qk * rq * rk;
    }
  }
  __syncthreads();

  // ---- 3. normalise; factors about this block's midpoint ---------------------
  // e_t = e^{G_t - G_mid} within [e^-40, e^40]; KX = k e, QX = q e (B operands),
  // KE = k / e (A operand base), QT = e^{G_mid} QX (record)
  float kx[16], qx[16];
  {
    float carry = 0.f;
    for (int b = 0; b < blk; ++b) carry += ms[MS_CARRY + b * D + ch];
    float G[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) G[r] = Gm[(r0 + r) * D + ch] + carry;
    const float gmid = G[8];
    ms[MS_GMID + blk * D + ch] = gmid;
    if (blk == 3) ms[MS_GC + ch] = G[15];
    const float egm = __expf(gmid);
    ms[MS_EGM + blk * D + ch] = egm;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const int t = r0 + r;
      const float e = __expf(G[r] - gmid);
      const float kh = Yk[t * D + ch] * ms[MS_RK + t], qh = Yq[t * D + ch] * ms[MS_RQ + t];
      kx[r] = kh * e;
      qx[r] = qh * e;
      Gm[t * D + ch] = kh / e;  // KE (own element)
      // QT tile image staged in the raw region (its tiles were consumed in step 1)
      *reinterpret_cast<float*>(sm + P_RAW + tc::sw128(t, ch, 64)) = tc::to_tf32(egm * qx[r]);
    }
  }
  tc::fence_async_smem();
  __syncthreads();  // conv(q), conv(k) are read; the KQX tile may overwrite them
  if (tid == 0) {
    tc::bulk_s2g(rec + REC_QT, sm + P_RAW, 32768);
    tc::bulk_commit();
  }
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    *reinterpret_cast<float*>(kqx + tc::sw128(32 * blk + r, ch, 128)) = tc::to_tf32(kx[r]);
    *reinterpret_cast<float*>(kqx + tc::sw128(32 * blk + 16 + r, ch, 128)) = tc::to_tf32(qx[r]);
  }
  __syncthreads();

  // ---- 4. block-to-block factors; record tiles KB and scalars ----------------
  {
    const float gc = ms[MS_GC + ch], gm = ms[MS_GMID + blk * D + ch];
    for (int J = 0; J < blk; ++J) ms[MS_Z + zidx(blk, J) * D + ch] = __expf(gm - ms[MS_GMID + J * D + ch]);
    const float egc = __expf(gc - gm);  // e^{G_C - G_mid}
    float kb[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) kb[r] = tc::to_tf32(egc * Gm[(r0 + r) * D + ch]);
    // row ch of KB, columns r0..r0+15 (half of a 128-byte slab row)
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<float4*>(rec + REC_KB + tc::sw128(ch, r0 + 4 * j, 128)) =
          make_float4(kb[4 * j], kb[4 * j + 1], kb[4 * j + 2], kb[4 * j + 3]);
    float* sc = reinterpret_cast<float*>(rec + REC_SC);
    if (tid < CH) { sc[tid] = ms[MS_BETA + tid]; sc[64 + tid] = ms[MS_PD + tid]; }
    if (blk == 0) sc[128 + ch] = __expf(gc);
  }
  if (tid == 0) tc::bulk_wait_read();  // the QT staging may be overwritten after this
  __syncthreads();

  // ---- 5. gated Gram blocks on the tensor core --------------------------------
  // pass kp covers channels 32kp..32kp+31.  Block rows are paired: pair p
  // stacks A_{2p} (rows 0..63) over A_{2p+1} (rows 64..127) into one M = 128
  // operand against B = KQX rows 64p..64p+63 (= B_{2p} | B_{2p+1}, N = 64); the
  // wanted products are the two diagonal 64 x 32 quadrants.  A_I rows j of
  // blocks J <= I are written (other rows are never read back).
  auto build_a = [&](int kp) {
    uint8_t* buf = sm + P_RAW + (kp & 1) * 32768;
    // (I, j, 4-channel group) with J(j) <= I: 160 rows x 8 groups
    for (int e = tid; e < 160 * 8; e += PREP_THREADS) {
      const int c4 = e & 7, rr = e >> 3;  // rr in [0, 160): I-major rows
      const int I = rr < 16 ? 0 : rr < 48 ? 1 : rr < 96 ? 2 : 3;
      const int j = rr - (I == 0 ? 0 : I == 1 ? 16 : I == 2 ? 48 : 96);
      const int J = j >> 4, c = 32 * kp + 4 * c4;
      float4 v = *reinterpret_cast<const float4*>(&Gm[j * D + c]);
      if (J < I) {
        const float4 z = *reinterpret_cast<const float4*>(&ms[MS_Z + zidx(I, J) * D + c]);
        v.x *= z.x; v.y *= z.y; v.z *= z.z; v.w *= z.w;
      }
      v = make_float4(tc::to_tf32(v.x), tc::to_tf32(v.y), tc::to_tf32(v.z), tc::to_tf32(v.w));
      *reinterpret_cast<float4*>(buf + (I >> 1) * 16384 + tc::sw128((I & 1) * 64 + j, 4 * c4, 128)) = v;
    }
    tc::fence_async_smem();
  };
  auto issue_gram = [&](int kp) {
    tc::fence_after();
    const uint64_t da = tc::desc(tc::smem_u32(sm + P_RAW + (kp & 1) * 32768));
    const uint64_t db = tc::desc(tc::smem_u32(kqx + kp * 16384));
#pragma unroll
    for (int pr = 0; pr < 2; ++pr)
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        tc::mma_ss(tm + 64 * pr, da + ((pr * 16384) >> 4) + tc::desc_step(128, ks),
                   db + ((pr * 64 * 128) >> 4) + tc::desc_step(128, ks), tc::idesc_tf32(128, 64),
                   (kp > 0 || ks > 0) ? 1 : 0);
    tc::commit(&bar_g[kp & 1]);
  };
  build_a(0);
  tc::fence_before();
  __syncthreads();
  if (tid == 0) issue_gram(0);
  build_a(1);
  tc::fence_before();
  __syncthreads();
  if (tid == 0) issue_gram(1);
  tc::bar_wait(&bar_g[0], 0);  // pass 0 done: buffer 0 free
  build_a(2);
  tc::fence_before();
  __syncthreads();
  if (tid == 0) issue_gram(2);
  tc::bar_wait(&bar_g[1], 0);  // pass 1 done: buffer 1 free
  build_a(3);
  tc::fence_before();
  __syncthreads();
  if (tid == 0) issue_gram(3);
  tc::bar_wait(&bar_g[1], 1);  // pass 3 done
  tc::bar_wait(&bar_g[0], 1);  // pass 2 done (each item uses two phases of each barrier)
  tc::fence_after();

  // ---- 6. read the diagonal quadrants (M = 128 layout: row m -> lane m) ------
  {
    const int sub = warp & 3, pr = (warp >> 2) & 1, part = warp >> 3;  // part 0: M columns, 1: P columns
    const int m = 32 * sub + lane;       // accumulator row
    const int I = 2 * pr + (m >> 6);     // block row
    const int j = m & 63;
    float v[16];
    tc::ld16(tm + ((uint32_t)(32 * sub) << 16) + 64 * pr + 32 * (m >> 6) + 16 * part, v);
    tc::ld_wait();
    float* dst = part == 0 ? Ms : Ps;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const int i = 16 * I + r;
      dst[i * CH + j] = i > j ? (part == 0 ? ms[MS_BETA + i] * v[r] : v[r]) : 0.f;  // diag(beta) M / P, strict
    }
  }
  __syncthreads();

  // ---- 7. X = (I + diag(beta) M)^-1, blocked forward substitution -------------
  float* Xd = (float*)(sm + P_RAW);         // [4][16][16] inverses of the diagonal blocks
  float* Yb = (float*)(sm + P_RAW) + 1024;  // [3][16][16]
  if (tid < 64) {
    const int I = tid >> 4, cc = tid & 15;  // column cc of X_II
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float s = (r == cc) ? 1.f : 0.f;
#pragma unroll
      for (int m = 0; m < r; ++m) s -= Ms[(16 * I + r) * CH + 16 * I + m] * x[m];
      x[r] = r < cc ? 0.f : s;
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) Xd[(I * 16 + r) * 16 + cc] = x[r];
  }
  __syncthreads();
#pragma unroll
  for (int I = 1; I < 4; ++I) {
    // Y_IJ = sum_{K=J}^{I-1} L_IK X_KJ  for J < I (X_KJ already in Ms for K < I)
    for (int e = tid; e < I * 256; e += PREP_THREADS) {
      const int J = e >> 8, r = (e >> 4) & 15, cc = e & 15;
      const float* Lrow = Ms + (16 * I + r) * CH;
      float s = 0.f;
#pragma unroll
      for (int m = 0; m < 16; ++m) s += Lrow[16 * J + m] * Xd[(J * 16 + m) * 16 + cc];
      for (int K = J + 1; K < I; ++K) {
#pragma unroll
        for (int m = 0; m < 16; ++m) s += Lrow[16 * K + m] * Ms[(16 * K + m) * CH + 16 * J + cc];
      }
      Yb[(J * 16 + r) * 16 + cc] = s;
    }
    __syncthreads();
    // X_IJ = -X_II Y_IJ, written over L_IJ
    for (int e = tid; e < I * 256; e += PREP_THREADS) {
      const int J = e >> 8, r = (e >> 4) & 15, cc = e & 15;
      float s = 0.f;
#pragma unroll
      for (int m = 0; m < 16; ++m) s += Xd[(I * 16 + r) * 16 + m] * Yb[(J * 16 + m) * 16 + cc];
      Ms[(16 * I + r) * CH + 16 * J + cc] = -s;
    }
    __syncthreads();
  }
  // diagonal blocks into Ms; Ms now holds X (unit lower triangular)
  for (int e = tid; e < 4 * 256; e += PREP_THREADS) {
    const int I = e >> 8, r = (e >> 4) & 15, cc = e & 15;
    Ms[(16 * I + r) * CH + 16 * I + cc] = Xd[(I * 16 + r) * 16 + cc];
  }
  __syncthreads();

  // ---- 8. T = X diag(beta); tiles for W = T K~ and the record's T_s, P_s -----
  uint8_t* tT = sm + P_RAW;          // [64 t][64 t'] tile, 16 KB
  uint8_t* tK = sm + P_RAW + 16384;  // [128 k][64 t'] tile (K~^T), 32 KB
  for (int e = tid; e < CH * 16; e += PREP_THREADS) {  // 4-column groups
    const int t = e >> 4, tp = 4 * (e & 15);
    float4 tv, pv;
    float* tvp = &tv.x;
    float* pvp = &pv.x;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = tp + u;
      tvp[u] = tc::to_tf32(c <= t ? Ms[t * CH + c] * ms[MS_BETA + c] : 0.f);
      pvp[u] = tc::to_tf32(Ps[t * CH + c]);
    }
    *reinterpret_cast<float4*>(tT + tc::sw128(t, tp, 64)) = tv;
    float4 ts = tv;
    float* tsp = &ts.x;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (tp + u >= t) tsp[u] = 0.f;  // strictly lower part only
    *reinterpret_cast<float4*>(rec + REC_B1 + tc::sw128(t, tp, 64)) = ts;
    *reinterpret_cast<float4*>(rec + REC_PS + tc::sw128(t, tp, 64)) = pv;
  }
  {
    // K~^T row ch, columns r0..r0+15: e^{G_t} k_t = e^{G_mid} * KX
    const float egm = ms[MS_EGM + blk * D + ch];
    float kt[16];
#pragma unroll
    for (int r = 0; r < 16; ++r)
      kt[r] = tc::to_tf32(egm * *reinterpret_cast<const float*>(kqx + tc::sw128(32 * blk + r, ch, 128)));
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<float4*>(tK + tc::sw128(ch, r0 + 4 * j, 128)) =
          make_float4(kt[4 * j], kt[4 * j + 1], kt[4 * j + 2], kt[4 * j + 3]);
  }
  tc::fence_async_smem();
  tc::fence_before();
  __syncthreads();
  if (tid == 0) {
    tc::fence_after();
    const uint64_t dt = tc::desc(tc::smem_u32(tT)), dk = tc::desc(tc::smem_u32(tK));
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
      tc::mma_ss(tm + 128, dt + tc::desc_step(64, ks), dk + tc::desc_step(128, ks), tc::idesc_tf32(64, 128),
                 ks > 0 ? 1 : 0);
    tc::commit(&bar_w);
  }
  tc::bar_wait(&bar_w, par);
  tc::fence_after();
  // the raw region (T and K~^T tiles) is free: fetch the next item's tiles
  // while this item finishes
  __syncthreads();
  if (tid == 0 && item + (int)gridDim.x < n_items) load_raw(item + gridDim.x);

  // ---- 9. -W rows into the record (columns 64..191 of B1) --------------------
  {
    const int sub = warp & 3, cb = warp >> 2;  // rows 16sub.., columns 32cb..32cb+31
    const int t = 16 * sub + (lane & 15);
    float w0[16], w1[16];
    tc::ld16(tm + ((uint32_t)(32 * sub) << 16) + 128 + 32 * cb, w0);
    tc::ld16(tm + ((uint32_t)(32 * sub) << 16) + 128 + 32 * cb + 16, w1);
    tc::ld_wait();
    if (lane < 16) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        *reinterpret_cast<float4*>(rec + REC_B1 + tc::sw128(t, 64 + 32 * cb + 4 * j, 64)) =
            make_float4(tc::to_tf32(-w0[4 * j]), tc::to_tf32(-w0[4 * j + 1]), tc::to_tf32(-w0[4 * j + 2]),
                        tc::to_tf32(-w0[4 * j + 3]));
        *reinterpret_cast<float4*>(rec + REC_B1 + tc::sw128(t, 64 + 32 * cb + 16 + 4 * j, 64)) =
            make_float4(tc::to_tf32(-w1[4 * j]), tc::to_tf32(-w1[4 * j + 1]), tc::to_tf32(-w1[4 * j + 2]),
                        tc::to_tf32(-w1[4 * j + 3]));
      }
    }
  }
  tc::fence_before();
  __syncthreads();  // TMEM columns and shared regions are reused by the next item
  tc::fence_after();
  }  // item loop
  if (tid == 0) tc::bulk_wait_all();
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem_base, 256);
}

}  // namespace kda
