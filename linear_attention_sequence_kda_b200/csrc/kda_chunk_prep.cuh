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

// shared memory plan of the prep kernel (bytes from a 1024-aligned base)
constexpr uint32_t PREP_YQ = 0;          // [64][128] f32: conv(q) -> q_hat
constexpr uint32_t PREP_YK = 32768;      // [64][128] f32: conv(k) -> k_hat
constexpr uint32_t PREP_E1 = 65536;      // [64][128] f32: Gamma -> e^{G_mid(J) - G_t}
constexpr uint32_t PREP_XF = 98304;      // [64][128] f32: e^{G_t - G_mid(J)}
constexpr uint32_t PREP_OPA = 131072;    // 4 x 8 KB Gram A (one 32-channel slab); later T tile
constexpr uint32_t PREP_OPB = 163840;    // 4 x 4 KB Gram B; (OPA+16K .. OPB+16K) later K~^T tile
constexpr uint32_t PREP_M = 180224;      // [64][64] f32: diag(beta) M strict -> X
constexpr uint32_t PREP_P = 196608;      // [64][64] f32: P strict
constexpr uint32_t PREP_MISC = 212992;   // scalars and solve temporaries (8 KB)
constexpr uint32_t PREP_SMEM = 221184 + 1024;  // + alignment slack

// misc region layout (floats; 2048 floats = 8 KB)
constexpr int MS_BETA = 0, MS_RQ = 64, MS_RK = 128, MS_PD = 192, MS_Z = 256 /*6x128*/,
              MS_EGM = 1024 /*4x128*/, MS_EGC = 1536 /*4x128*/;
// short-lived temporaries placed in regions that are idle at the time:
// block-midpoint Gammas in the Gram A region (steps 3-3b, before the Gram),
// solve temporaries in the Gram B region (step 7, after the Gram)
constexpr int GT_GMID = 0 /*4x128*/, GT_GC = 512 /*128*/;
constexpr int SV_XD = 0 /*4x16x16*/, SV_YB = 1024 /*3x16x16*/;

__device__ __forceinline__ int zidx(int I, int J) { return (I * (I - 1)) / 2 + J; }  // J < I

// raw input tiles: 3 halo rows + 64 chunk rows of one head (128 bf16 = 256 B)
constexpr int RAW_ROWS = CH + 3;
constexpr uint32_t RAW_BYTES = RAW_ROWS * D * 2;  // 17152

template <int ACT>
__global__ void __launch_bounds__(256, 1)
chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_g, const __nv_bfloat16* __restrict__ beta,
                  const float* __restrict__ conv_w, const __nv_bfloat16* __restrict__ init_conv,
                  const int32_t* __restrict__ cu, const int2* __restrict__ chunk_tab, int H,
                  uint8_t* __restrict__ records) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  float* Yq = (float*)(sm + PREP_YQ);
  float* Yk = (float*)(sm + PREP_YK);
  float* E1 = (float*)(sm + PREP_E1);
  float* Xf = (float*)(sm + PREP_XF);
  uint8_t* opA = sm + PREP_OPA;
  uint8_t* opB = sm + PREP_OPB;
  float* Ms = (float*)(sm + PREP_M);
  float* Ps = (float*)(sm + PREP_P);
  float* ms = (float*)(sm + PREP_MISC);
  float* gt = (float*)(sm + PREP_OPA);  // steps 3-3b only
  float* sv = (float*)(sm + PREP_OPB);  // step 7 only
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ch = tid & 127, half = tid >> 7;
  const int cid = blockIdx.x, h = blockIdx.y;
  const int2 nc = chunk_tab[cid];
  const int n = nc.x;
  const int64_t seg0 = cu[n], seg1 = cu[n + 1];
  const int64_t t0 = seg0 + (int64_t)CH * nc.y;
  const int L = (int)((seg1 - t0) < CH ? (seg1 - t0) : CH);
  const int64_t HD = (int64_t)H * D;
  const int64_t chan = (int64_t)h * D + ch;
  uint8_t* rec = records + ((int64_t)cid * H + h) * REC_BYTES;

  // raw tiles land in the region the Gram operands and M/P use later
  const __nv_bfloat16* rq_t = reinterpret_cast<const __nv_bfloat16*>(sm + PREP_OPA);
  const __nv_bfloat16* rk_t = reinterpret_cast<const __nv_bfloat16*>(sm + PREP_OPA + RAW_BYTES);
  const __nv_bfloat16* rg_t = reinterpret_cast<const __nv_bfloat16*>(sm + PREP_OPA + 2 * RAW_BYTES);
  if (warp == 0) tc::tmem_alloc(&tmem_base, 256);
  if (tid == 0) {
    tc::bar_init(&bar, 1);
    tc::bar_init_fence();
    // rows t0-3 .. t0+63 of head h (rows outside the tensor read as zero)
    tc::bar_expect_tx(&bar, 3 * RAW_BYTES);
    tc::tma_load_2d(sm + PREP_OPA, &tm_q, h * D, (int)(t0 - 3), &bar);
    tc::tma_load_2d(sm + PREP_OPA + RAW_BYTES, &tm_k, h * D, (int)(t0 - 3), &bar);
    tc::tma_load_2d(sm + PREP_OPA + 2 * RAW_BYTES, &tm_g, h * D, (int)(t0 - 3), &bar);
  }
  if (tid < CH) ms[MS_BETA + tid] = tid < L ? to_f(beta[(t0 + tid) * H + h]) : 0.f;
  const float4 wq = load4(conv_w + (0 * HD + chan) * 4);
  const float4 wk = load4(conv_w + (1 * HD + chan) * 4);
  __syncthreads();
  uint32_t phase = 0;
  tc::bar_wait(&bar, phase);
  phase ^= 1;

  // ---- 1. causal conv of q and k, clamped log-decay, half-local cumsum ------
  {
    const int r0 = 32 * half;
    float hq[3], hk[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int64_t p = t0 + r0 - 3 + j;  // absolute token of the halo row (tile row r0 + j)
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
#pragma unroll 8
    for (int r = 0; r < 32; ++r) {
      const int t = r0 + r;
      const float xq = to_f(rq_t[(t + 3) * D + ch]), xk = to_f(rk_t[(t + 3) * D + ch]);
      float yq = conv4(wq, hq[0], hq[1], hq[2], xq);
      float yk = conv4(wk, hk[0], hk[1], hk[2], xk);
      if (ACT == KDA_CONV_SILU) { yq = silu(yq); yk = silu(yk); }
      hq[0] = hq[1]; hq[1] = hq[2]; hq[2] = xq;
      hk[0] = hk[1]; hk[1] = hk[2]; hk[2] = xk;
      const bool valid = t < L;
      const float gl = valid ? fmaxf(to_f(rg_t[(t + 3) * D + ch]), LOG_DECAY_FLOOR) : 0.f;
      cum += gl;
      Yq[t * D + ch] = valid ? yq : 0.f;
      Yk[t * D + ch] = valid ? yk : 0.f;
      E1[t * D + ch] = cum;
    }
  }
  __syncthreads();

  // ---- 2. cumsum carry into the second half; L2 norms (warp per 8 rows) ----
  if (half == 1) {
    const float carry = E1[31 * D + ch];
    for (int t = 32; t < CH; ++t) E1[t * D + ch] += carry;
  }
  for (int t = warp * 8; t < warp * 8 + 8; ++t) {
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

  // ---- 3. normalise; block-midpoint factors ----------------------------------
  {
    const int r0 = 32 * half;
    // midpoints of this half's two blocks, and Gamma_C (row 63) from half 1
    for (int J = 2 * half; J < 2 * half + 2; ++J) gt[GT_GMID + J * D + ch] = E1[(16 * J + 8) * D + ch];
    if (half == 1) gt[GT_GC + ch] = E1[63 * D + ch];
    for (int r = 0; r < 32; ++r) {
      const int t = r0 + r;
      Yq[t * D + ch] *= ms[MS_RQ + t];
      Yk[t * D + ch] *= ms[MS_RK + t];
      const float d = E1[t * D + ch] - E1[(16 * (t >> 4) + 8) * D + ch];  // G_t - G_mid
      Xf[t * D + ch] = __expf(d);
    }
  }
  __syncthreads();
  {
    const int r0 = 32 * half;
    for (int r = 0; r < 32; ++r) {
      const int t = r0 + r;
      E1[t * D + ch] = 1.0f / Xf[t * D + ch];  // e^{G_mid - G_t}
    }
    // per-(block, channel) factors: e^{G_mid(J)}, e^{G_C - G_mid(J)}, and the
    // block-to-block factors e^{G_mid(I) - G_mid(J)} for J < I
    if (half == 0) {
      const float gc = gt[GT_GC + ch];
      for (int J = 0; J < 4; ++J) {
        const float gm = gt[GT_GMID + J * D + ch];
        ms[MS_EGM + J * D + ch] = __expf(gm);
        ms[MS_EGC + J * D + ch] = __expf(gc - gm);
      }
    } else {
      for (int I = 1; I < 4; ++I)
        for (int J = 0; J < I; ++J)
          ms[MS_Z + zidx(I, J) * D + ch] = __expf(gt[GT_GMID + I * D + ch] - gt[GT_GMID + J * D + ch]);
    }
  }
  __syncthreads();

  // ---- 4. record tiles that need no solve: QT, KB (thread = channel), scalars
  {
    const int r0 = 32 * half;
    float kb[32];
    for (int r = 0; r < 32; ++r) {
      const int t = r0 + r, J = t >> 4;
      const float xf = Xf[t * D + ch], e1 = E1[t * D + ch];
      const float qt = ms[MS_EGM + J * D + ch] * xf * Yq[t * D + ch];
      *reinterpret_cast<float*>(rec + REC_QT + tc::sw128(t, ch, 64)) = tc::to_tf32(qt);
      kb[r] = tc::to_tf32(ms[MS_EGC + J * D + ch] * e1 * Yk[t * D + ch]);
    }
    // row ch of KB, columns r0..r0+31 = one 128-byte slab row
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float4*>(rec + REC_KB + tc::sw128(ch, r0 + 4 * j, 128)) =
          make_float4(kb[4 * j], kb[4 * j + 1], kb[4 * j + 2], kb[4 * j + 3]);
    float* sc = reinterpret_cast<float*>(rec + REC_SC);
    if (tid < CH) { sc[tid] = ms[MS_BETA + tid]; sc[64 + tid] = ms[MS_PD + tid]; }
    if (half == 1) sc[128 + ch] = __expf(gt[GT_GC + ch]);  // gt is intact until step 5
  }

  // ---- 5. gated Gram blocks on the tensor core, 4 slabs of 32 channels -------
  const uint32_t tm = tmem_base;
  for (int kp = 0; kp < 4; ++kp) {
    // A_I: 4 x 64 rows x 32 channels (8192 elements), B_I: 4 x 32 rows x 32 (4096)
    for (int e = tid; e < 4 * 64 * 32; e += 256) {
      const int cc = e & 31, j = (e >> 5) & 63, I = e >> 11;
      const int c = kp * 32 + cc, J = j >> 4;
      float val = 0.f;
      if (J <= I) {
        val = Yk[j * D + c] * E1[j * D + c];
        if (J < I) val *= ms[MS_Z + zidx(I, J) * D + c];
      }
      *reinterpret_cast<float*>(opA + I * 8192 + tc::sw128(j, cc, 64)) = tc::to_tf32(val);
    }
    for (int e = tid; e < 4 * 32 * 32; e += 256) {
      const int cc = e & 31, r = (e >> 5) & 31, I = e >> 10;
      const int c = kp * 32 + cc, i = 16 * I + (r & 15);
      const float src = r < 16 ? Yk[i * D + c] : Yq[i * D + c];
      *reinterpret_cast<float*>(opB + I * 4096 + tc::sw128(r, cc, 32)) = tc::to_tf32(src * Xf[i * D + c]);
    }
    tc::fence_async_smem();
    tc::fence_before();
    __syncthreads();
    if (tid == 0) {
      tc::fence_after();
      const uint64_t da = tc::desc(tc::smem_u32(opA)), db = tc::desc(tc::smem_u32(opB));
#pragma unroll
      for (int I = 0; I < 4; ++I)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          tc::mma_ss(tm + 32 * I, da + ((I * 8192) >> 4) + tc::desc_step(64, ks),
                     db + ((I * 4096) >> 4) + tc::desc_step(32, ks), tc::idesc_tf32(64, 32),
                     (kp > 0 || ks > 0) ? 1 : 0);
      tc::commit(&bar);
    }
    tc::bar_wait(&bar, phase);
    phase ^= 1;
    tc::fence_after();
  }

  // ---- 6. read D_I (M = 64 layout: row j -> lane j%16 + 32*(j/16)) ---------
  if (warp < 4) {
    const int j = 16 * warp + (lane & 15);
    for (int I = 0; I < 4; ++I) {
      float mv[16], pv[16];
      tc::ld16(tm + ((uint32_t)(32 * warp) << 16) + 32 * I, mv);
      tc::ld16(tm + ((uint32_t)(32 * warp) << 16) + 32 * I + 16, pv);
      tc::ld_wait();
      if (lane < 16) {
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const int i = 16 * I + r;
          Ms[i * CH + j] = i > j ? ms[MS_BETA + i] * mv[r] : 0.f;  // diag(beta) M, strict
          Ps[i * CH + j] = i > j ? pv[r] : 0.f;
        }
      }
    }
  }
  __syncthreads();

  // ---- 7. X = (I + diag(beta) M)^-1, blocked forward substitution -------------
  float* Xd = sv + SV_XD;  // [4][16][16] inverses of the diagonal blocks
  float* Yb = sv + SV_YB;  // [3][16][16]
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
  for (int I = 1; I < 4; ++I) {
    // Y_IJ = sum_{K=J}^{I-1} L_IK X_KJ  for J < I (X_KJ already in Ms for K < I)
    for (int e = tid; e < I * 256; e += 256) {
      const int J = e >> 8, r = (e >> 4) & 15, cc = e & 15;
      float s = 0.f;
      for (int m = 16 * J; m < 16 * I; ++m) {
        const float xk = (m >> 4) == J ? Xd[(J * 16 + (m & 15)) * 16 + cc]   // X_JJ
                                       : Ms[m * CH + 16 * J + cc];           // X_KJ, K > J
        s += Ms[(16 * I + r) * CH + m] * xk;
      }
      Yb[(J * 16 + r) * 16 + cc] = s;
    }
    __syncthreads();
    // X_IJ = -X_II Y_IJ, written over L_IJ
    for (int e = tid; e < I * 256; e += 256) {
      const int J = e >> 8, r = (e >> 4) & 15, cc = e & 15;
      float s = 0.f;
#pragma unroll
      for (int m = 0; m < 16; ++m) s += Xd[(I * 16 + r) * 16 + m] * Yb[(J * 16 + m) * 16 + cc];
      Ms[(16 * I + r) * CH + 16 * J + cc] = -s;
    }
    __syncthreads();
  }
  // diagonal blocks into Ms; Ms now holds X (unit lower triangular)
  for (int e = tid; e < 4 * 256; e += 256) {
    const int I = e >> 8, r = (e >> 4) & 15, cc = e & 15;
    Ms[(16 * I + r) * CH + 16 * I + cc] = Xd[(I * 16 + r) * 16 + cc];
  }
  __syncthreads();

  // ---- 8. T = X diag(beta); tiles for W = T K~ and the record's T_s, P_s -----
  uint8_t* tT = opA;          // [64 t][64 t'] tile, 16 KB
  uint8_t* tK = opA + 16384;  // [128 k][64 t'] tile (K~^T), 32 KB
  for (int e = tid; e < CH * CH; e += 256) {
    const int t = e >> 6, tp = e & 63;
    const float tv = tp <= t ? Ms[t * CH + tp] * ms[MS_BETA + tp] : 0.f;
    const float tr = tc::to_tf32(tv);
    *reinterpret_cast<float*>(tT + tc::sw128(t, tp, 64)) = tr;
    *reinterpret_cast<float*>(rec + REC_B1 + tc::sw128(t, tp, 64)) = tp < t ? tr : 0.f;
    *reinterpret_cast<float*>(rec + REC_PS + tc::sw128(t, tp, 64)) = tc::to_tf32(Ps[t * CH + tp]);
  }
  {
    const int r0 = 32 * half;
    float kt[32];
    for (int r = 0; r < 32; ++r) {
      const int t = r0 + r;
      kt[r] = tc::to_tf32(ms[MS_EGM + (t >> 4) * D + ch] * Xf[t * D + ch] * Yk[t * D + ch]);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
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
    tc::commit(&bar);
  }
  tc::bar_wait(&bar, phase);
  phase ^= 1;
  tc::fence_after();

  // ---- 9. -W rows into the record (columns 64..191 of B1) --------------------
  if (warp < 4) {
    const int t = 16 * warp + (lane & 15);
    for (int cb = 0; cb < 8; ++cb) {
      float w[16];
      tc::ld16(tm + ((uint32_t)(32 * warp) << 16) + 128 + 16 * cb, w);
      tc::ld_wait();
      if (lane < 16) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<float4*>(rec + REC_B1 + tc::sw128(t, 64 + 16 * cb + 4 * j, 64)) =
              make_float4(tc::to_tf32(-w[4 * j]), tc::to_tf32(-w[4 * j + 1]), tc::to_tf32(-w[4 * j + 2]),
                          tc::to_tf32(-w[4 * j + 3]));
      }
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem_base, 256);
}

}  // namespace kda
