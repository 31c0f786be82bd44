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
// The record (kda_record.cuh), in the plainly normalised form (q_hat, k_hat;
// r = 1), all tiles fp32 values rounded to tf32, K-major 128-byte swizzled
// (kda_tc.cuh):
//   RA  [128][128 k]: -W and Q~ = e^{Gamma_t} * q_hat_t stacked by rows, -W
//                     first for even chunks of a segment, Q~ first for odd ones
//                     (so that one N = 128 product writes U next to the output
//                     buffer of the chunk's parity)
//   TS  [64 t][ 64]:  T strictly below the diagonal
//   B2  [192][64 t]:  P strictly below the diagonal and
//                     (e^{Gamma_C - Gamma_t} * k_hat_t)^T, in the same parity
//                     order
//   SC  fp32 b = beta[64], d = P_tt[64] (exact q_hat_t . k_hat_t), r = 1,
//       e^{Gamma_C}[128]
// The diagonal terms beta_t v_t (of T V) and P_tt u_t (of P U) are applied in
// fp32 by the scan kernel; they carry the largest single-token contributions.
//
// Gram blocks without overflow: the chunk is split into two 32-row halves b
// with reference rows m_b = 32b + 16.  For i in half I and j <= i in half J,
//   e^{G_i - G_j} = e^{G_i - G_{m_I}} * e^{G_{m_I} - G_j}
// where |G_i - G_{m_I}| <= 5 * 16 = 80 (fp32 and tf32 reach e^88) and
// e^{G_{m_I} - G_j} <= e^80 for j in half I, <= 1 for j in an earlier half.
// The tensor core computes one M = 128 product per Gram, rows (A, K-major):
//   0..31   k_j e^{G_{m_0} - G_j}, j = 0..31      (against half 0's columns)
//   32..95  k_j e^{G_{m_1} - G_j}, j = 0..63      (against half 1's columns)
//   96..127 not read back
// and columns (B) [x_i e^{G_i - G_{m_0}}]_{i<32} | [x_i e^{G_i - G_{m_1}}]_{i>=32}
// with x = q (the P Gram) or k (the M Gram); the wanted entries are the
// row-0..31 x column-0..31 and row-32..95 x column-32..63 blocks.
//
// Two blocks of 256 threads share an SM (90 KB of shared memory and 256 TMEM
// columns each), so that one block's barrier and tensor-core waits are covered
// by the other's work.  Thread (c, b) owns key/query channel c of token half b;
// the short-conv outputs of a chunk live in TMEM (lane = channel) rather than
// in shared memory, and row norms are reduced with warp shuffles.
#pragma once
#include "kda_common.cuh"
#include "kda_record.cuh"
#include "kda_tc.cuh"

namespace kda {

// shared memory plan (bytes from a 1024-aligned base); regions are reused
// phase by phase
constexpr int PREP_THREADS = 256;
constexpr uint32_t P_RAW = 0;                // steps 0-1: raw q, k, g tiles (3 x RAW_BYTES)
constexpr uint32_t P_GA = 0;                 // steps 3-5: Gram A tile, 4 slabs x 96 rows
constexpr uint32_t GA_ROWS = 96;
constexpr uint32_t P_GB = 49152;             // steps 3-5: Gram B tile, 4 slabs x 64 rows
constexpr uint32_t MS_LD = 68;               // row stride (floats) of the solve matrix: rows
                                             // 16-byte aligned, columns spread over all banks
constexpr uint32_t P_MS = 0;                 // step 6: diag(beta) M strict, [64][68] fp32
constexpr uint32_t P_TT = 17408;             // step 7: T tile [64 t][64 t'] (16 KB)
constexpr uint32_t P_KT = 33792;             // step 7: K~^T tile [128 k][64 t] (32 KB)
constexpr uint32_t P_TMP = 66560;            // steps 6-7: blocks of X (12.3 KB)
constexpr uint32_t P_WST = 52224;            // step 8: -W staged in its record image (32 KB), read by
                                             // bulk copies until the next item's step 3
constexpr uint32_t P_MISC = 84992;           // scalars (6 KB)
constexpr uint32_t PREP_SMEM = P_MISC + 6144 + 1024;
static_assert(P_GA + 3 * GA_ROWS * 128 + 128 * 128 <= P_MISC, "A tile reads past the Gram region");
static_assert(3 * RAW_BYTES <= P_MISC && P_TMP + (96 * 20 + 32 * 36 + 16) * 4 <= P_MISC,
              "shared regions overlap the scalars");
static_assert(P_MS + 64 * MS_LD * 4 <= P_TT, "solve matrix overlaps the T tile");
static_assert(P_WST >= 3 * RAW_BYTES && P_WST + 4 * 64 * 128 <= P_MISC && P_WST % 1024 == 0,
              "the -W staging overlaps the next item's raw tiles or the scalars");

// scalar region (floats)
constexpr int MB_BETA = 0, MB_RQ = 64, MB_RK = 128, MB_PD = 192, MB_CARRY = 256 /*128*/,
              MB_G1M = 384 /*128*/, MB_G1T = 512 /*128*/, MB_PART = 640 /*2 x 4 x 3 x 32*/;
static_assert((MB_PART + 768) * 4 <= 6144, "scalar region");

// TMEM columns: short-conv outputs, then stashes and accumulators
constexpr int TC_YQ = 0;    // conv(q) -> stash of k e^{G - G_m} (M Gram B operand)
constexpr int TC_YK = 64;   // conv(k) -> stash of e^{G} k (W operand)
constexpr int TC_G = 128;   // half-local cumulative gate
constexpr int TC_DP = 128;  // P Gram accumulator (64 columns)
constexpr int TC_DM = 192;  // M Gram accumulator (64 columns)
constexpr int TC_W = 128;   // W accumulator (M = 64, 128 columns)

// one 32-byte (256-bit) global store; dst 32-byte aligned
__device__ __forceinline__ void st_global_v8(float* dst, float a0, float a1, float a2, float a3, float a4, float a5,
                                             float a6, float a7) {
  asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "f"(a0), "f"(a1), "f"(a2),
               "f"(a3), "f"(a4), "f"(a5), "f"(a6), "f"(a7)
               : "memory");
}

// Sum over the 32 lanes of a warp of 16 per-lane vectors; lane l returns the
// total of entry l % 16 (recursive halving: 16 shuffles instead of 16 x 5).
__device__ __forceinline__ float lane_reduce16(float (&v)[16], int lane) {
#pragma unroll
  for (int m = 8; m >= 1; m >>= 1) {
    const bool up = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < m; ++i) {
      const float send = up ? v[i] : v[i + m];
      const float keep = up ? v[i + m] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
    }
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 16);
}

template <int ACT>
__global__ void __launch_bounds__(PREP_THREADS, 2)
chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_g, const __nv_bfloat16* __restrict__ beta,
                  const float* __restrict__ conv_w, const __nv_bfloat16* __restrict__ init_conv,
                  const int32_t* __restrict__ cu, const int2* __restrict__ chunk_tab, int H,
                  int n_items, uint8_t* __restrict__ records, int* __restrict__ work_counter,
                  int* __restrict__ ready, int vacate_below_smid, int vacate_after) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array itself so that the
  // compiler keeps the shared address space (32-bit shared loads and stores)
  uint8_t* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  float* ms = (float*)(sm + P_MISC);
  float* Ms = (float*)(sm + P_MS);
  __shared__ uint64_t bar_ld, bar_p, bar_m, bar_w;
  __shared__ uint32_t tmem_base;
  __shared__ int s_next;  // the block's next work item (claimed by thread 0)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ch = tid & 127, hb = tid >> 7;  // channel, 32-row half of the chunk
  const int q4 = warp & 3;                  // TMEM lane quarter (= ch / 32)
  const int r0 = 32 * hb;                   // first row of this thread's half
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

  // Work items are claimed in order from a global counter, so the records are
  // completed roughly chunk by chunk.  A block on an SM below
  // vacate_below_smid stops claiming once vacate_after items have been
  // handed out: those SMs then take the scan kernel, which runs concurrently
  // and consumes records as their ready flags are published.
  uint32_t smid;
  asm("mov.u32 %0, %%smid;" : "=r"(smid));
  const bool vacate = (int)smid < vacate_below_smid;
  auto claim = [&]() -> int {  // thread 0
    if (vacate && *reinterpret_cast<volatile int*>(work_counter) >= vacate_after) return n_items;
    return atomicAdd(work_counter, 1);
  };

  // ---- 0. once per block: TMEM, barriers, first item's tiles ----------------
  if (warp == 0) tc::tmem_alloc(&tmem_base, 256);
  if (tid == 0) {
    tc::bar_init(&bar_ld, 1); tc::bar_init(&bar_p, 1); tc::bar_init(&bar_m, 1); tc::bar_init(&bar_w, 1);
    tc::bar_init_fence();
    s_next = atomicAdd(work_counter, 1);  // every block takes at least one item
    if (s_next < n_items) load_raw(s_next);
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tm = tmem_base;
  const uint32_t tl = tm + ((uint32_t)(32 * q4) << 16);  // this warp's TMEM lanes
  uint32_t par = 0;  // phase parity of the per-item barriers
  // thread 0: the item whose -W bulk copies are in flight; its record is
  // published once they are complete (during the next item, or at exit)
  int pending = -1;
  auto publish = [&](int it) {
    tc::bulk_wait_all();
    tc::fence_async_global();
    if (ready) {  // every thread's stores of the item precede a barrier thread 0 has passed
      __threadfence();
      asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(ready + it), "r"(1) : "memory");
    }
  };

  // persistent loop over (chunk, head) work items, chunk-major
  for (int item = s_next; item < n_items; item = s_next, par ^= 1) {
  const int cid = item / H, h = item % H;
  const int2 nc = chunk_tab[cid];
  const int n = nc.x;
  const int64_t seg0 = cu[n], seg1 = cu[n + 1];
  const int64_t t0 = seg0 + (int64_t)CH * nc.y;
  const int L = (int)((seg1 - t0) < CH ? (seg1 - t0) : CH);
  const int64_t chan = (int64_t)h * D + ch;
  uint8_t* rec = records + ((int64_t)cid * H + h) * REC_BYTES;
  // row blocks of -W and Q~ in RA, of P and K-bar^T in B2, by chunk parity
  const int wrow0 = ra_w_row(nc.y & 1), qrow0 = ra_q_row(nc.y & 1);
  const int prow0 = b2_p_row(nc.y & 1), krow0 = b2_k_row(nc.y & 1);
  if (tid < CH) ms[MB_BETA + tid] = tid < L ? to_f(beta[(t0 + tid) * H + h]) : 0.f;
  const float4 wq = load4(conv_w + (0 * HD + chan) * 4);
  const float4 wk = load4(conv_w + (1 * HD + chan) * 4);
  tc::bar_wait(&bar_ld, par);

  // ---- 1. causal conv of q, k; half-local cumsum of the clamped gate; the
  //         row sums |q|^2, |k|^2, q.k over this warp's 32 channels ----------
  // cumulative gates are kept in base-2 units (Gamma * log2 e) so that every
  // e^x below is one ex2
  float gm_loc;  // half-local cumulative gate through row r0 + 16
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
    gm_loc = 0.f;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      float yq[16], yk[16], gl[16], sq[16], sk[16], sx[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const int t = r0 + 16 * g + r;
        const float xq = to_f(rq_t[(t + 3) * D + ch]), xk = to_f(rk_t[(t + 3) * D + ch]);
        float a = conv4(wq, hq[0], hq[1], hq[2], xq);
        float b = conv4(wk, hk[0], hk[1], hk[2], xk);
        if (ACT == KDA_CONV_SILU) { a = silu(a); b = silu(b); }
        hq[0] = hq[1]; hq[1] = hq[2]; hq[2] = xq;
        hk[0] = hk[1]; hk[1] = hk[2]; hk[2] = xk;
        const bool valid = t < L;
        cum += valid ? fmaxf(to_f(rg_t[(t + 3) * D + ch]), LOG_DECAY_FLOOR) * LOG2E : 0.f;
        yq[r] = valid ? a : 0.f;
        yk[r] = valid ? b : 0.f;
        gl[r] = cum;
        sq[r] = yq[r] * yq[r]; sk[r] = yk[r] * yk[r]; sx[r] = yq[r] * yk[r];
      }
      if (g == 1) gm_loc = gl[0];
      tc::st16(tl + TC_YQ + r0 + 16 * g, yq);
      tc::st16(tl + TC_YK + r0 + 16 * g, yk);
      tc::st16(tl + TC_G + r0 + 16 * g, gl);
      const float nq = lane_reduce16(sq, lane), nk = lane_reduce16(sk, lane), nx = lane_reduce16(sx, lane);
      if (lane < 16) {
        float* part = ms + MB_PART + (hb * 4 + q4) * 96 + 16 * g + lane;
        part[0] = nq; part[32] = nk; part[64] = nx;
      }
    }
    ms[(hb ? MB_G1T : MB_CARRY) + ch] = cum;  // half totals
    if (hb) ms[MB_G1M + ch] = gm_loc;
  }
  tc::st_wait();
  __syncthreads();

  // ---- 2. inverse row norms and the exact diagonal q_hat . k_hat ------------
  if (tid < CH) {
    const int hh = tid >> 5, rr = tid & 31;
    float nq = 0.f, nk = 0.f, nx = 0.f;
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      const float* part = ms + MB_PART + (hh * 4 + c4) * 96 + rr;
      nq += part[0]; nk += part[32]; nx += part[64];
    }
    const float rq = 1.0f / sqrtf(nq + NORM_EPS), rk = 1.0f / sqrtf(nk + NORM_EPS);
    ms[MB_RQ + tid] = rq; ms[MB_RK + tid] = rk; ms[MB_PD + tid] = nx * rq * rk;
  }
  if (tid == 0 && pending >= 0) tc::bulk_wait_read();  // step 3 overwrites the previous -W staging
  __syncthreads();

  // ---- 3. normalise; Gram operands, record tiles Q~ and K-bar^T, stashes ----
  const float carry = hb ? ms[MB_CARRY + ch] : 0.f;         // gate total of half 0
  const float g1m = ms[MB_CARRY + ch] + ms[MB_G1M + ch];     // G at row 48
  const float gC = ms[MB_CARRY + ch] + ms[MB_G1T + ch];      // G at the chunk end
  {
    const float gm = hb ? g1m : gm_loc;                      // this half's reference G_m
    const float egcm = tc::exp2_fast(gC - g1m);              // e^{G_C - G_{m_1}}, <= 1
#pragma unroll
    for (int g = 0; g < 4; ++g) {  // 8-row groups
      float yq[8], yk[8], gl[8];
      tc::ld8(tl + TC_YQ + r0 + 8 * g, yq);
      tc::ld8(tl + TC_YK + r0 + 8 * g, yk);
      tc::ld8(tl + TC_G + r0 + 8 * g, gl);
      const float4 rk0 = *reinterpret_cast<const float4*>(ms + MB_RK + r0 + 8 * g);
      const float4 rk1 = *reinterpret_cast<const float4*>(ms + MB_RK + r0 + 8 * g + 4);
      const float4 rq0 = *reinterpret_cast<const float4*>(ms + MB_RQ + r0 + 8 * g);
      const float4 rq1 = *reinterpret_cast<const float4*>(ms + MB_RQ + r0 + 8 * g + 4);
      const float rkv[8] = {rk0.x, rk0.y, rk0.z, rk0.w, rk1.x, rk1.y, rk1.z, rk1.w};
      const float rqv[8] = {rq0.x, rq0.y, rq0.z, rq0.w, rq1.x, rq1.y, rq1.z, rq1.w};
      tc::ld_wait();
      float kb[8];
      // rows r and r + 1 share each packed multiply and add (every lane rounded
      // as the scalar form rounds it); exponentials and tf32 roundings are per row
#pragma unroll
      for (int r = 0; r < 8; r += 2) {
        const float2 G = add2(make_float2(gl[r], gl[r + 1]), dup2(carry));
        const float2 d = add2(G, dup2(-gm));
        const float2 e1 = make_float2(tc::exp2_fast(d.x), tc::exp2_fast(d.y));
        const float2 e2 = make_float2(tc::exp2_fast(-d.x), tc::exp2_fast(-d.y));
        const float2 e3 = make_float2(tc::exp2_fast(G.x), tc::exp2_fast(G.y));
        const float2 kh = mul2(make_float2(yk[r], yk[r + 1]), make_float2(rkv[r], rkv[r + 1]));
        const float2 qh = mul2(make_float2(yq[r], yq[r + 1]), make_float2(rqv[r], rqv[r + 1]));
        // e^{G_{m_1} - G_t}: e2 for half 1; <= 1 for half 0
        const float2 a1 = hb ? e2 : make_float2(tc::exp2_fast(g1m - G.x), tc::exp2_fast(g1m - G.y));
        const float2 pb = mul2(qh, e1), pa = mul2(kh, a1), pq = mul2(qh, e3);
        // e^{G_C - G_t} = e^{G_C - G_{m_1}} e^{G_{m_1} - G_t}: for half 0 both
        // factors are <= 1 (an underflow only drops what is below fp32 anyway)
        const float2 kbr = mul2(kh, mul2(dup2(egcm), a1));
        const float2 ke1 = mul2(kh, e1), ke3 = mul2(kh, e3);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int rr = r + u;
          // B operand of the P Gram; A rows (block of the own half, and for
          // half 0 the rows read against half 1)
          *reinterpret_cast<float*>(sm + P_GB + tc::sw128o(r0 + 8 * g, rr, ch, 64)) = tc::to_tf32(u ? pb.y : pb.x);
          *reinterpret_cast<float*>(sm + P_GA + tc::sw128o(32 + r0 + 8 * g, rr, ch, GA_ROWS)) =
              tc::to_tf32(u ? pa.y : pa.x);
          if (!hb)
            *reinterpret_cast<float*>(sm + P_GA + tc::sw128o(r0 + 8 * g, rr, ch, GA_ROWS)) =
                tc::to_tf32((u ? kh.y : kh.x) * (u ? e2.y : e2.x));
          *reinterpret_cast<float*>(rec + REC_RA + tc::sw128o(qrow0 + r0 + 8 * g, rr, ch, 128)) =
              tc::to_tf32(u ? pq.y : pq.x);
          kb[rr] = tc::to_tf32(u ? kbr.y : kbr.x);
        }
        yq[r] = ke1.x; yq[r + 1] = ke1.y;  // stash: M Gram B operand
        yk[r] = ke3.x; yk[r + 1] = ke3.y;  // stash: e^{G} k for W
      }
      tc::st8(tl + TC_YQ + r0 + 8 * g, yq);
      tc::st8(tl + TC_YK + r0 + 8 * g, yk);
      // K-bar^T row ch (B2 row krow0 + ch), columns r0 + 8g .. +7: the two
      // 16-byte chunks (2g and 2g + 1 before the swizzle) fill one aligned
      // 32-byte sector, in swapped order on rows of odd swizzle phase; one
      // 256-bit store writes it
      {
        const bool swap = (ch & 1) != 0;  // swizzle phase of row krow0 + ch is ch % 8
        float* dst = reinterpret_cast<float*>(rec + REC_B2 + (tc::sw128(krow0 + ch, r0 + 8 * g, B2_ROWS) & ~16u));
        if (swap)
          st_global_v8(dst, kb[4], kb[5], kb[6], kb[7], kb[0], kb[1], kb[2], kb[3]);
        else
          st_global_v8(dst, kb[0], kb[1], kb[2], kb[3], kb[4], kb[5], kb[6], kb[7]);
      }
    }
  }
  tc::fence_async_smem();
  tc::st_wait();
  tc::fence_before();
  __syncthreads();

  // ---- 4. P Gram (A = GA, B = q operand) -------------------------------------
  const uint64_t d_ga = tc::desc(tc::smem_u32(sm + P_GA)), d_gb = tc::desc(tc::smem_u32(sm + P_GB));
  auto issue_gram = [&](uint32_t dcol, uint64_t* bar) {
    tc::fence_after();
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        tc::mma_ss(tm + dcol, d_ga + ((s * GA_ROWS * 128) >> 4) + tc::desc_step(0, ks),
                   d_gb + ((s * 64 * 128) >> 4) + tc::desc_step(0, ks), tc::idesc_tf32(128, 64),
                   (s | ks) ? 1 : 0);
    tc::commit(bar);
  };
  if (tid == 0) issue_gram(TC_DP, &bar_p);
  tc::bar_wait(&bar_p, par);
  tc::fence_after();
  // the B tile is free: k operand of the M Gram from the stash
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    float kx[16];
    tc::ld16(tl + TC_YQ + r0 + 16 * g, kx);
    tc::ld_wait();
#pragma unroll
    for (int r = 0; r < 16; ++r)
      *reinterpret_cast<float*>(sm + P_GB + tc::sw128o(r0 + 16 * g, r, ch, 64)) = tc::to_tf32(kx[r]);
  }
  tc::fence_async_smem();
  tc::fence_before();
  __syncthreads();
  if (tid == 0) issue_gram(TC_DM, &bar_m);

  // ---- 5. P into the record (while the M Gram runs) ---------------------------
  // accumulator row m = TMEM lane: A row (j = m for m < 32, j = m - 32 for
  // 32 <= m < 96); column n = query row i.  Warp (q4, hb) reads lanes of
  // quarter q4, columns 16 hb .. of the half that quarter pairs with.
  {
    const int j = q4 == 2 ? 32 + lane : (q4 == 3 ? 32 + lane : lane);
    const int ib = (q4 == 0 || q4 == 3 ? 0 : 32) + 16 * hb;  // first query row
    float v[16];
    if (q4 < 3) {
      tc::ld16(tl + TC_DP + ib, v);
      tc::ld_wait();
    }
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int i = ib + c;
      const float p = (q4 < 3 && i > j) ? v[c] : 0.f;  // strictly lower part; quarter 3 writes the zero block
      *reinterpret_cast<float*>(rec + REC_B2 + tc::sw128o(prow0 + ib, c, j, B2_ROWS)) = tc::to_tf32(p);
    }
  }
  tc::bar_wait(&bar_m, par);
  tc::fence_after();
  // ---- 5b. diag(beta) M (strictly lower) into the solve matrix ----------------
  if (q4 < 3) {
    const int j = q4 == 2 ? 32 + lane : lane;
    const int ib = (q4 == 0 ? 0 : 32) + 16 * hb;
    float v[16];
    tc::ld16(tl + TC_DM + ib, v);
    tc::ld_wait();
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int i = ib + c;
      Ms[i * MS_LD + j] = i > j ? ms[MB_BETA + i] * v[c] : 0.f;
    }
  }
  __syncthreads();

  // ---- 6. X = (I + diag(beta) M)^-1 (unit lower triangular) ------------------
  // Blocks of the 2 x 2 partitions, each X_ba = -X_bb L_ba X_aa:
  //   A  the four diagonal 16-blocks, by forward substitution   -> Xd[I]
  //   B  the off-diagonal 16-block of each 32-half               -> XB[P]
  //   C  the off-diagonal 32-block                               -> XC
  // Results go to their own buffers (nothing is overwritten while another
  // thread may still read it), so each stage needs one barrier.  Within B and
  // C a thread group computes a column of the intermediate product L X_aa and
  // shares it by shuffles before multiplying by X_bb.
  // Row strides of 20 (36) floats put 8 consecutive rows of a block in 8
  // distinct 4-bank groups, so the float4 row loads below are conflict-free.
  constexpr int XS = 20, XCS = 36;
  float* Xd = (float*)(sm + P_TMP);           // [4][16][XS]
  float* XB = Xd + 4 * 16 * XS;               // [2][16][XS]
  float* XC = XB + 2 * 16 * XS;               // [32][XCS]
  float* Zr = XC + 32 * XCS;                  // [16] zeros
  if (tid < 64) {
    const int I = tid >> 4, cc = tid & 15;  // column cc of X_II
    const float* Lb = Ms + (16 * I) * MS_LD + 16 * I;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float s = (r == cc) ? 1.f : 0.f;
#pragma unroll
      for (int m4 = 0; m4 < r; m4 += 4) {
        const float4 l = *reinterpret_cast<const float4*>(Lb + r * MS_LD + m4);
        s -= l.x * x[m4];
        if (m4 + 1 < r) s -= l.y * x[m4 + 1];
        if (m4 + 2 < r) s -= l.z * x[m4 + 2];
        if (m4 + 3 < r) s -= l.w * x[m4 + 3];
      }
      x[r] = r < cc ? 0.f : s;
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) Xd[(I * 16 + r) * XS + cc] = x[r];
  } else if (tid < 80) {
    Zr[tid - 64] = 0.f;
  }
  __syncthreads();
  {  // B: warp w -> half P = w / 4, column cc = 4 (w % 4) + lane / 8, rows k and k + 8 (k = lane % 8)
    const int P = warp >> 2, cc = 4 * (warp & 3) + (lane >> 3), k = lane & 7;
    const float* X0 = Xd + (2 * P) * 16 * XS;
    const float* X1 = Xd + (2 * P + 1) * 16 * XS;
    float xc[16];  // column cc of X_{2P,2P}
#pragma unroll
    for (int m = 0; m < 16; ++m) xc[m] = X0[m * XS + cc];
    float y[2];  // (L_{2P+1,2P} X_{2P,2P}) rows k, k + 8, column cc
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float* Lr = Ms + (32 * P + 16 + k + 8 * u) * MS_LD + 32 * P;
      float s = 0.f;
#pragma unroll
      for (int m4 = 0; m4 < 16; m4 += 4) {
        const float4 a = *reinterpret_cast<const float4*>(Lr + m4);
        s += a.x * xc[m4] + a.y * xc[m4 + 1] + a.z * xc[m4 + 2] + a.w * xc[m4 + 3];
      }
      y[u] = s;
    }
    float yc[16];  // the whole column cc, from the 8 lanes that share it
    const int base = lane & ~7;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      yc[kk] = __shfl_sync(0xffffffffu, y[0], base + kk);
      yc[kk + 8] = __shfl_sync(0xffffffffu, y[1], base + kk);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float* xr = X1 + (k + 8 * u) * XS;
      float s = 0.f;
#pragma unroll
      for (int m4 = 0; m4 < 16; m4 += 4) {
        const float4 a = *reinterpret_cast<const float4*>(xr + m4);
        s += a.x * yc[m4] + a.y * yc[m4 + 1] + a.z * yc[m4 + 2] + a.w * yc[m4 + 3];
      }
      XB[(P * 16 + k + 8 * u) * XS + cc] = -s;
    }
  }
  __syncthreads();
  {  // C: warp w -> column cc = 16 (w / 4) + 4 (w % 4) + lane / 8, rows k + 8u (k = lane % 8, u < 4)
    const int cc = 16 * (warp >> 2) + 4 * (warp & 3) + (lane >> 3), k = lane & 7;
    float y[4];
    if (warp < 4) {  // cc < 16: column of X_00 = [Xd0 ; XB0] column cc
      float xc[32];
#pragma unroll
      for (int m = 0; m < 16; ++m) { xc[m] = Xd[m * XS + cc]; xc[16 + m] = XB[m * XS + cc]; }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float* Lr = Ms + (32 + k + 8 * u) * MS_LD;
        float s = 0.f;
#pragma unroll
        for (int m4 = 0; m4 < 32; m4 += 4) {
          const float4 a = *reinterpret_cast<const float4*>(Lr + m4);
          s += a.x * xc[m4] + a.y * xc[m4 + 1] + a.z * xc[m4 + 2] + a.w * xc[m4 + 3];
        }
        y[u] = s;
      }
    } else {  // cc >= 16: column of X_00 = [0 ; Xd1] column cc - 16
      float xc[16];
#pragma unroll
      for (int m = 0; m < 16; ++m) xc[m] = Xd[(16 + m) * XS + (cc - 16)];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float* Lr = Ms + (32 + k + 8 * u) * MS_LD + 16;
        float s = 0.f;
#pragma unroll
        for (int m4 = 0; m4 < 16; m4 += 4) {
          const float4 a = *reinterpret_cast<const float4*>(Lr + m4);
          s += a.x * xc[m4] + a.y * xc[m4 + 1] + a.z * xc[m4 + 2] + a.w * xc[m4 + 3];
        }
        y[u] = s;
      }
    }
    float yc[32];  // column cc of L_10 X_00, from the 8 lanes that share it
    const int base = lane & ~7;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
#pragma unroll
      for (int u = 0; u < 4; ++u) yc[kk + 8 * u] = __shfl_sync(0xffffffffu, y[u], base + kk);
    // X_11 row r = [Xd2 row r, 0] (r < 16) or [XB1 row r - 16, Xd3 row r - 16]
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = k + 8 * u;  // u < 2: r < 16
      const float* ra = u < 2 ? Xd + (32 + r) * XS : XB + r * XS;  // Xd2 row r / XB1 row r - 16
      const float* rb = u < 2 ? Zr : Xd + (32 + r) * XS;             // zero / Xd3 row r - 16
      float s = 0.f;
#pragma unroll
      for (int m4 = 0; m4 < 16; m4 += 4) {
        const float4 a = *reinterpret_cast<const float4*>(ra + m4);
        s += a.x * yc[m4] + a.y * yc[m4 + 1] + a.z * yc[m4 + 2] + a.w * yc[m4 + 3];
        if (u >= 2) {
          const float4 b = *reinterpret_cast<const float4*>(rb + m4);
          s += b.x * yc[16 + m4] + b.y * yc[16 + m4 + 1] + b.z * yc[16 + m4 + 2] + b.w * yc[16 + m4 + 3];
        }
      }
      XC[r * XCS + cc] = -s;
    }
  }
  __syncthreads();

  // ---- 7. T = X diag(beta): record TS, T tile; K~^T tile; W = T K~ -----------
  if (tid == 0 && pending >= 0) {
    publish(pending);
    pending = -1;
  }
  for (int e = tid; e < CH * 16; e += PREP_THREADS) {  // 4-column groups
    const int t = e >> 4, tp = 4 * (e & 15);
    float4 tv, ts;
    float* tvp = &tv.x;
    float* tsp = &ts.x;
    // X row t, columns tp .. tp + 3 (one 16-block): diagonal block, off-diagonal
    // 16-block of a 32-half, the off-diagonal 32-block, or zero
    const int I = t >> 4, J = tp >> 4;
    const float* src = I == J ? Xd + (I * 16 + (t & 15)) * XS + (tp & 15)
                     : (I == J + 1 && (I & 1)) ? XB + ((I >> 1) * 16 + (t & 15)) * XS + (tp & 15)
                     : (I >= 2 && J <= 1) ? XC + (t - 32) * XCS + tp
                     : Zr;
    const float4 xr = *reinterpret_cast<const float4*>(src);
    const float* xrp = &xr.x;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = tp + u;
      const float x = c < t ? xrp[u] : (c == t ? 1.f : 0.f);
      tvp[u] = tc::to_tf32(x * ms[MB_BETA + c]);
      tsp[u] = c < t ? tvp[u] : 0.f;
    }
    *reinterpret_cast<float4*>(sm + P_TT + tc::sw128(t, tp, 64)) = tv;
    *reinterpret_cast<float4*>(rec + REC_TS + tc::sw128(t, tp, 64)) = ts;
  }
#pragma unroll
  for (int g = 0; g < 2; ++g) {  // K~^T row ch, columns r0 + 16g ..
    float kt[16];
    tc::ld16(tl + TC_YK + r0 + 16 * g, kt);
    tc::ld_wait();
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<float4*>(sm + P_KT + tc::sw128(ch, r0 + 16 * g + 4 * j, 128)) =
          make_float4(tc::to_tf32(kt[4 * j]), tc::to_tf32(kt[4 * j + 1]), tc::to_tf32(kt[4 * j + 2]),
                      tc::to_tf32(kt[4 * j + 3]));
  }
  tc::fence_async_smem();
  tc::fence_before();
  __syncthreads();
  if (tid == 0) {
    tc::fence_after();
    const uint64_t dt = tc::desc(tc::smem_u32(sm + P_TT)), dk = tc::desc(tc::smem_u32(sm + P_KT));
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
      tc::mma_ss(tm + TC_W, dt + tc::desc_step(64, ks), dk + tc::desc_step(128, ks), tc::idesc_tf32(64, 128),
                 ks > 0 ? 1 : 0);
    tc::commit(&bar_w);
  }
  {  // scalars of the record (normalised form: b = beta, d = q_hat . k_hat, r = 1)
    float* sc = reinterpret_cast<float*>(rec + REC_SC);
    if (tid < CH) { sc[SC_B + tid] = ms[MB_BETA + tid]; sc[SC_D + tid] = ms[MB_PD + tid]; sc[SC_R + tid] = 1.f; }
    if (hb == 0) sc[SC_G + ch] = tc::exp2_fast(gC);
  }
  tc::bar_wait(&bar_w, par);
  tc::fence_after();
  // the shared regions are free: fetch the next item's tiles while this one finishes
  __syncthreads();
  if (tid == 0) {
    const int nx = claim();
    s_next = nx;  // read by every thread after the item's last barrier
    if (nx < n_items) load_raw(nx);
  }

  // ---- 8. -W rows into the record (row block wrow0 of RA) -------------------
  // M = 64 accumulator: row t in lane 16 * (t / 16) ... of quarter t / 16.
  // The rows are staged in their record image (the swizzle phase of row
  // wrow0 + t is that of t) and leave in four 8 KB bulk copies, one per slab,
  // instead of one scattered 16-byte store per row and column group.
  {
    const int t = 16 * q4 + (lane & 15);
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      float w0[16], w1[16];
      const int c0 = 64 * hb + 32 * part;
      tc::ld16(tl + TC_W + c0, w0);
      tc::ld16(tl + TC_W + c0 + 16, w1);
      tc::ld_wait();
      if (lane < 16) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          *reinterpret_cast<float4*>(sm + P_WST + tc::sw128(t, c0 + 4 * j, 64)) =
              make_float4(tc::to_tf32(-w0[4 * j]), tc::to_tf32(-w0[4 * j + 1]), tc::to_tf32(-w0[4 * j + 2]),
                          tc::to_tf32(-w0[4 * j + 3]));
          *reinterpret_cast<float4*>(sm + P_WST + tc::sw128(t, c0 + 16 + 4 * j, 64)) =
              make_float4(tc::to_tf32(-w1[4 * j]), tc::to_tf32(-w1[4 * j + 1]), tc::to_tf32(-w1[4 * j + 2]),
                          tc::to_tf32(-w1[4 * j + 3]));
        }
      }
    }
  }
  tc::fence_async_smem();
  tc::fence_before();
  __syncthreads();  // TMEM columns and shared regions are reused by the next item
  tc::fence_after();
  if (tid == 0) {
#pragma unroll
    for (int sl = 0; sl < 4; ++sl)
      tc::bulk_s2g(rec + REC_RA + sl * 16384 + wrow0 * 128, sm + P_WST + sl * 8192, 8192);
    tc::bulk_commit();
    pending = item;
  }
  }  // item loop
  if (tid == 0 && pending >= 0) publish(pending);
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem_base, 256);
}

}  // namespace kda
