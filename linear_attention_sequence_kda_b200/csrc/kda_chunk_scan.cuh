// Chunk scan (the state-dependent half of the chunked KDA prefill): one thread
// block per (segment, head), serial over the segment's chunks, the 128 x 128
// fp32 state held in tensor memory the whole time (page "GLM-5.3-Flash im
// Detail", section "Sequenz-Mixing: 34 KDA-Schichten mit festem Zustand": a
// state is handed from chunk to chunk).
//
// Thread v (of 128) owns value column v: TMEM lane v holds row v of
//   V^T (cols 0..63) | S^T (cols 64..191) | U^T (192..255) | O^T (256..319)
// (tf32 MMA operands), in fp32 V^T (320..383) and U^T (384..447), and a second
// O^T buffer (448..511): chunk i's output is finalised while chunk i+1's first
// MMA group runs.
// Per chunk, with the record written by chunk_prep_kernel:
//   MMA1  U^T = [V^T | S^T] [T_s | -W]^T        (K = 64 + 128)
//         O^T = S^T Q~^T                          (K = 128)
//   fp32  U^T += beta * V^T (diagonal of T);  S^T <- S^T diag(e^{Gamma_C})
//   MMA2  O^T += U^T P_s^T;   S^T += U^T K-bar    (K = 64, A = U^T from TMEM)
//   fp32  o = O + P_tt u (diagonal of P), written to HBM.
// A operands are read from TMEM as tf32; the state itself stays fp32.
//
// Data movement: the raw value tile of chunk i+2 (TMA, 64 rows x 256 B) and the
// record halves of chunk i+1 (bulk copies) are in flight while chunk i runs;
// each record half is refilled as soon as the MMA group that reads it is done.
// The output rows of a chunk are staged in shared memory and leave with one
// TMA tensor store (full chunks) or one bulk store per valid row (a segment's
// last, partial chunk: rows past the segment end are never written).
#pragma once
#include "kda_chunk_prep.cuh"
#include "kda_common.cuh"
#include "kda_tc.cuh"

namespace kda {

constexpr uint32_t VT_BYTES = CH * D * 2;            // raw value tile (bf16)
constexpr uint32_t SCAN_A = 0;                       // record part A: B1 | QT (81920 B)
constexpr uint32_t SCAN_B = REC_TILES_A;             // record part B: PS | KB | SC (50176 B)
constexpr uint32_t SCAN_V0 = REC_TILES_A + REC_TILES_B;
constexpr uint32_t SCAN_V1 = SCAN_V0 + VT_BYTES;
constexpr uint32_t SCAN_O = SCAN_V1 + VT_BYTES;      // output staging [64 t][128] (fp32 or bf16)
constexpr uint32_t SCAN_SMEM = SCAN_O + CH * D * 4 + 1024;
constexpr int TM_V = 0, TM_S = 64, TM_U = 192;
constexpr int TM_VX = 320, TM_UX = 384;  // exact fp32 V and U for the diagonal terms
constexpr int TM_O0 = 256, TM_O1 = 448;  // output accumulators, alternating by chunk
__device__ __forceinline__ int o_col(int chunk) { return (chunk & 1) ? TM_O1 : TM_O0; }

template <typename Tout, int ACT>
__global__ void __launch_bounds__(128, 1)
chunk_scan_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const float* __restrict__ conv_w,
                  const float* init_state, const __nv_bfloat16* __restrict__ init_conv,
                  const int32_t* __restrict__ cu, const int32_t* __restrict__ chunk_base,
                  const int32_t* __restrict__ seq_order, int H, const uint8_t* __restrict__ records,
                  Tout* __restrict__ o, float* final_state) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t bar_a, bar_b, bar_v[2], bar_m1, bar_m2;
  __shared__ uint32_t tmem_base;
  __shared__ float scb[2][256];  // per chunk parity: beta[64], P_tt[64], e^{Gamma_C}[128]

  const int tid = threadIdx.x, warp = tid >> 5;
  const int n = seq_order[blockIdx.x / H], h = blockIdx.x % H;
  const int64_t seg0 = cu[n], T = cu[n + 1] - seg0;
  const int nchunks = (int)((T + CH - 1) / CH);
  const int64_t HD = (int64_t)H * D;
  const int64_t chan = (int64_t)h * D + tid;
  const uint8_t* rec0 = records + (int64_t)chunk_base[n] * H * REC_BYTES + (int64_t)h * REC_BYTES;
  const int64_t rec_stride = (int64_t)H * REC_BYTES;  // next chunk of the same head

  if (warp == 0) tc::tmem_alloc(&tmem_base, 512);
  if (tid == 0) {
    tc::bar_init(&bar_a, 1); tc::bar_init(&bar_b, 1);
    tc::bar_init(&bar_v[0], 1); tc::bar_init(&bar_v[1], 1);
    tc::bar_init(&bar_m1, 1); tc::bar_init(&bar_m2, 1);
    tc::bar_init_fence();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tm = tmem_base;
  const uint32_t lane_base = tm + ((uint32_t)(32 * warp) << 16);

  // initial state: row v of S^T = column v of S
  {
    const float* Si = init_state ? init_state + ((int64_t)n * H + h) * D * D + tid : nullptr;
    for (int g16 = 0; g16 < 8; ++g16) {
      float s[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) s[i] = Si ? Si[(int64_t)(16 * g16 + i) * D] : 0.f;
      tc::st16(lane_base + TM_S + 16 * g16, s);
    }
  }
  // value conv taps and history for channel tid
  const float4 wv = load4(conv_w + (2 * HD + chan) * 4);
  float hv0 = 0.f, hv1 = 0.f, hv2 = 0.f;
  if (init_conv) {
    const __nv_bfloat16* c = init_conv + ((int64_t)n * 9 + 6) * HD + chan;
    hv0 = to_f(c[0]); hv1 = to_f(c[HD]); hv2 = to_f(c[2 * HD]);
  }

  // issued counts per barrier (uniform across the block) for the exit drain
  int a_iss = 0, b_iss = 0, v_iss[2] = {0, 0}, m2 = 0;
  auto load_a = [&](int i) {
    tc::bar_expect_tx(&bar_a, REC_TILES_A);
    tc::bulk_g2s(sm + SCAN_A, rec0 + (int64_t)i * rec_stride, REC_TILES_A, &bar_a);
  };
  auto load_b = [&](int i) {
    tc::bar_expect_tx(&bar_b, REC_TILES_B);
    tc::bulk_g2s(sm + SCAN_B, rec0 + (int64_t)i * rec_stride + REC_PS, REC_TILES_B, &bar_b);
  };
  auto load_v = [&](int i) {
    tc::bar_expect_tx(&bar_v[i & 1], VT_BYTES);
    tc::tma_load_2d(sm + ((i & 1) ? SCAN_V1 : SCAN_V0), &tm_v, h * D, (int)(seg0 + (int64_t)CH * i),
                    &bar_v[i & 1]);
  };
  if (nchunks > 0) {
    if (tid == 0) {
      load_a(0);
      load_b(0);
      load_v(0);
      if (nchunks > 1) load_v(1);
    }
    a_iss = b_iss = 1; v_iss[0] = 1; v_iss[1] = nchunks > 1;
  }
  const uint64_t d_b1 = tc::desc(tc::smem_u32(sm + SCAN_A));
  const uint64_t d_qt = tc::desc(tc::smem_u32(sm + SCAN_A + REC_QT));
  const uint64_t d_ps = tc::desc(tc::smem_u32(sm + SCAN_B));
  const uint64_t d_kb = tc::desc(tc::smem_u32(sm + SCAN_B + (REC_KB - REC_PS)));

  // o = O + P_tt u for chunk j (O in its TMEM buffer, exact U still in UX):
  // staged as [t][v] rows in shared memory, then one tensor store (full chunk)
  // or one bulk store per valid row
  Tout* ost = reinterpret_cast<Tout*>(sm + SCAN_O);
  auto finalize = [&](int j) {
    const int Lj = (int)((T - (int64_t)CH * j) < CH ? (T - (int64_t)CH * j) : CH);
    const int64_t tj = seg0 + (int64_t)CH * j;
    const float* scj = scb[j & 1];
#pragma unroll
    for (int g16 = 0; g16 < 4; ++g16) {
      float r[16], ux[16];
      tc::ld16(lane_base + o_col(j) + 16 * g16, r);
      tc::ld16(lane_base + TM_UX + 16 * g16, ux);
      tc::ld_wait();
#pragma unroll
      for (int jj = 0; jj < 16; ++jj)
        ost[(16 * g16 + jj) * D + tid] = from_f<Tout>(fmaf(scj[64 + 16 * g16 + jj], ux[jj], r[jj]));
    }
    tc::fence_async_smem();
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (tid == 0) {
      if (Lj == CH)
        tc::tma_store_2d(&tm_o, h * D, (int)tj, ost);
      else
        for (int t = 0; t < Lj; ++t) tc::bulk_s2g(o + (tj + t) * HD + (int64_t)h * D, ost + t * D, D * sizeof(Tout));
      tc::bulk_commit();
    }
  };

  bool ok = true;
  for (int i = 0; i < nchunks && ok; ++i) {
    const int L = (int)((T - (int64_t)CH * i) < CH ? (T - (int64_t)CH * i) : CH);
    const int64_t t0 = seg0 + (int64_t)CH * i;

    // (a) causal conv of v for this chunk; V^T row into TMEM (tf32 and fp32)
    ok &= tc::bar_wait(&bar_v[i & 1], (i >> 1) & 1);
    {
      const __nv_bfloat16* vt = reinterpret_cast<const __nv_bfloat16*>(sm + ((i & 1) ? SCAN_V1 : SCAN_V0));
#pragma unroll
      for (int g16 = 0; g16 < 4; ++g16) {
        float vv[16], r[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int t = 16 * g16 + j;
          const float x = to_f(vt[t * D + tid]);
          float y = conv4(wv, hv0, hv1, hv2, x);
          if (ACT == KDA_CONV_SILU) y = silu(y);
          hv0 = hv1; hv1 = hv2; hv2 = x;
          vv[j] = t < L ? y : 0.f;
          r[j] = tc::to_tf32(vv[j]);
        }
        tc::st16(lane_base + TM_V + 16 * g16, r);
        tc::st16(lane_base + TM_VX + 16 * g16, vv);
      }
    }
    tc::st_wait();
    // (b) this chunk's record
    float* sc = scb[i & 1];
    ok &= tc::bar_wait(&bar_a, i & 1);
    ok &= tc::bar_wait(&bar_b, i & 1);
    sc[tid] = reinterpret_cast<const float*>(sm + SCAN_B + (REC_SC - REC_PS))[tid];
    sc[tid + 128] = reinterpret_cast<const float*>(sm + SCAN_B + (REC_SC - REC_PS))[tid + 128];
    if (tid == 0) tc::bulk_wait_read();  // the previous output store has read the staging tile
    tc::fence_before();
    ok = __syncthreads_and(ok);
    if (!ok) break;
    // (c) MMA group 1; the value tile buffer is free again
    if (tid == 0) {
      tc::fence_after();
#pragma unroll
      for (int ks = 0; ks < 24; ++ks)
        tc::mma_ts(tm + TM_U, tm + TM_V + 8 * ks, d_b1 + tc::desc_step(64, ks), tc::idesc_tf32(128, 64), ks > 0);
#pragma unroll
      for (int ks = 0; ks < 16; ++ks)
        tc::mma_ts(tm + o_col(i), tm + TM_S + 8 * ks, d_qt + tc::desc_step(64, ks), tc::idesc_tf32(128, 64),
                   ks > 0);
      tc::commit(&bar_m1);
      if (i + 2 < nchunks) load_v(i + 2);
    }
    if (i + 2 < nchunks) v_iss[i & 1]++;
    // while MMA group 1 runs: finish the previous chunk's output
    if (i > 0) finalize(i - 1);
    ok &= tc::bar_wait(&bar_m1, i & 1);
    tc::fence_after();
    if (!__syncthreads_and(ok)) { ok = false; break; }
    if (i + 1 < nchunks) {  // record part A is free again
      if (tid == 0) load_a(i + 1);
      a_iss++;
    }
    // (d) U += beta V (exact diagonal of T V), S^T <- S^T diag(gamma)
#pragma unroll
    for (int g16 = 0; g16 < 4; ++g16) {
      float r[16], vx[16], ux[16];
      tc::ld16(lane_base + TM_U + 16 * g16, r);
      tc::ld16(lane_base + TM_VX + 16 * g16, vx);
      tc::ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        ux[j] = fmaf(sc[16 * g16 + j], vx[j], r[j]);
        r[j] = tc::to_tf32(ux[j]);
      }
      tc::st16(lane_base + TM_U + 16 * g16, r);
      tc::st16(lane_base + TM_UX + 16 * g16, ux);
    }
#pragma unroll
    for (int g16 = 0; g16 < 8; g16 += 2) {
      float r0[16], r1[16];
      tc::ld16(lane_base + TM_S + 16 * g16, r0);
      tc::ld16(lane_base + TM_S + 16 * g16 + 16, r1);
      tc::ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        r0[j] *= sc[128 + 16 * g16 + j];
        r1[j] *= sc[128 + 16 * g16 + 16 + j];
      }
      tc::st16(lane_base + TM_S + 16 * g16, r0);
      tc::st16(lane_base + TM_S + 16 * g16 + 16, r1);
    }
    tc::st_wait();
    tc::fence_before();
    __syncthreads();
    // (e) MMA group 2
    if (tid == 0) {
      tc::fence_after();
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        tc::mma_ts(tm + o_col(i), tm + TM_U + 8 * ks, d_ps + tc::desc_step(64, ks), tc::idesc_tf32(128, 64), 1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        tc::mma_ts(tm + TM_S, tm + TM_U + 8 * ks, d_kb + tc::desc_step(128, ks), tc::idesc_tf32(128, 128), 1);
      tc::commit(&bar_m2);
    }
    ++m2;
    ok &= tc::bar_wait(&bar_m2, i & 1);
    tc::fence_after();
    if (!__syncthreads_and(ok)) { ok = false; break; }
    if (i + 1 < nchunks) {  // record part B is free again
      if (tid == 0) load_b(i + 1);
      b_iss++;
    }
  }
  if (ok && nchunks > 0) finalize(nchunks - 1);

  if (!ok) {
    // a wait gave up (status already recorded): drain what is still in flight
    // (each wait bounded; waiting on the parity of a completed phase returns at
    // once) so that TMEM and shared memory are idle before exit
    if (tid == 0) tc::commit(&bar_m2);
    tc::bar_wait(&bar_m2, m2 & 1);
    if (a_iss > 0) tc::bar_wait(&bar_a, (a_iss - 1) & 1);
    if (b_iss > 0) tc::bar_wait(&bar_b, (b_iss - 1) & 1);
    for (int b = 0; b < 2; ++b)
      if (v_iss[b] > 0) tc::bar_wait(&bar_v[b], (v_iss[b] - 1) & 1);
  }
  if (tid == 0) tc::bulk_wait_all();  // output rows are in global memory before exit
  // final state: column v of S = row v of S^T
  if (ok) {
    float* Sf = final_state + ((int64_t)n * H + h) * D * D + tid;
    for (int g16 = 0; g16 < 8; ++g16) {
      float s[16];
      tc::ld16(lane_base + TM_S + 16 * g16, s);
      tc::ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) Sf[(int64_t)(16 * g16 + i) * D] = s[i];
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tm, 512);
}

}  // namespace kda
