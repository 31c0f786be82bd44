// Chunk preparation (the state-independent half of the chunked KDA prefill):
// for every chunk of every (segment, head), in parallel, the record of
// kda_record.cuh.  Page "GLM-5.3-Flash im Detail", section "Sequenz-Mixing:
// 34 KDA-Schichten mit festem Zustand": prefill evaluates the tokens of a chunk
// in parallel and hands a state from chunk to chunk.
//
// Normalisation is deferred (kda_record.cuh): every per-element tile is built
// from the raw short-conv outputs y_q, y_k; the reciprocal norms r^q, r^k only
// scale 64-element vectors and 64 x 64 matrices.  Each element of q and k is
// thus touched once, by one pass that convolves, accumulates the gate and
// writes all of its scaled copies.
//
// Gram blocks without overflow: the chunk is split into two 32-row halves with
// reference rows m_0 = 16, m_1 = 48 (G = Gamma * log2 e, cumulative gate in
// base-2 units).  For i in half I and j <= i,
//   2^{G_i - G_j} = 2^{G_i - G_{m_I}} * 2^{G_{m_I} - G_j}
// where |G_i - G_{m_I}| <= 17 * 5 * log2 e < 123 (fp32 and tf32 reach 2^127)
// and 2^{G_{m_I} - G_j} <= 1 for j in an earlier half.  One tensor-core product
// gives both Grams, D = [Bq ; Bk] GA^T (M = 128, N = 96, K = 128 channels):
//   A rows   0..63  y^q_i 2^{G_i - G_{m(i)}}       (Bq)
//            64..127 y^k_i 2^{G_i - G_{m(i)}}      (Bk)
//   B rows   0..31  y^k_j 2^{G_{m_0} - G_j}, j = 0..31   (GA)
//            32..95 y^k_j 2^{G_{m_1} - G_j}, j = 0..63
// so that p_ij = D[i][j] (i < 32) or D[i][32 + j] (i >= 32), and m_ij likewise
// in rows 64 + i.
//
// The tiles of the 128 channels are built in two passes of 64 channels (the
// Gram accumulates over both), which keeps the shared-memory footprint small
// enough for two blocks per SM.  In a pass, lane l of warp w owns channels
// 4 (l % 16) .. + 3 of the pass and rows 8 w + 4 (l / 16) .. + 3: its global
// loads, packed products and 16-byte stores each cover four channels.
//
// After the Gram: the unit lower triangular X = (I + L)^-1 with
// L = diag(beta) Dk m Dk (blocked fp32 solve), T = X diag(beta),
// TS = Dk T (record) and T2 = Dk T Dk; the Bk rows are rescaled to
// K~' = y_k 2^G = Bk * 2^{G_{m(s)}} (into the Bq rows, no longer needed) and
// W' = T2 K~' is one more product that reads K~' as an MN-major operand (its
// channel index contiguous).
#pragma once
#include "kda_common.cuh"
#include "kda_record.cuh"
#include "kda_tc.cuh"

namespace kda {

constexpr int PREP_THREADS = 256;
// shared memory plan (bytes from a 1024-aligned base)
constexpr uint32_t P_AA = 0;                 // pass 0 [Bq ; Bk]: 2 slabs x (128 rows x 128 B)
constexpr uint32_t P_AB = 32768;             // pass 1 (K~' after the Gram: rows 64.. of both)
constexpr uint32_t P_GA = 65536;             // GA: 2 slabs x (96 rows x 128 B), reused per pass
constexpr uint32_t GA_ROWS = 96;
constexpr uint32_t GA_SLAB = GA_ROWS * 128;  // 12288
constexpr uint32_t P_MS = P_GA;              // after the Gram: solve matrix [64][MS_LD] fp32
constexpr uint32_t MS_LD = 68;               // rows 16-byte aligned, columns over all banks
constexpr uint32_t P_T2 = P_GA;              // after the solve: T2, slabs of 128 rows (0..63 used)
constexpr uint32_t P_TMP = 90112;            // solve blocks of X
constexpr uint32_t TMP_BYTES = (96 * 20 + 32 * 36 + 16) * 4;
constexpr uint32_t P_MISC = P_TMP + ((TMP_BYTES + 255) & ~255u);
// scalar region (floats)
constexpr int MB_XCH = 0;      // per pass [10][64]: warp totals of the gate, rows 16 and 48 (local)
constexpr int MB_NQ = 1280, MB_NK = 1344, MB_NX = 1408;  // row sums |y_q|^2, |y_k|^2, y_q . y_k
constexpr int MB_BETA = 1472, MB_RK = 1536;
constexpr int MB_FLOATS = 1600;
constexpr uint32_t PREP_SMEM = P_MISC + MB_FLOATS * 4 + 1024;
static_assert(P_MS + 64 * MS_LD * 4 <= P_TMP, "solve matrix overlaps the solve blocks");
static_assert(P_GA + 2 * GA_SLAB <= P_TMP, "GA overlaps the solve blocks");
static_assert(P_T2 + 16384 + 128 * 128 <= P_MISC, "the M = 128 read of T2 leaves the scratch regions");
static_assert(2 * (PREP_SMEM + 128) <= 233472, "two blocks per SM");

// TMEM columns
constexpr int TC_G = 0;  // Gram accumulator (96 columns)
constexpr int TC_W = 0;  // W accumulator (128 columns), after the Gram has been read

// Shared-memory matrix descriptor of an MN-major operand of 32-bit elements.
// For tf32 the tensor core reads MN-major tiles only in the 128-byte swizzle
// with 32-byte granules ("128B, base 32B"): rows of 128 bytes (32 MN-adjacent
// elements), 4 K-rows per 512-byte atom, and in K-row r the 32-byte granule j
// stored at granule position j ^ (r % 4).  Atoms of 32 MN elements are `lbo`
// bytes apart, atoms of 4 K-rows `sbo` bytes apart.
__device__ __forceinline__ uint64_t desc_mn32(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | ((uint64_t)1 << 46) | ((uint64_t)1 << 61);
}

// four bf16 (8 bytes, 8-byte aligned) -> float4
__device__ __forceinline__ float4 bf4(uint2 u) {
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xFFFF0000u));
}
__device__ __forceinline__ uint2 ldg8(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const uint2*>(p)); }
// conv taps of four channels, re-read (from L1) where they are used rather
// than held in registers across a loop: an opaque load that the compiler
// neither hoists nor merges
__device__ __forceinline__ void taps4(const float* p, float4 (&w)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(w[j].x), "=f"(w[j].y), "=f"(w[j].z), "=f"(w[j].w)
                 : "l"(p + 4 * j));
}
__device__ __forceinline__ float4 ex2_4(float4 x) {
  return make_float4(tc::exp2_fast(x.x), tc::exp2_fast(x.y), tc::exp2_fast(x.z), tc::exp2_fast(x.w));
}
__device__ __forceinline__ float4 add4(float4 a, float4 b) { return cat2(add2(lo2(a), lo2(b)), add2(hi2(a), hi2(b))); }
__device__ __forceinline__ float4 sub4(float4 a, float4 b) { return make_float4(a.x - b.x, a.y - b.y, a.z - b.z, a.w - b.w); }
__device__ __forceinline__ float4 mul4(float4 a, float4 b) { return cat2(mul2(lo2(a), lo2(b)), mul2(hi2(a), hi2(b))); }
__device__ __forceinline__ float4 tf32_4(float4 a) {
  return make_float4(tc::to_tf32(a.x), tc::to_tf32(a.y), tc::to_tf32(a.z), tc::to_tf32(a.w));
}
__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, a.x * b.x)));
}
// causal width-4 conv of four channels: taps w[c] (tap 3 = current token)
template <int ACT>
__device__ __forceinline__ float4 conv4x4(const float4 (&w)[4], float4 x0, float4 x1, float4 x2, float4 x3) {
  float4 y = make_float4(conv4(w[0], x0.x, x1.x, x2.x, x3.x), conv4(w[1], x0.y, x1.y, x2.y, x3.y),
                         conv4(w[2], x0.z, x1.z, x2.z, x3.z), conv4(w[3], x0.w, x1.w, x2.w, x3.w));
  if (ACT == KDA_CONV_SILU) y = make_float4(silu(y.x), silu(y.y), silu(y.z), silu(y.w));
  return y;
}

// Unit lower triangular X = (I + L)^-1 of a 64 x 64 strictly lower L held in
// Ms (row stride MS_LD), by blocks of the 2 x 2 partitions, each
// X_ba = -X_bb L_ba X_aa:
//   A  the four diagonal 16-blocks, by forward substitution   -> Xd[I]
//   B  the off-diagonal 16-block of each 32-half               -> XB[P]
//   C  the off-diagonal 32-block                               -> XC
// Results go to their own buffers, so each stage needs one barrier.  Within B
// and C a thread group computes a column of the intermediate product L X_aa and
// shares it by shuffles before multiplying by X_bb.  Row strides of 20 (36)
// floats put 8 consecutive rows of a block in 8 distinct 4-bank groups, so the
// float4 row loads are conflict-free.
constexpr int XS = 20, XCS = 36;
__device__ __forceinline__ void solve_unit_lower(const float* Ms, float* Xd, int tid, int warp, int lane) {
  float* XB = Xd + 4 * 16 * XS;  // [2][16][XS]
  float* XC = XB + 2 * 16 * XS;  // [32][XCS]
  float* Zr = XC + 32 * XCS;     // [16] zeros
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
    float xc[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) xc[m] = X0[m * XS + cc];
    float y[2];
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
    float yc[16];
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
    float yc[32];
    const int base = lane & ~7;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
#pragma unroll
      for (int u = 0; u < 4; ++u) yc[kk + 8 * u] = __shfl_sync(0xffffffffu, y[u], base + kk);
    // X_11 row r = [Xd2 row r, 0] (r < 16) or [XB1 row r - 16, Xd3 row r - 16]
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = k + 8 * u;
      const float* ra = u < 2 ? Xd + (32 + r) * XS : XB + r * XS;
      const float* rb = u < 2 ? Zr : Xd + (32 + r) * XS;
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
}
// X row t, columns tp .. tp + 3 (tp % 4 == 0): from the diagonal 16-block, the
// off-diagonal 16-block of a 32-half, the off-diagonal 32-block, or zero
__device__ __forceinline__ float4 x_row4(const float* Xd, int t, int tp) {
  const float* XB = Xd + 4 * 16 * XS;
  const float* XC = XB + 2 * 16 * XS;
  const float* Zr = XC + 32 * XCS;
  const int I = t >> 4, J = tp >> 4;
  const float* src = I == J ? Xd + (I * 16 + (t & 15)) * XS + (tp & 15)
                   : (I == J + 1 && (I & 1)) ? XB + ((I >> 1) * 16 + (t & 15)) * XS + (tp & 15)
                   : (I >= 2 && J <= 1) ? XC + (t - 32) * XCS + tp
                   : Zr;
  return *reinterpret_cast<const float4*>(src);
}

template <int ACT>
__global__ void __launch_bounds__(PREP_THREADS, 2)
chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_g, const __nv_bfloat16* __restrict__ qg,
                  const __nv_bfloat16* __restrict__ kg, const __nv_bfloat16* __restrict__ gg,
                  const __nv_bfloat16* __restrict__ beta, const float* __restrict__ conv_w,
                  const __nv_bfloat16* __restrict__ init_conv, const int32_t* __restrict__ cu,
                  const int2* __restrict__ chunk_tab, int H, int n_items, uint8_t* __restrict__ records,
                  int* __restrict__ work_counter, int* __restrict__ ready, int vacate_below_smid,
                  int vacate_after) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array itself so that the
  // compiler keeps the shared address space (32-bit shared loads and stores)
  uint8_t* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  float* ms = reinterpret_cast<float*>(sm + P_MISC);
  float* Ms = reinterpret_cast<float*>(sm + P_MS);
  float* Xd = reinterpret_cast<float*>(sm + P_TMP);
  __shared__ uint64_t bar_g, bar_w;
  __shared__ uint32_t tmem_base;
  __shared__ int s_next;  // the block's next work item (claimed by thread 0)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cq = lane & 15, rh = lane >> 4;
  const int r0 = 8 * warp + 4 * rh;  // first of this thread's 4 rows
  const int hf = warp >> 2;          // 32-row half of those rows
  const int64_t HD = (int64_t)H * D;
  // swizzle phase of this thread's row r0 + r in every K-major tile: 16-byte
  // chunk (cq % 8) lands at (cq % 8) ^ (4 rh + r) = c4 ^ r
  const int c4 = (cq & 7) ^ (4 * rh);

  uint32_t smid;
  asm("mov.u32 %0, %%smid;" : "=r"(smid));
  const bool vacate = (int)smid < vacate_below_smid;
  auto claim = [&]() -> int {  // thread 0
    if (vacate && *reinterpret_cast<volatile int*>(work_counter) >= vacate_after) return n_items;
    return atomicAdd(work_counter, 1);
  };
  // bring the raw q, k, g rows of item `it` (3 halo rows + 64) into L2
  auto prefetch = [&](int it) {  // thread 0
    const int2 c = chunk_tab[it / H];
    const int y = (int)(cu[c.x] + (int64_t)CH * c.y) - 3;
    const int x = (it % H) * D;
    const int yy = y < 0 ? 0 : y;
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(&tm_q)), "r"(x), "r"(yy) : "memory");
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(&tm_k)), "r"(x), "r"(yy) : "memory");
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(&tm_g)), "r"(x), "r"(yy) : "memory");
  };

  if (warp == 0) tc::tmem_alloc(&tmem_base, 256);
  if (tid == 0) {
    tc::bar_init(&bar_g, 1); tc::bar_init(&bar_w, 1);
    tc::bar_init_fence();
    s_next = atomicAdd(work_counter, 1);  // every block takes at least one item
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tm = tmem_base;
  uint32_t par_w = 0;  // phase parity of bar_w (one product per item); bar_g completes twice per item

  for (int item = s_next; item < n_items; item = s_next, par_w ^= 1) {
  int nxt = n_items;
  if (tid == 0) {  // claim the next item now and start its raw rows on their way to L2
    nxt = claim();
    if (nxt < n_items) prefetch(nxt);
  }
  const int cid = item / H, h = item % H;
  const int2 nc = chunk_tab[cid];
  const int n = nc.x, parity = nc.y & 1;
  const int64_t seg0 = cu[n], seg1 = cu[n + 1];
  const int64_t t0 = seg0 + (int64_t)CH * nc.y;
  const int L = (int)((seg1 - t0) < CH ? (seg1 - t0) : CH);
  uint8_t* rec = records + ((int64_t)cid * H + h) * REC_BYTES;
  if (tid < CH) ms[MB_BETA + tid] = tid < L ? to_f(beta[(t0 + tid) * H + h]) : 0.f;

  float nq[4] = {0.f, 0.f, 0.f, 0.f}, nk[4] = {0.f, 0.f, 0.f, 0.f}, nx[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    const int cl = 4 * cq;              // pass-local channel of this quad
    const int c = 64 * pass + cl;       // head channel
    const int64_t chan = (int64_t)h * D + c;
    float* xch = ms + MB_XCH + pass * 640;
    uint8_t* At = sm + (pass ? P_AB : P_AA);
    // raw rows r0-3 .. r0+3 of q or k (the 3 halo rows from the conv history
    // before the segment); rows past the chunk end are not needed
    // rows of the 7 that precede the segment (3 at most, in a segment's first chunk)
    const int before = (int)(seg0 - (t0 + r0 - 3));
    auto load_rows = [&](const __nv_bfloat16* x, int tensor, uint2 (&out)[7]) {
      const __nv_bfloat16* p = x + (t0 + r0 - 3) * HD + chan;
#pragma unroll
      for (int r = 0; r < 7; ++r) {
        uint2 a = make_uint2(0u, 0u);
        if (r0 - 3 + r < L) {
          if (r >= before) a = ldg8(p + r * HD);
          else if (init_conv) a = ldg8(init_conv + ((int64_t)n * 9 + tensor * 3 + (3 - before + r)) * HD + chan);
        }
        out[r] = a;
      }
    };
    // ---- g of rows r0 .. r0+3 and the k rows; the cumulative gate ---------
    uint2 rkv[7];
    float4 G[4];
    {
      uint2 rg[4];
      const __nv_bfloat16* pg = gg + (t0 + r0) * HD + chan;
#pragma unroll
      for (int r = 0; r < 4; ++r) rg[r] = (r0 + r < L) ? ldg8(pg + r * HD) : make_uint2(0u, 0u);
      load_rows(kg, 1, rkv);
      float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float4 gr = bf4(rg[r]);
        const float4 gp = make_float4(fmaxf(gr.x, LOG_DECAY_FLOOR), fmaxf(gr.y, LOG_DECAY_FLOOR),
                                      fmaxf(gr.z, LOG_DECAY_FLOOR), fmaxf(gr.w, LOG_DECAY_FLOOR));
        run = cat2(fma2(lo2(gp), dup2(LOG2E), lo2(run)), fma2(hi2(gp), dup2(LOG2E), hi2(run)));
        G[r] = run;  // rows past the chunk end add zero (their g was not loaded)
      }
      float4 below;  // total of rows 8w .. 8w+3 (the lane of the same quad, rh = 0)
      below.x = __shfl_sync(0xffffffffu, run.x, cq);
      below.y = __shfl_sync(0xffffffffu, run.y, cq);
      below.z = __shfl_sync(0xffffffffu, run.z, cq);
      below.w = __shfl_sync(0xffffffffu, run.w, cq);
      if (rh) {
#pragma unroll
        for (int r = 0; r < 4; ++r) G[r] = add4(G[r], below);
        *reinterpret_cast<float4*>(xch + warp * 64 + cl) = G[3];
      } else if (warp == 2 || warp == 6) {  // local gate at rows 16 and 48
        *reinterpret_cast<float4*>(xch + (warp == 2 ? 512 : 576) + cl) = G[0];
      }
    }
    __syncthreads();
    // ---- absolute gates, the reference gate and the chunk's total decay ----
    float4 gm, g48, egc;
    {
      float4 pre = make_float4(0.f, 0.f, 0.f, 0.f), gC = pre, g16 = pre;
#pragma unroll
      for (int w2 = 0; w2 < 8; ++w2) {
        const float4 t = *reinterpret_cast<const float4*>(xch + w2 * 64 + cl);
        if (w2 == 2) g16 = add4(gC, *reinterpret_cast<const float4*>(xch + 512 + cl));
        if (w2 == 6) g48 = add4(gC, *reinterpret_cast<const float4*>(xch + 576 + cl));
        if (w2 < warp) pre = add4(pre, t);
        gC = add4(gC, t);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) G[r] = add4(G[r], pre);
      if (warp == 0 && rh == 0)  // gamma = e^{Gamma_C} of these channels
        *reinterpret_cast<float4*>(rec + REC_SC + (SC_G + c) * 4) = ex2_4(gC);
      gm = hf ? g48 : g16;
      egc = ex2_4(sub4(gC, g48));  // 2^{G_C - G_48} <= 1
    }
    // the second pass rewrites GA: the first pass's Gram must have read it
    if (pass == 1) tc::bar_wait(&bar_g, 0);
    const uint32_t slab = (uint32_t)(cq >> 3);
    // ---- k rows: conv, |y_k|^2, Bk, GA, K-bar' -------------------------------
    // K-bar'^T: B2 row (b2_k_row + channel), tokens r0 .. r0+3 = one 16-byte
    // chunk, written as two 8-byte halves (rows r0, r0+1 and r0+2, r0+3)
    uint8_t* kbase = rec + REC_B2 + (uint32_t)(r0 >> 5) * (B2_ROWS * 128);
    {
      float4 kb0;  // K-bar' of the even row of the current pair
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = r0 + r;
        float4 wk[4];
        taps4(conv_w + (1 * HD + chan) * 4, wk);
        float4 yk = conv4x4<ACT>(wk, bf4(rkv[r]), bf4(rkv[r + 1]), bf4(rkv[r + 2]), bf4(rkv[r + 3]));
        if (row >= L) yk = make_float4(0.f, 0.f, 0.f, 0.f);
        nk[r] += dot4(yk, yk);
        const float4 d = sub4(G[r], gm);
        const uint32_t sw = (uint32_t)(((c4 ^ r) << 4) + row * 128);  // row offset + swizzled chunk
        *reinterpret_cast<float4*>(At + slab * 16384 + 64 * 128 + sw) = mul4(yk, ex2_4(d));  // Bk row
        const float4 ga = mul4(yk, ex2_4(make_float4(-d.x, -d.y, -d.z, -d.w)));
        float4 kx;
        if (hf) {  // half 1: reference m_1 only
          *reinterpret_cast<float4*>(sm + P_GA + slab * GA_SLAB + 32 * 128 + sw) = ga;
          kx = ga;
        } else {   // half 0: own reference, and m_1 for the later half's columns
          *reinterpret_cast<float4*>(sm + P_GA + slab * GA_SLAB + sw) = ga;
          kx = mul4(yk, ex2_4(sub4(g48, G[r])));
          *reinterpret_cast<float4*>(sm + P_GA + slab * GA_SLAB + 32 * 128 + sw) = kx;
        }
        const float4 kb = tf32_4(mul4(kx, egc));  // y_k 2^{G_C - G}
        if ((r & 1) == 0) {
          kb0 = kb;
        } else {
          const int ch2 = (r0 & 31) >> 2;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int R2 = b2_k_row(parity) + c + j;
            const float* a0 = &kb0.x;
            const float* a1 = &kb.x;
            *reinterpret_cast<float2*>(kbase + R2 * 128 + ((ch2 ^ (R2 & 7)) << 4) + (r >> 1) * 8) =
                make_float2(a0[j], a1[j]);
          }
        }
      }
    }
    // ---- q rows: conv, |y_q|^2, Bq, Q~'; y_q . y_k from Bq and the own-reference
    //      GA row (y_q 2^d . y_k 2^-d) ----------------------------------------
    {
      uint2 rqv[7];
      load_rows(qg, 0, rqv);
      // 2^G = 2^{G - G_m} 2^{G_m}; half 1 in two steps (2^{G_48} may be below
      // fp32's range while 2^G is not)
      const float4 sm1 = hf ? ex2_4(make_float4(gm.x + 120.f, gm.y + 120.f, gm.z + 120.f, gm.w + 120.f))
                            : ex2_4(gm);
      const float sm2 = hf ? 7.52316384526264e-37f : 1.f;  // 2^-120
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = r0 + r;
        float4 wq[4];
        taps4(conv_w + (0 * HD + chan) * 4, wq);
        float4 yq = conv4x4<ACT>(wq, bf4(rqv[r]), bf4(rqv[r + 1]), bf4(rqv[r + 2]), bf4(rqv[r + 3]));
        if (row >= L) yq = make_float4(0.f, 0.f, 0.f, 0.f);
        nq[r] += dot4(yq, yq);
        const float4 e1 = ex2_4(sub4(G[r], gm));
        const uint32_t sw = (uint32_t)(((c4 ^ r) << 4) + row * 128);
        const float4 bq = mul4(yq, e1);
        *reinterpret_cast<float4*>(At + slab * 16384 + sw) = bq;  // Bq row
        nx[r] += dot4(bq, *reinterpret_cast<const float4*>(sm + P_GA + slab * GA_SLAB + (hf ? 32 * 128 : 0) + sw));
        float4 qt = mul4(bq, sm1);
        qt = make_float4(qt.x * sm2, qt.y * sm2, qt.z * sm2, qt.w * sm2);
        // Q~' row of the record (rows ra_q_row .. of RA; slab = channel / 32)
        *reinterpret_cast<float4*>(rec + REC_RA + (uint32_t)(c >> 5) * 16384 + ra_q_row(parity) * 128 + sw) =
            tf32_4(qt);
      }
    }
    // ---- this pass's share of the Gram --------------------------------------
    tc::fence_async_smem();
    tc::fence_before();
    __syncthreads();
    if (tid == 0) {
      tc::fence_after();
      const uint64_t da = tc::desc(tc::smem_u32(At)), db = tc::desc(tc::smem_u32(sm + P_GA));
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        tc::mma_ss(tm + TC_G, da + tc::desc_step(128, ks), db + tc::desc_step(GA_ROWS, ks),
                   tc::idesc_tf32(128, GA_ROWS), (pass | ks) ? 1 : 0);
      tc::commit(&bar_g);
    }
  }

  // ---- row norms: sums over the 16 lanes of a row group (recursive halving)
  {
    float v[16] = {nq[0], nq[1], nq[2], nq[3], nk[0], nk[1], nk[2], nk[3],
                   nx[0], nx[1], nx[2], nx[3], 0.f, 0.f, 0.f, 0.f};
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
    const int e = lane & 15;  // entry: kind e / 4 (q.q, k.k, q.k), row r0 + e % 4
    if (e < 12) ms[MB_NQ + (e >> 2) * 64 + r0 + (e & 3)] = v[0];
  }
  __syncthreads();
  // reciprocal norms and the record's scalars
  if (tid < CH) {
    const float rq = 1.0f / sqrtf(ms[MB_NQ + tid] + NORM_EPS);
    const float rk = 1.0f / sqrtf(ms[MB_NK + tid] + NORM_EPS);
    ms[MB_RK + tid] = rk;
    float* sc = reinterpret_cast<float*>(rec + REC_SC);
    sc[SC_B + tid] = rk * ms[MB_BETA + tid];
    sc[SC_D + tid] = ms[MB_NX + tid];
    sc[SC_R + tid] = rq;
  }
  tc::bar_wait(&bar_g, 1);  // the Gram is complete; every A and GA tile is free
  tc::fence_after();
  // K~' = Bk 2^{G_m} (each thread its own rows and channels), written as the
  // MN-major operand of the W product into the Bq rows, which the Gram has
  // finished with: channel slab sg (32 channels) at sg * 16384, token row s at
  // s * 128, 32-byte granule swizzled by s % 4.  Half 1 scales in two steps, so
  // that 2^{G_48} below fp32's range cannot lose contributions that are
  // themselves representable.
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int cl = 4 * cq;
    const float* xch = ms + MB_XCH + pass * 640;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w2 = 0; w2 < 6; ++w2)
      if (w2 < (hf ? 6 : 2)) acc = add4(acc, *reinterpret_cast<const float4*>(xch + w2 * 64 + cl));
    const float4 gmr = add4(acc, *reinterpret_cast<const float4*>(xch + (hf ? 576 : 512) + cl));
    const float4 s1 = hf ? ex2_4(make_float4(gmr.x + 120.f, gmr.y + 120.f, gmr.z + 120.f, gmr.w + 120.f))
                         : ex2_4(gmr);
    const float s2 = hf ? 7.52316384526264e-37f : 1.f;  // 2^-120
    uint8_t* At = sm + (pass ? P_AB : P_AA) + (uint32_t)(cq >> 3) * 16384;
    const int gran = (cq & 7) >> 1;  // 32-byte granule of the quad in its 128-byte row
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int srow = r0 + r;
      const float4 x = mul4(*reinterpret_cast<const float4*>(At + 64 * 128 + (uint32_t)(((c4 ^ r) << 4) + srow * 128)),
                            s1);
      *reinterpret_cast<float4*>(At + srow * 128 + ((gran ^ (srow & 3)) << 5) + (cq & 1) * 16) =
          make_float4(x.x * s2, x.y * s2, x.z * s2, x.w * s2);
    }
  }
  __syncthreads();  // the reciprocal norms are visible to every thread
  // p into the record (B2 rows b2_p_row + i); L = diag(beta) Dk m Dk into Ms.
  // Accumulator lane: rows 0..63 of A (q) then 64..127 (k); warp (w % 4)
  // reads lanes 32 (w % 4) ..; the two warps of a lane quarter split the columns.
  {
    const int q4 = warp & 3, wh = warp >> 2;
    const int i = 32 * (q4 & 1) + lane;       // row within the q or the k block
    const bool kside = q4 >= 2;
    const int half = q4 & 1;
    // columns of this warp: half 0 rows read j 0..31 (D cols 0..31), half 1 rows
    // j 0..63 (D cols 32..95)
    const int jn = half ? 32 : 16;            // columns per warp
    const int j0 = wh * jn;
    const uint32_t col0 = (uint32_t)(half ? 32 + j0 : j0);
    const uint32_t taddr = tm + ((uint32_t)(32 * q4) << 16) + TC_G + col0;
    const float rki = kside ? ms[MB_RK + i] : 0.f;
    const float bri = kside ? rki * ms[MB_BETA + i] : 0.f;
    for (int j16 = 0; j16 < jn; j16 += 16) {
      float v[16];
      tc::ld16(taddr + j16, v);
      tc::ld_wait();
      const int jb = j0 + j16;
      if (!kside) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = jb + 4 * u;
          float4 o;
          o.x = j + 0 < i ? tc::to_tf32(v[4 * u + 0]) : 0.f;
          o.y = j + 1 < i ? tc::to_tf32(v[4 * u + 1]) : 0.f;
          o.z = j + 2 < i ? tc::to_tf32(v[4 * u + 2]) : 0.f;
          o.w = j + 3 < i ? tc::to_tf32(v[4 * u + 3]) : 0.f;
          const int R = b2_p_row(parity) + i;
          *reinterpret_cast<float4*>(rec + REC_B2 + (uint32_t)(j >> 5) * (B2_ROWS * 128) + R * 128 +
                                     ((((j & 31) >> 2) ^ (R & 7)) << 4)) = o;
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = jb + 4 * u;
          const float4 rk4 = *reinterpret_cast<const float4*>(ms + MB_RK + j);
          float4 o;
          o.x = j + 0 < i ? bri * rk4.x * v[4 * u + 0] : 0.f;
          o.y = j + 1 < i ? bri * rk4.y * v[4 * u + 1] : 0.f;
          o.z = j + 2 < i ? bri * rk4.z * v[4 * u + 2] : 0.f;
          o.w = j + 3 < i ? bri * rk4.w * v[4 * u + 3] : 0.f;
          *reinterpret_cast<float4*>(Ms + i * MS_LD + j) = o;
        }
      }
    }
    if (!kside && half == 0 && wh == 1) {  // rows 0..31: p is zero in columns 32..63
      const int R = b2_p_row(parity) + i;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        *reinterpret_cast<float4*>(rec + REC_B2 + (B2_ROWS * 128) + R * 128 + ((u ^ (R & 7)) << 4)) =
            make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  tc::fence_before();
  __syncthreads();
  // ---- X = (I + L)^-1 -----------------------------------------------------------
  solve_unit_lower(Ms, Xd, tid, warp, lane);
  // ---- T = X diag(beta): record TS = Dk T (strictly lower); T2 = Dk T Dk ---------
  for (int e = tid; e < CH * 16; e += PREP_THREADS) {  // (row t, 4-column group)
    const int t = e >> 4, tp = 4 * (e & 15);
    const float4 xr = x_row4(Xd, t, tp);
    const float* xrp = &xr.x;
    const float rkt = ms[MB_RK + t];
    float4 t1, t2;
    float* t1p = &t1.x;
    float* t2p = &t2.x;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int s = tp + u;
      const float x = s < t ? xrp[u] : (s == t ? 1.f : 0.f);
      const float tv = rkt * x * ms[MB_BETA + s];
      t1p[u] = s < t ? tc::to_tf32(tv) : 0.f;
      t2p[u] = tc::to_tf32(tv * ms[MB_RK + s]);
    }
    const uint32_t off = (uint32_t)(t * 128 + ((((tp & 31) >> 2) ^ (t & 7)) << 4));
    *reinterpret_cast<float4*>(rec + REC_TS + (uint32_t)(tp >> 5) * 8192 + off) = t1;
    *reinterpret_cast<float4*>(sm + P_T2 + (uint32_t)(tp >> 5) * 16384 + off) = t2;
  }
  tc::fence_async_smem();
  tc::fence_before();
  __syncthreads();
  // ---- W' = T2 K~' (M = 128, rows 64.. unused; N = 128 channels; K = 64) ------
  if (tid == 0) {
    tc::fence_after();
    const uint64_t dt = tc::desc(tc::smem_u32(sm + P_T2));
    const uint64_t dk = desc_mn32(tc::smem_u32(sm + P_AA), 16384, 512);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
      tc::mma_ss(tm + TC_W, dt + tc::desc_step(128, ks), dk + (uint64_t)((ks * 8 * 128) >> 4),
                 tc::idesc_tf32(128, 128) | (1u << 16), ks > 0 ? 1 : 0);
    tc::commit(&bar_w);
  }
  tc::bar_wait(&bar_w, par_w);
  tc::fence_after();
  // -W' into the record (RA rows ra_w_row + t): lanes 0..63 = rows t
  if ((warp & 3) < 2) {
    const int t = 32 * (warp & 1) + lane;
    const int cb = 64 * (warp >> 2);  // channels of this warp
    const int R = ra_w_row(parity) + t;
#pragma unroll
    for (int c16 = 0; c16 < 64; c16 += 16) {
      float v[16];
      tc::ld16(tm + ((uint32_t)(32 * (warp & 1)) << 16) + TC_W + cb + c16, v);
      tc::ld_wait();
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int ch = cb + c16 + 4 * u;
        *reinterpret_cast<float4*>(rec + REC_RA + (uint32_t)(ch >> 5) * 16384 + R * 128 +
                                   ((((ch & 31) >> 2) ^ (R & 7)) << 4)) =
            make_float4(tc::to_tf32(-v[4 * u]), tc::to_tf32(-v[4 * u + 1]), tc::to_tf32(-v[4 * u + 2]),
                        tc::to_tf32(-v[4 * u + 3]));
      }
    }
  }
  if (tid == 0) s_next = nxt;
  tc::fence_before();
  __syncthreads();  // TMEM columns and shared regions are reused by the next item
  tc::fence_after();
  if (tid == 0 && ready) {  // publish the record: every thread's stores precede the barrier above
    __threadfence();
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(ready + item), "r"(1) : "memory");
  }
  }  // item loop
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem_base, 256);
}

}  // namespace kda
