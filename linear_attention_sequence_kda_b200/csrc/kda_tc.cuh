// Blackwell (sm_100a) tensor-core helpers: tcgen05 MMA (kind::tf32), tensor
// memory (TMEM) allocation / loads / stores, shared-memory matrix descriptors,
// mbarriers with bounded waits, and bulk (non-tensor) async copies.
//
// Operand tiles in shared memory use the K-major, 128-byte-swizzled canonical
// layout for 32-bit elements: a tile of R rows (R % 8 == 0) and K columns is
// split into K/32 "slabs" of 32 columns; slab s occupies R * 128 contiguous
// bytes starting 1024-byte aligned; inside a slab row r is 128 bytes at
// r * 128 whose 16-byte chunk j is stored at chunk position j ^ (r % 8).  The
// hardware applies that XOR on address bits [4,7) ^ [7,10), so a descriptor
// may start at slab base + 32 * kstep bytes for the kstep-th 8-column step.
#pragma once
#include <cuda.h>
#include <stdint.h>

#include "kda_common.cuh"

namespace kda {
namespace tc {

// Default bound of a device-side wait, in nanoseconds of %globaltimer: four
// seconds.  Waits on another kernel's progress take a bound computed by the
// host for the problem at hand instead.
constexpr uint64_t kWaitNs = 4000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// byte offset of element (r, k) in a K-major SW128 tile of 32-bit elements
__host__ __device__ __forceinline__ uint32_t sw128(int r, int k, int R) {
  const int slab = k >> 5, kc = k & 31, c = kc >> 2;
  return (uint32_t)(slab * (R * 128) + r * 128 + ((c ^ (r & 7)) << 4) + ((kc & 3) << 2));
}

// the same offset for row rb + r where rb is a multiple of 8, so that the
// swizzle phase of the row is r % 8: with r a compile-time constant (unrolled
// loops) the row-dependent part folds into an immediate and one XOR
__host__ __device__ __forceinline__ uint32_t sw128o(int rb, int r, int k, int R) {
  const int slab = k >> 5, c = (k >> 2) & 7;
  return (uint32_t)(slab * (R * 128) + rb * 128 + r * 128 + ((c ^ (r & 7)) << 4) + ((k & 3) << 2));
}

// 2^x on the special-function unit (PTX ex2.approx, relative error ~2^-22)
__device__ __forceinline__ float exp2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// shared-memory matrix descriptor: SW128 K-major, SBO = 1024 B (8 rows x 128 B)
__device__ __forceinline__ uint64_t desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// descriptor of k-step `ks` (8 columns) of a tile with R rows at `base`
__device__ __forceinline__ uint64_t desc_k(uint32_t base, int R, int ks) {
  return desc(base + (uint32_t)((ks >> 2) * R * 128 + (ks & 3) * 32));
}
// the same as a constant added to desc(base): k-step ks of an R-row tile
// starts (ks / 4) slabs and (ks % 4) * 32 bytes further (address field is in
// 16-byte units and never overflows for shared-memory addresses)
__host__ __device__ constexpr uint64_t desc_step(int R, int ks) {
  return (uint64_t)(((ks >> 2) * R * 128 + (ks & 3) * 32) >> 4);
}

// instruction descriptor, kind::tf32, fp32 accumulate, both operands K-major
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, int neg_b = 0) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)neg_b << 14) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, int acc) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, int acc) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// make generic-proxy shared-memory writes visible to the tensor core (async proxy)
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---- TMEM ------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, int ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols));
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, int ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}

// 32 lanes x 16 columns of 32-bit: thread `lane` of the warp receives row
// (32 * (warp % 4) + lane), columns [col, col + 16).
__device__ __forceinline__ void ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// 32 lanes x 8 columns (same lane mapping as ld16)
__device__ __forceinline__ void ld8(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void st8(uint32_t taddr, const float* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
               "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
               "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
               : "memory");
}
__device__ __forceinline__ void ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// round an fp32 value to tf32 (nearest, ties away from zero); the low 13 bits
// become 0.  Adding half a tf32 unit (bit 12) to the magnitude bits and
// clearing the low 13 bits rounds the magnitude, carrying into the exponent
// (and to infinity past the largest finite value) exactly as rounding does;
// two integer instructions instead of a conversion on the quarter-rate pipe.
__device__ __forceinline__ float to_tf32(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

// ---- mbarriers ---------------------------------------------------------------
__device__ __forceinline__ void bar_init(uint64_t* bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void bar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void bar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool try_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait on phase parity.  Returns false (and records KDA_ERR_TIMEOUT in
// the device status word) if the phase did not complete within `limit_ns`
// nanoseconds.
__device__ __forceinline__ bool bar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns = kWaitNs) {
  const uint32_t a = smem_u32(bar);
  if (try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (try_wait(a, parity)) return true;
    if ((it & 255) == 0 && globaltimer() - t0 > limit_ns) break;
  }
  set_status(KDA_ERR_TIMEOUT);
  return false;
}

// Bounded wait that also gives up (without recording a status) once `*abort`
// is nonzero: another role of the block has already failed and will not
// produce what is awaited.
__device__ __forceinline__ bool bar_wait_or(uint64_t* bar, uint32_t parity, const volatile int* abort,
                                            uint64_t limit_ns = kWaitNs) {
  const uint32_t a = smem_u32(bar);
  if (try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (try_wait(a, parity)) return true;
    if ((it & 255) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > limit_ns) break;
    }
  }
  set_status(KDA_ERR_TIMEOUT);
  return false;
}
// Wait until another kernel publishes *flag != 0 (acquire at GPU scope), then
// order this thread's later bulk copies (async proxy) after that acquire, so
// that they read what the flag's writer stored before it.  Bounded: gives up
// after `limit_ns` nanoseconds (recording KDA_ERR_TIMEOUT), or without a
// status once `*abort` is set by another role of the block.
__device__ __forceinline__ bool flag_wait_or(const int* flag, const volatile int* abort, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 0;; ++it) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v) {
      asm volatile("fence.proxy.async.global;" ::: "memory");
      return true;
    }
    if ((it & 63) == 63) {
      if (*abort) return false;
      if (globaltimer() - t0 > limit_ns) break;
    }
    __nanosleep(64);
  }
  set_status(KDA_ERR_TIMEOUT);
  return false;
}
// plain arrival (release) on an mbarrier
__device__ __forceinline__ void bar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 2D tiled tensor copy global -> shared through a tensor map (TMA); (x, y) =
// (inner column, row) of the box origin, x * element size a multiple of 16 B.
// Rows outside the tensor (including negative y) are filled with zeros.
__device__ __forceinline__ void tma_load_2d(void* dst_smem, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst_smem)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 2D tiled tensor store shared -> global through a tensor map (bulk-group
// completion); the box must lie inside rows the caller owns
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int x, int y, const void* src_smem) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(smem_u32(src_smem))
               : "memory");
}

// bulk async copy shared -> global (bulk-group completion); both addresses
// 16-byte aligned, size a multiple of 16
__device__ __forceinline__ void bulk_s2g(void* dst, const void* src_smem, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src_smem)), "r"(bytes)
               : "memory");
}
// Per-thread asynchronous copy global -> shared of 4 or 8 bytes (both
// addresses aligned to the size); completion is awaited by the same thread
// with async_wait_all.
template <int BYTES>
__device__ __forceinline__ void async_copy(void* dst_smem, const void* src) {
  static_assert(BYTES == 4 || BYTES == 8, "cp.async.ca copies 4, 8 or 16 bytes");
  asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(smem_u32(dst_smem)), "l"(src), "n"(BYTES)
               : "memory");
}
__device__ __forceinline__ void async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until every committed bulk store of this thread has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// wait until every committed bulk store of this thread is complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// order completed bulk (async-proxy) global writes before this thread's later generic accesses
__device__ __forceinline__ void fence_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// hint: bring `bytes` (multiple of 16) of global memory at `src` into L2
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// bulk async copy global -> shared, completion signalled on `bar` (tx bytes)
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

}  // namespace tc
}  // namespace kda
