// Chunked bf16 prefill on the tensor cores: host-side scheduling and launches.
// chunk_prep_kernel (every chunk of every (segment, head) in parallel) writes
// one operand record per chunk-head into the workspace; chunk_scan_kernel (one
// block per (segment, head), longest segments first) carries the state across
// the segment's chunks.
//
// When the scan has few chains (at most OVERLAP_MAX_CHAINS (segment, head)
// pairs, e.g. one long sequence), it leaves most SMs idle, so the two kernels
// overlap: the scan runs on an internal stream forked from and joined back to
// the caller's stream, reading each chunk's record once prep publishes its
// ready flag, and the prep blocks on the first `chains` SMs stop claiming work
// once a share of the items is handed out, so that the scan blocks get those
// SMs while prep finishes on the others.  Prep claims items from a counter and
// never waits for the scan, so the pair cannot deadlock whichever kernel's
// blocks become resident first; with more chains the two run one after the
// other on the caller's stream.
#pragma once
#include <type_traits>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <numeric>
#include <vector>

#include "kda_chunk_prep.cuh"
#include "kda_chunk_scan.cuh"
#include "kda_common.cuh"
#include "kda_tmap.cuh"

namespace kda {

// workspace = header (chunk table, per-segment first chunk, segment order),
// then REC_BYTES per (chunk, head)
inline int64_t chunk_bound(int N, int64_t total_tokens) { return total_tokens / CH + N; }
inline size_t chunk_header_bytes(int N, int64_t nchunks) {
  const size_t b = (size_t)nchunks * sizeof(int2) + (size_t)(N + 1) * 4 + (size_t)N * 4 + (size_t)(N + 1) * 4;
  return (b + 1023) & ~(size_t)1023;
}
// work counter (16 B) and one ready flag per (chunk, head)
inline size_t chunk_sync_bytes(int64_t nchunks, int H) {
  return ((size_t)16 + (size_t)nchunks * H * 4 + 1023) & ~(size_t)1023;
}
// (+128: the records start on a 128-byte line whatever the workspace's
// 16-byte alignment, so that the scan can drop whole lines of a consumed
// record from L2)
inline size_t chunked_workspace_bytes(int N, int H, int64_t total_tokens) {
  const int64_t nc = chunk_bound(N, total_tokens);
  return chunk_header_bytes(N, nc) + chunk_sync_bytes(nc, H) + 128 + (size_t)nc * H * REC_BYTES;
}

// The optional output epilogue: the gated RMS normalisation of each head's
// output row, y = o / sqrt(mean o^2 + eps) * weight * sigmoid(gate).
struct OutputNorm {
  const void* gate = nullptr;    // [total_T, H, 128] bf16, or null for plain o
  const float* weight = nullptr;  // [128] fp32
  float eps = 0.f;
};

// What a chunked call runs: both kernels (the records are dropped from L2 as
// the scan consumes them), both keeping the records in the workspace, or the
// scan alone over records a keeping call left there.
enum class ChunkedMode { kFull, kKeepRecords, kScanOnly };

constexpr int OVERLAP_MAX_CHAINS = 96;  // leaves at least 52 of 148 SMs to prep
// Prep SM-time per chunk-head relative to the scan's time per chunk of a
// chain, used to pick when prep hands SMs over to the scan (the ratio that
// gave the shortest overlapped call on B200, 64 heads x 65,536 tokens, among
// 2.8 .. 4.4; the model value from the two kernels' separate timings is ~3).
constexpr double PREP_PER_SCAN_CHUNK = 3.2;
// The same with the output epilogue fused into the scan, whose chain is slower
// per chunk, so the scan takes its SMs earlier (best among 2.0 .. 3.6: 2.0 and
// 2.4 within noise of each other, 0.3-0.5 ms shorter than at 3.2).
constexpr double PREP_PER_SCAN_CHUNK_GATED = 2.2;

// Pending host-side fault (kda_inject_fault), taken by the first call that
// applies it.
inline std::atomic<int>& pending_fault() {
  static std::atomic<int> fault{KDA_FAULT_NONE};
  return fault;
}
inline bool take_fault(kda_fault kind) {
  int expected = kind;
  return pending_fault().compare_exchange_strong(expected, KDA_FAULT_NONE);
}

// Side stream and fork / join events of the overlapped mode, one set per
// device, created on first use.  fork_side() records the fork on `stream` and
// makes the side stream wait for it under one lock, so that two host threads
// forking at once cannot make a scan wait on the other thread's stream.
struct OverlapStreams {
  std::mutex mu;
  cudaStream_t streams[64] = {};
  cudaEvent_t forks[64] = {}, joins[64] = {};
};
inline OverlapStreams& overlap_streams() {
  static OverlapStreams o;
  return o;
}
inline kda_status fork_side(cudaStream_t stream, cudaStream_t* side, cudaEvent_t* join) {
  OverlapStreams& o = overlap_streams();
  int dev = 0;
  if (!cuda_ok(cudaGetDevice(&dev)) || dev < 0 || dev >= 64) return KDA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(o.mu);
  if (!o.streams[dev]) {
    if (!cuda_ok(cudaStreamCreateWithFlags(&o.streams[dev], cudaStreamNonBlocking)) ||
        !cuda_ok(cudaEventCreateWithFlags(&o.forks[dev], cudaEventDisableTiming)) ||
        !cuda_ok(cudaEventCreateWithFlags(&o.joins[dev], cudaEventDisableTiming)))
      return KDA_ERR_CUDA;
  }
  if (!cuda_ok(cudaEventRecord(o.forks[dev], stream)) ||
      !cuda_ok(cudaStreamWaitEvent(o.streams[dev], o.forks[dev], 0)))
    return KDA_ERR_CUDA;
  *side = o.streams[dev];
  *join = o.joins[dev];
  return KDA_OK;
}
// The join is recorded and awaited under the same lock for the same reason.
inline kda_status join_side(cudaStream_t stream, cudaStream_t side, cudaEvent_t join) {
  std::lock_guard<std::mutex> lock(overlap_streams().mu);
  if (!cuda_ok(cudaEventRecord(join, side)) || !cuda_ok(cudaStreamWaitEvent(stream, join, 0)))
    return KDA_ERR_CUDA;
  return KDA_OK;
}

// Bound of the scan's waits on the preparation kernel's progress: two seconds
// plus a microsecond per work item (prep publishes tens of items per
// microsecond on the whole GPU, so the bound is far above a legitimate wait
// even on a shared, time-sliced device).
inline uint64_t scan_wait_ns(int64_t items) { return 2000000000ull + (uint64_t)items * 1000ull; }

template <int ACT>
inline kda_status launch_chunked_t(const void* q, const void* k, const void* v, const void* g,
                                   const void* beta, const float* conv_w, const void* init_state,
                                   const void* init_conv, const int32_t* cu_dev,
                                   const int32_t* cu_host, int N, int H, kda_dtype o_dt,
                                   kda_dtype state_dt, void* o, void* final_state, void* workspace,
                                   const OutputNorm& norm, ChunkedMode mode, cudaStream_t stream,
                                   const int32_t** cu_used) {
  using T = __nv_bfloat16;
  (void)cu_dev;  // the kernels read the host offsets staged below, never the caller's device copy
  // The chunk table below is staged from host memory that this call owns and
  // releases on return; a captured graph would read it again on every replay,
  // long after it is gone, so stream capture is refused.
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (!cuda_ok(cudaStreamIsCapturing(stream, &cap))) return KDA_ERR_CUDA;
  if (cap != cudaStreamCaptureStatusNone) return KDA_ERR_UNSUPPORTED;
  // chunk table and longest-first segment order
  std::vector<int64_t> nch(N);
  int64_t total = 0;
  for (int n = 0; n < N; ++n) {
    nch[n] = ((int64_t)cu_host[n + 1] - cu_host[n] + CH - 1) / CH;
    total += nch[n];
  }
  const size_t hdr = chunk_header_bytes(N, total);
  std::vector<uint8_t> host(hdr, 0);
  int2* tab = reinterpret_cast<int2*>(host.data());
  int32_t* base = reinterpret_cast<int32_t*>(host.data() + (size_t)total * sizeof(int2));
  int32_t* order = base + (N + 1);
  // the segment offsets the kernels read: the host copy, staged with the chunk
  // table, so that the schedule and every kernel see the same segments even
  // if the caller's device copy differs from it
  int32_t* cu_stage = order + N;
  std::copy(cu_host, cu_host + N + 1, cu_stage);
  int64_t c = 0;
  for (int n = 0; n < N; ++n) {
    base[n] = (int32_t)c;
    for (int64_t i = 0; i < nch[n]; ++i) tab[c++] = make_int2(n, (int)i);
  }
  base[N] = (int32_t)c;
  std::iota(order, order + N, 0);
  std::stable_sort(order, order + N, [&](int a, int b) { return nch[a] > nch[b]; });
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // pageable source: the call returns after the bytes are staged, so `host`
  // may be released right after
  if (!cuda_ok(cudaMemcpyAsync(ws, host.data(), hdr, cudaMemcpyHostToDevice, stream)))
    return KDA_ERR_CUDA;
  const int2* d_tab = reinterpret_cast<const int2*>(ws);
  const int32_t* d_base = reinterpret_cast<const int32_t*>(ws + (size_t)total * sizeof(int2));
  const int32_t* d_order = d_base + (N + 1);
  const int32_t* d_cu = d_order + N;
  if (cu_used) *cu_used = d_cu;
  int* work_counter = reinterpret_cast<int*>(ws + hdr);
  int* ready = work_counter + 4;
  uint8_t* records = ws + hdr + chunk_sync_bytes(total, H);
  records += (128 - (reinterpret_cast<uintptr_t>(records) & 127)) & 127;
  const bool scan_only = mode == ChunkedMode::kScanOnly;
  if (!scan_only && !cuda_ok(cudaMemsetAsync(work_counter, 0, 16 + (size_t)total * H * 4, stream)))
    return KDA_ERR_CUDA;
  const int64_t items = total * H;
  const bool overlap = !scan_only && items > 0 && (int64_t)N * H <= OVERLAP_MAX_CHAINS;

  // TMA descriptors over the packed [total_T, H*128] tensors: 67-row boxes for
  // the inputs (3 halo rows + one chunk); 64-row boxes for the output tiles
  const uint64_t rows = (uint64_t)cu_host[N], cols = (uint64_t)H * D;
  CUtensorMap tq, tk, tg, tv, to, tz;
  if (!make_tmap_bf16_2d(&tq, q, rows, cols, RAW_ROWS, D) || !make_tmap_bf16_2d(&tk, k, rows, cols, RAW_ROWS, D) ||
      !make_tmap_bf16_2d(&tg, g, rows, cols, RAW_ROWS, D) || !make_tmap_bf16_2d(&tv, v, rows, cols, RAW_ROWS, D) ||
      !make_tmap_2d(&to, o, rows, cols, CH, D, o_dt == KDA_F32 ? 4 : 2) ||
      !make_tmap_bf16_2d(&tz, norm.gate ? norm.gate : v, rows, cols, CH, D))
    return KDA_ERR_CUDA;

  cudaStream_t scan_stream = stream, side = nullptr;
  cudaEvent_t join = nullptr;
  if (overlap) {
    if (fork_side(stream, &side, &join) != KDA_OK) return KDA_ERR_CUDA;
    scan_stream = side;
  }
  if (total > 0 && !scan_only) {
    auto prep = chunk_prep_kernel<ACT>;
    if (!cuda_ok(cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, PREP_SMEM)))
      return KDA_ERR_CUDA;
    // persistent blocks, two per SM, over the (chunk, head) items
    int dev = 0, sms = 148;
    if (!cuda_ok(cudaGetDevice(&dev)) ||
        !cuda_ok(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)))
      return KDA_ERR_CUDA;
    const unsigned blocks = (unsigned)(items < 2 * sms ? items : 2 * sms);
    int vacate_sms = 0, vacate_after = (int)items;
    if (overlap) {
      // prep hands the first `chains` SMs to the scan after a share f of the
      // items such that the scan's serial chain (longest segment) and prep's
      // remainder on the other SMs end together
      const int chains = N * H;
      const int64_t longest = *std::max_element(nch.begin(), nch.end());
      const double r = norm.gate ? PREP_PER_SCAN_CHUNK_GATED : PREP_PER_SCAN_CHUNK;
      double f = 1.0 - (double)longest * (sms - chains) / ((double)items * r);
      f = f < 0.0 ? 0.0 : (f > 1.0 ? 1.0 : f);
      vacate_sms = chains;
      vacate_after = (int)(f * (double)items);
    }
    // an injected KDA_FAULT_DROP_READY drops the publication of the flags the
    // scan waits on
    int* publish = overlap && !take_fault(KDA_FAULT_DROP_READY) ? ready : nullptr;
    prep<<<blocks, PREP_THREADS, PREP_SMEM, stream>>>(tq, tk, tg, (const T*)beta, conv_w, (const T*)init_conv,
                                                        d_cu, d_tab, H, (int)items, records, work_counter,
                                                        publish, vacate_sms, vacate_after);
    if (!cuda_ok(cudaGetLastError())) return KDA_ERR_CUDA;
  }
  // the scan, instantiated for the output and state element types
  auto launch_scan = [&](auto tout, auto ts, auto epi) -> bool {
    using Tout = decltype(tout);
    using Ts = decltype(ts);
    constexpr bool E = decltype(epi)::value;
    auto scan = chunk_scan_kernel<Tout, ACT, Ts, E>;
    if (!cuda_ok(cudaFuncSetAttribute(scan, cudaFuncAttributeMaxDynamicSharedMemorySize, SCAN_SMEM)))
      return false;
    scan<<<(unsigned)N * H, SCAN_THREADS, SCAN_SMEM, scan_stream>>>(
        tv, to, conv_w, (const Ts*)init_state, (const T*)init_conv, d_cu, d_base, d_order, H, records,
        overlap ? ready : nullptr, (Tout*)o, (Ts*)final_state, scan_wait_ns(items), tz, norm.weight,
        norm.eps, mode == ChunkedMode::kFull ? 0 : 1);
    return true;
  };
  using Plain = std::false_type;
  using Epi = std::true_type;
  bool ok;
  if (norm.gate)  // the epilogue writes bf16 (checked by the caller)
    ok = state_dt == KDA_F32 ? launch_scan(T{}, float{}, Epi{}) : launch_scan(T{}, T{}, Epi{});
  else if (o_dt == KDA_F32)
    ok = state_dt == KDA_F32 ? launch_scan(float{}, float{}, Plain{}) : launch_scan(float{}, T{}, Plain{});
  else
    ok = state_dt == KDA_F32 ? launch_scan(T{}, float{}, Plain{}) : launch_scan(T{}, T{}, Plain{});
  if (!ok || !cuda_ok(cudaGetLastError())) return KDA_ERR_CUDA;
  if (overlap && join_side(stream, side, join) != KDA_OK) return KDA_ERR_CUDA;
  return KDA_OK;
}

inline kda_status launch_chunked(const void* q, const void* k, const void* v, const void* g,
                                 const void* beta, const float* conv_w, const void* init_state,
                                 const void* init_conv, const int32_t* cu_dev,
                                 const int32_t* cu_host, int N, int H, kda_conv_act act,
                                 kda_dtype o_dt, kda_dtype state_dt, void* o, void* final_state,
                                 void* workspace, cudaStream_t stream,
                                 const OutputNorm& norm = OutputNorm{},
                                 ChunkedMode mode = ChunkedMode::kFull,
                                 const int32_t** cu_used = nullptr) {
  if (act == KDA_CONV_SILU)
    return launch_chunked_t<KDA_CONV_SILU>(q, k, v, g, beta, conv_w, init_state, init_conv, cu_dev,
                                           cu_host, N, H, o_dt, state_dt, o, final_state, workspace, norm,
                                           mode, stream, cu_used);
  return launch_chunked_t<KDA_CONV_NONE>(q, k, v, g, beta, conv_w, init_state, init_conv, cu_dev,
                                         cu_host, N, H, o_dt, state_dt, o, final_state, workspace, norm,
                                         mode, stream, cu_used);
}

}  // namespace kda
