// libkda.so: the C ABI declared in include/kda.h.  Host-side argument
// validation, then asynchronous launches on the caller's stream.
#include <stdio.h>

#include <mutex>

#include "kda_common.cuh"
#include "kda_decode.cuh"
#include "kda_decode_multi.cuh"
#include "kda_recurrent.cuh"
#include "kda_tail.cuh"
#include "kda_chunked.cuh"

using namespace kda;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t esize(kda_dtype dt) { return dt == KDA_F32 ? 4 : 2; }

struct PrefillArgs {
  const void *q, *k, *v, *g, *beta;
  const float* conv_w;
  const float* init_state;
  const void* init_conv;
  const int32_t *cu_dev, *cu_host;
  int N, H;
  kda_dtype dt;
  kda_conv_act act;
  kda_dtype o_dt;
  void* o;
  float* final_state;
  void* conv_tail;
  cudaStream_t stream;
  int64_t total_T;
  int max_len;
};

kda_status validate_prefill(PrefillArgs& a) {
  if (a.N < 0 || a.H < 1) return KDA_ERR_INVALID_ARG;
  if (a.dt != KDA_F32 && a.dt != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (a.act != KDA_CONV_NONE && a.act != KDA_CONV_SILU) return KDA_ERR_INVALID_ARG;
  if (a.o_dt != KDA_F32 && a.o_dt != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (a.N == 0) { a.total_T = 0; a.max_len = 0; return KDA_OK; }
  if (!a.cu_host || !a.cu_dev) return KDA_ERR_INVALID_ARG;
  if (a.cu_host[0] != 0) return KDA_ERR_INVALID_ARG;
  int max_len = 0;
  for (int n = 0; n < a.N; ++n) {
    const int64_t len = (int64_t)a.cu_host[n + 1] - a.cu_host[n];
    if (len < 0) return KDA_ERR_INVALID_ARG;
    if (len > max_len) max_len = (int)len;
  }
  a.total_T = a.cu_host[a.N];
  a.max_len = max_len;
  if (a.N > 65535) return KDA_ERR_UNSUPPORTED;
  if (!a.final_state || !a.conv_tail || !a.conv_w) return KDA_ERR_INVALID_ARG;
  if (a.total_T > 0 && (!a.q || !a.k || !a.v || !a.g || !a.beta || !a.o)) return KDA_ERR_INVALID_ARG;
  const void* al16[] = {a.q, a.k, a.v, a.g, a.o, a.conv_w, a.init_state, a.final_state,
                        a.init_conv, a.conv_tail};
  for (const void* p : al16)
    if (p && !aligned(p, 16)) return KDA_ERR_ALIGNMENT;
  if (a.beta && !aligned(a.beta, esize(a.dt))) return KDA_ERR_ALIGNMENT;
  if (a.total_T > 0 && (a.o == a.q || a.o == a.k || a.o == a.v || a.o == a.g))
    return KDA_ERR_INVALID_ARG;
  return KDA_OK;
}

template <typename Tin>
kda_status launch_tail(const PrefillArgs& a) {
  const int64_t total = (int64_t)a.N * 3 * a.H * D;
  if (total == 0) return KDA_OK;
  const int64_t want = (total + 255) / 256;
  const int64_t blocks = want < 148 * 16 ? want : 148 * 16;
  conv_tail_kernel<Tin><<<(unsigned)blocks, 256, 0, a.stream>>>(
      (const Tin*)a.q, (const Tin*)a.k, (const Tin*)a.v, (const Tin*)a.init_conv, a.cu_dev, a.N,
      a.H, (Tin*)a.conv_tail);
  return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

template <typename Tin, typename Tout, int ACT>
void launch_recurrent_t(const PrefillArgs& a) {
  recurrent_prefill_kernel<Tin, Tout, ACT><<<dim3(a.H, a.N), 128, 0, a.stream>>>(
      (const Tin*)a.q, (const Tin*)a.k, (const Tin*)a.v, (const Tin*)a.g, (const Tin*)a.beta,
      a.conv_w, a.init_state, (const Tin*)a.init_conv, a.cu_dev, a.H, (Tout*)a.o, a.final_state);
}

template <typename Tin>
kda_status launch_recurrent(const PrefillArgs& a) {
  const bool silu = a.act == KDA_CONV_SILU;
  if (a.o_dt == KDA_F32) {
    if (silu) launch_recurrent_t<Tin, float, KDA_CONV_SILU>(a);
    else launch_recurrent_t<Tin, float, KDA_CONV_NONE>(a);
  } else {
    if (silu) launch_recurrent_t<Tin, __nv_bfloat16, KDA_CONV_SILU>(a);
    else launch_recurrent_t<Tin, __nv_bfloat16, KDA_CONV_NONE>(a);
  }
  if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
  return launch_tail<Tin>(a);
}

kda_status run_recurrent(PrefillArgs& a) {
  if (a.N == 0) return KDA_OK;
  return a.dt == KDA_F32 ? launch_recurrent<float>(a) : launch_recurrent<__nv_bfloat16>(a);
}

template <typename Tin, typename Tout, int ACT>
void launch_decode_t(float* state, void* cache, const void* q, const void* k, const void* v,
                     const void* g, const void* beta, const float* conv_w, int N, int H, void* o,
                     cudaStream_t s) {
  decode_kernel<Tin, Tout, ACT><<<dim3(H, N), 256, 0, s>>>(
      state, (Tin*)cache, (const Tin*)q, (const Tin*)k, (const Tin*)v, (const Tin*)g,
      (const Tin*)beta, conv_w, H, (Tout*)o);
}

template <typename Tin>
void launch_decode(kda_conv_act act, kda_dtype o_dt, float* state, void* cache, const void* q,
                   const void* k, const void* v, const void* g, const void* beta,
                   const float* conv_w, int N, int H, void* o, cudaStream_t s) {
  const bool silu = act == KDA_CONV_SILU;
  if (o_dt == KDA_F32) {
    if (silu) launch_decode_t<Tin, float, KDA_CONV_SILU>(state, cache, q, k, v, g, beta, conv_w, N, H, o, s);
    else launch_decode_t<Tin, float, KDA_CONV_NONE>(state, cache, q, k, v, g, beta, conv_w, N, H, o, s);
  } else {
    if (silu) launch_decode_t<Tin, __nv_bfloat16, KDA_CONV_SILU>(state, cache, q, k, v, g, beta, conv_w, N, H, o, s);
    else launch_decode_t<Tin, __nv_bfloat16, KDA_CONV_NONE>(state, cache, q, k, v, g, beta, conv_w, N, H, o, s);
  }
}

template <typename Tin, typename Tout, int ACT>
void launch_verify_t(const float* state, const void* cache, const void* q, const void* k, const void* v,
                     const void* g, const void* beta, const float* conv_w, int N, int R, int H, void* o,
                     float* deltas, cudaStream_t s) {
  decode_verify_kernel<Tin, Tout, ACT><<<dim3(H, N), 256, 0, s>>>(
      state, (const Tin*)cache, (const Tin*)q, (const Tin*)k, (const Tin*)v, (const Tin*)g, (const Tin*)beta,
      conv_w, R, H, (Tout*)o, deltas);
}

template <typename Tin>
void launch_verify(kda_conv_act act, kda_dtype o_dt, const float* state, const void* cache, const void* q,
                   const void* k, const void* v, const void* g, const void* beta, const float* conv_w, int N,
                   int R, int H, void* o, float* deltas, cudaStream_t s) {
  const bool silu = act == KDA_CONV_SILU;
  if (o_dt == KDA_F32) {
    if (silu) launch_verify_t<Tin, float, KDA_CONV_SILU>(state, cache, q, k, v, g, beta, conv_w, N, R, H, o, deltas, s);
    else launch_verify_t<Tin, float, KDA_CONV_NONE>(state, cache, q, k, v, g, beta, conv_w, N, R, H, o, deltas, s);
  } else {
    if (silu)
      launch_verify_t<Tin, __nv_bfloat16, KDA_CONV_SILU>(state, cache, q, k, v, g, beta, conv_w, N, R, H, o, deltas, s);
    else
      launch_verify_t<Tin, __nv_bfloat16, KDA_CONV_NONE>(state, cache, q, k, v, g, beta, conv_w, N, R, H, o, deltas, s);
  }
}

// shared argument checks of the decode entry points
kda_status check_decode_common(int num_seqs, int num_heads, kda_dtype dt) {
  if (num_seqs < 0 || num_heads < 1) return KDA_ERR_INVALID_ARG;
  if (dt != KDA_F32 && dt != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (num_seqs > 65535) return KDA_ERR_UNSUPPORTED;
  return KDA_OK;
}

}  // namespace

extern "C" {

size_t kda_prefill_workspace_size(int num_seqs, int64_t total_tokens, int num_heads,
                                  int max_seqlen, kda_dtype dt) {
  if (num_seqs < 0 || total_tokens < 0 || num_heads < 1 || max_seqlen < 0) return 0;
  if (dt != KDA_BF16) return 0;
  return chunked_workspace_bytes(num_seqs, num_heads, total_tokens);
}

kda_status kda_prefill_recurrent(const void* q, const void* k, const void* v, const void* g,
                                 const void* beta, const float* conv_w,
                                 const float* init_state, const void* init_conv,
                                 const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host,
                                 int num_seqs, int num_heads, kda_dtype dt, kda_conv_act act,
                                 kda_dtype o_dt, void* o, float* final_state, void* conv_tail,
                                 void* stream) {
  PrefillArgs a{q, k, v, g, beta, conv_w, init_state, init_conv, cu_seqlens_dev,
                cu_seqlens_host, num_seqs, num_heads, dt, act, o_dt, o, final_state, conv_tail,
                (cudaStream_t)stream, 0, 0};
  kda_status st = validate_prefill(a);
  if (st != KDA_OK) return st;
  return run_recurrent(a);
}

kda_status kda_prefill(const void* q, const void* k, const void* v, const void* g,
                       const void* beta, const float* conv_w, const float* init_state,
                       const void* init_conv, const int32_t* cu_seqlens_dev,
                       const int32_t* cu_seqlens_host, int num_seqs, int num_heads,
                       kda_dtype dt, kda_conv_act act, kda_dtype o_dt, void* o,
                       float* final_state, void* conv_tail, void* workspace,
                       size_t workspace_bytes, void* stream) {
  PrefillArgs a{q, k, v, g, beta, conv_w, init_state, init_conv, cu_seqlens_dev,
                cu_seqlens_host, num_seqs, num_heads, dt, act, o_dt, o, final_state, conv_tail,
                (cudaStream_t)stream, 0, 0};
  kda_status st = validate_prefill(a);
  if (st != KDA_OK) return st;
  if (a.N == 0) return KDA_OK;
  if (dt == KDA_F32) return run_recurrent(a);
  const size_t need = chunked_workspace_bytes(a.N, a.H, a.total_T);
  if (need > 0 && (!workspace || workspace_bytes < need)) return KDA_ERR_WORKSPACE;
  if (workspace && !aligned(workspace, 16)) return KDA_ERR_ALIGNMENT;
  st = launch_chunked(a.q, a.k, a.v, a.g, a.beta, a.conv_w, a.init_state, a.init_conv, a.cu_dev,
                      a.cu_host, a.N, a.H, a.act, a.o_dt, a.o, a.final_state, workspace,
                      workspace_bytes, a.max_len, a.stream);
  if (st != KDA_OK) return st;
  return launch_tail<__nv_bfloat16>(a);
}

kda_status kda_decode_step(float* state, void* conv_cache, const void* q, const void* k,
                           const void* v, const void* g, const void* beta,
                           const float* conv_w, int num_seqs, int num_heads, kda_dtype dt,
                           kda_conv_act act, kda_dtype o_dt, void* o, void* stream) {
  if (num_seqs < 0 || num_heads < 1) return KDA_ERR_INVALID_ARG;
  if (dt != KDA_F32 && dt != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (o_dt != KDA_F32 && o_dt != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (act != KDA_CONV_NONE && act != KDA_CONV_SILU) return KDA_ERR_INVALID_ARG;
  if (num_seqs == 0) return KDA_OK;
  if (num_seqs > 65535) return KDA_ERR_UNSUPPORTED;
  if (!state || !conv_cache || !q || !k || !v || !g || !beta || !conv_w || !o)
    return KDA_ERR_INVALID_ARG;
  const void* al16[] = {state, conv_cache, q, k, v, g, conv_w, o};
  for (const void* p : al16)
    if (!aligned(p, 16)) return KDA_ERR_ALIGNMENT;
  if (!aligned(beta, esize(dt))) return KDA_ERR_ALIGNMENT;
  if (o == q || o == k || o == v || o == g) return KDA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (dt == KDA_F32)
    launch_decode<float>(act, o_dt, state, conv_cache, q, k, v, g, beta, conv_w, num_seqs,
                         num_heads, o, s);
  else
    launch_decode<__nv_bfloat16>(act, o_dt, state, conv_cache, q, k, v, g, beta, conv_w,
                                 num_seqs, num_heads, o, s);
  return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

size_t kda_decode_deltas_size(int num_seqs, int num_rows, int num_heads) {
  if (num_seqs < 0 || num_rows < 1 || num_rows > KDA_MAX_VERIFY_ROWS || num_heads < 1) return 0;
  return (size_t)num_seqs * num_heads * num_rows * 3 * D * sizeof(float);
}

kda_status kda_decode_verify(const float* state, const void* conv_cache, const void* q, const void* k,
                             const void* v, const void* g, const void* beta, const float* conv_w,
                             int num_seqs, int num_rows, int num_heads, kda_dtype dt, kda_conv_act act,
                             kda_dtype o_dt, void* o, float* deltas, void* stream) {
  kda_status st = check_decode_common(num_seqs, num_heads, dt);
  if (st != KDA_OK) return st;
  if (num_rows < 1 || num_rows > KDA_MAX_VERIFY_ROWS) return KDA_ERR_INVALID_ARG;
  if (o_dt != KDA_F32 && o_dt != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (act != KDA_CONV_NONE && act != KDA_CONV_SILU) return KDA_ERR_INVALID_ARG;
  if (num_seqs == 0) return KDA_OK;
  if (!state || !conv_cache || !q || !k || !v || !g || !beta || !conv_w || !o || !deltas)
    return KDA_ERR_INVALID_ARG;
  const void* al16[] = {state, conv_cache, q, k, v, g, conv_w, o, deltas};
  for (const void* p : al16)
    if (!aligned(p, 16)) return KDA_ERR_ALIGNMENT;
  if (!aligned(beta, esize(dt))) return KDA_ERR_ALIGNMENT;
  if (o == q || o == k || o == v || o == g || (const void*)deltas == (const void*)state) return KDA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (dt == KDA_F32)
    launch_verify<float>(act, o_dt, state, conv_cache, q, k, v, g, beta, conv_w, num_seqs, num_rows, num_heads, o,
                         deltas, s);
  else
    launch_verify<__nv_bfloat16>(act, o_dt, state, conv_cache, q, k, v, g, beta, conv_w, num_seqs, num_rows,
                                 num_heads, o, deltas, s);
  return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_decode_commit(float* state, void* conv_cache, const void* q, const void* k, const void* v,
                             const float* deltas, const int32_t* n_accept, int num_seqs, int num_rows,
                             int num_heads, kda_dtype dt, void* stream) {
  kda_status st = check_decode_common(num_seqs, num_heads, dt);
  if (st != KDA_OK) return st;
  if (num_rows < 1 || num_rows > KDA_MAX_VERIFY_ROWS) return KDA_ERR_INVALID_ARG;
  if (num_seqs == 0) return KDA_OK;
  if (!state || !conv_cache || !q || !k || !v || !deltas || !n_accept) return KDA_ERR_INVALID_ARG;
  const void* al16[] = {state, conv_cache, q, k, v, deltas};
  for (const void* p : al16)
    if (!aligned(p, 16)) return KDA_ERR_ALIGNMENT;
  if (!aligned(n_accept, 4)) return KDA_ERR_ALIGNMENT;
  cudaStream_t s = (cudaStream_t)stream;
  const dim3 grid(num_heads, num_seqs);
  if (dt == KDA_F32)
    decode_commit_kernel<float><<<grid, 256, 0, s>>>(state, (float*)conv_cache, (const float*)q, (const float*)k,
                                                      (const float*)v, deltas, n_accept, num_rows, num_heads);
  else
    decode_commit_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        state, (__nv_bfloat16*)conv_cache, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
        (const __nv_bfloat16*)v, deltas, n_accept, num_rows, num_heads);
  return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

const char* kda_status_string(kda_status s) {
  switch (s) {
    case KDA_OK: return "ok";
    case KDA_ERR_INVALID_ARG: return "invalid argument";
    case KDA_ERR_UNSUPPORTED: return "unsupported request";
    case KDA_ERR_ALIGNMENT: return "misaligned pointer";
    case KDA_ERR_WORKSPACE: return "workspace missing or too small";
    case KDA_ERR_CUDA: return "CUDA runtime error";
    case KDA_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

kda_status kda_check_async_status(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return KDA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return KDA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return KDA_ERR_CUDA;
  }
  return (kda_status)v;
}

int kda_version(void) { return (1 << 16) | 0; }

}  // extern "C"

// ---- prefill for callers that cannot allocate device memory ------------------
// The chunked path's scratch (chunk table + one operand record per chunk and
// head) lives in this file-scope device array instead of a caller workspace.
// In host code the name below is only a stand-in for the symbol; the device
// address is obtained with cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char kda_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// device address of kda_noalloc_scratch on the current device (looked up on
// the first call for that device, with that device current)
kda_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KDA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, kda_noalloc_scratch) != cudaSuccess || !p) return KDA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return KDA_OK;
}
}  // namespace

extern "C" kda_status kda_prefill_noalloc(const void* q, const void* k, const void* v, const void* g,
                                          const void* beta, const float* conv_w,
                                          const float* init_state, const void* init_conv,
                                          const int32_t* cu_seqlens_dev,
                                          const int32_t* cu_seqlens_host, int num_seqs,
                                          int num_heads, kda_dtype dt, kda_conv_act act,
                                          kda_dtype o_dt, void* o, float* final_state,
                                          void* conv_tail, void* stream) {
  PrefillArgs a{q, k, v, g, beta, conv_w, init_state, init_conv, cu_seqlens_dev,
                cu_seqlens_host, num_seqs, num_heads, dt, act, o_dt, o, final_state, conv_tail,
                (cudaStream_t)stream, 0, 0};
  kda_status st = validate_prefill(a);
  if (st != KDA_OK) return st;
  if (a.N == 0) return KDA_OK;
  if (dt == KDA_F32) return run_recurrent(a);  // the fp32 path uses no scratch
  const size_t need = chunked_workspace_bytes(a.N, a.H, a.total_T);
  if (need > KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != KDA_OK) return st;
  st = launch_chunked(a.q, a.k, a.v, a.g, a.beta, a.conv_w, a.init_state, a.init_conv, a.cu_dev,
                      a.cu_host, a.N, a.H, a.act, a.o_dt, a.o, a.final_state, scratch, need,
                      a.max_len, a.stream);
  if (st != KDA_OK) return st;
  return launch_tail<__nv_bfloat16>(a);
}
