// libkda.so: the C ABI declared in include/kda.h.  Host-side argument
// validation, then asynchronous launches on the caller's stream.
#include <stdio.h>

#include <mutex>
#include <type_traits>

#include "kda_common.cuh"
#include "kda_decode.cuh"
#include "kda_decode_multi.cuh"
#include "kda_recurrent.cuh"
#include "kda_tail.cuh"
#include "kda_chunked.cuh"
#include "kda_affine.cuh"
#include "kda_output_norm.cuh"

using namespace kda;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t esize(kda_dtype dt) { return dt == KDA_F32 ? 4 : 2; }
bool valid_dtype(kda_dtype t) { return t == KDA_F32 || t == KDA_BF16; }
bool valid_act(kda_conv_act a) { return a == KDA_CONV_NONE || a == KDA_CONV_SILU; }

// Runtime element type / activation -> template argument: f is called with a
// value of the matching type (float or __nv_bfloat16; an integral_constant
// holding the activation).
template <typename F> void by_type(kda_dtype t, F&& f) {
  if (t == KDA_F32) f(float{});
  else f(__nv_bfloat16{});
}
template <typename F> void by_act(kda_conv_act a, F&& f) {
  if (a == KDA_CONV_SILU) f(std::integral_constant<int, KDA_CONV_SILU>{});
  else f(std::integral_constant<int, KDA_CONV_NONE>{});
}

struct PrefillArgs {
  const void *q, *k, *v, *g, *beta;
  const float* conv_w;
  const void* init_state;
  const void* init_conv;
  const int32_t *cu_dev, *cu_host;
  int N, H;
  kda_dtype dt;
  kda_conv_act act;
  kda_dtype o_dt, state_dt;
  void* o;
  void* final_state;
  void* conv_tail;
  cudaStream_t stream;
  int64_t total_T;
  int max_len;
};

kda_status validate_prefill(PrefillArgs& a) {
  if (a.N < 0 || a.H < 1) return KDA_ERR_INVALID_ARG;
  if (!valid_dtype(a.dt) || !valid_dtype(a.o_dt) || !valid_dtype(a.state_dt) || !valid_act(a.act))
    return KDA_ERR_INVALID_ARG;
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
  return cuda_ok(cudaGetLastError()) ? KDA_OK : KDA_ERR_CUDA;
}

template <typename Tin>
kda_status launch_recurrent(const PrefillArgs& a) {
  by_type(a.o_dt, [&](auto tout) {
    by_type(a.state_dt, [&](auto ts) {
      by_act(a.act, [&](auto act) {
        using Tout = decltype(tout);
        using Ts = decltype(ts);
        recurrent_prefill_kernel<Tin, Tout, decltype(act)::value, Ts><<<dim3(a.H, a.N), 128, 0, a.stream>>>(
            (const Tin*)a.q, (const Tin*)a.k, (const Tin*)a.v, (const Tin*)a.g, (const Tin*)a.beta, a.conv_w,
            (const Ts*)a.init_state, (const Tin*)a.init_conv, a.cu_dev, a.H, (Tout*)a.o, (Ts*)a.final_state);
      });
    });
  });
  if (!cuda_ok(cudaGetLastError())) return KDA_ERR_CUDA;
  return launch_tail<Tin>(a);
}

kda_status run_recurrent(PrefillArgs& a) {
  if (a.N == 0) return KDA_OK;
  return a.dt == KDA_F32 ? launch_recurrent<float>(a) : launch_recurrent<__nv_bfloat16>(a);
}

// number of SMs of the current device (persistent grids)
kda_status sm_count(int* out) {
  int dev = 0;
  if (!cuda_ok(cudaGetDevice(&dev)) ||
      !cuda_ok(cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, dev)) || *out < 1)
    return KDA_ERR_CUDA;
  return KDA_OK;
}

// Launch a persistent decode-family kernel (256 threads, the prefetch buffers
// in `smem` bytes of dynamic shared memory) with two blocks per SM over N x H
// items.
template <typename Kern, typename... Args>
kda_status launch_persistent(Kern kern, uint32_t smem, int64_t items, cudaStream_t s, Args... args) {
  int sms = 0;
  if (sm_count(&sms) != KDA_OK) return KDA_ERR_CUDA;
  if (!cuda_ok(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)))
    return KDA_ERR_CUDA;
  const int blocks = (int)(items < 2 * sms ? items : 2 * sms);
  kern<<<blocks, 256, smem, s>>>(args...);
  return cuda_ok(cudaGetLastError()) ? KDA_OK : KDA_ERR_CUDA;
}

// shared argument checks of the decode entry points
kda_status check_decode_common(int num_seqs, int num_heads, kda_dtype dt, kda_dtype state_dt) {
  if (num_seqs < 0 || num_heads < 1) return KDA_ERR_INVALID_ARG;
  if (!valid_dtype(dt) || !valid_dtype(state_dt)) return KDA_ERR_INVALID_ARG;
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
                                 const void* init_state, const void* init_conv,
                                 const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host,
                                 int num_seqs, int num_heads, kda_dtype dt, kda_conv_act act,
                                 kda_dtype o_dt, kda_dtype state_dt, void* o, void* final_state,
                                 void* conv_tail, void* stream) {
  PrefillArgs a{q, k, v, g, beta, conv_w, init_state, init_conv, cu_seqlens_dev,
                cu_seqlens_host, num_seqs, num_heads, dt, act, o_dt, state_dt, o, final_state, conv_tail,
                (cudaStream_t)stream, 0, 0};
  kda_status st = validate_prefill(a);
  if (st != KDA_OK) return st;
  return run_recurrent(a);
}

namespace {
// kda_prefill and its record-keeping / scan-only forms
kda_status prefill_mode(const PrefillArgs& args, void* workspace, size_t workspace_bytes, ChunkedMode mode) {
  PrefillArgs a = args;
  kda_status st = validate_prefill(a);
  if (st != KDA_OK) return st;
  if (a.N == 0) return KDA_OK;
  if (a.dt == KDA_F32) {
    if (mode != ChunkedMode::kFull) return KDA_ERR_UNSUPPORTED;  // the recurrent path keeps no records
    return run_recurrent(a);
  }
  const size_t need = chunked_workspace_bytes(a.N, a.H, a.total_T);
  if (need > 0 && (!workspace || workspace_bytes < need)) return KDA_ERR_WORKSPACE;
  if (workspace && !aligned(workspace, 16)) return KDA_ERR_ALIGNMENT;
  const int32_t* cu_used = nullptr;
  st = launch_chunked(a.q, a.k, a.v, a.g, a.beta, a.conv_w, a.init_state, a.init_conv, a.cu_dev,
                      a.cu_host, a.N, a.H, a.act, a.o_dt, a.state_dt, a.o, a.final_state, workspace,
                      a.stream, OutputNorm{}, mode, &cu_used);
  if (st != KDA_OK) return st;
  a.cu_dev = cu_used;  // the staged host offsets, as the chunked kernels used
  return launch_tail<__nv_bfloat16>(a);
}
}  // namespace

#define KDA_PREFILL_ARGS_STRUCT                                                                          \
  PrefillArgs a{q, k, v, g, beta, conv_w, init_state, init_conv, cu_seqlens_dev,                        \
                cu_seqlens_host, num_seqs, num_heads, dt, act, o_dt, state_dt, o, final_state, conv_tail, \
                (cudaStream_t)stream, 0, 0}

kda_status kda_prefill(const void* q, const void* k, const void* v, const void* g,
                       const void* beta, const float* conv_w, const void* init_state,
                       const void* init_conv, const int32_t* cu_seqlens_dev,
                       const int32_t* cu_seqlens_host, int num_seqs, int num_heads,
                       kda_dtype dt, kda_conv_act act, kda_dtype o_dt, kda_dtype state_dt,
                       void* o, void* final_state, void* conv_tail, void* workspace,
                       size_t workspace_bytes, void* stream) {
  KDA_PREFILL_ARGS_STRUCT;
  return prefill_mode(a, workspace, workspace_bytes, ChunkedMode::kFull);
}

kda_status kda_prefill_records(const void* q, const void* k, const void* v, const void* g,
                               const void* beta, const float* conv_w, const void* init_state,
                               const void* init_conv, const int32_t* cu_seqlens_dev,
                               const int32_t* cu_seqlens_host, int num_seqs, int num_heads,
                               kda_dtype dt, kda_conv_act act, kda_dtype o_dt, kda_dtype state_dt,
                               void* o, void* final_state, void* conv_tail, void* workspace,
                               size_t workspace_bytes, void* stream) {
  KDA_PREFILL_ARGS_STRUCT;
  return prefill_mode(a, workspace, workspace_bytes, ChunkedMode::kKeepRecords);
}

kda_status kda_prefill_scan(const void* q, const void* k, const void* v, const void* g,
                            const void* beta, const float* conv_w, const void* init_state,
                            const void* init_conv, const int32_t* cu_seqlens_dev,
                            const int32_t* cu_seqlens_host, int num_seqs, int num_heads,
                            kda_dtype dt, kda_conv_act act, kda_dtype o_dt, kda_dtype state_dt,
                            void* o, void* final_state, void* conv_tail, void* workspace,
                            size_t workspace_bytes, void* stream) {
  KDA_PREFILL_ARGS_STRUCT;
  return prefill_mode(a, workspace, workspace_bytes, ChunkedMode::kScanOnly);
}
#undef KDA_PREFILL_ARGS_STRUCT

kda_status kda_prefill_gated(const void* q, const void* k, const void* v, const void* g,
                             const void* beta, const float* conv_w, const void* init_state,
                             const void* init_conv, const int32_t* cu_seqlens_dev,
                             const int32_t* cu_seqlens_host, int num_seqs, int num_heads,
                             kda_dtype dt, kda_conv_act act, kda_dtype o_dt, kda_dtype state_dt,
                             void* o, void* final_state, void* conv_tail, void* workspace,
                             size_t workspace_bytes, const void* gate, const float* norm_weight,
                             float norm_eps, void* stream) {
  PrefillArgs a{q, k, v, g, beta, conv_w, init_state, init_conv, cu_seqlens_dev,
                cu_seqlens_host, num_seqs, num_heads, dt, act, o_dt, state_dt, o, final_state, conv_tail,
                (cudaStream_t)stream, 0, 0};
  kda_status st = validate_prefill(a);
  if (st != KDA_OK) return st;
  if (o_dt != KDA_BF16 || !norm_weight || !(norm_eps >= 0.f) || norm_eps > 3.0e38f) return KDA_ERR_INVALID_ARG;
  if (a.total_T > 0 && (!gate || gate == o)) return KDA_ERR_INVALID_ARG;
  if ((gate && !aligned(gate, 16)) || !aligned(norm_weight, 16)) return KDA_ERR_ALIGNMENT;
  if (dt != KDA_BF16) return KDA_ERR_UNSUPPORTED;
  if (a.N == 0) return KDA_OK;
  const size_t need = chunked_workspace_bytes(a.N, a.H, a.total_T);
  if (need > 0 && (!workspace || workspace_bytes < need)) return KDA_ERR_WORKSPACE;
  if (workspace && !aligned(workspace, 16)) return KDA_ERR_ALIGNMENT;
  OutputNorm norm;
  norm.gate = gate;
  norm.weight = norm_weight;
  norm.eps = norm_eps;
  const int32_t* cu_used = nullptr;
  st = launch_chunked(a.q, a.k, a.v, a.g, a.beta, a.conv_w, a.init_state, a.init_conv, a.cu_dev,
                      a.cu_host, a.N, a.H, a.act, a.o_dt, a.state_dt, a.o, a.final_state, workspace,
                      a.stream, norm, ChunkedMode::kFull, &cu_used);
  if (st != KDA_OK) return st;
  a.cu_dev = cu_used;
  return launch_tail<__nv_bfloat16>(a);
}

kda_status kda_output_norm(const void* o, kda_dtype o_dt, const void* gate, const float* norm_weight,
                           float norm_eps, void* y, int64_t rows, int num_heads, void* stream) {
  if (rows < 0 || num_heads < 1 || !valid_dtype(o_dt)) return KDA_ERR_INVALID_ARG;
  if (!norm_weight || !(norm_eps >= 0.f) || norm_eps > 3.0e38f) return KDA_ERR_INVALID_ARG;
  if (rows == 0) return KDA_OK;
  if (!o || !gate || !y || gate == y || (y == o && o_dt != KDA_BF16)) return KDA_ERR_INVALID_ARG;
  const void* al16[] = {o, gate, y, norm_weight};
  for (const void* p : al16)
    if (!aligned(p, 16)) return KDA_ERR_ALIGNMENT;
  const int64_t row_heads = rows * num_heads;
  int sms = 0;
  kda_status st = sm_count(&sms);
  if (st != KDA_OK) return st;
  const int64_t want = (row_heads + NORM_THREADS / 32 - 1) / (NORM_THREADS / 32);
  const unsigned blocks = (unsigned)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
  cudaStream_t s = (cudaStream_t)stream;
  if (o_dt == KDA_F32)
    output_norm_kernel<float><<<blocks, NORM_THREADS, 0, s>>>(
        (const float*)o, (const __nv_bfloat16*)gate, norm_weight, norm_eps, (__nv_bfloat16*)y, row_heads);
  else
    output_norm_kernel<__nv_bfloat16><<<blocks, NORM_THREADS, 0, s>>>(
        (const __nv_bfloat16*)o, (const __nv_bfloat16*)gate, norm_weight, norm_eps, (__nv_bfloat16*)y,
        row_heads);
  return cuda_ok(cudaGetLastError()) ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_decode_step(void* state, void* conv_cache, const void* q, const void* k,
                           const void* v, const void* g, const void* beta,
                           const float* conv_w, int num_seqs, int num_heads, kda_dtype dt,
                           kda_conv_act act, kda_dtype o_dt, kda_dtype state_dt, void* o,
                           void* stream) {
  kda_status st = check_decode_common(num_seqs, num_heads, dt, state_dt);
  if (st != KDA_OK) return st;
  if (!valid_dtype(o_dt) || !valid_act(act)) return KDA_ERR_INVALID_ARG;
  if (num_seqs == 0) return KDA_OK;
  if (!state || !conv_cache || !q || !k || !v || !g || !beta || !conv_w || !o)
    return KDA_ERR_INVALID_ARG;
  const void* al16[] = {state, conv_cache, q, k, v, g, conv_w, o};
  for (const void* p : al16)
    if (!aligned(p, 16)) return KDA_ERR_ALIGNMENT;
  if (!aligned(beta, esize(dt))) return KDA_ERR_ALIGNMENT;
  if (o == q || o == k || o == v || o == g) return KDA_ERR_INVALID_ARG;
  if ((int64_t)num_seqs * num_heads > INT32_MAX) return KDA_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  kda_status rc = KDA_OK;
  by_type(dt, [&](auto tin) {
    by_type(o_dt, [&](auto tout) {
      by_type(state_dt, [&](auto ts) {
        by_act(act, [&](auto a) {
          using Tin = decltype(tin);
          using Ts = decltype(ts);
          rc = launch_persistent(decode_kernel<Tin, decltype(tout), decltype(a)::value, Ts>,
                                 DecodePrefetch<Tin, Ts, sizeof(Ts) == 2>::bytes(), (int64_t)num_seqs * num_heads, s, (Ts*)state, (Tin*)conv_cache, (const Tin*)q,
                                     (const Tin*)k, (const Tin*)v, (const Tin*)g, (const Tin*)beta, conv_w,
                                     num_seqs, num_heads, (decltype(tout)*)o);
        });
      });
    });
  });
  return rc;
}

size_t kda_decode_deltas_size(int num_seqs, int num_rows, int num_heads) {
  if (num_seqs < 0 || num_rows < 1 || num_rows > KDA_MAX_VERIFY_ROWS || num_heads < 1) return 0;
  return (size_t)num_seqs * num_heads * num_rows * 3 * D * sizeof(float);
}

kda_status kda_decode_verify(const void* state, const void* conv_cache, const void* q, const void* k,
                             const void* v, const void* g, const void* beta, const float* conv_w,
                             int num_seqs, int num_rows, int num_heads, kda_dtype dt, kda_conv_act act,
                             kda_dtype o_dt, kda_dtype state_dt, void* o, float* deltas, void* stream) {
  kda_status st = check_decode_common(num_seqs, num_heads, dt, state_dt);
  if (st != KDA_OK) return st;
  if (num_rows < 1 || num_rows > KDA_MAX_VERIFY_ROWS) return KDA_ERR_INVALID_ARG;
  if (!valid_dtype(o_dt) || !valid_act(act)) return KDA_ERR_INVALID_ARG;
  if (num_seqs == 0) return KDA_OK;
  if (!state || !conv_cache || !q || !k || !v || !g || !beta || !conv_w || !o || !deltas)
    return KDA_ERR_INVALID_ARG;
  const void* al16[] = {state, conv_cache, q, k, v, g, conv_w, o, deltas};
  for (const void* p : al16)
    if (!aligned(p, 16)) return KDA_ERR_ALIGNMENT;
  if (!aligned(beta, esize(dt))) return KDA_ERR_ALIGNMENT;
  if (o == q || o == k || o == v || o == g || (const void*)deltas == state) return KDA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  kda_status rc = KDA_OK;
  by_type(dt, [&](auto tin) {
    by_type(o_dt, [&](auto tout) {
      by_type(state_dt, [&](auto ts) {
        by_act(act, [&](auto a) {
          using Tin = decltype(tin);
          using Ts = decltype(ts);
          // no previous step: state and cache are only read
          decode_verify_kernel<Tin, decltype(tout), decltype(a)::value, Ts, false>
              <<<dim3(num_heads, num_seqs), 256, 0, s>>>((Ts*)state, (Tin*)conv_cache, (const Tin*)q, (const Tin*)k,
                                                         (const Tin*)v, (const Tin*)g, (const Tin*)beta, conv_w,
                                                         num_rows, num_heads, (decltype(tout)*)o, deltas, nullptr,
                                                         nullptr, nullptr, nullptr, nullptr, 0);
          rc = cuda_ok(cudaGetLastError()) ? KDA_OK : KDA_ERR_CUDA;
        });
      });
    });
  });
  return rc;
}

kda_status kda_decode_commit_verify(void* state, void* conv_cache, const void* prev_q, const void* prev_k,
                                    const void* prev_v, const float* prev_deltas, const int32_t* prev_n_accept,
                                    int prev_rows, const void* q, const void* k, const void* v, const void* g,
                                    const void* beta, const float* conv_w, int num_seqs, int num_rows,
                                    int num_heads, kda_dtype dt, kda_conv_act act, kda_dtype o_dt,
                                    kda_dtype state_dt, void* o, float* deltas, void* stream) {
  kda_status st = check_decode_common(num_seqs, num_heads, dt, state_dt);
  if (st != KDA_OK) return st;
  if (num_rows < 1 || num_rows > KDA_MAX_VERIFY_ROWS) return KDA_ERR_INVALID_ARG;
  if (prev_rows < 1 || prev_rows > KDA_MAX_VERIFY_ROWS) return KDA_ERR_INVALID_ARG;
  if (!valid_dtype(o_dt) || !valid_act(act)) return KDA_ERR_INVALID_ARG;
  if (num_seqs == 0) return KDA_OK;
  if (!state || !conv_cache || !prev_q || !prev_k || !prev_v || !prev_deltas || !prev_n_accept || !q || !k ||
      !v || !g || !beta || !conv_w || !o || !deltas)
    return KDA_ERR_INVALID_ARG;
  const void* al16[] = {state, conv_cache, prev_q, prev_k, prev_v, prev_deltas, q, k, v, g, conv_w, o, deltas};
  for (const void* p : al16)
    if (!aligned(p, 16)) return KDA_ERR_ALIGNMENT;
  if (!aligned(beta, esize(dt)) || !aligned(prev_n_accept, 4)) return KDA_ERR_ALIGNMENT;
  if (o == q || o == k || o == v || o == g || (const void*)deltas == state) return KDA_ERR_INVALID_ARG;
  {  // the new deltas may not overlap the previous step's (other blocks still read those)
    const uintptr_t d0 = (uintptr_t)deltas, d1 = d0 + kda_decode_deltas_size(num_seqs, num_rows, num_heads);
    const uintptr_t p0 = (uintptr_t)prev_deltas, p1 = p0 + kda_decode_deltas_size(num_seqs, prev_rows, num_heads);
    if (d0 < p1 && p0 < d1) return KDA_ERR_INVALID_ARG;
  }
  cudaStream_t s = (cudaStream_t)stream;
  kda_status rc = KDA_OK;
  by_type(dt, [&](auto tin) {
    by_type(o_dt, [&](auto tout) {
      by_type(state_dt, [&](auto ts) {
        by_act(act, [&](auto a) {
          using Tin = decltype(tin);
          using Ts = decltype(ts);
          decode_verify_kernel<Tin, decltype(tout), decltype(a)::value, Ts, true>
              <<<dim3(num_heads, num_seqs), 256, 0, s>>>((Ts*)state, (Tin*)conv_cache, (const Tin*)q, (const Tin*)k,
                                                         (const Tin*)v, (const Tin*)g, (const Tin*)beta, conv_w,
                                                         num_rows, num_heads, (decltype(tout)*)o, deltas,
                                                         (const Tin*)prev_q, (const Tin*)prev_k, (const Tin*)prev_v,
                                                         prev_deltas, prev_n_accept, prev_rows);
          rc = cuda_ok(cudaGetLastError()) ? KDA_OK : KDA_ERR_CUDA;
        });
      });
    });
  });
  return rc;
}

kda_status kda_decode_commit(void* state, void* conv_cache, const void* q, const void* k, const void* v,
                             const float* deltas, const int32_t* n_accept, int num_seqs, int num_rows,
                             int num_heads, kda_dtype dt, kda_dtype state_dt, void* stream) {
  kda_status st = check_decode_common(num_seqs, num_heads, dt, state_dt);
  if (st != KDA_OK) return st;
  if (num_rows < 1 || num_rows > KDA_MAX_VERIFY_ROWS) return KDA_ERR_INVALID_ARG;
  if (num_seqs == 0) return KDA_OK;
  if (!state || !conv_cache || !q || !k || !v || !deltas || !n_accept) return KDA_ERR_INVALID_ARG;
  const void* al16[] = {state, conv_cache, q, k, v, deltas};
  for (const void* p : al16)
    if (!aligned(p, 16)) return KDA_ERR_ALIGNMENT;
  if (!aligned(n_accept, 4)) return KDA_ERR_ALIGNMENT;
  cudaStream_t s = (cudaStream_t)stream;
  kda_status rc = KDA_OK;
  by_type(dt, [&](auto tin) {
    by_type(state_dt, [&](auto ts) {
      using Tin = decltype(tin);
      using Ts = decltype(ts);
      rc = launch_persistent(decode_commit_kernel<Tin, Ts>, CommitPrefetch<Ts>::bytes(num_rows),
                             (int64_t)num_seqs * num_heads, s, (Ts*)state, (Tin*)conv_cache, (const Tin*)q,
                             (const Tin*)k, (const Tin*)v, deltas, n_accept, num_seqs, num_rows, num_heads);
    });
  });
  return rc;
}

kda_status kda_state_affine(const float* A, const void* S_in, const float* B, void* S_out, int count,
                            kda_dtype state_dt, void* stream) {
  if (count < 0 || !valid_dtype(state_dt)) return KDA_ERR_INVALID_ARG;
  if (count == 0) return KDA_OK;
  if (!A || !S_in || !B || !S_out) return KDA_ERR_INVALID_ARG;
  const void* al16[] = {A, S_in, B, S_out};
  for (const void* p : al16)
    if (!aligned(p, 16)) return KDA_ERR_ALIGNMENT;
  if (S_out == (const void*)A || S_out == (const void*)B) return KDA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  kda_status rc = KDA_OK;
  by_type(state_dt, [&](auto ts) {
    using Ts = decltype(ts);
    auto kern = state_affine_kernel<Ts>;
    if (!cuda_ok(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, AFFINE_SMEM))) {
      rc = KDA_ERR_CUDA;
      return;
    }
    kern<<<count, 256, AFFINE_SMEM, s>>>(A, (const Ts*)S_in, B, (Ts*)S_out);
    rc = cuda_ok(cudaGetLastError()) ? KDA_OK : KDA_ERR_CUDA;
  });
  return rc;
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
  if (!cuda_ok(cudaStreamSynchronize((cudaStream_t)stream))) return KDA_ERR_CUDA;
  int v = 0;
  if (!cuda_ok(cudaMemcpyFromSymbol(&v, g_status, sizeof(int)))) return KDA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (!cuda_ok(cudaMemcpyToSymbol(g_status, &zero, sizeof(int)))) return KDA_ERR_CUDA;
  }
  return (kda_status)v;
}

kda_status kda_inject_fault(kda_fault kind) {
  if (kind != KDA_FAULT_NONE && kind != KDA_FAULT_DROP_READY) return KDA_ERR_INVALID_ARG;
  kda::pending_fault().store(kind);
  return KDA_OK;
}

int kda_version(void) { return (2 << 16) | 3; }

int kda_last_cuda_error(void) { return kda::t_last_cuda_error; }

}  // extern "C"

// ---- prefill for callers that cannot allocate device memory ------------------
// The chunked path's scratch (chunk table + one operand record per chunk and
// head) lives in this file-scope device array instead of a caller workspace.
// In host code the name below is only a stand-in for the symbol; the device
// address is obtained with cudaGetSymbolAddress, with the device current.
static __device__ __align__(256) unsigned char kda_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

namespace {
// device address of kda_noalloc_scratch on the current device, looked up on
// every call (cheap), so that a context torn down and created again never
// leaves a stale address behind
kda_status noalloc_scratch(void** out) {
  void* p = nullptr;
  if (!cuda_ok(cudaGetSymbolAddress(&p, kda_noalloc_scratch)) || !p) return KDA_ERR_CUDA;
  *out = p;
  return KDA_OK;
}
}  // namespace

extern "C" kda_status kda_prefill_noalloc(const void* q, const void* k, const void* v, const void* g,
                                          const void* beta, const float* conv_w,
                                          const void* init_state, const void* init_conv,
                                          const int32_t* cu_seqlens_dev,
                                          const int32_t* cu_seqlens_host, int num_seqs,
                                          int num_heads, kda_dtype dt, kda_conv_act act,
                                          kda_dtype o_dt, kda_dtype state_dt, void* o,
                                          void* final_state, void* conv_tail, void* stream) {
  PrefillArgs a{q, k, v, g, beta, conv_w, init_state, init_conv, cu_seqlens_dev,
                cu_seqlens_host, num_seqs, num_heads, dt, act, o_dt, state_dt, o, final_state, conv_tail,
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
  const int32_t* cu_used = nullptr;
  st = launch_chunked(a.q, a.k, a.v, a.g, a.beta, a.conv_w, a.init_state, a.init_conv, a.cu_dev,
                      a.cu_host, a.N, a.H, a.act, a.o_dt, a.state_dt, a.o, a.final_state, scratch,
                      a.stream, OutputNorm{}, ChunkedMode::kFull, &cu_used);
  if (st != KDA_OK) return st;
  a.cu_dev = cu_used;
  return launch_tail<__nv_bfloat16>(a);
}
