/*
 * kda.h -- C ABI of libkda.so, the B200 (sm_100a) KDA sequence-mixing library.
 *
 * Operation (page "GLM-5.3-Flash im Detail", section "Sequenz-Mixing:
 * 34 KDA-Schichten mit festem Zustand"; dimensions from "GLM-5.3-Flash
 * Internals - a measured profile", section "Anatomy"): per head, q, k and v pass a
 * causal depthwise convolution of width 4; q and k are L2-normalised; a
 * channel-wise forget gate alpha_t = exp(max(g_t, -5)) decays the state; a
 * scalar beta_t drives a delta-rule write; the query reads the updated state:
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t                    (S_t: 128 x 128 fp32 per head)
 *
 * Prefill evaluates many tokens per call (chunk-parallel inside, state handed
 * from chunk to chunk); decode applies one recurrent update per sequence.  The
 * same section states that prefill and decode use different kernel shapes, and
 * "GLM-5.3-Flash im Detail", section "FP8-Checkpoint und Betriebsgrenzen", that
 * disaggregated prefill and decode share identical KDA layouts: the final state
 * and conv tail written by kda_prefill are exactly the state and conv cache that
 * kda_decode_step consumes.
 *
 * Conventions for every entry point:
 *  - All pointers are caller-owned.  Tensor pointers are DEVICE pointers unless
 *    a parameter name ends in _host.  The library never allocates or frees.
 *  - Head dims are fixed at d_k = d_v = 128 (KDA_HEAD_DIM).
 *  - Per-token tensors are packed token-major, channel contiguous:
 *      q, k, v, g, o : [total_T, H, 128]   beta : [total_T, H]
 *    element type per `dt` (fp32 or bf16).  conv_w is always fp32:
 *      conv_w : [3, H*128, 4]  (q, k, v taps; tap 3 multiplies the current
 *               token, tap 0 the token three steps back; no bias)
 *  - States are [N, H, 128, 128], row = key channel, column = value channel
 *    (value index contiguous), stored with element type `state_dt`:
 *      KDA_F32  -- the state as computed (fp32);
 *      KDA_BF16 -- half the bytes.  All state arithmetic is still fp32; the
 *                  state is rounded to bf16 (nearest, ties to even) wherever
 *                  it is stored: by every decode step, after every committed
 *                  verify row, and once at the end of a prefill call (inside
 *                  a prefill call it stays fp32).  Each stored step moves an
 *                  element by at most half a bf16 ulp (2^-9 relative); the
 *                  rounding errors of successive decode steps add up until
 *                  the gate decays them, so a bf16 state drifts from the fp32
 *                  one by about 1e-2 of its rms within ten steps.
 *    The pages give the model's state as fp32 (page "GLM-5.3-Flash im
 *    Detail", section "Sequenz-Mixing: ...": 128 x 128 fp32 per head); page
 *    "Reading GLM 5.3 Flash from config.json: 6.0 KB of KV Cache per Token"
 *    counts a per-request KDA state of about half the fp32 size, i.e. two
 *    bytes per element.  Conv history / tail / cache is
 *    [N, 3 (q,k,v), 3 (time, oldest first), H*128] in the input dtype.
 *  - L2 norm: x / sqrt(sum x^2 + 1e-6).  No query scale.  Conv activation:
 *    KDA_CONV_NONE (default) or KDA_CONV_SILU (y * sigmoid(y)).
 *  - The output o has its own element type `o_dt` (fp32 or bf16).  Outputs of
 *    this layer are heavy-tailed (an aligned q_t, k_t pair makes |o_t| many
 *    times its rms), so rounding o to bf16 alone moves the largest elements
 *    by several percent of rms; fp32 keeps the full result.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream).  Argument errors are detected on the host before
 *    anything is launched and returned as a status; nothing aborts.
 *  - Alignment: q, k, v, g, o, states, conv tensors and workspace must be
 *    16-byte aligned; beta aligned to its element size.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KDA_HEAD_DIM 128
#define KDA_CHUNK 64
#define KDA_CONV_WIDTH 4

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad cu_seqlens, bad enum   */
  KDA_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement         */
  KDA_ERR_ALIGNMENT = 3,    /* a pointer violates the alignment rule above         */
  KDA_ERR_WORKSPACE = 4,    /* workspace missing or smaller than required          */
  KDA_ERR_CUDA = 5,         /* a CUDA runtime call failed (launch, attribute, ...) */
  KDA_ERR_TIMEOUT = 6       /* a bounded device-side wait gave up (async status)   */
} kda_status;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;
typedef enum { KDA_CONV_NONE = 0, KDA_CONV_SILU = 1 } kda_conv_act;

/* Bytes of device workspace kda_prefill needs for this problem (0 if none).
 * Pure host function; never fails (returns 0 for invalid sizes). */
size_t kda_prefill_workspace_size(int num_seqs, int64_t total_tokens, int num_heads,
                                  int max_seqlen, kda_dtype dt);

/*
 * kda_prefill -- one KDA mixing step over N packed segments (varlen prefill).
 *   q, k, v, g, beta : inputs as laid out above; segment n is rows
 *                      [cu_seqlens[n], cu_seqlens[n+1]).  May be NULL only when
 *                      total_T == 0.
 *   conv_w           : [3, H*128, 4] fp32 conv taps.
 *   init_state       : [N, H, 128, 128] (state_dt), or NULL for zero states.
 *   init_conv        : [N, 3, 3, H*128] raw q/k/v of the 3 tokens before each
 *                      segment (oldest first), or NULL for zeros.
 *   cu_seqlens_dev   : [N+1] int32 device copy of the segment offsets.
 *   cu_seqlens_host  : [N+1] int32 host copy; must equal the device copy.
 *                      cu[0] == 0, non-decreasing.  The chunked (bf16) path
 *                      validates and schedules from this copy and stages it
 *                      in the workspace with its chunk table, and its kernels
 *                      read only that staged copy; the fp32 recurrent path's
 *                      kernels read cu_seqlens_dev.
 *   o_dt             : element type of o (KDA_F32 or KDA_BF16).
 *   state_dt         : element type of init_state and final_state.
 *   o                : out [total_T, H, 128] (o_dt).  Must not alias inputs.
 *   final_state      : out [N, H, 128, 128] (state_dt); may equal init_state
 *                      (in place).
 *   conv_tail        : out [N, 3, 3, H*128] (dt): last 3 raw tokens of
 *                      concat(init_conv, segment); may equal init_conv.
 *   workspace        : device scratch of kda_prefill_workspace_size() bytes
 *                      (may be NULL when that size is 0).
 * Returns KDA_OK once all work is enqueued.  bf16 inputs run the chunked
 * tensor-core path; fp32 inputs run the fp32 recurrent path.
 *
 * Scheduling of the chunked path: when N * H <= 96 (one long sequence, say),
 * its two kernels overlap.  The second runs on a library-owned stream of the
 * current device that is forked from `stream` after the workspace is set up
 * and joined back to it with events before the call's last launch, so all work
 * is still ordered on `stream` as seen from the caller.  Calls from several
 * host threads at once are correct (each fork and join is recorded and
 * awaited under one lock) and their second kernels serialise on that stream.
 * The chunked path stages a chunk table from host memory owned by the call, so
 * it cannot be captured into a CUDA graph: a call on a capturing stream returns
 * KDA_ERR_UNSUPPORTED and enqueues nothing.  The fp32 recurrent path and the
 * decode entry points copy nothing from the host.
 */
kda_status kda_prefill(const void* q, const void* k, const void* v, const void* g,
                       const void* beta, const float* conv_w, const void* init_state,
                       const void* init_conv, const int32_t* cu_seqlens_dev,
                       const int32_t* cu_seqlens_host, int num_seqs, int num_heads,
                       kda_dtype dt, kda_conv_act act, kda_dtype o_dt, kda_dtype state_dt,
                       void* o, void* final_state, void* conv_tail, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * kda_prefill_recurrent -- same contract as kda_prefill, always evaluated by
 * the token-by-token fp32 kernel (one thread block per (segment, head), the
 * state held in registers).  Exact to fp32 rounding for any dtype; slower.
 * Needs no workspace (pass NULL, 0).
 */
kda_status kda_prefill_recurrent(const void* q, const void* k, const void* v, const void* g,
                                 const void* beta, const float* conv_w,
                                 const void* init_state, const void* init_conv,
                                 const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host,
                                 int num_seqs, int num_heads, kda_dtype dt, kda_conv_act act,
                                 kda_dtype o_dt, kda_dtype state_dt, void* o, void* final_state,
                                 void* conv_tail, void* stream);

/*
 * kda_prefill_records / kda_prefill_scan -- the chunked prefill in two halves,
 * for callers that run several scans over the same chunks with different
 * values or initial states (context parallelism: one prefill from S = 0 and
 * one from S = I with v = 0 give a segment's affine carry S_out = A S_in + B,
 * and a third from the carried-in state gives its outputs; page
 * "GLM-5.3-Flash im Detail", section "Sequenz-Mixing: ...": a state is handed
 * from chunk to chunk, linearly).  The chunk records (everything the scan
 * reads that does not involve v or the state) depend on q, k, g, beta, the
 * segments, the heads, conv_w's q and k taps and the q and k rows of
 * init_conv only.
 *   kda_prefill_records : exactly kda_prefill, and the records stay valid in
 *                         `workspace` after the call (kda_prefill drops them
 *                         from L2 without writing them back as they are read).
 *   kda_prefill_scan    : the scan half only: o, final_state and conv_tail of
 *                         a kda_prefill with these arguments, provided that
 *                         `workspace` holds the records of a kda_prefill_records
 *                         call with the same q, k, g, beta, cu_seqlens,
 *                         num_heads, act, conv_w and q/k conv history (v,
 *                         init_state, the v history and the output types may
 *                         differ).  Results are then bit-identical to
 *                         kda_prefill's; with other records they are
 *                         meaningless but every access stays inside
 *                         `workspace`.  Any number of scans may follow one
 *                         records call, until the workspace is reused.
 * Arguments, workspace size and errors are kda_prefill's; fp32 inputs (the
 * recurrent path, which keeps no records) return KDA_ERR_UNSUPPORTED.
 */
kda_status kda_prefill_records(const void* q, const void* k, const void* v, const void* g,
                               const void* beta, const float* conv_w, const void* init_state,
                               const void* init_conv, const int32_t* cu_seqlens_dev,
                               const int32_t* cu_seqlens_host, int num_seqs, int num_heads,
                               kda_dtype dt, kda_conv_act act, kda_dtype o_dt, kda_dtype state_dt,
                               void* o, void* final_state, void* conv_tail, void* workspace,
                               size_t workspace_bytes, void* stream);
kda_status kda_prefill_scan(const void* q, const void* k, const void* v, const void* g,
                            const void* beta, const float* conv_w, const void* init_state,
                            const void* init_conv, const int32_t* cu_seqlens_dev,
                            const int32_t* cu_seqlens_host, int num_seqs, int num_heads,
                            kda_dtype dt, kda_conv_act act, kda_dtype o_dt, kda_dtype state_dt,
                            void* o, void* final_state, void* conv_tail, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * kda_prefill_gated -- kda_prefill followed by the output epilogue, fused into
 * the chunked path's output store, so that the unnormalised o never reaches
 * HBM.  Page "GLM-5.3-Flash Internals - a measured profile", section
 * "Findings": the mixer output passes o_norm, gated by the g_b_proj output,
 * before o_proj.  The pages name these modules only; the reading taken is a
 * gated RMS normalisation over each head's 128 value channels:
 *     o[t, h, :] = x / sqrt(mean_c x_c^2 + norm_eps) * norm_weight * sigmoid(gate[t, h, :])
 * where x is the mixer output kda_prefill would write for (t, h).
 *   gate        : [total_T, H, 128] bf16, the g_b_proj output; must not alias o.
 *   norm_weight : [128] fp32 (shared by the heads), 16-byte aligned.
 *   norm_eps    : >= 0 and finite.
 *   o_dt        : must be KDA_BF16 (the epilogue writes bf16).
 * Every other argument, the workspace and the scheduling are those of
 * kda_prefill.  Errors: as kda_prefill; KDA_ERR_INVALID_ARG for a NULL gate or
 * weight, gate == o, o_dt != KDA_BF16 or a negative / non-finite eps;
 * KDA_ERR_UNSUPPORTED for fp32 inputs (the recurrent path has no fused
 * epilogue: run kda_prefill and then kda_output_norm).
 */
kda_status kda_prefill_gated(const void* q, const void* k, const void* v, const void* g,
                             const void* beta, const float* conv_w, const void* init_state,
                             const void* init_conv, const int32_t* cu_seqlens_dev,
                             const int32_t* cu_seqlens_host, int num_seqs, int num_heads,
                             kda_dtype dt, kda_conv_act act, kda_dtype o_dt, kda_dtype state_dt,
                             void* o, void* final_state, void* conv_tail, void* workspace,
                             size_t workspace_bytes, const void* gate, const float* norm_weight,
                             float norm_eps, void* stream);

/*
 * kda_output_norm -- the same output epilogue on its own, for mixer outputs
 * produced by the decode entry points or the recurrent path:
 *     y[r, h, :] = o[r, h, :] / sqrt(mean_c o[r, h, c]^2 + norm_eps) * norm_weight * sigmoid(gate[r, h, :])
 *   o           : [rows, H, 128] of element type o_dt.
 *   gate        : [rows, H, 128] bf16.
 *   norm_weight : [128] fp32.
 *   y           : out [rows, H, 128] bf16; may equal o when o_dt is KDA_BF16,
 *                 must not alias gate.
 * All pointers 16-byte aligned (KDA_ERR_ALIGNMENT otherwise).  rows == 0
 * enqueues nothing.  Errors: KDA_ERR_INVALID_ARG for a bad size, enum or eps,
 * a NULL pointer or a forbidden alias.
 */
kda_status kda_output_norm(const void* o, kda_dtype o_dt, const void* gate, const float* norm_weight,
                           float norm_eps, void* y, int64_t rows, int num_heads, void* stream);

/*
 * kda_decode_step -- one recurrent update per sequence (page "GLM-5.3-Flash im
 * Detail", section "Sequenz-Mixing: ...": decode of a single token performs a
 * recurrent update), in place.
 *   state      : [N, H, 128, 128] (state_dt), read and overwritten with S_t.
 *   conv_cache : [N, 3, 3, H*128] (dt), read (3 previous raw tokens) and
 *                shifted in place so that it ends with this step's raw token.
 *   q, k, v, g : [N, H, 128] raw inputs of the new token (dt); beta : [N, H].
 *   conv_w     : [3, H*128, 4] fp32.
 *   o_dt, o    : out [N, H, 128] with element type o_dt.
 *   state_dt   : element type of state (o reads the loaded state; the
 *                updated state is rounded when stored).
 * Each (sequence, head) state is streamed through registers exactly once.
 * Errors: KDA_ERR_INVALID_ARG for a bad size or enum, a NULL pointer, or o
 * aliasing an input; KDA_ERR_ALIGNMENT for a pointer that is not 16-byte
 * aligned (beta: element aligned); KDA_ERR_UNSUPPORTED for N > 65535.
 */
kda_status kda_decode_step(void* state, void* conv_cache, const void* q, const void* k,
                           const void* v, const void* g, const void* beta,
                           const float* conv_w, int num_seqs, int num_heads, kda_dtype dt,
                           kda_conv_act act, kda_dtype o_dt, kda_dtype state_dt, void* o,
                           void* stream);

/*
 * Multi-token decode for speculative serving (page "GLM-5.3-Flash Internals -
 * a measured profile": the model serves with multi-token prediction, k = 5
 * drafts, so one verify step carries 6 rows, and about four of them are
 * accepted).  A step verifies R rows against each sequence's state without
 * changing it, and a second call keeps the accepted prefix:
 *
 *   kda_decode_verify(state, cache, rows 0..R-1) -> o for every row, deltas
 *   kda_decode_commit(state, cache, rows, deltas, n_accept) -> state and cache
 *       after the first n_accept[n] rows of sequence n
 *
 * Row t of a sequence is decoded exactly as kda_decode_step would decode it
 * after rows 0..t-1 (same arithmetic in the same order), so verify outputs and
 * the committed state and cache equal those of n single-token steps, bit for
 * bit.  The state is read once by verify and read and written once by commit,
 * instead of once per row.
 *
 * Common arguments:
 *   num_seqs N, num_rows R (1 <= R <= KDA_MAX_VERIFY_ROWS), num_heads H.
 *   q, k, v, g : [N, R, H, 128] raw rows (dt), row t of sequence n at
 *                (n * R + t); beta : [N, R, H].
 *   deltas     : device scratch of kda_decode_deltas_size(N, R, H) bytes,
 *                [N, H, R, 3, 128] fp32 (k_hat, u, alpha of each row), written
 *                by verify and read by commit; caller-owned.
 */
#define KDA_MAX_VERIFY_ROWS 8
size_t kda_decode_deltas_size(int num_seqs, int num_rows, int num_heads);

/*
 * kda_decode_verify -- decode rows 0..R-1 of every sequence in turn from
 * `state` and `conv_cache`, neither of which is modified.
 *   state      : [N, H, 128, 128] (state_dt), read only.  With a bf16 state,
 *                row t + 1 starts from the state after row t rounded to bf16,
 *                as the single step of row t would have stored it.
 *   conv_cache : [N, 3, 3, H*128] (dt), read only.
 *   conv_w     : [3, H*128, 4] fp32.
 *   o_dt, o    : out [N, R, H, 128], row t = o of that row.
 *   deltas     : out, see above.
 * Errors: KDA_ERR_INVALID_ARG for R outside [1, KDA_MAX_VERIFY_ROWS], a NULL
 * pointer, or outputs aliasing inputs; KDA_ERR_ALIGNMENT for a pointer that
 * is not 16-byte aligned (beta: element aligned); KDA_ERR_UNSUPPORTED for
 * N > 65535.  Nothing is launched on error.
 */
kda_status kda_decode_verify(const void* state, const void* conv_cache, const void* q, const void* k,
                             const void* v, const void* g, const void* beta, const float* conv_w,
                             int num_seqs, int num_rows, int num_heads, kda_dtype dt, kda_conv_act act,
                             kda_dtype o_dt, kda_dtype state_dt, void* o, float* deltas, void* stream);

/*
 * kda_decode_commit -- apply the first n_accept[n] verified rows of sequence
 * n: state and conv_cache (same layouts as kda_decode_verify) are updated in
 * place to what n_accept[n] calls of kda_decode_step would leave.
 *   q, k, v  : the same raw rows that were verified (the conv cache takes the
 *              last three raw tokens of [cache, accepted rows]).
 *   deltas   : as written by kda_decode_verify for these rows and this state.
 *   n_accept : [N] int32 on the device, each in [0, R]; 0 leaves that
 *              sequence untouched.  A value outside [0, R] is clamped to it
 *              and recorded as KDA_ERR_INVALID_ARG in the device status word
 *              (kda_check_async_status).
 * Errors as for kda_decode_verify.
 */
kda_status kda_decode_commit(void* state, void* conv_cache, const void* q, const void* k, const void* v,
                             const float* deltas, const int32_t* n_accept, int num_seqs, int num_rows,
                             int num_heads, kda_dtype dt, kda_dtype state_dt, void* stream);

/*
 * kda_decode_commit_verify -- kda_decode_commit of the previous speculative
 * step followed by kda_decode_verify of the next one, in one pass over each
 * state: the state is read once and written once (not at all when no row of
 * the previous step is kept), where the two separate calls read it twice.
 *   1. The first prev_n_accept[n] rows of the previous step are kept, with
 *      exactly the arithmetic of kda_decode_commit: state and conv_cache are
 *      updated in place and stored.
 *   2. The num_rows new rows are verified from the updated state and cache
 *      exactly as kda_decode_verify would verify them: o and deltas.
 * So the results equal kda_decode_commit(prev ...) then kda_decode_verify(...),
 * bit for bit.
 *   prev_q, prev_k, prev_v : the previous step's raw rows [N, prev_rows, H, 128]
 *                            (dt), as given to its verify.
 *   prev_deltas            : the deltas its verify wrote.
 *   prev_n_accept          : [N] int32 on the device, each in [0, prev_rows];
 *                            out-of-range values are clamped and recorded as
 *                            for kda_decode_commit.
 *   prev_rows              : rows of the previous step, 1..KDA_MAX_VERIFY_ROWS.
 *   deltas                 : out, the new rows' deltas; must not overlap
 *                            prev_deltas (callers alternate two buffers).
 * Other arguments as for kda_decode_verify.  A first step (no previous step)
 * is a plain kda_decode_verify.
 * Errors: as for kda_decode_verify, and KDA_ERR_INVALID_ARG for prev_rows out
 * of range, a NULL previous-step pointer or overlapping deltas.
 */
kda_status kda_decode_commit_verify(void* state, void* conv_cache, const void* prev_q, const void* prev_k,
                                    const void* prev_v, const float* prev_deltas, const int32_t* prev_n_accept,
                                    int prev_rows, const void* q, const void* k, const void* v, const void* g,
                                    const void* beta, const float* conv_w, int num_seqs, int num_rows,
                                    int num_heads, kda_dtype dt, kda_conv_act act, kda_dtype o_dt,
                                    kda_dtype state_dt, void* o, float* deltas, void* stream);

/*
 * kda_prefill_noalloc -- kda_prefill for callers that cannot allocate device
 * memory.  (Not an operation of the method: the pages have no counterpart; it
 * only changes where the scratch lives.)
 *
 * Some callers cannot call cudaMalloc or hand the library a workspace: an
 * inference server that has carved all device memory into its own pools
 * before serving starts, or a plugin whose host application owns every device
 * allocation.  This entry point takes the same arguments as kda_prefill
 * without the workspace and allocates nothing (no cudaMalloc, cudaFree or
 * allocating library call).  Its scratch is one static device array of
 * KDA_NOALLOC_SCRATCH_BYTES that the library holds on every GPU that loads it,
 * until the process exits.
 *   - Problems whose kda_prefill_workspace_size() exceeds
 *     KDA_NOALLOC_SCRATCH_BYTES are rejected with KDA_ERR_WORKSPACE before any
 *     launch (about 1000 chunk-heads: (sum over segments of ceil(T_n / 64))
 *     x num_heads <= 1000 fits).
 *   - Every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress; no allocation).
 *   - All calls share the one array and it keeps the last call's contents
 *     (every byte a call reads is written earlier in that same call, so
 *     nothing needs clearing).  Calls whose work overlaps on the GPU (other
 *     streams, other host threads) race on it: serialise them.
 *   - fp32 inputs use the recurrent path, which needs no scratch.
 */
#define KDA_NOALLOC_SCRATCH_BYTES ((size_t)128 << 20)
kda_status kda_prefill_noalloc(const void* q, const void* k, const void* v, const void* g,
                               const void* beta, const float* conv_w, const void* init_state,
                               const void* init_conv, const int32_t* cu_seqlens_dev,
                               const int32_t* cu_seqlens_host, int num_seqs, int num_heads,
                               kda_dtype dt, kda_conv_act act, kda_dtype o_dt, kda_dtype state_dt,
                               void* o, void* final_state, void* conv_tail, void* stream);

/*
 * kda_state_affine -- S_out = A S_in + B for `count` (sequence, head) states:
 * the exchange step of one long sequence split into contiguous segments
 * (context parallelism).  Page "GLM-5.3-Flash im Detail", section
 * "Sequenz-Mixing: ...": the state is handed from chunk to chunk, and that
 * hand-over is linear in the state, so a whole segment maps its initial state
 * as S_out = A S_in + B.  B is the segment's final state from S_in = 0; A
 * (key x key) is its final state from S_in = I with v = 0 (each value column a
 * probe; the v part of the conv history zero as well), both from kda_prefill.
 * A rank composes its segment's initial state from the (A, B) of every
 * earlier segment, one call per segment.
 *   A, B        : [count, 128, 128] fp32, row = key channel.
 *   S_in, S_out : [count, 128, 128] (state_dt); S_out may equal S_in (every
 *                 state is read before it is written), not A or B.
 * fp32 arithmetic with a k-ascending sum.  Errors: KDA_ERR_INVALID_ARG for a
 * NULL pointer, count < 0, a bad state_dt or S_out aliasing A or B;
 * KDA_ERR_ALIGNMENT for a pointer that is not 16-byte aligned.
 */
kda_status kda_state_affine(const float* A, const void* S_in, const float* B, void* S_out, int count,
                            kda_dtype state_dt, void* stream);

/* Static description of a status code (never NULL). */
const char* kda_status_string(kda_status s);

/*
 * Synchronises `stream`, then returns and clears the library's device status
 * word on the current device: KDA_OK, or KDA_ERR_TIMEOUT if a bounded
 * device-side wait gave up since the last call (the kernel that gave up
 * stopped early, so its outputs are invalid), KDA_ERR_INVALID_ARG if
 * kda_decode_commit met an n_accept outside [0, R], or KDA_ERR_CUDA if the
 * synchronisation itself failed.
 */
kda_status kda_check_async_status(void* stream);

/*
 * Host-side fault injection, for tests of the failure path only.
 *   KDA_FAULT_DROP_READY : the next kda_prefill / kda_prefill_noalloc call
 *       that takes the overlapped chunked mode (at most 96 (sequence, head)
 *       pairs) launches its preparation kernel without the per-chunk ready
 *       flags, so the flags the scan waits on are never published.  The scan's
 *       bounded waits give up (after 2 s plus 1 us per (chunk, head) work
 *       item of the call, timed by %globaltimer), every block drains its own copies
 *       and tensor-core work, frees its tensor memory and returns; the call's
 *       outputs are invalid and kda_check_async_status reports
 *       KDA_ERR_TIMEOUT.  The context stays usable.
 *   KDA_FAULT_NONE       : clears a pending fault.
 * A fault is pending until one call applies it (one-shot); process-wide.
 * Errors: KDA_ERR_INVALID_ARG for an unknown kind.  Pure host function.
 */
typedef enum { KDA_FAULT_NONE = 0, KDA_FAULT_DROP_READY = 1 } kda_fault;
kda_status kda_inject_fault(kda_fault kind);

/*
 * The cudaError_t value behind the last KDA_ERR_CUDA that an entry point
 * returned on the calling host thread (0 if none has been returned yet).  Pure
 * host function; the value is not cleared by later successful calls.
 */
int kda_last_cuda_error(void);

/* Library ABI version: (major << 16) | minor. */
int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
