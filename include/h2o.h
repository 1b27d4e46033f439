/*
 * h2o.h -- C ABI of the chunked H2O sparse-attention step on one B200.
 *
 * The operation (from "Learning how to Forget: Fine-tuning for Long-Context
 * Sparse Attention", arXiv 2608.19920):
 *   - §1 Introduction: keys and values live in a fixed-size KV cache of C
 *     slots; when the cache is full, a policy evicts slots.  H2O (heavy-hitter
 *     oracle) is the policy the paper optimises, with dedicated SDPA kernels.
 *   - §1, second contribution: the SDPA kernel also returns the attention
 *     weight each key received, summed over queries (and heads).
 *   - §2 Related work: the summed attention weights are H2O's score input.
 *   - Summary page, glossary "H2O": cache entries are scored by how often and
 *     how strongly they were attended; the less important ones are evicted.
 *
 * One step, for each independent cache b and KV head g, with G = H_q / H_kv
 * query heads per KV head, n valid slots and a chunk of n_q tokens at
 * positions t0 .. t0+n_q-1:
 *   1. O = softmax(scale * Q K^T) V, where query i of head h (KV head h / G)
 *      sees the n valid cache slots and chunk keys j <= i.
 *   2. colsum[b,g,key] = sum over the G heads and the n_q queries of the
 *      softmax probability that key received.
 *   3. score[s] += colsum (fp32) for every valid slot s; new token i gets
 *      candidate score colsum of chunk key i.
 *   4. If n + n_q <= C the new tokens fill slots n .. n+n_q-1.  Otherwise keep
 *      every candidate at position >= t0 + n_q - W (recent window) and the
 *      highest-scoring others up to C entries; ties go to the lower candidate
 *      index (slot s -> s, new token i -> C + i).  The kept new tokens, in
 *      ascending order, move into the freed and empty slots in ascending
 *      order; kept entries stay in place.
 *   5. n <- min(C, n + n_q); t0 <- t0 + n_q.
 *
 * Layouts (row-major, contiguous, every base pointer 16-byte aligned; the
 * workspace 256-byte aligned):
 *   q, out            [batch, n_q, H_q, head_dim]      element type = dtype
 *   k_new, v_new      [batch, n_q, H_kv, head_dim]     element type = dtype
 *   cache k, v        [batch, H_kv, capacity, head_dim] element type = dtype
 *                     (Q8: int8 codes, then [batch, H_kv, capacity] float32
 *                     scales, see h2o_dtype)
 *   scores            [batch, H_kv, capacity]          float32
 *   pos               [batch, H_kv, capacity]          int32, -1 = empty slot
 *   state             [4] int32: n, t0, device error bits, reserved
 *   colsum (in/out)   [batch, H_kv, capacity + n_q]    float32; entry s < n is
 *                     cache slot s, entries n .. capacity-1 are 0, entry
 *                     capacity + j is chunk key j.
 *
 * Conventions:
 *   - Every call is asynchronous on the given CUDA stream (NULL = legacy
 *     default stream).  Argument errors are returned synchronously, before
 *     anything is launched.  Errors detected on the device (a bounded wait
 *     that expired, an inconsistent eviction plan) are latched in state[2]
 *     and returned by h2o_cache_check().
 *   - All memory is owned by the caller; the library allocates nothing on
 *     the device.  h2o_cache_destroy() frees the host handle and the copy
 *     streams and events that h2o_chunk_step_host creates on first use.
 *   - All caches of a handle advance together (one n_q per call).  A handle
 *     must not be used from two host threads at once.
 *   - Supported: head_dim 64 or 128; dtype BF16 or Q8 (tensor-core path) or
 *     F32 (fp32 FMA path); H_q a multiple of H_kv; 0 <= recent_window <=
 *     capacity; capacity + max_chunk <= 50176 (the selection keeps one fp32
 *     key per candidate in shared memory).
 */
#ifndef H2O_H_
#define H2O_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define H2O_API __attribute__((visibility("default")))
#else
#define H2O_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  H2O_OK = 0,
  H2O_ERR_INVALID_ARG = 1, /* null pointer, n_q out of range, bad handle     */
  H2O_ERR_SHAPE = 2,       /* unsupported sizes, buffer too small            */
  H2O_ERR_DTYPE = 3,       /* unknown dtype                                  */
  H2O_ERR_ALIGN = 4,       /* pointer not 16-byte (workspace: 256-byte) aligned */
  H2O_ERR_CUDA = 5,        /* a CUDA runtime call failed                     */
  H2O_ERR_TIMEOUT = 6,     /* a kernel's bounded wait expired (device bit 1) */
  H2O_ERR_STATE = 7        /* inconsistent eviction plan (device bit 2), a
                              kernel's shared-memory layout check (bit 4), or,
                              in the H2O_DEBUG build libh2o_debug.so, a failed
                              bounds check (bit 8; the access is skipped)    */
} h2o_status;

/* Element types.  BF16 and F32: q, k_new, v_new, out and the cache's K and V
 * all of that type.  Q8 (the quantised cache of Q-Hitter, page 1 §2 Related
 * Work: "Q-Hitter combines H2O with quantisation"; summary page Table 5,
 * qh2o rows -- the pages give no format, this is the one read here): q,
 * k_new, v_new and out are bf16; every cache row (one slot of one KV head, K
 * and V separately) is stored as head_dim int8 codes and one fp32 scale,
 *   s = fl32(max|x| / 127),  code = clamp(rint(fl32(x / s)), -127, 127)
 * (ties to even; an all-zero row has s = 0), and the attention reads
 * bf16(fl32(code * s)).  A new token is quantised when it is placed into the
 * cache; within the step that brings it, it is attended at its bf16 input
 * value.  The cache K (and V) buffer holds the codes
 * [batch, H_kv, capacity, head_dim] int8 followed by the scales
 * [batch, H_kv, capacity] float32. */
typedef enum { H2O_BF16 = 0, H2O_F32 = 1, H2O_Q8 = 2 } h2o_dtype;

/* Eviction policy.  H2O ranks the unprotected candidates by their
 * accumulated attention (the summed weights added to the score each step);
 * LR and SLR are score-free: they rank by position (the most recent stay),
 * SLR also always keeps the sequence's first sink_tokens positions.  The
 * recent window protects in every policy; placement is the same.  LR and SLR
 * keep no scores (placed tokens get 0) and skip the summed-weights kernel
 * unless colsum_out asks for them. */
typedef enum { H2O_POLICY_H2O = 0, H2O_POLICY_LR = 1, H2O_POLICY_SLR = 2 } h2o_policy;

typedef struct {
  int32_t batch;          /* independent caches (layers x sequences), >= 1   */
  int32_t n_q_heads;      /* H_q                                             */
  int32_t n_kv_heads;     /* H_kv, divides H_q                               */
  int32_t head_dim;       /* 64 or 128                                       */
  int32_t capacity;       /* C, slots per (cache, KV head)                   */
  int32_t max_chunk;      /* largest n_q accepted by the step calls          */
  int32_t recent_window;  /* W, 0 <= W <= C                                  */
  h2o_dtype dtype;        /* element type of q, k, v, out and the cache      */
  float softmax_scale;    /* <= 0 selects 1/sqrt(head_dim)                   */
  int32_t policy;         /* h2o_policy                                      */
  int32_t sink_tokens;    /* SLR: positions < sink_tokens always stay;
                             0 <= sink_tokens, sink_tokens + recent_window
                             <= capacity; ignored by the other policies      */
} h2o_config;

/* Byte sizes of the caller-owned device buffers for a configuration. */
typedef struct {
  size_t k_bytes, v_bytes;  /* cache K and V                                 */
  size_t scores_bytes;      /* float32 scores                                */
  size_t pos_bytes;         /* int32 positions                               */
  size_t state_bytes;       /* 4 x int32                                     */
  size_t workspace_bytes;   /* row statistics, summed weights, eviction plan,
                               the logits and split-KV partials of n_q = 1
                               calls, and staging for h2o_chunk_step_host    */
} h2o_sizes;

/* Caller-owned device buffers (sizes from h2o_required_bytes). */
typedef struct {
  void* k;
  void* v;
  float* scores;
  int32_t* pos;
  int32_t* state;
  void* workspace;
  size_t workspace_bytes;
} h2o_buffers;

typedef struct h2o_cache h2o_cache;

/* Validates cfg and fills *out.  Host only; touches no device. */
H2O_API h2o_status h2o_required_bytes(const h2o_config* cfg, h2o_sizes* out);

/* Creates a handle over caller-owned buffers and, on `stream`, clears the
 * cache to the empty state (K, V, scores = 0; pos = -1; n = t0 = 0; no
 * error).  The buffers must stay valid until h2o_cache_destroy. */
H2O_API h2o_status h2o_cache_create(const h2o_config* cfg, const h2o_buffers* bufs,
                            void* stream, h2o_cache** out);

/* The whole step (attention with summed weights, score update, selection,
 * placement) for all caches.  q, k_new, v_new, out: device pointers in the
 * layouts above with 1 <= n_q <= max_chunk (n_q = 0 is a no-op).
 * colsum_out (device, may be NULL) receives the summed weights in the colsum
 * layout.  Advances n and t0.  A decode step (n_q = 1, at most 8 query heads
 * per KV head) runs as two launches (split-KV attention; merge, summed
 * weights and the single-token eviction), other steps as three. */
H2O_API h2o_status h2o_chunk_step(h2o_cache* c, const void* q, const void* k_new,
                          const void* v_new, int32_t n_q, void* out,
                          float* colsum_out, void* stream);

/* Same step with HOST buffers (pinned memory recommended).  The inputs are
 * uploaded into one of two staging sets of the workspace (alternate calls
 * use alternate sets), the step runs on `stream`, and out is downloaded
 * back.  The uploads and downloads run on two streams the cache owns, one
 * per direction, ordered with `stream` by events, so one call's copies
 * overlap the kernels of the calls before and after it.
 *   - The input host buffers must stay untouched until `stream` has passed
 *     this call's step (the step waits for the upload).
 *   - out_host is complete once h2o_cache_host_join has been called on a
 *     stream and that stream has passed the join; until then it may still
 *     be in transfer.
 *   - colsum_out_host (may be NULL) is copied on `stream` itself, after the
 *     step.
 * The workspace holds both staging sets (h2o_required_bytes counts them). */
H2O_API h2o_status h2o_chunk_step_host(h2o_cache* c, const void* q_host,
                               const void* k_new_host, const void* v_new_host,
                               int32_t n_q, void* out_host,
                               float* colsum_out_host, void* stream);

/* Makes `stream` wait until every download issued by h2o_chunk_step_host
 * on this cache so far has landed in host memory (no-op before the first
 * host call).  Does not block the host. */
H2O_API h2o_status h2o_cache_host_join(h2o_cache* c, void* stream);

/* Steps 1-2 only: out and colsum_out (both device; colsum_out may be NULL)
 * for the current cache contents.  The cache state does not change. */
H2O_API h2o_status h2o_attention(h2o_cache* c, const void* q, const void* k_new,
                         const void* v_new, int32_t n_q, void* out,
                         float* colsum_out, void* stream);

/* Backward of h2o_attention for fine-tuning through the cache: the
 * gradients of O with respect to q, the cache's K and V and the chunk's
 * k_new and v_new, with the cache contents and visibility held fixed (the
 * eviction that follows is a discrete decision and is not differentiated).
 * Call it after h2o_attention with the same q, k_new, v_new, n_q and before
 * anything changes the cache (h2o_evict, a step, h2o_cache_write); it reads
 * that call's row statistics from the workspace (else H2O_ERR_STATE).
 * out, d_out: device [batch, n_q, H_q, d] bf16 (O of that call and dL/dO).
 * Outputs, device float32, 16-byte aligned: dq [batch, n_q, H_q, d];
 * dk_cache, dv_cache [batch, H_kv, C, d] (rows of slots >= n are zero);
 * dk_new, dv_new [batch, n_q, H_kv, d].  BF16 caches only (F32 and Q8:
 * H2O_ERR_DTYPE); n_q >= 2 (a one-token h2o_attention runs the decode
 * kernels, which keep no row statistics).  Deterministic (fixed reduction
 * order). */
H2O_API h2o_status h2o_attention_backward(h2o_cache* c, const void* q, const void* k_new,
                                          const void* v_new, int32_t n_q, const void* out,
                                          const void* d_out, float* dq, float* dk_cache,
                                          float* dv_cache, float* dk_new, float* dv_new,
                                          void* stream);

/* Steps 3-5 only, with caller-supplied summed weights `colsum` (device,
 * colsum layout for this n_q, float32).  Advances n and t0. */
H2O_API h2o_status h2o_evict(h2o_cache* c, const float* colsum, const void* k_new,
                     const void* v_new, int32_t n_q, void* stream);

/* Copies the cache state out.  k, v, scores, pos may each be NULL or a
 * device or host pointer (the copy kind is inferred); n_t0 (host, may be
 * NULL) receives {n, t0}. */
H2O_API h2o_status h2o_cache_read(const h2o_cache* c, void* k, void* v, float* scores,
                          int32_t* pos, int32_t* n_t0, void* stream);

/* Replaces the cache state (checkpoint restore).  Pointers as in
 * h2o_cache_read (all four required); n_t0 (host) = {n, t0} with
 * 0 <= n <= capacity and t0 >= n.  Clears the device error bits. */
H2O_API h2o_status h2o_cache_write(h2o_cache* c, const void* k, const void* v,
                           const float* scores, const int32_t* pos,
                           const int32_t* n_t0, void* stream);

/* Synchronises `stream` and returns the device error bits as a status:
 * H2O_OK, H2O_ERR_TIMEOUT or H2O_ERR_STATE (or H2O_ERR_CUDA). */
H2O_API h2o_status h2o_cache_check(h2o_cache* c, void* stream);

/* Host-side view of the handle: n, t0 and the number of kernels launched
 * through it so far (each may be NULL). */
H2O_API h2o_status h2o_cache_info(const h2o_cache* c, int32_t* n, int32_t* t0,
                          uint64_t* kernel_launches);

/* Per-kernel timing.  While enabled, every step records a CUDA event on its
 * stream before its first kernel and after each kernel.  h2o_cache_kernel_ms
 * waits for the last recorded event and writes the device durations (ms) of
 * the last step's kernels: [0] attention forward, [1] summed weights,
 * [2] score update + selection + K/V scatter (one kernel), [3] reserved,
 * reads 0 (a kernel that did not run reads 0).  Disabled by default; enabling creates the events on the
 * current device. */
H2O_API h2o_status h2o_cache_set_timing(h2o_cache* c, int enable);
H2O_API h2o_status h2o_cache_kernel_ms(h2o_cache* c, float* ms4);

/* Attention with summed weights (steps 1-2 of the step) that allocates
 * nothing and needs no handle or workspace.  The paper has no counterpart:
 * this entry point exists for callers that cannot allocate device memory --
 * engines or plugin hosts that own the whole memory budget and pass a
 * plugin only its inputs and outputs, and serving loops that must not
 * allocate once running.  The row statistics the two kernels share live in
 * a static device array of the library (16 MiB per GPU that loads it, held
 * until the process exits), so
 *   batch * n_q_heads * (n_q rounded up to a multiple of 128) <= 4194304
 * or the call returns H2O_ERR_SHAPE before launching anything.
 * Inputs: cfg (capacity, heads, head_dim, dtype BF16 or F32 (Q8:
 * H2O_ERR_DTYPE), scale; max_chunk bounds
 * n_q; recent_window unused), k_cache / v_cache (device, cache layout) with
 * n valid slots, q, k_new, v_new (device, chunk layouts).  Outputs (device):
 * out, and colsum_out in the colsum layout for this n_q (required).
 * The first call on a device looks up the array's device address on the
 * current device (cudaGetSymbolAddress; safe if several host threads make
 * it at once); make that first call before any stream capture.  All calls
 * on a device share the array and it keeps the last call's contents
 * (nothing in it needs clearing between calls), so calls that overlap on
 * the GPU race on it: serialise them.  A static error word beside it is
 * cleared at the start of every call (cudaMemsetAsync on `stream`) and
 * latches an expired bounded wait of that call's kernels, in which case out
 * and colsum_out are incomplete: h2o_static_scratch_check reports it. */
H2O_API h2o_status h2o_attention_static_scratch(const h2o_config* cfg, const void* k_cache,
                                                const void* v_cache, int32_t n, const void* q,
                                                const void* k_new, const void* v_new,
                                                int32_t n_q, void* out, float* colsum_out,
                                                void* stream);

/* Status of the last h2o_attention_static_scratch call on the current
 * device: synchronises `stream` (the stream of that call), then returns
 * H2O_ERR_TIMEOUT if one of its kernels' bounded waits expired (its outputs
 * are then incomplete), H2O_OK otherwise (or H2O_ERR_CUDA).  No counterpart
 * in the paper; allocates nothing. */
H2O_API h2o_status h2o_static_scratch_check(void* stream);

/* Diagnostic of the failure path: one warp waits, with the same bounded
 * wait the kernels use, on a barrier nothing completes.  After limit_us
 * (1 .. 2,000,000) the wait gives up, ORs the timeout bit (1) into
 * *err_word (device int32; NULL selects the error word that
 * h2o_static_scratch_check reports) and the kernel returns; the context
 * stays usable.  No trap, no hang. */
H2O_API h2o_status h2o_selftest_wait_timeout(int32_t* err_word, uint32_t limit_us,
                                             void* stream);

/* Diagnostic of the kernels' FMA-pipe exponential: y[i] = 2^x[i] computed
 * the way the attention kernels compute part of their exponentials without
 * the special function unit (Cody-Waite range reduction and a degree-3
 * minimax polynomial: relative error below 7.5e-5 for -125 <= x <= 0; x
 * below -125, -inf included, gives about 2^-125).  x, y: device float32 arrays
 * of n elements.  No counterpart in the paper. */
H2O_API h2o_status h2o_selftest_exp2(const float* x, float* y, int32_t n, void* stream);

/* Waits for the copies h2o_chunk_step_host still has in flight, then frees
 * the host handle and its copy streams and events.  Device buffers stay the
 * caller's. */
H2O_API void h2o_cache_destroy(h2o_cache* c);

H2O_API const char* h2o_status_string(h2o_status s);

#ifdef __cplusplus
}
#endif

#endif /* H2O_H_ */
