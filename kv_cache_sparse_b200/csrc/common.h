// common.h -- definitions shared by the host API and the kernels.
#pragma once

#include <cuda.h>
#include <stdint.h>
#include <string.h>

namespace h2o {

// Device error bits, latched in state[2].
constexpr int kDevErrTimeout = 1;  // a bounded mbarrier wait expired
constexpr int kDevErrPlan = 2;     // freed-slot and kept-token counts disagree
constexpr int kDevErrSmem = 4;     // dynamic shared memory too small after alignment
constexpr int kDevErrBounds = 8;   // H2O_DEBUG builds: an index failed its bounds check

// Bounds checks of the H2O_DEBUG build (libh2o_debug.so): a failed check
// latches kDevErrBounds in the error word and the access is skipped; it never
// traps.  In the normal build the checks compile to nothing.
#if defined(__CUDACC__)
#ifdef H2O_DEBUG
__device__ __forceinline__ bool debug_in_bounds(bool ok, int* err) {
  if (!ok) atomicOr(err, kDevErrBounds);
  return ok;
}
#define H2O_IN_BOUNDS(cond, err) ::h2o::debug_in_bounds((cond), (err))
#else
#define H2O_IN_BOUNDS(cond, err) true
#endif
#endif

// Largest dynamic shared memory a CTA may request on sm_100 (227 KiB).
constexpr int kMaxDynSmem = 232448;

// Longest time a kernel thread waits on one mbarrier phase before it gives up.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

constexpr int kTileRows = 128;  // query rows per attention tile (TMEM lanes)
constexpr int kTileKeys = 128;  // keys per attention tile

// Largest capacity + max_chunk the selection kernel keeps in shared memory.
constexpr int kMaxCandidates = 50176;

__host__ __device__ inline int cdiv(int a, int b) { return (a + b - 1) / b; }

// A 32-bit key that orders like the fp32 value, negative values included:
// non-negative values get the sign bit set, negative ones all bits flipped;
// -0 is +0.  The largest key (0xFFFFFFFF) is left free for the selection's
// "protected" mark (only a NaN pattern would map there).
__host__ __device__ inline uint32_t ordered_key(float v) {
  uint32_t u;
  memcpy(&u, &v, sizeof(u));
  if (u == 0x80000000u) u = 0u;
  const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return k == 0xFFFFFFFFu ? 0xFFFFFFFEu : k;
}

// ---------------------------------------------------------------- attention

// Arguments of the tensor-core attention kernel and the column-sum kernel.
struct AttnParams {
  int B, Hq, Hkv, G;    // caches, query heads, KV heads, heads per group
  int nq;               // chunk length of this call
  int n;                // valid cache slots
  int C;                // capacity
  int nq_pad;           // row stride of the row statistics (multiple of 128)
  float scale_log2;     // softmax scale * log2(e)
  void* out;            // [B, nq, Hq, d]
  float* nlse2;         // [B, Hq, nq_pad]: minus the log2-domain log-sum-exp of
                        // each row (-inf for padding rows), so 2^(x + nlse2)
                        // is the row's normalised probability
  float* colsum;        // [B, Hkv, colsum_ld]
  int colsum_ld;        // row stride of colsum (>= C + nq)
  int* err;             // device error word (state + 2)
  // int8 cache (Q8): one fp32 scale per (cache, KV head, slot) of K and V,
  // [B*Hkv, C]; null for the bf16 cache
  const float* k_scale;
  const float* v_scale;
};

// Arguments of the backward kernels (attn_bwd.cu).
struct BwdParams {
  int B, Hq, Hkv, G, nq, n, C, nq_pad;
  float scale;            // softmax scale (natural)
  float scale_log2;       // scale * log2(e)
  const float* nlse2;     // [B, Hq, nq_pad]: the forward's -lse2 (-inf for padding rows)
  float* dsum;            // [B, Hq, nq_pad]: -scale * D_i, D_i = <dO_i, O_i> (0 past nq)
  float* dq;              // [B, nq, Hq, d]
  float* dk_cache;        // [B, Hkv, C, d]
  float* dv_cache;
  float* dk_new;          // [B, nq, Hkv, d]
  float* dv_new;
  int* err;               // device error word (state + 2)
};

// ---------------------------------------------------------------- eviction

constexpr int kPolicyH2O = 0;
constexpr int kPolicyLR = 1;
constexpr int kPolicySLR = 2;

struct EvictParams {
  int B, Hkv, C, d, esize;  // esize: bytes per element of K/V
  int n, t0, nq, W;
  const float* colsum;      // [B, Hkv, colsum_ld]
  int colsum_ld;
  float* scores;            // [B, Hkv, C]
  int* pos;                 // [B, Hkv, C]
  int* plan_slots;          // [B, Hkv, max_chunk]
  int* plan_tokens;         // [B, Hkv, max_chunk]
  int* plan_count;          // [B, Hkv]
  int plan_ld;              // max_chunk
  const void* k_new;        // [B, nq, Hkv, d]
  const void* v_new;
  void* k_cache;            // [B, Hkv, C, d]
  void* v_cache;
  int* state;               // [4]: n, t0, err, reserved
  int policy;               // kPolicyH2O (rank by score), kPolicyLR / kPolicySLR (by position)
  int sinks;                // kPolicySLR: positions < sinks are protected
  // int8 cache (Q8): new rows (bf16, esize 2 in k_new / v_new) are quantised
  // into the cache's int8 codes (esize is then 1) and per-slot scales
  int q8;
  float* k_scale;           // [B*Hkv, C]
  float* v_scale;
};

// ---------------------------------------------------------------- decode (n_q = 1)

constexpr int kDecodeMaxG = 8;        // largest GQA group the decode kernels take
constexpr int kDecodeSliceKeys = 1024;  // keys per CTA of the merge kernel

// Keys per split-KV partial: 32 KiB of K (and of V) rows, at most 256 keys.
__host__ __device__ constexpr int decode_chunk_keys(int head_dim, int esize) {
  return 32768 / (head_dim * esize) < 256 ? 32768 / (head_dim * esize) : 256;
}

struct DecodeParams {
  int B, Hkv, G, C;         // caches, KV heads, heads per group, capacity
  int n, t0, W;             // valid slots, position of the new token, window
  int n_chunks;             // cdiv(n + 1, decode_chunk_keys): key n is the new token
  int part_ld;              // chunks per (cache, KV head) in part
  int n_slices;             // cdiv(n + 1, kDecodeSliceKeys): CTAs of the merge per head
  int slices_ld;            // entries per (cache, KV head) in best
  unsigned long long* best; // [B*Hkv, slices_ld]: each merge CTA's eviction candidate
  int* ticket;              // [B*Hkv]: merge CTAs done (zero between steps)
  int spread_o;             // 1: every merge CTA of a head merges part of O
  float scale_log2;         // softmax scale * log2(e)
  const void* q;            // [B, 1, Hq, d]
  const void* k_new;        // [B, 1, Hkv, d]
  const void* v_new;
  void* k_cache;            // [B, Hkv, C, d]
  void* v_cache;
  void* out;                // [B, 1, Hq, d]
  float* logits;            // [B*Hkv, G, C + 1]: x = scale*log2(e)*<q, k>, key n = new token
  float* part;              // [B*Hkv, part_ld, G, d + 2]: unnormalised O, max, sum per chunk
  float* colsum;            // [B*Hkv, colsum_ld]: slots, zeros up to C, then the new key at C
  int colsum_ld;
  float* scores;            // [B, Hkv, C]   (eviction only)
  int* pos;                 // [B, Hkv, C]
  int* state;               // [4]: n, t0, err, reserved
  int evict;                // 1: score update and placement after the attention
  int policy;               // as in EvictParams
  int sinks;
  float* k_scale;           // int8 cache (Q8): per-slot scales [B*Hkv, C]; else null
  float* v_scale;
};


}  // namespace h2o
