// decode.cu -- the step for one new token per cache (n_q = 1): attention that
// also returns the summed weights, then the single-token eviction
// ("Learning how to Forget", §1: the SDPA kernel returns summed attention
// weights for the H2O scores; §2: FlashInfer's 1 << N_q << N_k regime, here
// at N_q = 1, the generation step after a chunked prefill).
//
// With one query per head the step is a pass over the cache's K and V: 4·d
// bytes per (slot, KV head) for 4·d·G FLOPs, so it is bound by HBM, not by
// the tensor cores, and runs on the FMA pipe.  The keys are split over many
// CTAs (split-KV):
//   decode_partial  grid (cdiv(n + 1, KC), B*Hkv), 256 threads; KC keys per
//                   CTA (32 KiB of rows: 128 for bf16, d = 128).  Two bulk
//                   copies (cp.async.bulk) bring the chunk's K and V rows into
//                   shared memory; the new token's row (key n) is copied by a
//                   warp.  Logits: each lane holds d/32 elements of the G
//                   query rows; a warp takes 32/G keys at a time, so that its
//                   32 lanes hold partial sums of 32 (key, head) pairs, and a
//                   transposing butterfly (5 shuffle rounds, each lane giving
//                   away half of its values) leaves lane l with the full dot
//                   product of pair l.  The logits are stored for the summed
//                   weights; one warp per head takes the chunk's max and sum;
//                   P V is accumulated per lane over the head-dim slice, the
//                   eight warps' partial sums (over the K rows, which are no
//                   longer needed) added in a fixed order.  Then an atomic
//                   ticket per (cache, KV head) elects the last CTA to
//                   finish, which merges the unit (merge_unit): per-head
//                   lse2 over the chunks, O, the summed weights of all n + 1
//                   keys with the score update and the eviction candidate on
//                   the way, and the new token's placement.  One launch per
//                   step.
//   decode_finish   (the two-launch form, kDecodeFused = false) grid
//                   (cdiv(n + 1, 1024), B*Hkv), 256 threads, programmatic
//                   dependent launch.  Every CTA merges the chunk statistics
//                   of each head (lse2) and a share of the outputs O.  Each CTA
//                   writes the summed weights colsum[j] = sum_h 2^(x_hj -
//                   lse2_h) of its 1024 keys and, when evicting, adds them to
//                   its slots' scores and finds its eviction candidate; the
//                   last CTA of the (cache, KV head) to finish (atomic ticket)
//                   takes the minimum over the slices and places the new
//                   token.  Each pass needs data from HBM or L2, so every
//                   load is issued up front: the slots' scores and positions
//                   and the new token's rows before the wait for the
//                   split-KV grid, the chunk statistics, partial outputs and
//                   logits together right after it.  The rule is the top-C
//                   rule of the chunk step with
//                   N_q = 1: the unprotected candidate last in (score desc,
//                   index asc) order leaves -- the lowest score, the highest
//                   index among equal scores (for the score-free policies the
//                   position takes the place of the score).
// Both are deterministic (fixed reduction orders; the atomic only elects the
// CTA that finishes).
#include <cuda_bf16.h>

#include "attn.h"
#include "q8.cuh"
#include "sm100.cuh"

namespace h2o {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxChunks = (kMaxCandidates + 1 + 63) / 64;  // smallest chunk: 64 keys

template <typename T, int E>
__device__ __forceinline__ void lds_row(const uint8_t* src, float (&f)[E]);

template <>
__device__ __forceinline__ void lds_row<__nv_bfloat16, 4>(const uint8_t* src, float (&f)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(src);
  f[0] = __uint_as_float(u.x << 16);
  f[1] = __uint_as_float(u.x & 0xffff0000u);
  f[2] = __uint_as_float(u.y << 16);
  f[3] = __uint_as_float(u.y & 0xffff0000u);
}

template <>
__device__ __forceinline__ void lds_row<__nv_bfloat16, 2>(const uint8_t* src, float (&f)[2]) {
  const uint32_t u = *reinterpret_cast<const uint32_t*>(src);
  f[0] = __uint_as_float(u << 16);
  f[1] = __uint_as_float(u & 0xffff0000u);
}

template <>
__device__ __forceinline__ void lds_row<float, 4>(const uint8_t* src, float (&f)[4]) {
  const float4 v = *reinterpret_cast<const float4*>(src);
  f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}

template <>
__device__ __forceinline__ void lds_row<float, 2>(const uint8_t* src, float (&f)[2]) {
  const float2 v = *reinterpret_cast<const float2*>(src);
  f[0] = v.x; f[1] = v.y;
}

// E codes of an int8 cache row (Q8) and its scale -> the values the
// attention reads (q8.cuh).
template <int E>
__device__ __forceinline__ void lds_q8(const uint8_t* src, float s, float (&f)[E]) {
  if (E == 4) {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(src);
#pragma unroll
    for (int e = 0; e < E; ++e) f[e] = q8_value(static_cast<int8_t>((u >> (8 * e)) & 0xFF), s);
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) f[e] = q8_value(static_cast<int8_t>(src[e]), s);
  }
}

__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_float(float v) { return v; }
__device__ __forceinline__ void store(__nv_bfloat16* dst, float v) { *dst = __float2bfloat16_rn(v); }
__device__ __forceinline__ void store(float* dst, float v) { *dst = v; }

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ unsigned long long warp_min64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w < v ? w : v;
  }
  return v;
}

// Copies `bytes` (a multiple of 16) with the lanes of a warp.
__device__ __forceinline__ void copy_row(void* dst, const void* src, int bytes, int lane) {
  for (int o = lane * 16; o < bytes; o += 32 * 16)
    *reinterpret_cast<uint4*>(static_cast<char*>(dst) + o) =
        *reinterpret_cast<const uint4*>(static_cast<const char*>(src) + o);
}

// T: element type of q, out and the new rows; Q8: the cache holds int8 codes
// with one fp32 scale per row instead of T.
template <typename T, int D, int G, bool Q8>
struct PartialLayout {
  static constexpr int kCode = Q8 ? 1 : static_cast<int>(sizeof(T));  // bytes per cache element
  static constexpr int KC = decode_chunk_keys(D, kCode);
  static constexpr int kRow = D * kCode;
  static constexpr int kK = 0;                          // [KC][D] cache rows of K; after the
                                                        // logits: [warps][G][D] float sums of P V
  static constexpr int kV = kK + KC * kRow;             // [KC][D] of V
  static constexpr int kX = kV + KC * kRow;             // [G][KC] float logits, then
                                                        // [KC][G] float P (key-major)
  static constexpr int kS = kX + 2 * G * KC * 4;        // Q8: [2][KC] float scales of K, V
  static constexpr int kN = kS + (Q8 ? 2 * KC * 4 : 0);  // Q8: the new token's K, V rows (T)
  static constexpr int kBytes = kN + (Q8 ? 2 * D * static_cast<int>(sizeof(T)) : 0);
  static_assert(kWarps * G * D * 4 <= KC * kRow, "the P V sums must fit over the K rows");
  // the merge (last CTA of a unit) reuses the K and V rows for 2 x [G][chunks] floats
  static constexpr int kMaxChunksL = (kMaxCandidates + 1 + KC - 1) / KC;
  static_assert(2 * G * kMaxChunksL * 4 <= kX, "merge scratch must fit over the K and V rows");
};

// The merge of one (cache, KV head) unit by one CTA, once every split-KV
// partial and logit of the unit is written: per-head log-sum-exp over the
// chunks, O, the summed weights of the n + 1 keys and, when evicting, the
// score update, the eviction candidate (the lowest rank value, the highest
// index among equals) and the new token's placement.  Data the other CTAs
// wrote is read through L2 (__ldcg); each pass issues its loads in batches
// before using them, so that one CTA keeps many in flight.  scratch: shared
// memory for 2 * G * n_chunks floats.
// Loads per thread per batch: G * kMergeBatch<G> logits (keys) or kR *
// kMergeBatch<G> partial outputs (chunks).
template <int G>
constexpr int kMergeBatch = G >= 8 ? 2 : 16 / G;

template <typename T, int D, int G, bool Q8>
__device__ __forceinline__ void merge_unit(const DecodeParams& p, int bg, float* scratch) {
  __shared__ float lse[G], lh[G];
  __shared__ unsigned long long wmin[kWarps];
  __shared__ float s_new;  // the new token's summed weight
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NCk = p.n_chunks, C = p.C, n = p.n;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  constexpr size_t kChunkStride = static_cast<size_t>(G) * (D + 2);
  const float* part = p.part + static_cast<size_t>(bg) * p.part_ld * kChunkStride;
  float* fac = scratch;                // [G][NCk]: chunk max, then 2^(chunk max - head max)
  float* csum = scratch + G * NCk;     // [G][NCk]: chunk sums

  // ---- per-head log-sum-exp over the chunks: the chunk statistics into
  //      shared memory (all loads in flight), then one warp per head
  for (int i = tid; i < G * NCk; i += kThreads) {
    const int h = i / NCk, c = i % NCk;
    const float* st = part + c * kChunkStride + h * (D + 2) + D;
    fac[i] = __ldcg(st);
    csum[i] = __ldcg(st + 1);
  }
  __syncthreads();
  if (warp < G) {
    float m = -INFINITY;
    for (int c = lane; c < NCk; c += 32) m = fmaxf(m, fac[warp * NCk + c]);
    m = warp_max(m);
    float l = 0.f;
    for (int c = lane; c < NCk; c += 32) {
      const float f = ex2_approx(fac[warp * NCk + c] - m);
      fac[warp * NCk + c] = f;
      l = fmaf(csum[warp * NCk + c], f, l);
    }
    l = warp_sum(l);
    if (lane == 0) {
      lh[warp] = l;
      lse[warp] = m + __log2f(l);
    }
  }
  __syncthreads();

  // ---- O: thread t merges outputs t, t + 256, ... (kR of them) over the
  //      chunks, kMergeBatch<G> chunks of loads at a time
  {
    constexpr int kR = (G * D + kThreads - 1) / kThreads;
    T* out = static_cast<T*>(p.out) + (static_cast<size_t>(b) * p.Hkv * G + g * G) * D;
    float acc[kR];
#pragma unroll
    for (int r = 0; r < kR; ++r) acc[r] = 0.f;
    for (int c0 = 0; c0 < NCk; c0 += kMergeBatch<G>) {
      float v[kMergeBatch<G>][kR];
#pragma unroll
      for (int u = 0; u < kMergeBatch<G>; ++u)
#pragma unroll
        for (int r = 0; r < kR; ++r) {
          const int i = tid + r * kThreads;
          v[u][r] = (c0 + u < NCk && i < G * D)
                        ? __ldcg(part + (c0 + u) * kChunkStride + (i / D) * (D + 2) + (i % D))
                        : 0.f;
        }
#pragma unroll
      for (int u = 0; u < kMergeBatch<G>; ++u)
#pragma unroll
        for (int r = 0; r < kR; ++r) {
          const int i = tid + r * kThreads;
          if (c0 + u < NCk && i < G * D) acc[r] = fmaf(v[u][r], fac[(i / D) * NCk + c0 + u], acc[r]);
        }
    }
#pragma unroll
    for (int r = 0; r < kR; ++r) {
      const int i = tid + r * kThreads;
      if (i < G * D) store(out + i, acc[r] / lh[i / D]);
    }
  }

  // ---- summed weights of the n + 1 keys, with the score update and this
  //      thread's eviction candidate on the way; kMergeBatch<G> keys per thread
  //      per batch, their loads issued before any of them is used
  const float* lg = p.logits + static_cast<size_t>(bg) * G * (C + 1);
  float* cs = p.colsum + static_cast<size_t>(bg) * p.colsum_ld;
  float* score = p.scores + static_cast<size_t>(bg) * C;
  int* pos = p.pos + static_cast<size_t>(bg) * C;
  const bool by_score = p.policy == kPolicyH2O;
  const int sinks = p.policy == kPolicySLR ? p.sinks : 0;
  const bool full = p.evict && n >= C;
  // unprotected: position < t0 + 1 - W (and, under SLR, >= the sink count).
  // Candidate key: rank value (the score as an order-preserving key, or the
  // position) then the inverted index, so that the minimum is the lowest
  // value with the highest index.
  const long long limit = static_cast<long long>(p.t0) + 1 - p.W;
  float lse_r[G];
#pragma unroll
  for (int h = 0; h < G; ++h) lse_r[h] = lse[h];
  unsigned long long best = ~0ull;
  for (int j0 = tid; j0 <= n; j0 += kMergeBatch<G> * kThreads) {
    float x[kMergeBatch<G>][G], sc[kMergeBatch<G>];
    int ps[kMergeBatch<G>];
#pragma unroll
    for (int u = 0; u < kMergeBatch<G>; ++u) {
      const int j = j0 + u * kThreads;
      const bool key = j <= n, slot = j < n;
#pragma unroll
      for (int h = 0; h < G; ++h) x[u][h] = key ? __ldcg(lg + static_cast<size_t>(h) * (C + 1) + j) : 0.f;
      sc[u] = (slot && p.evict && by_score) ? score[j] : 0.f;
      ps[u] = (slot && full) ? pos[j] : 0;
    }
#pragma unroll
    for (int u = 0; u < kMergeBatch<G>; ++u) {
      const int j = j0 + u * kThreads;
      if (j > n) continue;
      float sw = 0.f;
#pragma unroll
      for (int h = 0; h < G; ++h) sw += ex2_approx(x[u][h] - lse_r[h]);
      if (j == n) {
        cs[C] = sw;
        s_new = sw;
        continue;
      }
      cs[j] = sw;
      if (!p.evict) continue;
      if (!full) {
        if (by_score) score[j] = __fadd_rn(sc[u], sw);
        continue;
      }
      uint32_t rank;
      if (by_score) {
        const float v = __fadd_rn(sc[u], sw);
        score[j] = v;
        rank = ordered_key(v);
      } else {
        rank = static_cast<uint32_t>(ps[u]);
      }
      if (ps[u] < limit && ps[u] >= sinks) {
        const unsigned long long key = (static_cast<unsigned long long>(rank) << 32) | (0xffffffffu - j);
        best = key < best ? key : best;
      }
    }
  }
  for (int j = n + tid; j < C; j += kThreads) cs[j] = 0.f;  // empty slots received nothing
  __syncthreads();  // s_new
  if (!p.evict) return;

  // ---- eviction
  const size_t row_bytes = static_cast<size_t>(D) * (Q8 ? 1 : sizeof(T));  // cache rows
  const size_t new_bytes = static_cast<size_t>(D) * sizeof(T);
  char* kc = static_cast<char*>(p.k_cache) + static_cast<size_t>(bg) * C * row_bytes;
  char* vc = static_cast<char*>(p.v_cache) + static_cast<size_t>(bg) * C * row_bytes;
  const char* kn = static_cast<const char*>(p.k_new) + static_cast<size_t>(bg) * new_bytes;
  const char* vn = static_cast<const char*>(p.v_new) + static_cast<size_t>(bg) * new_bytes;
  // the new token's rows into slot `slot`: copied, or quantised (Q8); one warp
  auto place_new = [&](int slot) {
    if (!H2O_IN_BOUNDS(slot >= 0 && slot < C, p.state + 2)) return;
    if (Q8) {
      q8_quantize_row_warp<D>(reinterpret_cast<const __nv_bfloat16*>(kn),
                              reinterpret_cast<int8_t*>(kc + static_cast<size_t>(slot) * row_bytes),
                              p.k_scale + static_cast<size_t>(bg) * C + slot, lane);
      q8_quantize_row_warp<D>(reinterpret_cast<const __nv_bfloat16*>(vn),
                              reinterpret_cast<int8_t*>(vc + static_cast<size_t>(slot) * row_bytes),
                              p.v_scale + static_cast<size_t>(bg) * C + slot, lane);
    } else {
      copy_row(kc + static_cast<size_t>(slot) * row_bytes, kn, static_cast<int>(row_bytes), lane);
      copy_row(vc + static_cast<size_t>(slot) * row_bytes, vn, static_cast<int>(row_bytes), lane);
    }
  };
  if (bg == 0 && tid == 0) {
    p.state[0] = min(C, n + 1);
    p.state[1] = p.t0 + 1;
  }
  if (!full) {  // room left: the new token takes slot n
    if (tid == 0) {
      score[n] = by_score ? s_new : 0.f;
      pos[n] = p.t0;
    }
    if (warp == 0) place_new(n);
    return;
  }
  if (tid == 0 && p.t0 < limit && p.t0 >= sinks) {  // W = 0: the new token competes
    const uint32_t rank = by_score ? ordered_key(s_new) : static_cast<uint32_t>(p.t0);
    const unsigned long long key = (static_cast<unsigned long long>(rank) << 32) | (0xffffffffu - C);
    best = key < best ? key : best;
  }
  best = warp_min64(best);
  if (lane == 0) wmin[warp] = best;
  __syncthreads();  // also: every slot's score is updated before one is replaced
  if (warp != 0) return;
  unsigned long long m = lane < kWarps ? wmin[lane] : ~0ull;
  m = warp_min64(m);
  if (m == ~0ull) {  // cannot happen: W + sinks <= C leaves an unprotected candidate
    if (lane == 0) atomicOr(&p.state[2], kDevErrPlan);
    return;
  }
  const int e = static_cast<int>(0xffffffffu - static_cast<uint32_t>(m & 0xffffffffu));
  if (e < C) {  // an old slot leaves; the new token takes it
    if (lane == 0) {
      score[e] = by_score ? s_new : 0.f;
      pos[e] = p.t0;
    }
    place_new(e);
  }
}

// The split-KV partial of one chunk (keys [chunk*KC, +KC) of the n + 1 of a
// (cache, KV head) unit bg): logits (stored for the summed weights), the
// chunk's max and sum per head, and the unnormalised P V, written to the
// unit's partials.  The caller has issued the bulk copies of the chunk's
// cache rows into sK / sV (completing bK / bV with the given parity) when
// the chunk holds cache slots; this copies the new token's rows (when key n
// is in the chunk) and, int8 cache, the rows' scales.  sK is reused for the
// warps' P V sums once the logits are done.  Returns false when a wait gave
// up (after letting the copies land).
template <typename T, int D, int G, bool Q8>
__device__ __forceinline__ bool chunk_partial(const DecodeParams& p, int bg, int chunk,
                                              uint8_t* sK, uint8_t* sV, uint8_t* sN,
                                              float* sScale, float* xs, uint32_t bK, uint32_t bV,
                                              uint32_t parity, int* abort_flag,
                                              const float (&qf)[G][D / 32]) {
  using L = PartialLayout<T, D, G, Q8>;
  constexpr int KC = L::KC;
  constexpr int E = D / 32;   // row elements per lane
  constexpr int KB = 32 / G;  // keys per warp batch: 32 (key, head) pairs
  __shared__ float hstat[G][2];  // chunk max, chunk sum
  float* ored = reinterpret_cast<float*>(sK);  // written once the K rows are used
  const int j0 = chunk * KC;
  const int nk = p.n + 1;
  const int nkc = min(KC, nk - j0);           // keys of this chunk (>= 1)
  const int rows = max(0, min(KC, p.n - j0));  // of them cache slots
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int* err = p.state + 2;
  constexpr int kNewRow = D * static_cast<int>(sizeof(T));  // the new rows are T
  uint8_t* sNK = Q8 ? sN : sK + rows * L::kRow;  // the new token's rows
  uint8_t* sNV = Q8 ? sN + kNewRow : sV + rows * L::kRow;
  if (warp == 0 && nkc > rows) {  // the new token is key n, in this chunk
    copy_row(sNK, static_cast<const uint8_t*>(p.k_new) + bg * kNewRow, kNewRow, lane);
    copy_row(sNV, static_cast<const uint8_t*>(p.v_new) + bg * kNewRow, kNewRow, lane);
  }
  if (Q8) {
    for (int i = tid; i < KC; i += kThreads) {
      const size_t at = static_cast<size_t>(bg) * p.C + j0 + i;
      sScale[i] = i < rows ? p.k_scale[at] : 0.f;
      sScale[KC + i] = i < rows ? p.v_scale[at] : 0.f;
    }
  }
  // this lane's slice of key (value) row k of the chunk as floats
  auto kv_row = [&](int k, bool is_v, float (&f)[E]) {
    if (Q8) {
      if (k == rows)
        lds_row<T, E>((is_v ? sNV : sNK) + lane * E * sizeof(T), f);
      else
        lds_q8<E>((is_v ? sV : sK) + k * L::kRow + lane * E, sScale[(is_v ? KC : 0) + k], f);
    } else {
      lds_row<T, E>((is_v ? sV : sK) + k * L::kRow + lane * E * sizeof(T), f);
    }
  };
  __syncthreads();  // the new token's rows and the scales are in place
  bool ok = rows == 0 || mbar_wait(bK, parity, err, abort_flag);
  ok = __all_sync(0xffffffffu, ok);

  // ---- logits: a warp batch is KB keys x G heads = 32 dot products
  if (ok) {
    float* lg = p.logits + static_cast<size_t>(bg) * G * (p.C + 1);
    for (int k0 = warp * KB; k0 < nkc; k0 += kWarps * KB) {
      float v[32];
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        float kf[E];
        kv_row(min(k0 + k, KC - 1), false, kf);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float a = 0.f;
#pragma unroll
          for (int e = 0; e < E; ++e) a = fmaf(qf[h][e], kf[e], a);
          v[k * G + h] = a;
        }
      }
      // transposing butterfly: after round r a lane keeps the half of its
      // values whose index bit (4 - r) equals its own lane bit, and adds the
      // partner's copy of them; at the end lane l holds pair l
#pragma unroll
      for (int r = 0; r < 5; ++r) {
        const int off = 16 >> r;
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
          const float send = up ? v[i] : v[i + off];
          const float keep = up ? v[i + off] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      const int kl = k0 + lane / G, h = lane % G;
      const bool valid = kl < nkc;  // rows past the chunk's keys hold stale data
      if (kl < KC) xs[h * KC + kl] = valid ? v[0] * p.scale_log2 : -INFINITY;
      if (valid) lg[static_cast<size_t>(h) * (p.C + 1) + j0 + kl] = v[0] * p.scale_log2;
    }
  }
  __syncthreads();
  // ---- chunk max and sum per head (one warp per head), P key-major into
  // pk, so that P V reads a key's G weights at once
  float* pk = xs + G * KC;
  if (ok && warp < G) {
    float m = -INFINITY;
    for (int k = lane; k < nkc; k += 32) m = fmaxf(m, xs[warp * KC + k]);
    m = warp_max(m);
    float l = 0.f;
    for (int k = lane; k < nkc; k += 32) {
      const float pw = ex2_approx(xs[warp * KC + k] - m);
      pk[k * G + warp] = pw;
      l += pw;
    }
    l = warp_sum(l);
    if (lane == 0) {
      hstat[warp][0] = m;
      hstat[warp][1] = l;
    }
  }
  if (ok && rows > 0) ok = mbar_wait(bV, parity, err, abort_flag);
  ok = __all_sync(0xffffffffu, ok);
  __syncthreads();
  // ---- P V: each lane its head-dim slice, warps over the keys
  float o[G][E];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < E; ++e) o[h][e] = 0.f;
  if (ok) {
#pragma unroll 2
    for (int k = warp; k < nkc; k += kWarps) {
      float vf[E];
      kv_row(k, true, vf);
      float pw[G];
      if constexpr (G % 4 == 0) {
#pragma unroll
        for (int h = 0; h < G; h += 4) {
          const float4 w = *reinterpret_cast<const float4*>(pk + k * G + h);
          pw[h] = w.x;
          pw[h + 1] = w.y;
          pw[h + 2] = w.z;
          pw[h + 3] = w.w;
        }
      } else if constexpr (G == 2) {
        const float2 w = *reinterpret_cast<const float2*>(pk + k * G);
        pw[0] = w.x;
        pw[1] = w.y;
      } else {
        pw[0] = pk[k];
      }
      // o += P V two elements at a time (the same fused multiply-adds)
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < E; e += 2)
          ffma2(o[h][e], o[h][e + 1], pw[h], pw[h], vf[e], vf[e + 1], o[h][e], o[h][e + 1]);
    }
  }
  if (!ok && tid == 0 && rows > 0) {  // a wait gave up: the copies land before their
    mbar_wait_drain(bK, parity, err);  // buffers are written or reused
    mbar_wait_drain(bV, parity, err);
  }
  __syncthreads();  // every warp is done with the K rows
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < E; ++e) ored[(warp * G + h) * D + lane * E + e] = o[h][e];
  __syncthreads();
  if (ok && H2O_IN_BOUNDS(chunk < p.part_ld, err)) {
    float* part = p.part + (static_cast<size_t>(bg) * p.part_ld + chunk) * G * (D + 2);
    for (int i = tid; i < G * D; i += kThreads) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += ored[w * G * D + i];
      part[(i / D) * (D + 2) + (i % D)] = s;
    }
    if (tid < G) {
      part[tid * (D + 2) + D] = hstat[tid][0];
      part[tid * (D + 2) + D + 1] = hstat[tid][1];
    }
  }
  return ok;
}

// Ticket of unit bg after one of its chunks: true in the CTA that finished
// the unit's last chunk, after which every chunk's logits and partials are
// visible to it (and the ticket is reset for the next step).
__device__ __forceinline__ bool last_of_unit(const DecodeParams& p, int bg) {
  __shared__ int is_last;
  __threadfence();  // this CTA's logits and partials, before the ticket
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(&p.ticket[bg], 1) == p.n_chunks - 1;
  __syncthreads();
  const bool last = is_last != 0;
  if (last) {
    __threadfence();  // every CTA of the unit took its ticket after its writes
    if (threadIdx.x == 0) p.ticket[bg] = 0;  // ready for the next step
  }
  return last;
}

// This lane's slice of the G query rows of unit bg.
template <typename T, int D, int G>
__device__ __forceinline__ void load_q(const DecodeParams& p, int bg, float (&qf)[G][D / 32]) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const T* q = static_cast<const T*>(p.q) + (static_cast<size_t>(b) * p.Hkv * G + g * G) * D;
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < E; ++e) qf[h][e] = to_float(q[h * D + lane * E + e]);
}

// Bulk copies of the cache rows of chunk `chunk` of unit bg (cache slots
// only; nothing when the chunk holds just the new token).
template <typename T, int D, int G, bool Q8>
__device__ __forceinline__ void load_chunk(const DecodeParams& p, int bg, int chunk, uint8_t* sK,
                                           uint8_t* sV, uint32_t bK, uint32_t bV) {
  using L = PartialLayout<T, D, G, Q8>;
  const int j0 = chunk * L::KC;
  const int rows = max(0, min(L::KC, p.n - j0));
  if (rows == 0) {  // nothing to copy: the phases still complete, so that a
    mbar_arrive(bK);  // reused stage keeps its parity
    mbar_arrive(bV);
    return;
  }
  const size_t off = (static_cast<size_t>(bg) * p.C + j0) * L::kRow;
  const uint32_t bytes = static_cast<uint32_t>(rows) * L::kRow;
  mbar_arrive_expect_tx(bK, bytes);
  bulk_load(smem_u32(sK), static_cast<const uint8_t*>(p.k_cache) + off, bytes, bK);
  mbar_arrive_expect_tx(bV, bytes);
  bulk_load(smem_u32(sV), static_cast<const uint8_t*>(p.v_cache) + off, bytes, bV);
}

// One CTA per chunk; kFused: the last CTA of each (cache, KV head) also
// merges it (merge_unit), so that the step is one launch; otherwise
// decode_finish follows.
template <typename T, int D, int G, bool Q8, bool kFused>
__global__ void __launch_bounds__(kThreads, 3) decode_partial(const DecodeParams p) {
  using L = PartialLayout<T, D, G, Q8>;
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int abort_flag;
  const int bg = blockIdx.y;
  const int chunk = blockIdx.x;
  const uint32_t bK = smem_u32(&bars[0]), bV = smem_u32(&bars[1]);
  if (threadIdx.x == 0) {
    mbar_init(bK, 1);
    mbar_init(bV, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) load_chunk<T, D, G, Q8>(p, bg, chunk, dsm + L::kK, dsm + L::kV, bK, bV);
  float qf[G][D / 32];
  load_q<T, D, G>(p, bg, qf);
  chunk_partial<T, D, G, Q8>(p, bg, chunk, dsm + L::kK, dsm + L::kV, dsm + L::kN,
                             reinterpret_cast<float*>(dsm + L::kS),
                             reinterpret_cast<float*>(dsm + L::kX), bK, bV, 0u, &abort_flag, qf);
  // the merge kernel may start now (its CTAs wait for this grid before
  // reading; triggered at the start instead, they take SM slots from this
  // grid's second wave: 31.7 against 29.7 us per step on one cache)
  griddep_launch_dependents();
  if (!kFused) return;
  // the merge's scratch reuses the K and V rows (every copy has landed)
  if (last_of_unit(p, bg)) merge_unit<T, D, G, Q8>(p, bg, reinterpret_cast<float*>(dsm));
}

template <typename T, int D, int G, bool Q8>
__global__ void __launch_bounds__(kThreads) decode_finish(const DecodeParams p) {
  constexpr int kPer = kDecodeSliceKeys / kThreads;  // keys of the slice per thread
  constexpr int kStatB = 4;  // chunk statistics per lane read at once (128 chunks a warp)
  constexpr int kOB = 24;    // partial outputs per thread read at once
  static_assert(kDecodeSliceKeys % kThreads == 0, "slice keys per thread");
  __shared__ float fac[G][kMaxChunks];  // 2^(chunk max - head max)
  __shared__ float lse[G], lh[G];
  __shared__ unsigned long long wmin[kWarps];
  __shared__ int is_last;
  const int slice = blockIdx.x;
  const int bg = blockIdx.y;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NCk = p.n_chunks;
  const int C = p.C, n = p.n;
  const int ja = slice * kDecodeSliceKeys;      // this slice's keys [ja, jb): thread tid
  const int jb = min(n + 1, ja + kDecodeSliceKeys);  // takes ja + tid + r * kThreads
  const int sb = min(jb, n);                     // of them cache slots: [ja, sb)
  const bool by_score = p.policy == kPolicyH2O;
  const bool last_slice = slice == static_cast<int>(gridDim.x) - 1;
  // Every pass below needs data from HBM or L2, so the loads are issued up
  // front, all at once: a dependent round trip per pass made the kernel
  // latency bound.  First what the split-KV kernel does not write, read
  // while it still runs: this thread's slots' scores and positions, and the
  // new token's rows (warp 0, 16 bytes a lane; the int8 cache quantises them
  // from global memory instead).
  float sc_old[kPer];
  int ps_old[kPer];
  uint4 k_row = make_uint4(0, 0, 0, 0), v_row = make_uint4(0, 0, 0, 0);
  constexpr int kNewBytes = D * static_cast<int>(sizeof(T));
  static_assert(kNewBytes <= 32 * 16, "a new row is at most 16 bytes a lane");
  if (p.evict) {
    const float* score = p.scores + static_cast<size_t>(bg) * C;
    const int* pos = p.pos + static_cast<size_t>(bg) * C;
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
      const int s = ja + tid + r * kThreads;
      sc_old[r] = (by_score && s < sb) ? score[s] : 0.f;
      ps_old[r] = (n >= C && s < sb) ? pos[s] : 0;
    }
    if (!Q8 && warp == 0 && lane * 16 < kNewBytes) {
      k_row = *reinterpret_cast<const uint4*>(static_cast<const char*>(p.k_new) +
                                              static_cast<size_t>(bg) * kNewBytes + lane * 16);
      v_row = *reinterpret_cast<const uint4*>(static_cast<const char*>(p.v_new) +
                                              static_cast<size_t>(bg) * kNewBytes + lane * 16);
    }
  }
  griddep_wait();  // the partials and logits come from the preceding kernel
  const float* part = p.part + static_cast<size_t>(bg) * p.part_ld * G * (D + 2);
  auto pidx = [&](int c, int h) { return (static_cast<size_t>(c) * G + h) * (D + 2); };

  // ---- then the split-KV kernel's outputs, together: (a) the chunk
  // statistics of head `warp` (warps < G); (b) the first partial outputs of
  // this thread's share of O; (c) the logits of this thread's keys
  float cm[kStatB], cl[kStatB];
#pragma unroll
  for (int t = 0; t < kStatB; ++t) {
    const int c = lane + 32 * t;
    const bool v = warp < G && c < NCk;
    cm[t] = v ? part[pidx(c, warp) + D] : -INFINITY;
    cl[t] = v ? part[pidx(c, warp) + D + 1] : 0.f;
  }
  // O: the CTAs that merge it are all slices when there are few (cache, KV
  // head) units (latency), else the first only (less repeated work); tpo
  // lanes per output, each summing chunks cg, cg + tpo, ... in order, then a
  // fixed butterfly over the tpo lanes
  const int o_slices = p.spread_o ? static_cast<int>(gridDim.x) : 1;
  const bool do_o = slice < o_slices;
  const int GD = G * D;
  const int per = (GD + o_slices - 1) / o_slices;
  const int o_begin = slice * per, o_end = min(GD, o_begin + per);
  int tpo = 1;
  while (tpo < 32 && 2 * tpo * per <= kThreads) tpo *= 2;
  const int cg = tid % tpo;
  const int o_stride = kThreads / tpo;  // outputs per pass
  float ov[kOB];
  auto load_o = [&](int i, int c0) {  // output i (if valid), chunks c0, c0 + tpo, ...
    const bool valid = do_o && i < o_end;
    const int h = valid ? i / D : 0, d = valid ? i % D : 0;
#pragma unroll
    for (int u = 0; u < kOB; ++u) {
      const int c = c0 + u * tpo;
      ov[u] = (valid && c < NCk) ? part[pidx(c, h) + d] : 0.f;
    }
  };
  load_o(o_begin + tid / tpo, cg);
  const float* lg = p.logits + static_cast<size_t>(bg) * G * (C + 1);
  float lv[kPer][G];
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int j = ja + tid + r * kThreads;
#pragma unroll
    for (int h = 0; h < G; ++h) lv[r][h] = j < jb ? lg[static_cast<size_t>(h) * (C + 1) + j] : 0.f;
  }

  // ---- per-head log-sum-exp over the chunks (one warp per head)
  if (warp < G) {
    float m = -INFINITY;
#pragma unroll
    for (int t = 0; t < kStatB; ++t) m = fmaxf(m, cm[t]);
    for (int c = lane + 32 * kStatB; c < NCk; c += 32) m = fmaxf(m, part[pidx(c, warp) + D]);
    m = warp_max(m);
    float l = 0.f;
#pragma unroll
    for (int t = 0; t < kStatB; ++t) {
      const int c = lane + 32 * t;
      if (c < NCk) {
        const float f = ex2_approx(cm[t] - m);
        if (do_o) fac[warp][c] = f;
        l = fmaf(cl[t], f, l);
      }
    }
    for (int c = lane + 32 * kStatB; c < NCk; c += 32) {
      const float f = ex2_approx(part[pidx(c, warp) + D] - m);
      if (do_o) fac[warp][c] = f;
      l = fmaf(part[pidx(c, warp) + D + 1], f, l);
    }
    l = warp_sum(l);
    if (lane == 0) {
      lh[warp] = l;
      lse[warp] = m + __log2f(l);
    }
  }
  __syncthreads();
  if (do_o) {
    T* out = static_cast<T*>(p.out) + (static_cast<size_t>(b) * p.Hkv * G + g * G) * D;
    for (int base = o_begin; base < o_end; base += o_stride) {
      const int i = base + tid / tpo;
      const bool valid = i < o_end;
      const int h = valid ? i / D : 0;
      if (base != o_begin) load_o(i, cg);
      float acc = 0.f;
      for (int c0 = cg;;) {
#pragma unroll
        for (int u = 0; u < kOB; ++u) {
          const int c = c0 + u * tpo;
          if (valid && c < NCk) acc = fmaf(ov[u], fac[h][c], acc);
        }
        c0 += kOB * tpo;
        if (c0 >= NCk) break;
        load_o(i, c0);
      }
      for (int o = tpo / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (valid && cg == 0) store(out + i, acc / lh[h]);
    }
  }

  // ---- summed weights of this slice's keys: slots, then the new key at C
  float* cs = p.colsum + static_cast<size_t>(bg) * p.colsum_ld;
  float csv[kPer];
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int j = ja + tid + r * kThreads;
    float s = 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) s += ex2_approx(lv[r][h] - lse[h]);
    csv[r] = s;
    if (j < jb) cs[j < n ? j : C] = s;
  }
  if (last_slice)  // empty slots received nothing
    for (int j = n + tid; j < C; j += kThreads) cs[j] = 0.f;
  if (!p.evict) return;

  // ---- eviction
  __syncthreads();  // this CTA's summed weights are written
  const int sinks = p.policy == kPolicySLR ? p.sinks : 0;
  float* score = p.scores + static_cast<size_t>(bg) * C;
  int* pos = p.pos + static_cast<size_t>(bg) * C;
  const size_t row_bytes = static_cast<size_t>(D) * (Q8 ? 1 : sizeof(T));  // cache rows
  char* kc = static_cast<char*>(p.k_cache) + static_cast<size_t>(bg) * C * row_bytes;
  char* vc = static_cast<char*>(p.v_cache) + static_cast<size_t>(bg) * C * row_bytes;
  // the new token's rows into slot `slot`: stored from registers, or
  // quantised (Q8); warp 0
  auto place_new = [&](int slot) {
    if (!H2O_IN_BOUNDS(slot >= 0 && slot < C, p.state + 2)) return;
    if (Q8) {
      const size_t new_off = static_cast<size_t>(bg) * kNewBytes;
      q8_quantize_row_warp<D>(
          reinterpret_cast<const __nv_bfloat16*>(static_cast<const char*>(p.k_new) + new_off),
          reinterpret_cast<int8_t*>(kc + static_cast<size_t>(slot) * row_bytes),
          p.k_scale + static_cast<size_t>(bg) * C + slot, lane);
      q8_quantize_row_warp<D>(
          reinterpret_cast<const __nv_bfloat16*>(static_cast<const char*>(p.v_new) + new_off),
          reinterpret_cast<int8_t*>(vc + static_cast<size_t>(slot) * row_bytes),
          p.v_scale + static_cast<size_t>(bg) * C + slot, lane);
    } else if (lane * 16 < kNewBytes) {
      *reinterpret_cast<uint4*>(kc + static_cast<size_t>(slot) * row_bytes + lane * 16) = k_row;
      *reinterpret_cast<uint4*>(vc + static_cast<size_t>(slot) * row_bytes + lane * 16) = v_row;
    }
  };
  if (bg == 0 && slice == 0 && tid == 0) {
    p.state[0] = min(C, n + 1);
    p.state[1] = p.t0 + 1;
  }
  if (n < C) {  // room left: the new token takes slot n (key n is in the last slice)
    if (by_score) {
#pragma unroll
      for (int r = 0; r < kPer; ++r) {
        const int s = ja + tid + r * kThreads;
        if (s < sb) score[s] = __fadd_rn(sc_old[r], csv[r]);
      }
    }
    if (last_slice) {
      if (tid == 0) {
        score[n] = by_score ? cs[C] : 0.f;
        pos[n] = p.t0;
      }
      if (warp == 0) place_new(n);
    }
    return;
  }
  // full: this slice's candidate.  Unprotected: position < t0 + 1 - W (and,
  // under SLR, >= the sink count).  Key: rank value (the score as an
  // order-preserving key, or the position) then the inverted index, so that
  // the minimum is the lowest value with the highest index.
  const long long limit = static_cast<long long>(p.t0) + 1 - p.W;
  unsigned long long best = ~0ull;
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int s = ja + tid + r * kThreads;
    if (s >= sb) continue;
    const int ps = ps_old[r];
    uint32_t rank;
    if (by_score) {
      const float sc = __fadd_rn(sc_old[r], csv[r]);
      score[s] = sc;
      rank = ordered_key(sc);
    } else {
      rank = static_cast<uint32_t>(ps);
    }
    if (ps < limit && ps >= sinks) {
      const unsigned long long key = (static_cast<unsigned long long>(rank) << 32) | (0xffffffffu - s);
      best = key < best ? key : best;
    }
  }
  if (last_slice && tid == 0 && p.t0 < limit && p.t0 >= sinks) {  // W = 0: the new token competes
    const uint32_t rank = by_score ? ordered_key(cs[C]) : static_cast<uint32_t>(p.t0);
    const unsigned long long key = (static_cast<unsigned long long>(rank) << 32) | (0xffffffffu - C);
    best = key < best ? key : best;
  }
  best = warp_min64(best);
  if (lane == 0) wmin[warp] = best;
  __syncthreads();
  if (tid == 0) {
    unsigned long long m = wmin[0];
    for (int w = 1; w < kWarps; ++w) m = wmin[w] < m ? wmin[w] : m;
    if (H2O_IN_BOUNDS(slice < p.slices_ld, p.state + 2))
      p.best[static_cast<size_t>(bg) * p.slices_ld + slice] = m;
    __threadfence();  // candidate, scores and summed weights before the ticket
    is_last = atomicAdd(&p.ticket[bg], 1) == static_cast<int>(gridDim.x) - 1;
  }
  __syncthreads();
  if (!is_last || warp != 0) return;
  // the last CTA of this (cache, KV head): every slice's writes are visible
  __threadfence();
  unsigned long long m = ~0ull;
  for (int sl = lane; sl < static_cast<int>(gridDim.x); sl += 32) {
    const unsigned long long v = __ldcg(&p.best[static_cast<size_t>(bg) * p.slices_ld + sl]);
    m = v < m ? v : m;
  }
  m = warp_min64(m);
  if (lane == 0) p.ticket[bg] = 0;  // ready for the next step
  if (m == ~0ull) {  // cannot happen: W + sinks <= C leaves an unprotected candidate
    if (lane == 0) atomicOr(&p.state[2], kDevErrPlan);
    return;
  }
  const int e = static_cast<int>(0xffffffffu - static_cast<uint32_t>(m & 0xffffffffu));
  if (e < C) {  // an old slot leaves; the new token takes it
    if (lane == 0) {
      score[e] = by_score ? __ldcg(&cs[C]) : 0.f;
      pos[e] = p.t0;
    }
    place_new(e);
  }
}

// One launch per step (the merge in each unit's last CTA) or two (a merge
// kernel over slices of the keys).  Measured on one Qwen-shaped cache (C 8192,
// 8 KV heads): 47.1 us with one launch against 31.7 us with two -- one CTA per
// (cache, KV head) merging 8193 keys is slower than 72 CTAs behind a
// programmatic dependent launch -- and 1719 against 1680 us on 144 caches;
// so two.
constexpr bool kDecodeFused = false;

template <typename T, int D, int G, bool Q8>
cudaError_t launch_partial(const DecodeParams& p, cudaStream_t st) {
  using L = PartialLayout<T, D, G, Q8>;
  static int attr_bits[2] = {0, 0};
  const void* fn = reinterpret_cast<const void*>(decode_partial<T, D, G, Q8, kDecodeFused>);
  cudaError_t e = ensure_smem_attr(fn, L::kBytes, attr_bits);
  if (e != cudaSuccess) return e;
  decode_partial<T, D, G, Q8, kDecodeFused>
      <<<dim3(p.n_chunks, p.B * p.Hkv), kThreads, L::kBytes, st>>>(p);
  return cudaGetLastError();
}

template <typename T, int D, int G, bool Q8>
cudaError_t launch_finish(const DecodeParams& p, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.n_slices, p.B * p.Hkv);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_finish<T, D, G, Q8>, p);
}

template <typename T, int D, int G, bool Q8>
cudaError_t launch_group(const DecodeParams& p, cudaStream_t st) {
  const cudaError_t e = launch_partial<T, D, G, Q8>(p, st);
  if (e != cudaSuccess || kDecodeFused) return e;
  return launch_finish<T, D, G, Q8>(p, st);
}

template <typename T, int D, bool Q8 = false>
cudaError_t launch(const DecodeParams& p, cudaStream_t st) {
  switch (p.G) {
    case 1: return launch_group<T, D, 1, Q8>(p, st);
    case 2: return launch_group<T, D, 2, Q8>(p, st);
    case 4: return launch_group<T, D, 4, Q8>(p, st);
    case 8: return launch_group<T, D, 8, Q8>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool decode_supported(int G) { return G == 1 || G == 2 || G == 4 || G == 8; }

int decode_launches() { return kDecodeFused ? 1 : 2; }

cudaError_t launch_decode(const DecodeParams& p, int esize, int head_dim, cudaStream_t st) {
  if (p.n_chunks > kMaxChunks || !decode_supported(p.G) || p.n_slices > p.slices_ld)
    return cudaErrorInvalidValue;
  if (esize == 1)  // int8 cache, bf16 activations
    return head_dim == 128 ? launch<__nv_bfloat16, 128, true>(p, st)
                           : launch<__nv_bfloat16, 64, true>(p, st);
  if (esize == 2)
    return head_dim == 128 ? launch<__nv_bfloat16, 128>(p, st) : launch<__nv_bfloat16, 64>(p, st);
  return head_dim == 128 ? launch<float, 128>(p, st) : launch<float, 64>(p, st);
}

}  // namespace h2o
