// evict.cu -- H2O score accumulation, top-C selection and K/V slot scatter.
//
// "Learning how to Forget", §1: a fixed-size KV cache whose slots a policy
// evicts when it is full; summary page glossary "H2O": entries are scored by
// the attention they accumulated and the less important ones evicted.
//
// Per (cache, KV head), with the candidates' keys in shared memory -- one
// CTA (h2o_select: 1024 threads, or 256 when the units outnumber the SMs
// twice) or, for up to 16 units, a cluster of 8 CTAs (h2o_select_cluster,
// below) -- the selection runs these steps:
//   1. score[s] <- fl32(score[s] + colsum[s]) for the n valid slots; new token
//      i's candidate score is colsum[C + i].  The score-free policies (LR,
//      SLR) rank by position instead: a candidate's key is its position, no
//      score is accumulated and placed tokens get score 0; SLR also protects
//      positions below the sink count.
//   2. If n + nq <= C every new token is kept and goes to slot n + i.
//   3. Otherwise a candidate at position >= t0 + nq - W is protected.  Each
//      candidate gets a 32-bit key: 0xFFFFFFFF when protected, else its fp32
//      score mapped to a key that orders like the score (negative scores
//      included), or its position for LR / SLR.
//      A 4 x 8-bit MSB-first radix select finds the C-th largest key T and
//      how many keys equal to T are kept; those are the ones of lowest
//      candidate index (slot s -> s, new token i -> n + i; same order as the
//      C + i numbering).  So exactly C candidates stay, ties go to the lower
//      index, and the protected ones always stay (there are at most W <= C).
//   4. Ordered compaction (one block scan over contiguous per-thread ranges)
//      lists the free slots (evicted or empty) and the kept new tokens in
//      ascending order; the k-th kept token goes to the k-th free slot.  The
//      CTA writes the score and position of the placed tokens and the plan,
//      then copies their K and V rows into the slots (16-byte vector loads
//      and stores, whole rows per warp, several loads in flight per thread).
#include "attn.h"
#include "q8.cuh"
#include "sm100.cuh"

namespace h2o {

constexpr uint32_t kProtectedKey = 0xFFFFFFFFu;

__device__ __forceinline__ uint32_t score_key(float s) { return ordered_key(s); }

// Exclusive scan of one 64-bit value per thread over the block (four packed
// 16-bit counters: no field carries into the next while every block total
// stays below 2^16); returns the prefix, writes the block total to *total.
template <int NT>
__device__ __forceinline__ uint64_t block_excl_scan64(uint64_t v, uint64_t* warp_sums,
                                                      uint64_t* total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) warp_sums[w] = x;
  __syncthreads();
  if (w == 0) {
    uint64_t s = lane < NW ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < NW) warp_sums[lane] = s;  // inclusive
  }
  __syncthreads();
  const uint64_t before = (w > 0 ? warp_sums[w - 1] : 0) + x - v;
  *total = warp_sums[NW - 1];
  return before;
}

// Copies the K and V rows of the placed tokens: the k-th token tok_of(k)
// goes to slot slot_of(k), k < count.  A token's K row and V row are
// per_tok = 2 * (16-byte vectors per row) consecutive vectors; thread t always
// moves vector t % per_tok of tokens t / per_tok, + NT / per_tok, ... (per_tok
// is 16, 32 or 64 and divides NT), so a warp reads and writes whole rows and
// each thread keeps kCopyBatch loads in flight before it stores.
constexpr int kCopyBatch = 8;

template <int NT, class SlotOf, class TokOf>
__device__ __forceinline__ void copy_rows(const EvictParams& e, int b, int g, int count,
                                          SlotOf slot_of, TokOf tok_of) {
  const int vpr = e.d * e.esize / 16;  // vectors per row
  const int per_tok = 2 * vpr;
  const int r = static_cast<int>(threadIdx.x) % per_tok;
  const int tok_step = NT / per_tok;
  const bool is_v = r >= vpr;
  const int c = is_v ? r - vpr : r;
  const size_t vpr_s = static_cast<size_t>(vpr);
  // this thread's vector of new token 0 of (b, g), and of slot 0 of (b, g)
  const uint4* src0 = static_cast<const uint4*>(is_v ? e.v_new : e.k_new) +
                      (static_cast<size_t>(b) * e.nq * e.Hkv + g) * vpr_s + c;
  uint4* dst0 = static_cast<uint4*>(is_v ? e.v_cache : e.k_cache) +
                (static_cast<size_t>(b) * e.Hkv + g) * e.C * vpr_s + c;
  const size_t src_tok = static_cast<size_t>(e.Hkv) * vpr_s;  // vectors between new tokens
  for (int q0 = static_cast<int>(threadIdx.x) / per_tok; q0 < count; q0 += kCopyBatch * tok_step) {
    uint4 buf[kCopyBatch];
#pragma unroll
    for (int u = 0; u < kCopyBatch; ++u) {
      const int q = q0 + u * tok_step;
      if (q < count && H2O_IN_BOUNDS(tok_of(q) >= 0 && tok_of(q) < e.nq, e.state + 2))
        buf[u] = __ldg(src0 + static_cast<size_t>(tok_of(q)) * src_tok);
    }
#pragma unroll
    for (int u = 0; u < kCopyBatch; ++u) {
      const int q = q0 + u * tok_step;
      if (q < count && H2O_IN_BOUNDS(slot_of(q) >= 0 && slot_of(q) < e.C, e.state + 2))
        dst0[static_cast<size_t>(slot_of(q)) * vpr_s] = buf[u];
    }
  }
}

// The int8 cache (Q8): the placed tokens' rows are quantised on the way in.
// One warp per (token, K or V) row: the row's scale from a warp maximum, its
// codes written by every lane (q8.cuh).
template <int NT, int D, class SlotOf, class TokOf>
__device__ __forceinline__ void quantize_rows(const EvictParams& e, int b, int g, int count,
                                              SlotOf slot_of, TokOf tok_of) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t bg = static_cast<size_t>(b) * e.Hkv + g;
  for (int j = warp; j < 2 * count; j += NT / 32) {
    const int q = j >> 1;
    const bool is_v = j & 1;
    const int tok = tok_of(q), slot = slot_of(q);
    if (!H2O_IN_BOUNDS(tok >= 0 && tok < e.nq && slot >= 0 && slot < e.C, e.state + 2)) continue;
    const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(is_v ? e.v_new : e.k_new) +
                               ((static_cast<size_t>(b) * e.nq + tok) * e.Hkv + g) * D;
    int8_t* dst = static_cast<int8_t*>(is_v ? e.v_cache : e.k_cache) + (bg * e.C + slot) * D;
    float* sc = (is_v ? e.v_scale : e.k_scale) + bg * e.C + slot;
    q8_quantize_row_warp<D>(src, dst, sc, lane);
  }
}

// The K/V rows of the placed tokens: copied, or quantised for the int8 cache.
template <int NT, class SlotOf, class TokOf>
__device__ __forceinline__ void place_rows(const EvictParams& e, int b, int g, int count,
                                           SlotOf slot_of, TokOf tok_of) {
  if (!e.q8)
    copy_rows<NT>(e, b, g, count, slot_of, tok_of);
  else if (e.d == 128)
    quantize_rows<NT, 128>(e, b, g, count, slot_of, tok_of);
  else
    quantize_rows<NT, 64>(e, b, g, count, slot_of, tok_of);
}

constexpr int kLoadBatch = 8;  // global loads in flight per thread in the first pass
constexpr int kVecBatch = 2;   // 16-byte loads per array in flight per thread (four slots each)
constexpr int kNewPre = 4;     // new tokens' summed weights loaded per thread before the old slots
constexpr int kBins = 256;     // radix passes of 8 bits, most significant first

// What the selection of one (cache, KV head) needs to know.
struct SelectCtx {
  float* score;        // [C] of this (cache, KV head)
  const int* pos;      // [C]
  const float* cs;     // summed weights: [n] cache slots, then [C + i] new token i
  int n, nq, C, t0, sinks;
  long long limit;     // positions >= limit are in the protected window
  bool evict, by_score, old_protectable, need_pos;
};

// Step 1 for the candidates x in [x_lo, x_hi) (cache slot x < n, new token
// x - n otherwise): accumulates the slots' scores and writes each
// candidate's key to keys[x - x_lo].  kLoadBatch loads in flight per thread.
template <int NT>
__device__ __forceinline__ void build_keys(const SelectCtx& s, int x_lo, int x_hi,
                                           uint32_t* keys) {
  const int o_hi = min(x_hi, s.n);
  for (int x0 = x_lo + static_cast<int>(threadIdx.x); x0 < o_hi; x0 += kLoadBatch * NT) {
    float sc[kLoadBatch], cv[kLoadBatch];
    int ps[kLoadBatch];
#pragma unroll
    for (int k = 0; k < kLoadBatch; ++k) {
      const int x = x0 + k * NT;
      sc[k] = 0.f;
      cv[k] = 0.f;
      ps[k] = -1;
      if (x < o_hi) {
        if (s.by_score) {
          sc[k] = s.score[x];
          cv[k] = s.cs[x];
        }
        if (s.need_pos) ps[k] = s.pos[x];
      }
    }
#pragma unroll
    for (int k = 0; k < kLoadBatch; ++k) {
      const int x = x0 + k * NT;
      if (x < o_hi) {
        const bool prot = s.old_protectable && (ps[k] >= s.limit || ps[k] < s.sinks);
        uint32_t key;
        if (s.by_score) {
          const float v = sc[k] + cv[k];
          s.score[x] = v;
          key = score_key(v);
        } else {
          key = static_cast<uint32_t>(ps[k]);  // the most recent rank highest
        }
        keys[x - x_lo] = prot ? kProtectedKey : key;
      }
    }
  }
  for (int x0 = max(x_lo, s.n) + static_cast<int>(threadIdx.x); x0 < x_hi; x0 += kLoadBatch * NT) {
    float cv[kLoadBatch];
#pragma unroll
    for (int k = 0; k < kLoadBatch; ++k) {
      const int x = x0 + k * NT;
      cv[k] = (s.by_score && x < x_hi) ? s.cs[s.C + (x - s.n)] : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kLoadBatch; ++k) {
      const int x = x0 + k * NT;
      if (x < x_hi) {
        const long long p = static_cast<long long>(s.t0) + (x - s.n);
        const bool prot = s.evict && (p >= s.limit || p < s.sinks);
        keys[x - x_lo] = prot ? kProtectedKey
                              : (s.by_score ? score_key(cv[k]) : static_cast<uint32_t>(p));
      }
    }
  }
}

// Warp 0 of the CTA: the bin of histogram h (scanned from the top) that holds
// the k-th largest key, and the count of keys in the bins above it.
__device__ __forceinline__ void find_bin(const int* h, int k, int lane, int* sel_bin,
                                         int* sel_above) {
  constexpr int per = kBins / 32;  // lane L looks at bins 255-8L .. 248-8L
  int loc = 0;
#pragma unroll
  for (int e8 = 0; e8 < per; ++e8) loc += h[kBins - 1 - lane * per - e8];
  int inc = loc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  int run = inc - loc;  // keys in higher bins than this lane's
  if (run < k && run + loc >= k) {
    for (int e8 = 0; e8 < per; ++e8) {
      const int bin = kBins - 1 - lane * per - e8;
      const int cnt = h[bin];
      if (run + cnt >= k) {
        *sel_bin = bin;
        *sel_above = run;
        break;
      }
      run += cnt;
    }
  }
}

// The single-CTA selection finds the C-th largest key in three digits of
// 11, 11 and 10 bits (most significant first).  The first digit's histogram
// is built while the keys are made; the second pass also copies the keys of
// the chosen first-digit bin into a short list (when they fit), and the last
// digit is counted over that list only.
constexpr int kWideBins = 2048;  // 11-bit digits
constexpr int kListCap = 1024;   // keys of the chosen first-digit bin kept for the last pass

// Adds one to hist[bin] for every lane of the warp with bin >= 0 (lanes with
// the same bin add together).
__device__ __forceinline__ void warp_hist_add(int* hist, int bin, int lane) {
  const unsigned same = __match_any_sync(0xffffffffu, bin);
  if (bin >= 0 && (__ffs(same) - 1) == lane) atomicAdd(&hist[bin], __popc(same));
}

// Block-wide: the bin of hist[0, nbins) (counted from the top) that holds the
// k-th largest key, and the number of keys in the bins above it.  nbins is a
// multiple of NT; every thread takes nbins / NT consecutive bins.
template <int NT>
__device__ __forceinline__ void find_bin_block(const int* hist, int nbins, int k,
                                               uint64_t* warp_sums, int* sel_bin,
                                               int* sel_above) {
  const int per = nbins / NT;
  const int top = nbins - 1 - static_cast<int>(threadIdx.x) * per;  // this thread: top .. top-per+1
  int loc = 0;
  for (int e8 = 0; e8 < per; ++e8) loc += hist[top - e8];
  uint64_t tot;
  int run = static_cast<int>(block_excl_scan64<NT>(static_cast<uint64_t>(loc), warp_sums, &tot));
  if (run < k && run + loc >= k) {
    for (int e8 = 0; e8 < per; ++e8) {
      const int cnt = hist[top - e8];
      if (run + cnt >= k) {
        *sel_bin = top - e8;
        *sel_above = run;
        break;
      }
      run += cnt;
    }
  }
}

// Step 1 for the old slots [0, n_vec), four at a time (16-byte loads and
// stores): accumulates their scores, writes their keys, and tracks the lowest
// unprotected key and the protected count.  kB 16-byte loads per array in
// flight per thread; kPos: the positions are needed (the score-free
// policies, or a window or sinks that can protect an old slot).
template <int NT, int kB, bool kPos>
__device__ __forceinline__ void vec_pass(float* __restrict__ score, const float* __restrict__ cs,
                                         const int* __restrict__ pos, uint32_t* keys, int n_vec,
                                         bool by_score, bool old_protectable, long long limit,
                                         int sinks, uint32_t& old_min, int& n_prot) {
  const int tid = threadIdx.x;
  for (int v0 = tid; 4 * v0 < n_vec; v0 += kB * NT) {
    float4 sc[kB], cv[kB];
    int4 ps[kPos ? kB : 1];
#pragma unroll
    for (int k = 0; k < kB; ++k) {
      const int v = v0 + k * NT;
      sc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      cv[k] = sc[k];
      if (kPos) ps[k] = make_int4(-1, -1, -1, -1);
      if (4 * v < n_vec) {
        if (by_score) {
          sc[k] = reinterpret_cast<const float4*>(score)[v];
          cv[k] = reinterpret_cast<const float4*>(cs)[v];
        }
        if (kPos) ps[k] = reinterpret_cast<const int4*>(pos)[v];
      }
    }
#pragma unroll
    for (int k = 0; k < kB; ++k) {
      const int v = v0 + k * NT;
      if (4 * v >= n_vec) continue;
      const float s4[4] = {sc[k].x + cv[k].x, sc[k].y + cv[k].y, sc[k].z + cv[k].z,
                           sc[k].w + cv[k].w};
      int p4[4] = {-1, -1, -1, -1};
      if (kPos) {
        p4[0] = ps[k].x; p4[1] = ps[k].y; p4[2] = ps[k].z; p4[3] = ps[k].w;
      }
      uint32_t key4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool prot = kPos && old_protectable && (p4[e] >= limit || p4[e] < sinks);
        const uint32_t key = by_score ? score_key(s4[e]) : static_cast<uint32_t>(p4[e]);
        key4[e] = prot ? kProtectedKey : key;
        if (prot) ++n_prot; else old_min = min(old_min, key);
      }
      if (by_score) reinterpret_cast<float4*>(score)[v] = make_float4(s4[0], s4[1], s4[2], s4[3]);
      reinterpret_cast<uint4*>(keys)[v] = make_uint4(key4[0], key4[1], key4[2], key4[3]);
    }
  }
}

template <int NT>
__global__ void __launch_bounds__(NT, (NT == 256 ? 4 : 1))
    h2o_select(const EvictParams e, int plan_smem) {
  extern __shared__ uint32_t keys[];          // [n + nq], then (plan_smem) the plan [2][nq]
  __shared__ int hist[kWideBins];
  __shared__ uint32_t list[kListCap];
  __shared__ int list_n;
  __shared__ uint64_t warp_sums[32];
  __shared__ int sel_bin, sel_above;

  const int bg = blockIdx.x;
  const int b = bg / e.Hkv, g = bg % e.Hkv;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int n = e.n, nq = e.nq, C = e.C;
  const int NC = n + nq;
  float* __restrict__ score = e.scores + static_cast<size_t>(bg) * C;
  int* __restrict__ pos = e.pos + static_cast<size_t>(bg) * C;
  const float* __restrict__ cs = e.colsum + static_cast<size_t>(bg) * e.colsum_ld;
  int* __restrict__ slots = e.plan_slots + static_cast<size_t>(bg) * e.plan_ld;
  int* __restrict__ toks = e.plan_tokens + static_cast<size_t>(bg) * e.plan_ld;
  const bool evict = NC > C;
  const long long limit = static_cast<long long>(e.t0) + nq - e.W;
  const bool by_score = e.policy == kPolicyH2O;
  const int sinks = e.policy == kPolicySLR ? e.sinks : 0;
  // an old slot (position < t0) can be protected by the window only when
  // W > nq, by the sinks only under SLR
  const bool old_protectable = evict && (e.W > nq || sinks > 0);
  const bool need_pos = old_protectable || !by_score;
  for (int i = tid; i < kWideBins; i += NT) hist[i] = 0;
  if (tid == 0) list_n = 0;
  __syncthreads();
  griddep_wait();  // the summed weights come from the preceding kernel
  if (bg == 0 && tid == 0) {
    e.state[0] = min(C, n + nq);
    e.state[1] = e.t0 + nq;
  }

  // 1. accumulate scores and build the keys; loads are batched so that
  //    kLoadBatch of them are in flight per thread.  On the way: the lowest
  //    unprotected old key, the highest unprotected new key, the protected
  //    count (for the shortcut below).
  uint32_t old_min = 0xFFFFFFFFu, new_max = 0u;
  int n_prot = 0;
  // the old slots four at a time (16-byte loads and stores) when the unit's
  // scores, summed weights and positions are 16-byte aligned; the rest below
  const bool vec = ((reinterpret_cast<uintptr_t>(score) | reinterpret_cast<uintptr_t>(cs) |
                     reinterpret_cast<uintptr_t>(pos)) & 15) == 0;
  const int n_vec = vec ? (n & ~3) : 0;
  // the new tokens' summed weights (the first kNewPre per thread) are loaded
  // now, so that their latency overlaps the old slots' pass
  float cv_pre[kNewPre];
#pragma unroll
  for (int k = 0; k < kNewPre; ++k) {
    const int i = tid + k * NT;
    cv_pre[k] = (by_score && i < nq) ? cs[C + i] : 0.f;
  }
  if (need_pos)
    vec_pass<NT, kVecBatch, true>(score, cs, pos, keys, n_vec, by_score, old_protectable, limit,
                                  sinks, old_min, n_prot);
  else
    vec_pass<NT, 2 * kVecBatch, false>(score, cs, pos, keys, n_vec, by_score, old_protectable,
                                       limit, sinks, old_min, n_prot);
  for (int x0 = n_vec + tid; x0 < n; x0 += kLoadBatch * NT) {
    float sc[kLoadBatch], cv[kLoadBatch];
    int ps[kLoadBatch];
#pragma unroll
    for (int k = 0; k < kLoadBatch; ++k) {
      const int x = x0 + k * NT;
      sc[k] = 0.f;
      cv[k] = 0.f;
      ps[k] = -1;
      if (x < n) {
        if (by_score) {
          sc[k] = score[x];
          cv[k] = cs[x];
        }
        if (need_pos) ps[k] = pos[x];
      }
    }
#pragma unroll
    for (int k = 0; k < kLoadBatch; ++k) {
      const int x = x0 + k * NT;
      if (x < n) {
        const bool prot = old_protectable && (ps[k] >= limit || ps[k] < sinks);
        uint32_t key;
        if (by_score) {
          const float s = sc[k] + cv[k];
          score[x] = s;
          key = score_key(s);
        } else {
          key = static_cast<uint32_t>(ps[k]);  // the most recent rank highest
        }
        keys[x] = prot ? kProtectedKey : key;
        if (prot) ++n_prot; else old_min = min(old_min, key);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < kNewPre; ++k) {
    const int i = tid + k * NT;
    if (i < nq) {
      const long long p = static_cast<long long>(e.t0) + i;
      const bool prot = evict && (p >= limit || p < sinks);
      const uint32_t key = by_score ? score_key(cv_pre[k]) : static_cast<uint32_t>(p);
      keys[n + i] = prot ? kProtectedKey : key;
      if (prot) ++n_prot; else new_max = max(new_max, key);
    }
  }
  for (int i0 = kNewPre * NT + tid; i0 < nq; i0 += kLoadBatch * NT) {
    float cv[kLoadBatch];
#pragma unroll
    for (int k = 0; k < kLoadBatch; ++k) {
      const int i = i0 + k * NT;
      cv[k] = (by_score && i < nq) ? cs[C + i] : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kLoadBatch; ++k) {
      const int i = i0 + k * NT;
      if (i < nq) {
        const long long p = static_cast<long long>(e.t0) + i;
        const bool prot = evict && (p >= limit || p < sinks);
        const uint32_t key = by_score ? score_key(cv[k]) : static_cast<uint32_t>(p);
        keys[n + i] = prot ? kProtectedKey : key;
        if (prot) ++n_prot; else new_max = max(new_max, key);
      }
    }
  }
  if (!evict) {
    // fill phase: every new token goes to slot n + i
    for (int i = tid; i < nq; i += NT) {
      slots[i] = n + i;
      toks[i] = i;
      score[n + i] = by_score ? cs[C + i] : 0.f;
      pos[n + i] = e.t0 + i;
    }
    if (tid == 0) e.plan_count[bg] = nq;
    place_rows<NT>(e, b, g, nq, [n](int q) { return n + q; }, [](int q) { return q; });
    return;
  }
  // A full cache, nothing protected, and no new key above the lowest old key:
  // the C old entries are the top C (an old slot also wins a tie: its index
  // is lower), so nothing moves and the scores are already updated.  This is
  // the steady state of caches without a recent window, where one chunk's
  // summed weights stay below the weights the cache's entries have gathered.
  {
    uint32_t a = old_min, z = new_max;
    int pr = n_prot;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
      z = max(z, __shfl_xor_sync(0xffffffffu, z, o));
      pr += __shfl_xor_sync(0xffffffffu, pr, o);
    }
    __shared__ uint32_t red_min[NT / 32], red_max[NT / 32];
    __shared__ int red_prot[NT / 32];
    if (lane == 0) {
      red_min[tid >> 5] = a;
      red_max[tid >> 5] = z;
      red_prot[tid >> 5] = pr;
    }
    __syncthreads();
    if (tid < 32) {
      a = tid < NT / 32 ? red_min[tid] : 0xFFFFFFFFu;
      z = tid < NT / 32 ? red_max[tid] : 0u;
      pr = tid < NT / 32 ? red_prot[tid] : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
        z = max(z, __shfl_xor_sync(0xffffffffu, z, o));
        pr += __shfl_xor_sync(0xffffffffu, pr, o);
      }
      if (tid == 0) sel_bin = (n == C && pr == 0 && z <= a) ? 1 : 0;
    }
    __syncthreads();
    if (sel_bin) {
      if (tid == 0) e.plan_count[bg] = 0;
      return;
    }
  }

  // 2. the C-th largest key, three digits: bits 31..21 over every key;
  //    bits 20..10 over the keys of the chosen first-digit bin, which are also
  //    listed (when they fit); bits 9..0 over that list (or, when it
  //    overflowed, over every key with the chosen 22-bit prefix)
  const int iters = (NC + NT - 1) / NT;
  for (int it = 0; it < iters; ++it) {
    const int x = it * NT + tid;
    warp_hist_add(hist, x < NC ? static_cast<int>(keys[x] >> 21) : -1, lane);
  }
  __syncthreads();
  int k = C;  // rank (1-based, descending) still to locate
  find_bin_block<NT>(hist, kWideBins, k, warp_sums, &sel_bin, &sel_above);
  __syncthreads();
  const uint32_t d1 = static_cast<uint32_t>(sel_bin);
  k -= sel_above;
  for (int i = tid; i < kWideBins; i += NT) hist[i] = 0;
  __syncthreads();
  for (int it = 0; it < iters; ++it) {
    const int x = it * NT + tid;
    const uint32_t key = x < NC ? keys[x] : 0u;
    const bool in = x < NC && (key >> 21) == d1;
    warp_hist_add(hist, in ? static_cast<int>((key >> 10) & (kWideBins - 1)) : -1, lane);
    const unsigned ball = __ballot_sync(0xffffffffu, in);
    int base = 0;
    if (lane == 0 && ball) base = atomicAdd(&list_n, __popc(ball));
    base = __shfl_sync(0xffffffffu, base, 0);
    const int at = base + __popc(ball & ((1u << lane) - 1u));
    if (in && at < kListCap) list[at] = key;
  }
  __syncthreads();
  find_bin_block<NT>(hist, kWideBins, k, warp_sums, &sel_bin, &sel_above);
  __syncthreads();
  const uint32_t pre22 = (d1 << 11) | static_cast<uint32_t>(sel_bin);  // key >> 10
  k -= sel_above;
  const int listed = list_n;
  for (int i = tid; i < 1024; i += NT) hist[i] = 0;
  __syncthreads();
  const bool use_list = listed <= kListCap;
  const int m = use_list ? listed : NC;
  for (int it = 0; it < (m + NT - 1) / NT; ++it) {
    const int x = it * NT + tid;
    const uint32_t key = x < m ? (use_list ? list[x] : keys[x]) : 0u;
    const bool in = x < m && (key >> 10) == pre22;
    warp_hist_add(hist, in ? static_cast<int>(key & 1023u) : -1, lane);
  }
  __syncthreads();
  find_bin_block<NT>(hist, 1024, k, warp_sums, &sel_bin, &sel_above);
  __syncthreads();
  const uint32_t prefix = (pre22 << 10) | static_cast<uint32_t>(sel_bin);
  k -= sel_above;

  // when no new token is kept (so n == C and nothing moves: the scores are
  // already updated) the ordered pass below is not needed.  Kept new tokens:
  // those above T, and of the keys equal to T the first k in candidate order,
  // where the old slots come first.
  {
    const uint32_t T0 = prefix;
    int gt_new = 0, eq_old = 0, eq_new = 0;
    for (int x = tid; x < NC; x += NT) {
      const uint32_t key = keys[x];
      if (x < n) {
        eq_old += key == T0;
      } else {
        gt_new += key > T0;
        eq_new += key == T0;
      }
    }
    uint64_t tot;
    block_excl_scan64<NT>(static_cast<uint64_t>(gt_new) | (static_cast<uint64_t>(eq_old) << 16) |
                              (static_cast<uint64_t>(eq_new) << 32),
                          warp_sums, &tot);
    const int t_gt_new = static_cast<int>(tot & 0xFFFF);
    const int t_eq_old = static_cast<int>((tot >> 16) & 0xFFFF);
    const int t_eq_new = static_cast<int>((tot >> 32) & 0xFFFF);
    const int kept_new = t_gt_new + max(0, min(t_eq_new, k - t_eq_old));
    if (kept_new == 0 && n == C) {
      if (tid == 0) e.plan_count[bg] = 0;
      return;
    }
  }
  const uint32_t T = prefix;  // C-th largest key; keep the first k keys equal to T

  // 3. ordered pass over contiguous ranges.  Keys above T stay, keys below
  //    go, and of the keys equal to T the first k in candidate-index order
  //    stay.  One scan of four counters per thread (freed old slots and kept
  //    new tokens among the keys != T, keys == T, keys == T that are old
  //    slots) places every thread's output: old slots precede new tokens in
  //    index order, so the kept T-keys before a range are the first
  //    min(eq, k) of them, and the old ones among those min(eq_old, k).
  const int per = (NC + NT - 1) / NT;
  const int lo = min(NC, tid * per), hi = min(NC, lo + per);
  int fo_s = 0, nn_s = 0, eq = 0, eq_old = 0;
  for (int x = lo; x < hi; ++x) {
    const uint32_t key = keys[x];
    if (key == T) {
      ++eq;
      eq_old += x < n;
    } else if (key > T) {
      nn_s += x >= n;
    } else {
      fo_s += x < n;
    }
  }
  // counts and totals stay below 2^16 (candidates <= kMaxCandidates)
  uint64_t pk_tot;
  const uint64_t pk_before = block_excl_scan64<NT>(
      static_cast<uint64_t>(fo_s) | (static_cast<uint64_t>(nn_s) << 16) |
          (static_cast<uint64_t>(eq) << 32) | (static_cast<uint64_t>(eq_old) << 48),
      warp_sums, &pk_tot);
  auto field = [](uint64_t v, int f) { return static_cast<int>((v >> (16 * f)) & 0xFFFF); };
  const int eq_b = field(pk_before, 2), eqo_b = field(pk_before, 3);
  const int fo_before = field(pk_before, 0) + eqo_b - min(eqo_b, k);
  const int nw_before = field(pk_before, 1) + min(eq_b, k) - min(eqo_b, k);
  const int eq_t = field(pk_tot, 2), eqo_t = field(pk_tot, 3);
  const int tot_free_old = field(pk_tot, 0) + eqo_t - min(eqo_t, k);
  const int tot_new = field(pk_tot, 1) + min(eq_t, k) - min(eqo_t, k);
  // empty slots n .. C-1 are free too: thread t takes a fixed share, in order
  const int empty = C - n;
  const int e_per = (empty + NT - 1) / NT;
  const int e_lo = n + min(empty, tid * e_per), e_hi = n + min(empty, (tid + 1) * e_per);
  if (tot_free_old + empty != tot_new) {
    if (tid == 0) {
      atomicOr(e.state + 2, kDevErrPlan);
      e.plan_count[bg] = 0;
    }
    return;
  }
  // free slots in order (evicted old slots (< n) first, then the empty ones)
  // and kept new tokens in order; in shared memory when it has room
  int* p_slots = plan_smem ? reinterpret_cast<int*>(keys + NC) : slots;
  int* p_toks = plan_smem ? p_slots + nq : toks;
  int fo = fo_before, nw = nw_before, eq_rank = eq_b;
  for (int x = lo; x < hi; ++x) {
    const uint32_t key = keys[x];
    bool kept = key > T;
    if (key == T) kept = eq_rank++ < k;
    if (x < n) {
      if (!kept && H2O_IN_BOUNDS(fo < nq, e.state + 2)) p_slots[fo++] = x;
    } else if (kept && H2O_IN_BOUNDS(nw < nq, e.state + 2)) {
      p_toks[nw++] = x - n;
    }
  }
  int em = tot_free_old + (e_lo - n);
  for (int s = e_lo; s < e_hi; ++s)
    if (H2O_IN_BOUNDS(em < nq, e.state + 2)) p_slots[em++] = s;
  __syncthreads();
  // 4. scores and positions of the placed tokens (and the plan, when it was
  //    built in shared memory), then their K/V rows
  for (int q = tid; q < tot_new; q += NT) {
    const int s = p_slots[q], i = p_toks[q];
    if (!H2O_IN_BOUNDS(s >= 0 && s < C && i >= 0 && i < nq, e.state + 2)) continue;
    score[s] = by_score ? cs[C + i] : 0.f;
    pos[s] = e.t0 + i;
    if (plan_smem) {
      slots[q] = s;
      toks[q] = i;
    }
  }
  if (tid == 0) e.plan_count[bg] = tot_new;
  place_rows<NT>(e, b, g, tot_new, [p_slots](int q) { return p_slots[q]; },
                [p_toks](int q) { return p_toks[q]; });
}

// h2o_select_cluster: the same selection for few (cache, KV head) units,
// spread over a cluster of CL CTAs each, so that one unit's work runs on CL
// SMs.  CTA r of the cluster holds the keys of candidates [r*share,
// (r+1)*share).  Each radix pass counts into the CTA's own histogram (two
// buffers, alternating between passes, so that one cluster barrier per pass
// suffices), then every CTA sums the CL histograms through distributed shared
// memory and finds the same digit.  The ordered compaction scans each CTA's
// range, exchanges the CTA totals the same way and writes the plan to global
// memory; after a cluster barrier (release / acquire) each CTA places its
// share of the kept tokens.  Every CTA takes the same cluster barriers; none
// leaves before the last one, after which no CTA reads another's memory.
template <int NT, int CL>
__global__ void __launch_bounds__(NT, 1) h2o_select_cluster(const EvictParams e) {
  extern __shared__ uint32_t keys[];  // [share]: this CTA's candidates
  __shared__ int hist[2][kBins];      // this CTA's counts, alternating buffers
  __shared__ int tot[kBins];          // the cluster's counts of the current pass
  __shared__ uint64_t warp_sums[32];
  __shared__ uint64_t cta_total;      // this CTA's packed counters, read by the cluster
  __shared__ uint64_t cl_before, cl_total;
  __shared__ int sel_bin, sel_above;

  const int rank = static_cast<int>(cluster_ctarank());
  const int bg = blockIdx.x / CL;
  const int b = bg / e.Hkv, g = bg % e.Hkv;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int n = e.n, nq = e.nq, C = e.C;
  const int NC = n + nq;
  float* __restrict__ score = e.scores + static_cast<size_t>(bg) * C;
  int* __restrict__ pos = e.pos + static_cast<size_t>(bg) * C;
  const float* __restrict__ cs = e.colsum + static_cast<size_t>(bg) * e.colsum_ld;
  int* __restrict__ slots = e.plan_slots + static_cast<size_t>(bg) * e.plan_ld;
  int* __restrict__ toks = e.plan_tokens + static_cast<size_t>(bg) * e.plan_ld;
  SelectCtx sx;
  sx.score = score;
  sx.pos = pos;
  sx.cs = cs;
  sx.n = n;
  sx.nq = nq;
  sx.C = C;
  sx.t0 = e.t0;
  sx.evict = NC > C;
  sx.by_score = e.policy == kPolicyH2O;
  sx.sinks = e.policy == kPolicySLR ? e.sinks : 0;
  sx.limit = static_cast<long long>(e.t0) + nq - e.W;
  sx.old_protectable = sx.evict && (e.W > nq || sx.sinks > 0);
  sx.need_pos = sx.old_protectable || !sx.by_score;
  const int share = (NC + CL - 1) / CL;
  const int x_lo = min(NC, rank * share), x_hi = min(NC, x_lo + share);
  const int len = x_hi - x_lo;
  griddep_wait();  // the summed weights come from the preceding kernel
  if (bg == 0 && rank == 0 && tid == 0) {
    e.state[0] = min(C, n + nq);
    e.state[1] = e.t0 + nq;
  }

  // 1. scores and keys of this CTA's candidates
  build_keys<NT>(sx, x_lo, x_hi, keys);
  if (!sx.evict) {
    // fill phase: new token i goes to slot n + i; CTA r takes the tokens of
    // its own share (no cluster barrier on this path)
    const int qs = (nq + CL - 1) / CL;
    const int i_lo = min(nq, rank * qs), i_hi = min(nq, i_lo + qs);
    for (int i = i_lo + tid; i < i_hi; i += NT) {
      slots[i] = n + i;
      toks[i] = i;
      score[n + i] = sx.by_score ? cs[C + i] : 0.f;
      pos[n + i] = e.t0 + i;
    }
    if (rank == 0 && tid == 0) e.plan_count[bg] = nq;
    place_rows<NT>(e, b, g, i_hi - i_lo, [n, i_lo](int q) { return n + i_lo + q; },
                  [i_lo](int q) { return i_lo + q; });
    return;
  }
  __syncthreads();

  // 2. radix select of the C-th largest key over the whole cluster
  uint32_t prefix = 0, pmask = 0;
  int k = C;  // rank (1-based, descending) still to locate
  const int iters = (len + NT - 1) / NT;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    int* my_hist = hist[pass & 1];
    for (int i = tid; i < kBins; i += NT) my_hist[i] = 0;
    __syncthreads();
    for (int it = 0; it < iters; ++it) {
      const int x = it * NT + tid;
      int bin = -1;
      if (x < len) {
        const uint32_t key = keys[x];
        if ((key & pmask) == prefix) bin = static_cast<int>((key >> shift) & (kBins - 1));
      }
      const unsigned same = __match_any_sync(0xffffffffu, bin);
      if (bin >= 0 && (__ffs(same) - 1) == lane) atomicAdd(&my_hist[bin], __popc(same));
    }
    cluster_sync_all();  // every CTA's counts of this pass are complete
    for (int i = tid; i < kBins; i += NT) {
      const uint32_t a = smem_u32(&my_hist[i]);
      int t = 0;
#pragma unroll
      for (int r = 0; r < CL; ++r) t += static_cast<int>(ld_dsmem_u32(dsmem_map(a, r)));
      tot[i] = t;
    }
    __syncthreads();
    if (warp == 0) find_bin(tot, k, lane, &sel_bin, &sel_above);
    __syncthreads();
    prefix |= static_cast<uint32_t>(sel_bin) << shift;
    pmask |= static_cast<uint32_t>(kBins - 1) << shift;
    k -= sel_above;
    // the buffer read above is cleared again two passes later, after the
    // next pass's cluster barrier: every CTA has finished reading it by then
  }
  const uint32_t T = prefix;  // C-th largest key; keep the first k keys equal to T

  // 3. ordered compaction (the packed counters of the single-CTA kernel),
  //    first within the CTA, then across the cluster in rank order
  const int per = (len + NT - 1) / NT;
  const int lo = min(len, tid * per), hi = min(len, lo + per);
  int fo_s = 0, nn_s = 0, eq = 0, eq_old = 0;
  for (int j = lo; j < hi; ++j) {
    const uint32_t key = keys[j];
    const int x = x_lo + j;
    if (key == T) {
      ++eq;
      eq_old += x < n;
    } else if (key > T) {
      nn_s += x >= n;
    } else {
      fo_s += x < n;
    }
  }
  uint64_t cta_sum;
  const uint64_t in_cta = block_excl_scan64<NT>(
      static_cast<uint64_t>(fo_s) | (static_cast<uint64_t>(nn_s) << 16) |
          (static_cast<uint64_t>(eq) << 32) | (static_cast<uint64_t>(eq_old) << 48),
      warp_sums, &cta_sum);
  if (tid == 0) cta_total = cta_sum;
  cluster_sync_all();  // every CTA's total is published
  if (warp == 0) {
    const uint64_t v = lane < CL ? ld_dsmem_u64(dsmem_map(smem_u32(&cta_total), lane)) : 0;
    uint64_t before = 0, all = 0;
#pragma unroll
    for (int r = 0; r < CL; ++r) {
      const uint64_t t = __shfl_sync(0xffffffffu, v, r);
      all += t;
      if (r < rank) before += t;
    }
    if (lane == 0) {
      cl_before = before;
      cl_total = all;
    }
  }
  __syncthreads();
  auto field = [](uint64_t v, int f) { return static_cast<int>((v >> (16 * f)) & 0xFFFF); };
  const uint64_t pk_before = cl_before + in_cta, pk_tot = cl_total;
  const int eq_b = field(pk_before, 2), eqo_b = field(pk_before, 3);
  const int fo_before = field(pk_before, 0) + eqo_b - min(eqo_b, k);
  const int nw_before = field(pk_before, 1) + min(eq_b, k) - min(eqo_b, k);
  const int eq_t = field(pk_tot, 2), eqo_t = field(pk_tot, 3);
  const int tot_free_old = field(pk_tot, 0) + eqo_t - min(eqo_t, k);
  const int tot_new = field(pk_tot, 1) + min(eq_t, k) - min(eqo_t, k);
  // empty slots n .. C-1 are free too: the cluster's threads take fixed shares
  const int empty = C - n;
  const int gt = rank * NT + tid;
  const int e_per = (empty + CL * NT - 1) / (CL * NT);
  const int e_lo = n + min(empty, gt * e_per), e_hi = n + min(empty, (gt + 1) * e_per);
  const bool bad = tot_free_old + empty != tot_new;  // the same in every CTA
  if (!bad) {
    int fo = fo_before, nw = nw_before, eq_rank = eq_b;
    for (int j = lo; j < hi; ++j) {
      const uint32_t key = keys[j];
      const int x = x_lo + j;
      bool kept = key > T;
      if (key == T) kept = eq_rank++ < k;
      if (x < n) {
        if (!kept && H2O_IN_BOUNDS(fo < e.plan_ld, e.state + 2)) slots[fo++] = x;
      } else if (kept && H2O_IN_BOUNDS(nw < e.plan_ld, e.state + 2)) {
        toks[nw++] = x - n;
      }
    }
    int em = tot_free_old + (e_lo - n);
    for (int s2 = e_lo; s2 < e_hi; ++s2)
      if (H2O_IN_BOUNDS(em < e.plan_ld, e.state + 2)) slots[em++] = s2;
  }
  cluster_sync_all();  // the plan is complete; no CTA reads another's shared memory after this
  if (bad) {
    if (rank == 0 && tid == 0) {
      atomicOr(e.state + 2, kDevErrPlan);
      e.plan_count[bg] = 0;
    }
    return;
  }
  // 4. this CTA's share of the placed tokens: scores, positions, K/V rows
  const int qs = (tot_new + CL - 1) / CL;
  const int q_lo = min(tot_new, rank * qs), q_hi = min(tot_new, q_lo + qs);
  for (int q = q_lo + tid; q < q_hi; q += NT) {
    const int s2 = slots[q], i = toks[q];
    if (!H2O_IN_BOUNDS(s2 >= 0 && s2 < C && i >= 0 && i < nq, e.state + 2)) continue;
    score[s2] = sx.by_score ? cs[C + i] : 0.f;
    pos[s2] = e.t0 + i;
  }
  if (rank == 0 && tid == 0) e.plan_count[bg] = tot_new;
  place_rows<NT>(e, b, g, q_hi - q_lo, [slots, q_lo](int q) { return slots[q_lo + q]; },
                [toks, q_lo](int q) { return toks[q_lo + q]; });
}

// Dynamic shared memory the selection kernel can take next to its static
// arrays (histograms, scan sums).
template <int NT>
static size_t select_dyn_limit() {
  static const size_t limit = [] {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, h2o_select<NT>) != cudaSuccess) return size_t{0};
    return static_cast<size_t>(kMaxDynSmem) - fa.sharedSizeBytes;
  }();
  return limit;
}

template <int NT>
static cudaError_t launch_select(const EvictParams& e, cudaStream_t st) {
  const size_t limit = select_dyn_limit<NT>();
  if (limit < static_cast<size_t>(kMaxCandidates) * sizeof(uint32_t)) return cudaErrorInvalidValue;
  // the keys, then the plan when it fits next to them
  const size_t keys_bytes = static_cast<size_t>(e.n + e.nq) * sizeof(uint32_t);
  const size_t plan_bytes = static_cast<size_t>(2) * e.nq * sizeof(int);
  const int plan_smem = keys_bytes + plan_bytes <= limit ? 1 : 0;
  const size_t smem = keys_bytes + (plan_smem ? plan_bytes : 0);
  static int attr_bits[2] = {0, 0};
  cudaError_t err = ensure_smem_attr(reinterpret_cast<const void*>(h2o_select<NT>),
                                     static_cast<int>(limit), attr_bits);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(e.B * e.Hkv);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, h2o_select<NT>, e, plan_smem);
}

// Cluster variant: kClusterCtas CTAs of kClusterThreads per (cache, KV head),
// used while the units fill at most kClusterUnits * kClusterCtas SMs.
constexpr int kClusterCtas = 8;
constexpr int kClusterThreads = 512;
constexpr int kClusterUnits = 16;

static cudaError_t launch_select_cluster(const EvictParams& e, cudaStream_t st) {
  constexpr int CL = kClusterCtas, NT = kClusterThreads;
  const int share = (e.n + e.nq + CL - 1) / CL;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(e.B * e.Hkv * CL);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = static_cast<size_t>(share) * sizeof(uint32_t);  // <= 25 KiB
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, h2o_select_cluster<NT, CL>, e);
}

cudaError_t launch_evict(const EvictParams& e, int max_chunk, cudaStream_t st) {
  (void)max_chunk;
  // few (cache, KV head) units: a cluster of CTAs each, so that a unit's
  // selection runs on several SMs; many units: one CTA each (smaller CTAs,
  // several per SM, once the units outnumber the SMs twice)
  if (e.B * e.Hkv <= kClusterUnits) return launch_select_cluster(e, st);
  if (e.B * e.Hkv >= 2 * 148) return launch_select<256>(e, st);
  return launch_select<1024>(e, st);
}

}  // namespace h2o
