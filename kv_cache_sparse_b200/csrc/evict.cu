// evict.cu -- H2O score accumulation, top-C selection and K/V slot scatter.
//
// "Learning how to Forget", §1: a fixed-size KV cache whose slots a policy
// evicts when it is full; summary page glossary "H2O": entries are scored by
// the attention they accumulated and the less important ones evicted.
//
// h2o_select (one 1024-thread CTA per (cache, KV head); candidates in shared
// memory):
//   1. score[s] <- fl32(score[s] + colsum[s]) for the n valid slots; new token
//      i's candidate score is colsum[C + i].
//   2. If n + nq <= C every new token is kept and goes to slot n + i.
//   3. Otherwise a candidate at position >= t0 + nq - W is protected.  Each
//      candidate gets a 32-bit key: 0xFFFFFFFF when protected, else the bit
//      pattern of its (non-negative) fp32 score, which orders like the score.
//      A 4 x 8-bit MSB-first radix select finds the C-th largest key T and
//      how many keys equal to T are kept; those are the ones of lowest
//      candidate index (slot s -> s, new token i -> n + i; same order as the
//      C + i numbering).  So exactly C candidates stay, ties go to the lower
//      index, and the protected ones always stay (there are at most W <= C).
//   4. Ordered compaction (block scans over contiguous per-thread ranges)
//      lists the free slots (evicted or empty) and the kept new tokens in
//      ascending order; the k-th kept token goes to the k-th free slot.  The
//      CTA writes the score and position of the placed tokens and the plan.
// h2o_scatter (many CTAs per (cache, KV head)): copies the K and V rows of the
// placed tokens into their slots with 16-byte vector loads and stores.
#include "attn.h"
#include "sm100.cuh"

namespace h2o {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr uint32_t kProtectedKey = 0xFFFFFFFFu;

__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  return u == 0x80000000u ? 0u : u;  // -0 orders as +0
}

// Exclusive scan of one value per thread over the block; returns the prefix,
// writes the block total to *total.  All threads must call it.
__device__ __forceinline__ int block_excl_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) warp_sums[w] = x;
  __syncthreads();
  if (w == 0) {
    int s = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;  // inclusive
  }
  __syncthreads();
  const int before = (w > 0 ? warp_sums[w - 1] : 0) + x - v;
  *total = warp_sums[kSelWarps - 1];
  return before;
}

__global__ void __launch_bounds__(kSelThreads, 1) h2o_select(const EvictParams e) {
  extern __shared__ uint32_t keys[];  // [n + nq]
  __shared__ int hist[256];
  __shared__ int warp_sums[kSelWarps];
  __shared__ int sel_bin, sel_above;

  const int bg = blockIdx.x;
  const int tid = threadIdx.x;
  const int n = e.n, nq = e.nq, C = e.C;
  const int NC = n + nq;
  float* score = e.scores + static_cast<size_t>(bg) * C;
  int* pos = e.pos + static_cast<size_t>(bg) * C;
  const float* cs = e.colsum + static_cast<size_t>(bg) * e.colsum_ld;
  int* slots = e.plan_slots + static_cast<size_t>(bg) * e.plan_ld;
  int* toks = e.plan_tokens + static_cast<size_t>(bg) * e.plan_ld;
  const bool evict = NC > C;
  const long long limit = static_cast<long long>(e.t0) + nq - e.W;

  // 1. accumulate scores, build the keys
  for (int x = tid; x < NC; x += kSelThreads) {
    float s;
    long long ps;
    if (x < n) {
      s = score[x] + cs[x];
      score[x] = s;
      ps = pos[x];
    } else {
      s = cs[C + (x - n)];
      ps = static_cast<long long>(e.t0) + (x - n);
    }
    keys[x] = (evict && ps >= limit) ? kProtectedKey : score_key(s);
  }
  if (!evict) {
    for (int i = tid; i < nq; i += kSelThreads) {
      slots[i] = n + i;
      toks[i] = i;
      score[n + i] = cs[C + i];
      pos[n + i] = e.t0 + i;
    }
    if (tid == 0) e.plan_count[bg] = nq;
    return;
  }
  __syncthreads();

  // 2. radix select of the C-th largest key
  uint32_t prefix = 0, pmask = 0;
  int k = C;  // rank (1-based, descending) still to locate
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    const int iters = (NC + kSelThreads - 1) / kSelThreads;
    for (int it = 0; it < iters; ++it) {
      const int x = it * kSelThreads + tid;
      int bin = 256;
      if (x < NC) {
        const uint32_t key = keys[x];
        if ((key & pmask) == prefix) bin = (key >> shift) & 255;
      }
      const unsigned same = __match_any_sync(0xffffffffu, bin);
      if (bin < 256 && (__ffs(same) - 1) == (tid & 31)) atomicAdd(&hist[bin], __popc(same));
    }
    __syncthreads();
    if (tid < 32) {
      // lane L looks at bins 255-8L .. 248-8L (descending)
      int cnt[8], loc = 0;
#pragma unroll
      for (int e8 = 0; e8 < 8; ++e8) {
        cnt[e8] = hist[255 - 8 * tid - e8];
        loc += cnt[e8];
      }
      int inc = loc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (tid >= o) inc += y;
      }
      int run = inc - loc;  // keys in higher bins than this lane's
#pragma unroll
      for (int e8 = 0; e8 < 8; ++e8) {
        if (run < k && run + cnt[e8] >= k) {
          sel_bin = 255 - 8 * tid - e8;
          sel_above = run;
        }
        run += cnt[e8];
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(sel_bin) << shift;
    pmask |= 0xFFu << shift;
    k -= sel_above;
    __syncthreads();
  }
  const uint32_t T = prefix;  // C-th largest key; keep the first k keys equal to T

  // 3. ordered pass over contiguous ranges: rank the T-keys, count free slots
  //    and kept new tokens
  const int per = (NC + kSelThreads - 1) / kSelThreads;
  const int lo = min(NC, tid * per), hi = min(NC, lo + per);
  int n_eq = 0;
  for (int x = lo; x < hi; ++x) n_eq += (keys[x] == T);
  int tot;
  int eq_before = block_excl_scan(n_eq, warp_sums, &tot);
  int n_free = 0, n_new = 0;
  for (int x = lo; x < hi; ++x) {
    const uint32_t key = keys[x];
    bool kept = key > T;
    if (key == T) kept = (eq_before++ < k);
    if (x < n) n_free += !kept;
    else n_new += kept;
    keys[x] = kept ? 1u : 0u;  // from here on: kept flag
  }
  // empty slots n .. C-1 are free too; give them to the threads in order
  const int empty = C - n;
  const int e_per = (empty + kSelThreads - 1) / kSelThreads;
  const int e_lo = n + min(empty, tid * e_per), e_hi = n + min(empty, (tid + 1) * e_per);
  n_free += e_hi - e_lo;
  // free slots are ordered: evicted slots (< n) of threads 0..1023, then the
  // empty slots (>= n) of threads 0..1023; scan the two parts separately
  const int free_old = n_free - (e_hi - e_lo);
  int tot_free_old, tot_empty, tot_new;
  const int fo_before = block_excl_scan(free_old, warp_sums, &tot_free_old);
  const int em_before = block_excl_scan(e_hi - e_lo, warp_sums, &tot_empty);
  const int nw_before = block_excl_scan(n_new, warp_sums, &tot_new);
  if (tot_free_old + tot_empty != tot_new) {
    if (tid == 0) {
      atomicOr(e.state + 2, kDevErrPlan);
      e.plan_count[bg] = 0;
    }
    return;
  }
  int fo = fo_before, nw = nw_before;
  for (int x = lo; x < hi; ++x) {
    if (x < n) {
      if (!keys[x]) slots[fo++] = x;
    } else if (keys[x]) {
      toks[nw++] = x - n;
    }
  }
  int em = tot_free_old + em_before;
  for (int s = e_lo; s < e_hi; ++s) slots[em++] = s;
  __syncthreads();
  // 4. scores and positions of the placed tokens
  for (int q = tid; q < tot_new; q += kSelThreads) {
    const int s = slots[q], i = toks[q];
    score[s] = cs[C + i];
    pos[s] = e.t0 + i;
  }
  if (tid == 0) e.plan_count[bg] = tot_new;
}

// One 16-byte vector per thread; rows of d * esize bytes (a multiple of 16).
__global__ void __launch_bounds__(256) h2o_scatter(const EvictParams e) {
  const int bg = blockIdx.x;
  const int b = bg / e.Hkv, g = bg % e.Hkv;
  const int count = e.plan_count[bg];
  const int vpr = e.d * e.esize / 16;  // vectors per row
  const int total = 2 * count * vpr;   // K rows then V rows
  const int* slots = e.plan_slots + static_cast<size_t>(bg) * e.plan_ld;
  const int* toks = e.plan_tokens + static_cast<size_t>(bg) * e.plan_ld;
  const size_t row_bytes = static_cast<size_t>(e.d) * e.esize;
  for (int w = blockIdx.y * blockDim.x + threadIdx.x; w < total; w += gridDim.y * blockDim.x) {
    const int which = w / (count * vpr);  // 0: K, 1: V
    const int r = w % (count * vpr);
    const int q = r / vpr, v = r % vpr;
    const int s = slots[q], i = toks[q];
    const uint8_t* src = static_cast<const uint8_t*>(which ? e.v_new : e.k_new) +
                         ((static_cast<size_t>(b) * e.nq + i) * e.Hkv + g) * row_bytes;
    uint8_t* dst = static_cast<uint8_t*>(which ? e.v_cache : e.k_cache) +
                   ((static_cast<size_t>(b) * e.Hkv + g) * e.C + s) * row_bytes;
    const uint4 val = __ldg(reinterpret_cast<const uint4*>(src) + v);
    reinterpret_cast<uint4*>(dst)[v] = val;
  }
  if (bg == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    e.state[0] = min(e.C, e.n + e.nq);
    e.state[1] = e.t0 + e.nq;
  }
}

cudaError_t launch_evict(const EvictParams& e, int max_chunk, cudaStream_t st,
                         cudaEvent_t between) {
  const size_t smem = static_cast<size_t>(e.n + e.nq) * sizeof(uint32_t);
  static int attr_bits[2] = {0, 0};
  if (!smem_attr_done(reinterpret_cast<const void*>(h2o_select), attr_bits)) {
    cudaError_t err = cudaFuncSetAttribute(h2o_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kMaxCandidates * 4);
    if (err != cudaSuccess) return err;
  }
  const int units = e.B * e.Hkv;
  h2o_select<<<units, kSelThreads, smem, st>>>(e);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (between) cudaEventRecord(between, st);
  const int vpr = e.d * e.esize / 16;
  const int work = 2 * e.nq * vpr;
  int gy = cdiv(work, 256);
  const int target = 4 * 148;  // spread the copy over every SM
  gy = max(1, min(gy, cdiv(target, units)));
  h2o_scatter<<<dim3(units, gy), 256, 0, st>>>(e);
  (void)max_chunk;
  return cudaGetLastError();
}

}  // namespace h2o
