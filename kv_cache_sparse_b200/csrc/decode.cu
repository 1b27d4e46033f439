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
//   decode_partial  grid (cdiv(n + 1, 256), B*Hkv), 256 threads.  The keys
//                   [256k, 256k + 256) of one (cache, KV head); key n is the
//                   new token.  Thread = key: the G logits x = c<q_h, k>
//                   (fp32 FMA over 16-byte loads of the K row), stored for
//                   the summed weights; the chunk's max and sum of 2^(x - m)
//                   per head.  Then thread = (8 head-dim elements, key
//                   group): the chunk's unnormalised P V for the G heads,
//                   summed over the key groups in a fixed order.
//   decode_finish   grid B*Hkv, 512 threads.  Merges the chunks of each head
//                   (max, sum, O) in chunk order, writes O and the summed
//                   weights colsum[j] = sum_h 2^(x_hj - lse2_h), and when
//                   evicting adds them to the scores (one fp32 add each) and
//                   places the new token: the top-C rule of the chunk step
//                   with N_q = 1 keeps all but one candidate, the unprotected
//                   one last in (score desc, index asc) order -- the lowest
//                   score, the highest index among equal scores.
// Both are deterministic (fixed reduction orders, no atomics).
#include <cuda_bf16.h>

#include "attn.h"
#include "sm100.cuh"

namespace h2o {

namespace {

constexpr int kPartialThreads = 256;
constexpr int kFinishThreads = 512;
constexpr int kMaxChunks = (kMaxCandidates + kDecodeChunk - 1) / kDecodeChunk;

__device__ __forceinline__ void load8(const __nv_bfloat16* src, float (&f)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(src);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // element 2i is the low half of word i
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ void load8(const float* src, float (&f)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(src);
  const float4 b = *reinterpret_cast<const float4*>(src + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
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

// Copies one row of `bytes` bytes (a multiple of 16) with the lanes of a warp.
__device__ __forceinline__ void copy_row(void* dst, const void* src, int bytes, int lane) {
  for (int o = lane * 16; o < bytes; o += 32 * 16)
    *reinterpret_cast<uint4*>(static_cast<char*>(dst) + o) =
        *reinterpret_cast<const uint4*>(static_cast<const char*>(src) + o);
}

template <typename T, int D>
__global__ void __launch_bounds__(kPartialThreads) decode_partial(const DecodeParams p) {
  constexpr int U = D / 8;                         // 8-element pieces of a row
  constexpr int KG = kPartialThreads / U;          // key groups of the P V phase
  constexpr int KPG = kDecodeChunk / KG;           // keys per group
  extern __shared__ __align__(16) float dsm[];
  const int G = p.G;
  float* qs = dsm;                                 // [G][D]
  float* ps = qs + G * D;                          // [G][kDecodeChunk]
  float* ored = ps + G * kDecodeChunk;             // [KG][G][D]
  __shared__ float wred[kDecodeMaxG][kPartialThreads / 32];
  __shared__ float hstat[kDecodeMaxG][2];          // chunk max, chunk sum
  // the merge kernel may start; it waits for this grid before reading
  griddep_launch_dependents();

  const int bg = blockIdx.y;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int chunk = blockIdx.x;
  const int j0 = chunk * kDecodeChunk;
  const int nk = p.n + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const T* q = static_cast<const T*>(p.q) + (static_cast<size_t>(b) * p.Hkv * G + g * G) * D;
  for (int i = tid; i < G * D; i += kPartialThreads) qs[i] = to_float(q[i]);
  __syncthreads();

  // ---- thread = key: logits of the G heads
  const int j = j0 + tid;
  const bool valid = j < nk;
  float x[kDecodeMaxG];
#pragma unroll
  for (int h = 0; h < kDecodeMaxG; ++h) x[h] = 0.f;
  if (valid) {
    const T* krow = j < p.n
                        ? static_cast<const T*>(p.k_cache) + (static_cast<size_t>(bg) * p.C + j) * D
                        : static_cast<const T*>(p.k_new) + static_cast<size_t>(bg) * D;
#pragma unroll 4
    for (int d0 = 0; d0 < D; d0 += 8) {
      float kf[8];
      load8(krow + d0, kf);
#pragma unroll
      for (int h = 0; h < kDecodeMaxG; ++h) {
        if (h < G) {
          const float4 qa = *reinterpret_cast<const float4*>(qs + h * D + d0);
          const float4 qb = *reinterpret_cast<const float4*>(qs + h * D + d0 + 4);
          float a = x[h];
          a = fmaf(qa.x, kf[0], a);
          a = fmaf(qa.y, kf[1], a);
          a = fmaf(qa.z, kf[2], a);
          a = fmaf(qa.w, kf[3], a);
          a = fmaf(qb.x, kf[4], a);
          a = fmaf(qb.y, kf[5], a);
          a = fmaf(qb.z, kf[6], a);
          a = fmaf(qb.w, kf[7], a);
          x[h] = a;
        }
      }
    }
  }
  float* lg = p.logits + static_cast<size_t>(bg) * G * (p.C + 1);
#pragma unroll
  for (int h = 0; h < kDecodeMaxG; ++h) {
    if (h < G) {
      x[h] = valid ? x[h] * p.scale_log2 : -INFINITY;
      if (valid) lg[static_cast<size_t>(h) * (p.C + 1) + j] = x[h];
      const float m = warp_max(x[h]);
      if (lane == 0) wred[h][warp] = m;
    }
  }
  __syncthreads();
  if (tid < G) {
    float m = wred[tid][0];
    for (int w = 1; w < kPartialThreads / 32; ++w) m = fmaxf(m, wred[tid][w]);
    hstat[tid][0] = m;  // finite: every chunk holds at least one valid key
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < kDecodeMaxG; ++h) {
    if (h < G) {
      const float pw = valid ? ex2_approx(x[h] - hstat[h][0]) : 0.f;
      ps[h * kDecodeChunk + tid] = pw;
      const float s = warp_sum(pw);
      if (lane == 0) wred[h][warp] = s;
    }
  }
  __syncthreads();
  if (tid < G) {
    float s = 0.f;
    for (int w = 0; w < kPartialThreads / 32; ++w) s += wred[tid][w];
    hstat[tid][1] = s;
  }

  // ---- thread = (8 head-dim elements, key group): unnormalised P V
  const int u = tid % U, kg = tid / U;
  float o[kDecodeMaxG][8];
#pragma unroll
  for (int h = 0; h < kDecodeMaxG; ++h)
#pragma unroll
    for (int e = 0; e < 8; ++e) o[h][e] = 0.f;
  for (int jj = 0; jj < KPG; ++jj) {
    const int jl = kg * KPG + jj;
    const int jv = j0 + jl;
    if (jv >= nk) break;
    const T* vrow = jv < p.n
                        ? static_cast<const T*>(p.v_cache) + (static_cast<size_t>(bg) * p.C + jv) * D
                        : static_cast<const T*>(p.v_new) + static_cast<size_t>(bg) * D;
    float vf[8];
    load8(vrow + u * 8, vf);
#pragma unroll
    for (int h = 0; h < kDecodeMaxG; ++h) {
      if (h < G) {
        const float pw = ps[h * kDecodeChunk + jl];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[h][e] = fmaf(pw, vf[e], o[h][e]);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < kDecodeMaxG; ++h) {
    if (h < G) {
      float4* dst = reinterpret_cast<float4*>(ored + (static_cast<size_t>(kg) * G + h) * D + u * 8);
      dst[0] = make_float4(o[h][0], o[h][1], o[h][2], o[h][3]);
      dst[1] = make_float4(o[h][4], o[h][5], o[h][6], o[h][7]);
    }
  }
  __syncthreads();
  float* part = p.part + (static_cast<size_t>(bg) * p.part_ld + chunk) * G * (D + 2);
  for (int i = tid; i < G * D; i += kPartialThreads) {
    float s = 0.f;
    for (int k = 0; k < KG; ++k) s += ored[static_cast<size_t>(k) * G * D + i];
    part[(i / D) * (D + 2) + (i % D)] = s;
  }
  if (tid < G) {
    part[tid * (D + 2) + D] = hstat[tid][0];
    part[tid * (D + 2) + D + 1] = hstat[tid][1];
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kFinishThreads) decode_finish(const DecodeParams p) {
  __shared__ float fac[kDecodeMaxG][kMaxChunks];   // 2^(chunk max - head max)
  __shared__ float psum[kDecodeMaxG][kMaxChunks];  // chunk sums
  __shared__ float mh[kDecodeMaxG], lh[kDecodeMaxG], lse[kDecodeMaxG];
  __shared__ unsigned long long wmin[kFinishThreads / 32];
  const int G = p.G;
  const int bg = blockIdx.x;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NCk = p.n_chunks;
  const int C = p.C, n = p.n;
  griddep_wait();  // the partials come from the preceding kernel
  const float* part = p.part + static_cast<size_t>(bg) * p.part_ld * G * (D + 2);
  auto pidx = [&](int c, int h) { return (static_cast<size_t>(c) * G + h) * (D + 2); };

  // ---- merge the chunks: chunk maxima and sums into shared memory, then
  // one warp per head reduces them (fixed tree order)
  for (int i = tid; i < NCk * G; i += kFinishThreads) {
    const int c = i / G, h = i % G;
    fac[h][c] = part[pidx(c, h) + D];       // chunk max, turned into the factor below
    psum[h][c] = part[pidx(c, h) + D + 1];  // chunk sum
  }
  __syncthreads();
  if (warp < G) {
    float m = -INFINITY;
    for (int c = lane; c < NCk; c += 32) m = fmaxf(m, fac[warp][c]);
    m = warp_max(m);
    float l = 0.f;
    for (int c = lane; c < NCk; c += 32) {
      const float f = ex2_approx(fac[warp][c] - m);
      fac[warp][c] = f;
      l = fmaf(psum[warp][c], f, l);
    }
    l = warp_sum(l);
    if (lane == 0) {
      mh[warp] = m;
      lh[warp] = l;
      lse[warp] = m + __log2f(l);
    }
  }
  __syncthreads();
  T* out = static_cast<T*>(p.out) + (static_cast<size_t>(b) * p.Hkv * G + g * G) * D;
  for (int i = tid; i < G * D; i += kFinishThreads) {
    const int h = i / D, d = i % D;
    float acc = 0.f;
#pragma unroll 8
    for (int c = 0; c < NCk; ++c) acc = fmaf(part[pidx(c, h) + d], fac[h][c], acc);
    store(out + i, acc / lh[h]);
  }

  // ---- summed weights: slots, zeros up to C, the new key at C
  const float* lg = p.logits + static_cast<size_t>(bg) * G * (C + 1);
  float* cs = p.colsum + static_cast<size_t>(bg) * p.colsum_ld;
#pragma unroll 4
  for (int j = tid; j <= n; j += kFinishThreads) {
    float s = 0.f;
    for (int h = 0; h < G; ++h) s += ex2_approx(lg[static_cast<size_t>(h) * (C + 1) + j] - lse[h]);
    cs[j < n ? j : C] = s;
  }
  for (int j = n + tid; j < C; j += kFinishThreads) cs[j] = 0.f;
  if (!p.evict) return;

  // ---- eviction of one candidate
  __syncthreads();  // the row of summed weights is complete
  float* score = p.scores + static_cast<size_t>(bg) * C;
  int* pos = p.pos + static_cast<size_t>(bg) * C;
  const float cnew = cs[C];
  const size_t row_bytes = static_cast<size_t>(D) * sizeof(T);
  char* kc = static_cast<char*>(p.k_cache) + static_cast<size_t>(bg) * C * row_bytes;
  char* vc = static_cast<char*>(p.v_cache) + static_cast<size_t>(bg) * C * row_bytes;
  const char* kn = static_cast<const char*>(p.k_new) + static_cast<size_t>(bg) * row_bytes;
  const char* vn = static_cast<const char*>(p.v_new) + static_cast<size_t>(bg) * row_bytes;
  if (bg == 0 && tid == 0) {
    p.state[0] = min(C, n + 1);
    p.state[1] = p.t0 + 1;
  }
  const bool by_score = p.policy == kPolicyH2O;
  const int sinks = p.policy == kPolicySLR ? p.sinks : 0;
  const float snew = by_score ? cnew : 0.f;  // the score-free policies keep none
  if (n < C) {  // room left: the new token takes slot n
    if (by_score)
      for (int s = tid; s < n; s += kFinishThreads) score[s] = __fadd_rn(score[s], cs[s]);
    if (tid == 0) {
      score[n] = snew;
      pos[n] = p.t0;
    }
    if (warp == 0) {
      copy_row(kc + n * row_bytes, kn, static_cast<int>(row_bytes), lane);
      copy_row(vc + n * row_bytes, vn, static_cast<int>(row_bytes), lane);
    }
    return;
  }
  // full: candidates with position < t0 + 1 - W (and, under SLR, >= the sink
  // count) are unprotected; the one with the lowest rank value (then the
  // highest index: slot s -> s, new token -> C) leaves.  The rank value is the
  // score (>= 0, so its bit pattern orders like the value) or, for the
  // score-free policies, the position.
  const long long limit = static_cast<long long>(p.t0) + 1 - p.W;
  unsigned long long best = ~0ull;
  for (int s = tid; s < C; s += kFinishThreads) {
    const int ps = pos[s];
    uint32_t rank;
    if (by_score) {
      const float sc = __fadd_rn(score[s], cs[s]);
      score[s] = sc;
      rank = __float_as_uint(sc);
    } else {
      rank = static_cast<uint32_t>(ps);
    }
    if (ps < limit && ps >= sinks) {
      const unsigned long long key = (static_cast<unsigned long long>(rank) << 32) | (0xffffffffu - s);
      best = key < best ? key : best;
    }
  }
  if (tid == 0 && p.t0 < limit && p.t0 >= sinks) {  // W = 0: the new token competes too
    const uint32_t rank = by_score ? __float_as_uint(cnew) : static_cast<uint32_t>(p.t0);
    const unsigned long long key = (static_cast<unsigned long long>(rank) << 32) | (0xffffffffu - C);
    best = key < best ? key : best;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
    best = other < best ? other : best;
  }
  if (lane == 0) wmin[warp] = best;
  __syncthreads();
  if (warp == 0) {
    best = lane < kFinishThreads / 32 ? wmin[lane] : ~0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
      best = other < best ? other : best;
    }
    if (best == ~0ull) {  // cannot happen: W <= C leaves an unprotected candidate
      if (lane == 0) atomicOr(&p.state[2], kDevErrPlan);
      return;
    }
    const int e = static_cast<int>(0xffffffffu - static_cast<uint32_t>(best & 0xffffffffu));
    if (e < C) {  // an old slot leaves; the new token takes it
      if (lane == 0) {
        score[e] = snew;
        pos[e] = p.t0;
      }
      copy_row(kc + static_cast<size_t>(e) * row_bytes, kn, static_cast<int>(row_bytes), lane);
      copy_row(vc + static_cast<size_t>(e) * row_bytes, vn, static_cast<int>(row_bytes), lane);
    }
  }
}

template <typename T, int D>
cudaError_t launch(const DecodeParams& p, cudaStream_t st) {
  constexpr int U = D / 8, KG = kPartialThreads / U;
  const size_t smem = static_cast<size_t>(p.G) * (D + kDecodeChunk + KG * D) * sizeof(float);
  static int attr_bits[2] = {0, 0};
  if (!smem_attr_done(reinterpret_cast<const void*>(decode_partial<T, D>), attr_bits)) {
    const int most = kDecodeMaxG * (D + kDecodeChunk + KG * D) * static_cast<int>(sizeof(float));
    cudaError_t e = cudaFuncSetAttribute(decode_partial<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e != cudaSuccess) return e;
  }
  decode_partial<T, D><<<dim3(p.n_chunks, p.B * p.Hkv), kPartialThreads, smem, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.B * p.Hkv);
  cfg.blockDim = dim3(kFinishThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_finish<T, D>, p);
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, int esize, int head_dim, cudaStream_t st) {
  if (p.n_chunks > kMaxChunks || p.G > kDecodeMaxG) return cudaErrorInvalidValue;
  if (esize == 2)
    return head_dim == 128 ? launch<__nv_bfloat16, 128>(p, st) : launch<__nv_bfloat16, 64>(p, st);
  return head_dim == 128 ? launch<float, 128>(p, st) : launch<float, 64>(p, st);
}

}  // namespace h2o
