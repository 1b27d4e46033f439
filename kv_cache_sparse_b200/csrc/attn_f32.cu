// attn_f32.cu -- the attention step for float32 inputs, in fp32 FMA arithmetic.
//
// Same operation as the bf16 tensor-core kernels ("Learning how to Forget",
// §1: SDPA over cache ++ chunk that also returns summed attention weights),
// for float inputs: tf32 tensor cores would round the inputs to 10 mantissa
// bits, which costs more accuracy than the summed-weight tolerance allows on
// keys seen by few queries, so this path keeps every product in fp32.  It is
// meant for small configurations.
//
//   attn_f32_rows:   one CTA per (cache, head, query): logits against every
//                    visible key, max / sum, O = P V / l, and lse2.
//   attn_f32_colsum: one CTA per (cache, KV head, key): the probabilities of
//                    that key over the G heads and the queries that see it,
//                    rebuilt from lse2 and summed in a fixed tree order.
#include "attn.h"
#include "sm100.cuh"

namespace h2o {

constexpr int kF32Threads = 128;

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < kF32Threads / 32; ++i) r = fmaxf(r, red[i]);
  return r;
}

__device__ __forceinline__ float block_reduce_sum(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < kF32Threads / 32; ++i) r += red[i];
  return r;
}

// key j of the visible list of query i: cache slot j (j < n) or chunk key j - n
__device__ __forceinline__ const float* key_row(const float* kc, const float* kn, int j, int n,
                                                const AttnParams& p, int b, int g, int d) {
  return j < n ? kc + ((static_cast<size_t>(b) * p.Hkv + g) * p.C + j) * d
               : kn + ((static_cast<size_t>(b) * p.nq + (j - n)) * p.Hkv + g) * d;
}

__global__ void __launch_bounds__(kF32Threads)
    attn_f32_rows(const float* __restrict__ q, const float* __restrict__ kc,
                  const float* __restrict__ vc, const float* __restrict__ kn,
                  const float* __restrict__ vn, const AttnParams p, int d) {
  __shared__ float qs[256];
  __shared__ float ps[kF32Threads];
  __shared__ float red[kF32Threads / 32];
  const int i = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / p.Hq, h = bh % p.Hq, g = h / p.G;
  const float* qrow = q + ((static_cast<size_t>(b) * p.nq + i) * p.Hq + h) * d;
  for (int t = threadIdx.x; t < d; t += blockDim.x) qs[t] = qrow[t];
  __syncthreads();
  const int nk = p.n + i + 1;  // visible keys
  const float c = p.scale_log2;
  // pass 1: running max / sum per thread, then across the block
  float m = -INFINITY, l = 0.f;
  for (int j = threadIdx.x; j < nk; j += blockDim.x) {
    const float* kr = key_row(kc, kn, j, p.n, p, b, g, d);
    float s = 0.f;
    for (int t = 0; t < d; ++t) s = fmaf(qs[t], kr[t], s);
    const float x = s * c;
    const float mn = fmaxf(m, x);
    l = l * exp2f(m - mn) + exp2f(x - mn);
    m = mn;
  }
  const float M = block_reduce_max(m, red);
  const float Lsum = block_reduce_sum(m == -INFINITY ? 0.f : l * exp2f(m - M), red);
  const float lse2 = M + log2f(Lsum);
  // pass 2: O = sum_j 2^(x_j - lse2) V_j, 128 keys at a time
  float o0 = 0.f, o1 = 0.f;  // elements threadIdx.x and threadIdx.x + 128 (d <= 256)
  for (int j0 = 0; j0 < nk; j0 += blockDim.x) {
    const int j = j0 + threadIdx.x;
    float pr = 0.f;
    if (j < nk) {
      const float* kr = key_row(kc, kn, j, p.n, p, b, g, d);
      float s = 0.f;
      for (int t = 0; t < d; ++t) s = fmaf(qs[t], kr[t], s);
      pr = exp2f(s * c - lse2);
    }
    __syncthreads();
    ps[threadIdx.x] = pr;
    __syncthreads();
    const int cnt = min(static_cast<int>(blockDim.x), nk - j0);
    for (int jj = 0; jj < cnt; ++jj) {
      const float* vr = key_row(vc, vn, j0 + jj, p.n, p, b, g, d);
      if (threadIdx.x < d) o0 = fmaf(ps[jj], vr[threadIdx.x], o0);
      if (threadIdx.x + 128 < d) o1 = fmaf(ps[jj], vr[threadIdx.x + 128], o1);
    }
  }
  float* orow = reinterpret_cast<float*>(p.out) + ((static_cast<size_t>(b) * p.nq + i) * p.Hq + h) * d;
  if (threadIdx.x < d) orow[threadIdx.x] = o0;
  if (threadIdx.x + 128 < d) orow[threadIdx.x + 128] = o1;
  if (threadIdx.x == 0) p.nlse2[(static_cast<size_t>(b) * p.Hq + h) * p.nq_pad + i] = -lse2;
}

__global__ void __launch_bounds__(kF32Threads)
    attn_f32_colsum(const float* __restrict__ q, const float* __restrict__ kc,
                    const float* __restrict__ kn, const AttnParams p, int d) {
  __shared__ float ks[256];
  __shared__ float red[kF32Threads / 32];
  const int key = blockIdx.x;  // 0..n-1 cache slots, n..n+nq-1 chunk keys
  const int bg = blockIdx.y;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const float* kr = key_row(kc, kn, key, p.n, p, b, g, d);
  for (int t = threadIdx.x; t < d; t += blockDim.x) ks[t] = kr[t];
  __syncthreads();
  const int i_min = key < p.n ? 0 : key - p.n;  // queries that see this key
  const int rows = p.G * (p.nq - i_min);
  const float c = p.scale_log2;
  float acc = 0.f;
  for (int r = threadIdx.x; r < rows; r += blockDim.x) {
    const int h = g * p.G + r / (p.nq - i_min);
    const int i = i_min + r % (p.nq - i_min);
    const float* qr = q + ((static_cast<size_t>(b) * p.nq + i) * p.Hq + h) * d;
    float s = 0.f;
    for (int t = 0; t < d; ++t) s = fmaf(qr[t], ks[t], s);
    acc += exp2f(s * c + p.nlse2[(static_cast<size_t>(b) * p.Hq + h) * p.nq_pad + i]);
  }
  const float total = block_reduce_sum(acc, red);
  if (threadIdx.x == 0) {
    float* out = p.colsum + static_cast<size_t>(bg) * p.colsum_ld;
    out[key < p.n ? key : p.C + (key - p.n)] = total;
  }
}

__global__ void zero_empty_slots(const AttnParams p) {
  float* out = p.colsum + static_cast<size_t>(blockIdx.x) * p.colsum_ld;
  for (int j = p.n + threadIdx.x; j < p.C; j += blockDim.x) out[j] = 0.f;
}

cudaError_t launch_attn_f32(int head_dim, const float* q, const float* kc, const float* vc,
                            const float* kn, const float* vn, const AttnParams& p,
                            cudaStream_t st) {
  attn_f32_rows<<<dim3(p.nq, p.B * p.Hq), kF32Threads, 0, st>>>(q, kc, vc, kn, vn, p, head_dim);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_f32_colsum<<<dim3(p.n + p.nq, p.B * p.Hkv), kF32Threads, 0, st>>>(q, kc, kn, p, head_dim);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (p.n < p.C) {
    zero_empty_slots<<<p.B * p.Hkv, 256, 0, st>>>(p);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace h2o
