// q8.cuh -- the int8 cache format of the Q-Hitter variant ("Learning how to
// Forget", page 1 §2 Related Work: Q-Hitter combines H2O with quantisation;
// summary page, Table 5, qh2o rows).  The pages give no format; the one used
// here: each cache row (one slot of one KV head, K and V separately) holds d
// int8 codes and one fp32 scale, symmetric,
//   s = fl32(max_i |x_i| / 127),  code_i = clamp(rint(fl32(x_i / s)), -127, 127)
// (ties to even; an all-zero row has s = 0 and zero codes), and the attention
// reads bf16(fl32(code_i * s)) (round to nearest even).  A token is quantised
// when it is placed into the cache.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace h2o {

// The value the attention reads for one code.
__device__ __forceinline__ float q8_value(int code, float s) {
  return __bfloat162float(__float2bfloat16_rn(__fmul_rn(static_cast<float>(code), s)));
}

// Quantises one row of D bf16 values with a warp: lane l holds elements
// [l * D/32, (l+1) * D/32).  Writes the D codes (lane l its D/32 bytes) and,
// from lane 0, the scale.
template <int D>
__device__ __forceinline__ void q8_quantize_row_warp(const __nv_bfloat16* src, int8_t* dst,
                                                     float* scale, int lane) {
  constexpr int E = D / 32;
  float x[E];
#pragma unroll
  for (int e = 0; e < E; ++e) x[e] = __bfloat162float(src[lane * E + e]);
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = __fdiv_rn(amax, 127.0f);
  uint32_t packed[(E + 3) / 4] = {};
#pragma unroll
  for (int e = 0; e < E; ++e) {
    int c = 0;
    if (s > 0.f) c = max(-127, min(127, __float2int_rn(__fdiv_rn(x[e], s))));
    packed[e / 4] |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * (e % 4));
  }
  if (E == 4) {
    *reinterpret_cast<uint32_t*>(dst + lane * E) = packed[0];
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) dst[lane * E + e] = static_cast<int8_t>((packed[e / 4] >> (8 * (e % 4))) & 0xFF);
  }
  if (lane == 0) *scale = s;
}

// 16 codes (one 16-byte chunk) times the row scale -> 16 bf16 values packed in
// 8 words, ready for a 128-byte-swizzled MMA operand.  The codes go through
// fp32 exactly: 2^23 + (code + 128) built by byte permutes, minus 2^23 + 128.
__device__ __forceinline__ void q8_dequant16(uint4 codes, float s, uint32_t (&out)[8]) {
  const uint32_t w[4] = {codes.x ^ 0x80808080u, codes.y ^ 0x80808080u, codes.z ^ 0x80808080u,
                         codes.w ^ 0x80808080u};  // offset binary: code + 128
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float f[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // 0x4B0000uu: 2^23 + u
      const uint32_t bits = __byte_perm(w[i], 0x4B000000u, 0x7650 + j);
      f[j] = __fmul_rn(__uint_as_float(bits) - 8388736.0f, s);
    }
    out[2 * i] = (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f[1]))) << 16) |
                 __bfloat16_as_ushort(__float2bfloat16_rn(f[0]));
    out[2 * i + 1] = (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f[3]))) << 16) |
                     __bfloat16_as_ushort(__float2bfloat16_rn(f[2]));
  }
}

}  // namespace h2o
