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

// (a0, a1) - (b0, b1) and (a0, a1) * (b0, b1), packed f32x2, round to nearest.
__device__ __forceinline__ void q8_sub2(float& d0, float& d1, float a0, float a1, float b) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b));
}

__device__ __forceinline__ void q8_mul2(float& d0, float& d1, float a0, float a1, float b) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b));
}

// 16 codes (one 16-byte chunk) times the row scale -> 16 bf16 values packed in
// 8 words (element 2k in the low half of word k), ready for an MMA operand.
// A code c goes through fp32 exactly: the bytes c + 128 are placed under the
// exponent of 2^23 by byte permutes (2^23 + c + 128) and 2^23 + 128 is
// subtracted; then one rounding for c * s (fp32) and one for bf16.
__device__ __forceinline__ void q8_dequant16(uint4 codes, float s, uint32_t (&out)[8]) {
  const uint32_t w[4] = {codes.x ^ 0x80808080u, codes.y ^ 0x80808080u, codes.z ^ 0x80808080u,
                         codes.w ^ 0x80808080u};  // offset binary: code + 128
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float f[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) f[j] = __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7650 + j));
    q8_sub2(f[0], f[1], f[0], f[1], 8388736.0f);  // 2^23 + 128
    q8_sub2(f[2], f[3], f[2], f[3], 8388736.0f);
    q8_mul2(f[0], f[1], f[0], f[1], s);
    q8_mul2(f[2], f[3], f[2], f[3], s);
    uint32_t lo, hi;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(lo) : "f"(f[1]), "f"(f[0]));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(hi) : "f"(f[3]), "f"(f[2]));
    out[2 * i] = lo;
    out[2 * i + 1] = hi;
  }
}

}  // namespace h2o
