// attn_bwd.cu -- backward of the chunk step's attention on sm_100a tensor
// cores: dQ, dK and dV for the cache slots and the chunk's keys, with the
// eviction decision held fixed ("Learning how to Forget", §1: fine-tuning
// through the KV cache with the policy in place; summary page, Tables 1 and
// 6: training with each cache policy).
//
// With P = softmax(scale Q K^T) over the visible keys (the forward's row
// statistic lse2 rebuilds it: P = 2^(x - lse2), x = scale*log2(e)*<q, k>),
//   dV = P^T dO,  dP = dO V^T,  dS = P (dP - D) with D_i = <dO_i, O_i>,
//   dQ = scale dS K,  dK = scale dS^T Q,
// dK and dV summed over the G query heads of a KV head.  Three kernels:
//   bwd_rowdot   -scale * D_i for every (cache, head, query): one warp per
//                row (0 for the padding rows up to the next multiple of 128).
//   bwd_dkdv     key-stationary, like the column-sum kernel: one CTA per
//                (cache, KV head, 128 keys), looping over the (head, query
//                tile) units that see its keys.  The MMAs compute
//                S^T = K Q^T and dP^T = V dO^T with the keys on the TMEM
//                lanes; one thread per key turns its rows into P^T and
//                scale*dS^T (bf16, written back over the first columns of S^T
//                and dP^T), and the MMAs accumulate dV += P^T dO and
//                dK += dS^T Q in TMEM (A operand from TMEM, B the dO / Q tile
//                as an MN-major operand).
//   bwd_dq       query-stationary, like the forward: one CTA per (cache,
//                head, 128 queries), looping over the key tiles it sees:
//                S = Q K^T, dP = dO V^T, one thread per query row forms
//                scale*dS (bf16, over S), and dQ += dS K accumulates in TMEM.
// Every reduction has a fixed order (no atomics): the results are
// deterministic.  Roles in the two tensor-core kernels: warp 0 TMA producer,
// warp 1 TMEM allocation and the MMA-issuing thread, warps 2..9 the rows in
// two warpgroups, one per half of the 128 columns of S (queries in bwd_dkdv,
// keys in bwd_dq).  Each half has its own ready barriers, so the tensor core
// accumulates one half and computes the next unit's first half while the
// other warpgroup still works on the second.
#include <cuda_bf16.h>

#include "attn.h"
#include "sm100.cuh"

namespace h2o {

// ---------------------------------------------------------------- D_i

__global__ void bwd_rowdot(const __nv_bfloat16* __restrict__ out,
                           const __nv_bfloat16* __restrict__ dout, const BwdParams p, int d) {
  // one warp per row (b, h, i) of the padded statistic; i >= nq gets 0
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int rows = p.B * p.Hq * p.nq_pad;
  if (row >= rows) return;
  const int i = row % p.nq_pad;
  const int h = (row / p.nq_pad) % p.Hq;
  const int b = row / (p.nq_pad * p.Hq);
  float s = 0.f;
  if (i < p.nq) {
    const size_t at = ((static_cast<size_t>(b) * p.nq + i) * p.Hq + h) * d;
    for (int e = lane; e < d; e += 32) s = fmaf(__bfloat162float(out[at + e]), __bfloat162float(dout[at + e]), s);
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o2);
  }
  // stored as -scale * D_i, the term the row arithmetic adds to scale * dP
  if (lane == 0) p.dsum[row] = -p.scale * s;
}

// ---------------------------------------------------------------- dK, dV

template <int D>
struct DkdvLayout {
  static constexpr int kRegions = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kStages = 2;  // units in flight (Q, dO, lse2, D)
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kKOff + kTileBytes;
  static constexpr int kQOff = kVOff + kTileBytes;                  // [stage]
  static constexpr int kDOOff = kQOff + kStages * kTileBytes;       // [stage]
  static constexpr int kRowOff = kDOOff + kStages * kTileBytes;     // [stage][2][128] float
  static constexpr int kBarOff = kRowOff + kStages * 1024;
  // kv_full, u_full[S], u_empty[S], s_full[2], p_full[2], o_done, drain
  static constexpr int kNumBars = 1 + 2 * kStages + 6;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

// Both tensor-core kernels: warp 0 TMA, warp 1 TMEM + MMA, then two
// warpgroups of row threads, one per half of the 128 columns of S.
// Row warps per TMEM lane quadrant and half of a unit: 1 (a warp takes the
// half's 64 columns) or 2 (32 columns each, so that one warp's TMEM loads
// and exponentials overlap the other's).  Measured on the C 8192 cache: the
// row work of a half drops from ~1650 to ~1270 cycles with 2, but the MMA
// thread, sharing its SM sub-partition with twice the row warps, notices
// the ready rows ~750 cycles late instead of ~300 (spinning or not), and the
// backward takes 609-611 us against 595-597 with 1.
constexpr int kRowSplit = 1;
constexpr int kBwdThreads = 64 + 2 * 128 * kRowSplit;

// TMEM column of the bf16 pairs of 16 columns ks (0..3) of half hf: each row
// warp writes the pairs of its own columns over the first of them.
__device__ __forceinline__ uint32_t pair_col(int hf, int ks) {
  return kRowSplit == 2 ? 64 * hf + 32 * (ks >> 1) + 8 * (ks & 1) : 64 * hf + 8 * ks;
}

// Row arithmetic shared by the two kernels: from 32 logits s and 32 dP
// values of one row (or one key), the bf16 pairs of P and of scale * dS =
// P (scale dP - scale D).  Column c's statistics: -lse2 in nls and -scale*D
// in nds, either per column (kCol: 32 floats each in shared memory, read 16
// bytes at a time) or one value for the whole row (nls[0], nds[0]).  Pairs
// of columns go through packed f32x2 arithmetic.
template <int NV, bool kMask, bool kCol>
__device__ __forceinline__ void p_ds(const uint32_t (&s)[NV], const uint32_t (&dp)[NV],
                                     const float* nls, const float* nds, float c, float scale,
                                     int first_valid, int last_valid, uint32_t (&pp)[NV / 2],
                                     uint32_t (&dd)[NV / 2]) {
#pragma unroll
  for (int k = 0; k < NV; k += 4) {
    float4 nl, nd;
    if (kCol) {
      nl = *reinterpret_cast<const float4*>(nls + k);
      nd = *reinterpret_cast<const float4*>(nds + k);
    } else {
      nl = make_float4(nls[0], nls[0], nls[0], nls[0]);
      nd = make_float4(nds[0], nds[0], nds[0], nds[0]);
    }
    float x0, x1, x2, x3;
    ffma2(x0, x1, __uint_as_float(s[k]), __uint_as_float(s[k + 1]), c, c, nl.x, nl.y);
    ffma2(x2, x3, __uint_as_float(s[k + 2]), __uint_as_float(s[k + 3]), c, c, nl.z, nl.w);
    float p0 = ex2_approx(x0), p1 = ex2_approx(x1), p2 = ex2_approx(x2), p3 = ex2_approx(x3);
    if (kMask) {
      p0 = (k >= first_valid && k <= last_valid) ? p0 : 0.f;
      p1 = (k + 1 >= first_valid && k + 1 <= last_valid) ? p1 : 0.f;
      p2 = (k + 2 >= first_valid && k + 2 <= last_valid) ? p2 : 0.f;
      p3 = (k + 3 >= first_valid && k + 3 <= last_valid) ? p3 : 0.f;
    }
    // every term is finite (padding rows have P = 0 and -scale*D = 0), so a
    // zero P gives a zero dS
    float t0, t1, t2, t3, d0, d1, d2, d3;
    ffma2(t0, t1, __uint_as_float(dp[k]), __uint_as_float(dp[k + 1]), scale, scale, nd.x, nd.y);
    ffma2(t2, t3, __uint_as_float(dp[k + 2]), __uint_as_float(dp[k + 3]), scale, scale, nd.z, nd.w);
    fmul2(d0, d1, p0, p1, t0, t1);
    fmul2(d2, d3, p2, p3, t2, t3);
    pp[k >> 1] = pack_bf16x2(p0, p1);
    pp[(k >> 1) + 1] = pack_bf16x2(p2, p3);
    dd[k >> 1] = pack_bf16x2(d0, d1);
    dd[(k >> 1) + 1] = pack_bf16x2(d2, d3);
  }
}

// The row work of NSUB x 16 columns of a unit's S and dP in TMEM (S at
// s_col, dP at s_col + 128, the block's columns starting at c0): sub-blocks
// of 16 columns whose TMEM loads are issued one ahead of the arithmetic; the
// bf16 pairs of sub-block k go over columns [c0 + 8k, +8) of S (P) and of dP
// (scale dS) -- or, kDsOverS, scale dS over S and P nowhere -- which hold
// values this thread has already read.  Column statistics at nls / nds (per
// column, kCol) or the row's own (nls[0], nds[0]); masking as in p_ds, the
// bounds relative to column c0.
template <bool kCol, bool kDsOverS, int NSUB>
__device__ __forceinline__ void rows_block(uint32_t s_col, int c0, const float* nls,
                                           const float* nds, float c, float scale, bool masked,
                                           int first_valid, int last_valid) {
  uint32_t sv[2][16], dp[2][16];
  tmem_ld16(s_col + c0, sv[0]);
  tmem_ld16(s_col + 128 + c0, dp[0]);
  tmem_wait_ld();
#pragma unroll
  for (int k = 0; k < NSUB; ++k) {
    const int cur = k & 1;
    if (k + 1 < NSUB) {
      tmem_ld16(s_col + c0 + 16 * (k + 1), sv[cur ^ 1]);
      tmem_ld16(s_col + 128 + c0 + 16 * (k + 1), dp[cur ^ 1]);
    }
    uint32_t pp[8], dd[8];
    const float* nl = kCol ? nls + 16 * k : nls;
    const float* nd = kCol ? nds + 16 * k : nds;
    if (masked)
      p_ds<16, true, kCol>(sv[cur], dp[cur], nl, nd, c, scale, first_valid - 16 * k,
                           last_valid - 16 * k, pp, dd);
    else
      p_ds<16, false, kCol>(sv[cur], dp[cur], nl, nd, c, scale, 0, 0, pp, dd);
    if (kDsOverS) {
      tmem_st8(s_col + c0 + 8 * k, dd);
    } else {
      tmem_st8(s_col + c0 + 8 * k, pp);
      tmem_st8(s_col + 128 + c0 + 8 * k, dd);
    }
    if (k + 1 < NSUB) tmem_wait_ld();
  }
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
             const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc,
             const __grid_constant__ CUtensorMap tm_kn, const __grid_constant__ CUtensorMap tm_vn,
             const BwdParams p) {
  using L = DkdvLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bg = blockIdx.y;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int NCTC = cdiv(p.C, 128);
  const int NQT = cdiv(p.nq, 128);
  const bool is_chunk = static_cast<int>(blockIdx.x) >= NCTC;
  const int kt = is_chunk ? blockIdx.x - NCTC : blockIdx.x;
  const int j0 = kt * 128;
  const size_t row_stride = static_cast<size_t>(D);
  if (!is_chunk && j0 >= p.n) {
    // slots past the valid ones have no gradient
    for (int r = threadIdx.x; r < min(128, p.C - j0) * D; r += blockDim.x) {
      const size_t at = (static_cast<size_t>(bg) * p.C + j0) * row_stride + r;
      p.dk_cache[at] = 0.f;
      p.dv_cache[at] = 0.f;
    }
    griddep_wait();  // see the end of the kernel
    return;
  }
  const int qt_min = is_chunk ? kt : 0;
  const int span = NQT - qt_min;
  const int R = p.G * span;

  const uint32_t bar_kv = sbase + L::kBarOff;
  const uint32_t bar_full0 = bar_kv + 8;
  const uint32_t bar_empty0 = bar_full0 + 8 * L::kStages;
  const uint32_t bar_s0 = bar_empty0 + 8 * L::kStages;  // [half]
  const uint32_t bar_p0 = bar_s0 + 16;                  // [half]
  const uint32_t bar_o = bar_p0 + 16;
  const uint32_t bar_drain = bar_o + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar_full0 + 8 * s, 1);
      mbar_init(bar_empty0 + 8 * s, 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(bar_s0 + 8 * h, 1);
      mbar_init(bar_p0 + 8 * h, 128 * kRowSplit);
    }
    mbar_init(bar_o, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S^T [0,128), dP^T [128,256), dV [256, 256+D), dK [384, 384+D).
  // Half hf of a unit is its queries [64 hf, +64): S^T columns [64 hf, +64),
  // dP^T columns [128 + 64 hf, +64); its P^T and scale*dS^T (bf16 pairs) go
  // over the first 32 of those columns.

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_kv, 2 * L::kTileBytes);
      for (int r = 0; r < L::kRegions; ++r) {
        if (is_chunk) {
          tma_load_4d(sbase + L::kKOff + r * 16384, &tm_kn, bar_kv, r * 64, g, j0, b);
          tma_load_4d(sbase + L::kVOff + r * 16384, &tm_vn, bar_kv, r * 64, g, j0, b);
        } else {
          tma_load_3d(sbase + L::kKOff + r * 16384, &tm_kc, bar_kv, r * 64, j0, bg);
          tma_load_3d(sbase + L::kVOff + r * 16384, &tm_vc, bar_kv, r * 64, j0, bg);
        }
      }
      int issued = 0;
      for (int u = 0; u < R; ++u) {
        const int h = g * p.G + u / span;
        const int qt = qt_min + u % span;
        const int s = u % L::kStages;
        if (u >= L::kStages &&
            !mbar_wait(bar_empty0 + 8 * s, ((u / L::kStages) + 1) & 1, p.err, abort_flag))
          break;
        const uint32_t full = bar_full0 + 8 * s;
        mbar_arrive_expect_tx(full, 2 * L::kTileBytes + 1024);
        for (int r = 0; r < L::kRegions; ++r) {
          tma_load_4d(sbase + L::kQOff + s * L::kTileBytes + r * 16384, &tm_q, full, r * 64, h,
                      qt * 128, b);
          tma_load_4d(sbase + L::kDOOff + s * L::kTileBytes + r * 16384, &tm_do, full, r * 64, h,
                      qt * 128, b);
        }
        const size_t roff = (static_cast<size_t>(b) * p.Hq + h) * p.nq_pad + qt * 128;
        bulk_load(sbase + L::kRowOff + s * 1024, p.nlse2 + roff, 512, full);
        bulk_load(sbase + L::kRowOff + s * 1024 + 512, p.dsum + roff, 512, full);
        issued = u + 1;
      }
      mbar_wait_drain(bar_kv, 0, p.err);
      for (int u = (issued > L::kStages ? issued - L::kStages : 0); u < issued; ++u)
        mbar_wait_drain(bar_full0 + 8 * (u % L::kStages), (u / L::kStages) & 1, p.err);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, D, false, true);
      // S^T and dP^T of one half of unit u (stage s): contraction over the
      // head dim, the half's 64 query rows of the Q / dO tiles as B
      auto issue_s = [&](int s, int hf) {
        const uint32_t qb = sbase + L::kQOff + s * L::kTileBytes + hf * 8192;
        const uint32_t db = sbase + L::kDOOff + s * L::kTileBytes + hf * 8192;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_bf16_ss(tmem + 64 * hf, sw128_desc(sbase + L::kKOff + off, 16, 1024),
                      sw128_desc(qb + off, 16, 1024), kIdescS, ks > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_bf16_ss(tmem + 128 + 64 * hf, sw128_desc(sbase + L::kVOff + off, 16, 1024),
                      sw128_desc(db + off, 16, 1024), kIdescS, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar_s0 + 8 * hf);
      };
      // dV += P^T dO and dK += (scale dS)^T Q over the half's 64 queries (16
      // per MMA = 8 TMEM columns of bf16 pairs; B the dO / Q rows MN-major)
      auto issue_acc = [&](int s, int hf, bool first) {
        const uint32_t qb = sbase + L::kQOff + s * L::kTileBytes;
        const uint32_t db = sbase + L::kDOOff + s * L::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          mma_bf16_ts(tmem + 256, tmem + pair_col(hf, ks),
                      sw128_desc(db + (4 * hf + ks) * 2048, 16384, 1024), kIdescAcc,
                      (first && ks == 0) ? 0u : 1u);
        }
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          mma_bf16_ts(tmem + 384, tmem + 128 + pair_col(hf, ks),
                      sw128_desc(qb + (4 * hf + ks) * 2048, 16384, 1024), kIdescAcc,
                      (first && ks == 0) ? 0u : 1u);
        }
      };
      bool ok = mbar_wait(bar_kv, 0, p.err, abort_flag);
      if (ok && R > 0) ok = mbar_wait(bar_full0, 0, p.err, abort_flag);
      if (ok && R > 0) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(0, 1);
      }
      // per unit: the accumulation of half 0 and the next unit's half-0 S^T
      // run on the tensor core while the row threads work on half 1
      for (int u = 0; u < R && ok; ++u) {
        const int s = u % L::kStages;
        const bool more = u + 1 < R;
        const int s1 = (u + 1) % L::kStages;
        ok = mbar_wait(bar_p0, u & 1, p.err, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_acc(s, 0, u == 0);
        if (more) {
          ok = mbar_wait(bar_full0 + 8 * s1, ((u + 1) / L::kStages) & 1, p.err, abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_s(s1, 0);
        }
        ok = mbar_wait(bar_p0 + 8, u & 1, p.err, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_acc(s, 1, false);
        mma_commit(bar_empty0 + 8 * s);
        if (more) issue_s(s1, 1);
      }
      mma_commit(bar_o);
      mma_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0, p.err);
    }
  } else {
    const int rw = warp - 2;
    const int hf = rw / (4 * kRowSplit);       // half of the unit's queries
    const int sub = (rw >> 2) % kRowSplit;     // kRowSplit 2: its 32 of the half's columns
    const int quad = warp & 3;
    const int row = quad * 32 + lane;  // key j0 + row
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float c = p.scale_log2, scale = p.scale;
    bool ok = true;
    for (int u = 0; u < R; ++u) {
      const int s = u % L::kStages;
      ok = mbar_wait(bar_s0 + 8 * hf, u & 1, p.err, abort_flag);
      if (ok) ok = mbar_wait(bar_full0 + 8 * s, (u / L::kStages) & 1, p.err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float* nls = reinterpret_cast<const float*>(smem + L::kRowOff + s * 1024);
      const float* nds = nls + 128;
      const int qt = qt_min + u % span;
      const bool diag = is_chunk && qt == kt;  // query col sees key row iff row <= col
      // queries [c0, +64 / kRowSplit); bf16 pairs over the first of them
      const int c0 = 64 * hf + (64 / kRowSplit) * sub;
      rows_block<true, false, 4 / kRowSplit>(lane_base, c0, nls + c0, nds + c0, c, scale, diag,
                                            row - c0, 1 << 30);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p0 + 8 * hf);
    }
    if (ok) {
      ok = mbar_wait(bar_o, 0, p.err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      // half 0 writes dK, half 1 dV (kRowSplit 2: each warp half of the columns)
      tc_fence_after();
      const int key = j0 + row;
      float* dst = nullptr;
      if (is_chunk) {
        if (key < p.nq)
          dst = (hf == 0 ? p.dk_new : p.dv_new) +
                ((static_cast<size_t>(b) * p.nq + key) * p.Hkv + g) * row_stride;
      } else if (key < p.C) {
        dst = (hf == 0 ? p.dk_cache : p.dv_cache) + (static_cast<size_t>(bg) * p.C + key) * row_stride;
      }
      const bool valid = is_chunk ? key < p.nq : key < p.n;
      const uint32_t col = hf == 0 ? 384 : 256;
      constexpr int kW = D / kRowSplit;  // columns of the row this warp writes
#pragma unroll
      for (int c0 = sub * kW; c0 < (sub + 1) * kW; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(lane_base + col + c0, v);
        tmem_wait_ld();
        if (dst) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 x = valid ? make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                                 __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4*>(dst + c0 + e) = x;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // this grid may overlap the dQ grid before it (programmatic launch: they
  // share no data); it completes only after that grid has, so the stream's
  // later work sees both
  griddep_wait();
}

// ---------------------------------------------------------------- dQ

template <int D>
struct DqLayout {
  static constexpr int kRegions = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kStages = 2;
  static constexpr int kQOff = 0;
  static constexpr int kDOOff = kQOff + kTileBytes;
  static constexpr int kKOff = kDOOff + kTileBytes;            // [stage]
  static constexpr int kVOff = kKOff + kStages * kTileBytes;   // [stage]
  static constexpr int kBarOff = kVOff + kStages * kTileBytes;
  // qd_full, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_done, drain
  static constexpr int kNumBars = 1 + 2 * kStages + 6;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
           const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc,
           const __grid_constant__ CUtensorMap tm_kn, const __grid_constant__ CUtensorMap tm_vn,
           const BwdParams p) {
  using L = DqLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NQT = cdiv(p.nq, 128);
  const int qt = blockIdx.x % NQT;
  const int bh = blockIdx.x / NQT;
  const int b = bh / p.Hq, h = bh % p.Hq, g = h / p.G;
  const int NCT = cdiv(p.n, 128);
  const int T = NCT + qt + 1;  // cache tiles, then chunk tiles 0..qt
  // the dK/dV grid (launched next, programmatically) may fill the SMs this
  // grid's last wave leaves idle
  griddep_launch_dependents();

  const uint32_t bar_qd = sbase + L::kBarOff;
  const uint32_t bar_full0 = bar_qd + 8;
  const uint32_t bar_empty0 = bar_full0 + 8 * L::kStages;
  const uint32_t bar_s0 = bar_empty0 + 8 * L::kStages;  // [half]
  const uint32_t bar_p0 = bar_s0 + 16;                  // [half]
  const uint32_t bar_o = bar_p0 + 16;
  const uint32_t bar_drain = bar_o + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  if (threadIdx.x == 0) {
    mbar_init(bar_qd, 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar_full0 + 8 * s, 1);
      mbar_init(bar_empty0 + 8 * s, 1);
    }
    for (int hf = 0; hf < 2; ++hf) {
      mbar_init(bar_s0 + 8 * hf, 1);
      mbar_init(bar_p0 + 8 * hf, 128 * kRowSplit);
    }
    mbar_init(bar_o, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S [0,128), dP [128,256), dQ [256, 256+D).  Half hf of a
  // key tile is its keys [64 hf, +64): S columns [64 hf, +64), dP columns
  // [128 + 64 hf, +64); its scale*dS (bf16 pairs) goes over the first 32 S
  // columns of the half.

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_qd, 2 * L::kTileBytes);
      for (int r = 0; r < L::kRegions; ++r) {
        tma_load_4d(sbase + L::kQOff + r * 16384, &tm_q, bar_qd, r * 64, h, qt * 128, b);
        tma_load_4d(sbase + L::kDOOff + r * 16384, &tm_do, bar_qd, r * 64, h, qt * 128, b);
      }
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const bool chunk = t >= NCT;
        const int j0 = (chunk ? t - NCT : t) * 128;
        const int s = t % L::kStages;
        if (t >= L::kStages &&
            !mbar_wait(bar_empty0 + 8 * s, ((t / L::kStages) + 1) & 1, p.err, abort_flag))
          break;
        const uint32_t full = bar_full0 + 8 * s;
        mbar_arrive_expect_tx(full, 2 * L::kTileBytes);
        for (int r = 0; r < L::kRegions; ++r) {
          const uint32_t kd = sbase + L::kKOff + s * L::kTileBytes + r * 16384;
          const uint32_t vd = sbase + L::kVOff + s * L::kTileBytes + r * 16384;
          if (chunk) {
            tma_load_4d(kd, &tm_kn, full, r * 64, g, j0, b);
            tma_load_4d(vd, &tm_vn, full, r * 64, g, j0, b);
          } else {
            tma_load_3d(kd, &tm_kc, full, r * 64, j0, b * p.Hkv + g);
            tma_load_3d(vd, &tm_vc, full, r * 64, j0, b * p.Hkv + g);
          }
        }
        issued = t + 1;
      }
      mbar_wait_drain(bar_qd, 0, p.err);
      for (int t = (issued > L::kStages ? issued - L::kStages : 0); t < issued; ++t)
        mbar_wait_drain(bar_full0 + 8 * (t % L::kStages), (t / L::kStages) & 1, p.err);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, D, false, true);
      // S = Q K^T and dP = dO V^T for one half of key tile t (stage s): the
      // half's 64 key rows of the K / V tiles as B
      auto issue_s = [&](int s, int hf) {
        const uint32_t kb = sbase + L::kKOff + s * L::kTileBytes + hf * 8192;
        const uint32_t vb = sbase + L::kVOff + s * L::kTileBytes + hf * 8192;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_bf16_ss(tmem + 64 * hf, sw128_desc(sbase + L::kQOff + off, 16, 1024),
                      sw128_desc(kb + off, 16, 1024), kIdescS, ks > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_bf16_ss(tmem + 128 + 64 * hf, sw128_desc(sbase + L::kDOOff + off, 16, 1024),
                      sw128_desc(vb + off, 16, 1024), kIdescS, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar_s0 + 8 * hf);
      };
      // dQ += (scale dS) K over the half's 64 keys (B the K rows, MN-major)
      auto issue_acc = [&](int s, int hf, bool first) {
        const uint32_t kb = sbase + L::kKOff + s * L::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          mma_bf16_ts(tmem + 256, tmem + pair_col(hf, ks),
                      sw128_desc(kb + (4 * hf + ks) * 2048, 16384, 1024), kIdescAcc,
                      (first && ks == 0) ? 0u : 1u);
        }
      };
      bool ok = mbar_wait(bar_qd, 0, p.err, abort_flag);
      if (ok) ok = mbar_wait(bar_full0, 0, p.err, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(0, 1);
      }
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % L::kStages;
        const bool more = t + 1 < T;
        const int s1 = (t + 1) % L::kStages;
        ok = mbar_wait(bar_p0, t & 1, p.err, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_acc(s, 0, t == 0);
        if (more) {
          ok = mbar_wait(bar_full0 + 8 * s1, ((t + 1) / L::kStages) & 1, p.err, abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_s(s1, 0);
        }
        ok = mbar_wait(bar_p0 + 8, t & 1, p.err, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_acc(s, 1, false);
        mma_commit(bar_empty0 + 8 * s);
        if (more) issue_s(s1, 1);
      }
      mma_commit(bar_o);
      mma_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0, p.err);
    }
  } else {
    const int rw = warp - 2;
    const int hf = rw / (4 * kRowSplit);       // half of each key tile
    const int sub = (rw >> 2) % kRowSplit;     // kRowSplit 2: its 32 of the half's columns
    const int quad = warp & 3;
    const int row = quad * 32 + lane;  // query qt*128 + row
    const int i = qt * 128 + row;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float c = p.scale_log2, scale = p.scale;
    const size_t ridx = (static_cast<size_t>(b) * p.Hq + h) * p.nq_pad + i;
    const float nls[1] = {p.nlse2[ridx]};  // -inf for padding rows: P = 0
    const float nds[1] = {p.dsum[ridx]};   // -scale * D_i (0 for padding rows)
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      ok = mbar_wait(bar_s0 + 8 * hf, t & 1, p.err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // visible keys of this tile for this row
      int last = 127;
      bool masked = false;
      if (t < NCT) {
        if (t == NCT - 1 && p.n - t * 128 < 128) {
          masked = true;
          last = p.n - t * 128 - 1;
        }
      } else if (t - NCT == qt) {
        masked = true;
        last = row;
      }
      // keys [c0, +64 / kRowSplit); scale*dS over S's first of them
      const int c0 = 64 * hf + (64 / kRowSplit) * sub;
      rows_block<false, true, 4 / kRowSplit>(lane_base, c0, nls, nds, c, scale, masked, 0,
                                             last - c0);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p0 + 8 * hf);
    }
    if (ok) {
      ok = mbar_wait(bar_o, 0, p.err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      // each warp writes its share of the row's dQ columns
      tc_fence_after();
      float* dqr = p.dq + ((static_cast<size_t>(b) * p.nq + i) * p.Hq + h) * D;
      constexpr int kW = D / (2 * kRowSplit);  // 16, 32 or 64 columns
      const int part = hf * kRowSplit + sub;
#pragma unroll
      for (int c0 = part * kW; c0 < (part + 1) * kW; c0 += 16) {
        uint32_t qv[16];
        tmem_ld16(lane_base + 256 + c0, qv);
        tmem_wait_ld();
        if (i < p.nq) {
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(dqr + c0 + e) =
                make_float4(__uint_as_float(qv[e]), __uint_as_float(qv[e + 1]),
                            __uint_as_float(qv[e + 2]), __uint_as_float(qv[e + 3]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- launch

template <int D>
static cudaError_t launch_bwd_d(const BwdMaps& m, const BwdParams& p, const void* out,
                                const void* dout, cudaStream_t st) {
  const int rows = p.B * p.Hq * p.nq_pad;
  bwd_rowdot<<<cdiv(rows, 8), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(out),
                                            static_cast<const __nv_bfloat16*>(dout), p, D);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  static int bits_a[2] = {0, 0}, bits_b[2] = {0, 0};
  e = ensure_smem_attr(reinterpret_cast<const void*>(bwd_dkdv<D>), DkdvLayout<D>::kAlloc, bits_a);
  if (e != cudaSuccess) return e;
  e = ensure_smem_attr(reinterpret_cast<const void*>(bwd_dq<D>), DqLayout<D>::kAlloc, bits_b);
  if (e != cudaSuccess) return e;
  // dQ first (256 CTAs on the headline cache: 1.7 waves), then dK/dV, which
  // needs nothing from dQ and starts its CTAs on the SMs dQ's last wave
  // leaves idle
  bwd_dq<D><<<p.B * p.Hq * cdiv(p.nq, 128), kBwdThreads, DqLayout<D>::kAlloc, st>>>(
      m.q, m.dout, m.kc, m.vc, m.kn, m.vn, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cdiv(p.C, 128) + cdiv(p.nq, 128), p.B * p.Hkv);
  cfg.blockDim = dim3(kBwdThreads);
  cfg.dynamicSmemBytes = DkdvLayout<D>::kAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, bwd_dkdv<D>, m.q, m.dout, m.kc, m.vc, m.kn, m.vn, p);
}

cudaError_t launch_attn_bwd_bf16(int head_dim, const BwdMaps& m, const BwdParams& p,
                                 const void* out, const void* dout, cudaStream_t st) {
  return head_dim == 128 ? launch_bwd_d<128>(m, p, out, dout, st)
                         : launch_bwd_d<64>(m, p, out, dout, st);
}

}  // namespace h2o
