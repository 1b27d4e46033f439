// attn_colsum.cu -- summed attention weights per key on sm_100a tensor cores.
//
// colsum[b, g, key] = sum over the G query heads of KV head g and the chunk's
// queries of softmax probability P[h, i, key] ("Learning how to Forget", §1:
// the SDPA kernel returns summed attention weights, the H2O score input).
// P is rebuilt from the logits and the row statistic written by the forward
// kernel (minus lse2): P = 2^(x - lse2), x = scale*log2(e)*<q, k>.  Nothing
// of P is stored.
//
// Key-stationary: one CTA per (cache, KV head, tile of 128 keys).  The MMA
// computes S^T = K_tile Q_rows^T with the keys on the 128 TMEM lanes, so every
// thread owns one key and sums its probabilities along its own TMEM row: the
// column sum needs no cross-thread reduction.  Rows are processed in tiles of
// 128 queries of one head; the sum order is fixed, so results are
// deterministic (no atomics).
//   warp 0      TMA producer: the key tile once, then Q tiles + their lse2
//   warp 1      TMEM allocation; one thread issues the tcgen05.mma, S of row
//               tile u into the 128-column TMEM buffer u % 4
//   warps 2..17 four summing warpgroups; group g takes row tiles u = g, g+4,
//               g+8, ...: one thread per key, all 128 query columns of the
//               tile, read from TMEM in two halves of 64.  A group frees its
//               S buffer as soon as the second half is in registers, so the
//               MMA of its next tile runs while it sums; with four groups the
//               waits and loads of one are covered by the others, and the
//               exponential units stay busy.
// With the int8 cache (Q8) a cache key tile arrives as int8 codes (TMA, no
// swizzle) and the summing warps dequantise it once, into the same
// 128-byte-swizzled bf16 operand, before the first MMA (q8.cuh).
#include "attn.h"
#include "q8.cuh"
#include "sm100.cuh"

namespace h2o {

template <int D, bool Q8 = false>
struct ColLayout {
  static constexpr int kRegions = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kCodeBytes = Q8 ? 128 * D : 0;  // int8 codes of a cache key tile
  static constexpr int kGroups = 4;                // summing warpgroups
  static constexpr int kQStages = 5;               // Q tiles, released when their MMA completes
  static constexpr int kLseStages = 2 * kGroups;   // row statistics, released by the summing group
  static constexpr int kSBufs = kGroups;           // TMEM S buffers, one per summing group
  static constexpr int kKOff = 0;
  static constexpr int kQOff = kKOff + kTileBytes;
  static constexpr int kLseOff = kQOff + kQStages * kTileBytes;  // 512 bytes per stage
  static constexpr int kBarOff = kLseOff + kLseStages * 512;
  // k_full, q_full[QS], q_empty[QS], lse_full[LS], lse_empty[LS], s_full[SB], s_empty[SB], drain
  static constexpr int kNumBars = 1 + 2 * kQStages + 2 * kLseStages + 2 * kSBufs + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kRedOff = kMiscOff + 16;
  static constexpr int kCodeOff = (kRedOff + (kGroups - 1) * 128 * 4 + 1023) / 1024 * 1024;
  static constexpr int kBytes = kCodeOff + kCodeBytes + (Q8 ? 8 : 0);  // + the codes' barrier
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr int kTmemCols = 512;
  static constexpr int kThreads = 64 + 128 * kGroups;
};

// Pairs of query columns (of every eight) whose exponentials run on the FMA
// pipe (exp2_fma2) instead of the special function unit, which the rest
// keep busy: the kernel issues one MUFU op per exponential otherwise and is
// bound by that unit.
constexpr int kEmuPairsOf8 = 2;
// Each CTA starts its sweep over the row tiles at a tile of its own (and
// wraps around), so that the CTAs resident at one time read different Q
// tiles from L2 instead of all the same one.  The order is fixed per CTA, so
// the sums stay deterministic.
constexpr bool kRotateRows = true;

template <bool kDiag>
__device__ __forceinline__ void sum_tile(const uint32_t (&v0)[32], const uint32_t (&v1)[32],
                                         const float4* nlse4, float c, int first_col,
                                         float (&part)[4]) {
  // x = s * c + (-lse2) two columns at a time (packed f32x2), then 2^x and
  // the running sums, also packed
#pragma unroll
  for (int q4 = 0; q4 < 16; ++q4) {
    const float4 nl = nlse4[q4];
    const int col = q4 * 4;
    const uint32_t s0 = q4 < 8 ? v0[col] : v1[col - 32];
    const uint32_t s1 = q4 < 8 ? v0[col + 1] : v1[col - 31];
    const uint32_t s2 = q4 < 8 ? v0[col + 2] : v1[col - 30];
    const uint32_t s3 = q4 < 8 ? v0[col + 3] : v1[col - 29];
    float x0, x1, x2, x3;
    ffma2(x0, x1, __uint_as_float(s0), __uint_as_float(s1), c, c, nl.x, nl.y);
    ffma2(x2, x3, __uint_as_float(s2), __uint_as_float(s3), c, c, nl.z, nl.w);
    float p0, p1, p2, p3;
    if (((2 * q4) & 7) < kEmuPairsOf8) {
      exp2_fma2(p0, p1, x0, x1);
    } else {
      p0 = ex2_approx(x0);
      p1 = ex2_approx(x1);
    }
    if (((2 * q4 + 1) & 7) < kEmuPairsOf8) {
      exp2_fma2(p2, p3, x2, x3);
    } else {
      p2 = ex2_approx(x2);
      p3 = ex2_approx(x3);
    }
    if (kDiag) {  // query i0+col sees key j0+row iff row <= col
      p0 = (col >= first_col) ? p0 : 0.f;
      p1 = (col + 1 >= first_col) ? p1 : 0.f;
      p2 = (col + 2 >= first_col) ? p2 : 0.f;
      p3 = (col + 3 >= first_col) ? p3 : 0.f;
    }
    fadd2(part[0], part[1], part[0], part[1], p0, p1);
    fadd2(part[2], part[3], part[2], part[3], p2, p3);
  }
}

template <int D, bool Q8>
__global__ void __launch_bounds__(64 + 128 * ColLayout<D>::kGroups, 1)
    attn_colsum_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_kc,
                       const __grid_constant__ CUtensorMap tm_kn, const AttnParams p) {
  using L = ColLayout<D, Q8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int bg = blockIdx.y;
  const int b = bg / p.Hkv;
  const int g = bg % p.Hkv;
  const int NCTC = cdiv(p.C, 128);  // key tiles covering the whole capacity
  const int NQT = cdiv(p.nq, 128);
  const bool is_chunk = static_cast<int>(blockIdx.x) >= NCTC;
  const int kt = is_chunk ? blockIdx.x - NCTC : blockIdx.x;
  const int j0 = kt * 128;
  float* out = p.colsum + static_cast<size_t>(bg) * p.colsum_ld;

  if (!is_chunk && j0 >= p.n) {
    // slots beyond the valid ones received no weight
    for (int j = j0 + threadIdx.x; j < min(j0 + 128, p.C); j += blockDim.x) out[j] = 0.f;
    return;
  }
  const int qt_min = is_chunk ? kt : 0;  // a chunk key is seen by queries i >= key
  const int span = NQT - qt_min;
  const int R = p.G * span;
  // row tile of sweep step v: (v + rot) mod R
  const int rot = kRotateRows ? static_cast<int>((blockIdx.x * 7u + blockIdx.y * 13u) % R) : 0;
  auto tile_of = [&](int v) { return v + rot < R ? v + rot : v + rot - R; };

  const uint32_t bar_k = sbase + L::kBarOff;
  const uint32_t bar_q_full0 = bar_k + 8;
  const uint32_t bar_q_empty0 = bar_q_full0 + 8 * L::kQStages;
  const uint32_t bar_l_full0 = bar_q_empty0 + 8 * L::kQStages;
  const uint32_t bar_l_empty0 = bar_l_full0 + 8 * L::kLseStages;
  const uint32_t bar_s_full0 = bar_l_empty0 + 8 * L::kLseStages;
  const uint32_t bar_s_empty0 = bar_s_full0 + 8 * L::kSBufs;
  const uint32_t bar_drain = bar_s_empty0 + 8 * L::kSBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  float* red = reinterpret_cast<float*>(smem + L::kRedOff);
  // Q8 cache tile: the codes land at kCodeOff (barrier bar_codes); the
  // summing threads dequantise them and then arrive on bar_k themselves
  const bool dequant = Q8 && !is_chunk;
  const uint32_t bar_codes = sbase + L::kCodeOff + L::kCodeBytes;

  if (threadIdx.x == 0) {
    mbar_init(bar_k, dequant ? 128 * L::kGroups : 1);
    if (dequant) mbar_init(bar_codes, 1);
    for (int s = 0; s < L::kQStages; ++s) {
      mbar_init(bar_q_full0 + 8 * s, 1);
      mbar_init(bar_q_empty0 + 8 * s, 1);  // the MMA's commit
    }
    for (int s = 0; s < L::kLseStages; ++s) {
      mbar_init(bar_l_full0 + 8 * s, 1);
      mbar_init(bar_l_empty0 + 8 * s, 128);  // the summing group of that tile
    }
    for (int s = 0; s < L::kSBufs; ++s) {
      mbar_init(bar_s_full0 + 8 * s, 1);
      mbar_init(bar_s_empty0 + 8 * s, 128);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      if (dequant) {  // int8 codes of the key tile: one box of 128 rows x D bytes
        mbar_arrive_expect_tx(bar_codes, L::kCodeBytes);
        tma_load_3d(sbase + L::kCodeOff, &tm_kc, bar_codes, 0, j0, b * p.Hkv + g);
      } else {
        mbar_arrive_expect_tx(bar_k, L::kTileBytes);
        for (int r = 0; r < L::kRegions; ++r) {
          if (is_chunk)
            tma_load_4d(sbase + L::kKOff + r * 16384, &tm_kn, bar_k, r * 64, g, j0, b);
          else
            tma_load_3d(sbase + L::kKOff + r * 16384, &tm_kc, bar_k, r * 64, j0, b * p.Hkv + g);
        }
      }
      int issued_q = 0, issued_l = 0;
      bool waited = false;
      for (int u = 0; u < R; ++u) {
        const int h = g * p.G + tile_of(u) / span;
        const int qt = qt_min + tile_of(u) % span;
        const int s = u % L::kQStages;
        if (u >= L::kQStages &&
            !mbar_wait(bar_q_empty0 + 8 * s, ((u / L::kQStages) + 1) & 1, p.err, abort_flag))
          break;
        mbar_arrive_expect_tx(bar_q_full0 + 8 * s, L::kTileBytes);
        for (int r = 0; r < L::kRegions; ++r)
          tma_load_4d(sbase + L::kQOff + s * L::kTileBytes + r * 16384, &tm_q, bar_q_full0 + 8 * s,
                      r * 64, h, qt * 128, b);
        issued_q = u + 1;
        const int sl = u % L::kLseStages;
        if (u >= L::kLseStages &&
            !mbar_wait(bar_l_empty0 + 8 * sl, ((u / L::kLseStages) + 1) & 1, p.err, abort_flag))
          break;
        if (!waited) {  // the row statistics come from the preceding forward kernel
          griddep_wait();
          waited = true;
        }
        mbar_arrive_expect_tx(bar_l_full0 + 8 * sl, 512);
        bulk_load(sbase + L::kLseOff + sl * 512,
                  p.nlse2 + (static_cast<size_t>(b) * p.Hq + h) * p.nq_pad + qt * 128, 512,
                  bar_l_full0 + 8 * sl);
        issued_l = u + 1;
      }
      // drain: every issued copy has landed before the CTA can exit
      mbar_wait_drain(dequant ? bar_codes : bar_k, 0, p.err);
      for (int u = (issued_q > L::kQStages ? issued_q - L::kQStages : 0); u < issued_q; ++u)
        mbar_wait_drain(bar_q_full0 + 8 * (u % L::kQStages), (u / L::kQStages) & 1, p.err);
      for (int u = (issued_l > L::kLseStages ? issued_l - L::kLseStages : 0); u < issued_l; ++u)
        mbar_wait_drain(bar_l_full0 + 8 * (u % L::kLseStages), (u / L::kLseStages) & 1, p.err);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, false, false);
      bool ok = mbar_wait(bar_k, 0, p.err, abort_flag);
      for (int u = 0; u < R && ok; ++u) {
        const int s = u % L::kQStages;
        const int sb = u % L::kSBufs;
        ok = mbar_wait(bar_q_full0 + 8 * s, (u / L::kQStages) & 1, p.err, abort_flag);
        if (ok && u >= L::kSBufs)
          ok = mbar_wait(bar_s_empty0 + 8 * sb, ((u / L::kSBufs) + 1) & 1, p.err, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qbase = sbase + L::kQOff + s * L::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_bf16_ss(tmem + sb * 128, sw128_desc(sbase + L::kKOff + off, 16, 1024),
                      sw128_desc(qbase + off, 16, 1024), kIdesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar_s_full0 + 8 * sb);
        mma_commit(bar_q_empty0 + 8 * s);
      }
      mma_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0, p.err);
    }
  } else {
    const int quad = warp & 3;
    const int grp = (warp - 2) >> 2;   // row tiles u with u % kGroups == grp
    const int row = quad * 32 + lane;  // key j0 + row
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float c = p.scale_log2;
    float acc = 0.f;
    bool ok = true;
    if (dequant) {
      // the tile's 128 x D codes -> bf16 in the swizzled K operand: chunks of
      // 16 codes (16-byte pieces of a row), each to two 16-byte chunks of its
      // 128-byte region row at chunk index ^ (row & 7)
      const int t = threadIdx.x - 64;  // 0 .. 128 * kGroups - 1
      ok = mbar_wait(bar_codes, 0, p.err, abort_flag);
      if (ok) {
        constexpr int kChunks = 128 * D / 16;
        for (int job = t; job < kChunks; job += 128 * L::kGroups) {
          const int r = job / (D / 16), i = job % (D / 16);  // key row, 16-code piece
          const float sc = j0 + r < p.n ? p.k_scale[static_cast<size_t>(bg) * p.C + j0 + r] : 0.f;
          const uint4 codes = *reinterpret_cast<const uint4*>(smem + L::kCodeOff + r * D + 16 * i);
          uint32_t w[8];
          q8_dequant16(codes, sc, w);
          const int e = 16 * i;                  // first element
          const int reg = e / 64, c16 = (e % 64) / 8;  // region, 16-byte chunk in its row
          uint8_t* rowp = smem + L::kKOff + reg * 16384 + r * 128;
          *reinterpret_cast<uint4*>(rowp + ((c16 ^ (r & 7)) * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(rowp + (((c16 + 1) ^ (r & 7)) * 16)) =
              make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
      fence_proxy_async_smem();  // the MMA reads the operand through the async proxy
      mbar_arrive(bar_k);
    }
    for (int u = grp; u < R; u += L::kGroups) {
      const int sl = u % L::kLseStages;
      const int sb = u % L::kSBufs;
      ok = mbar_wait(bar_s_full0 + 8 * sb, (u / L::kSBufs) & 1, p.err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t v[2][32];
      tmem_ld32(lane_base + sb * 128, v[0]);
      tmem_ld32(lane_base + sb * 128 + 32, v[1]);
      tmem_wait_ld();
      ok = mbar_wait(bar_l_full0 + 8 * sl, (u / L::kLseStages) & 1, p.err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const float4* nlse4 = reinterpret_cast<const float4*>(smem + L::kLseOff + sl * 512);
      const int qt = qt_min + tile_of(u) % span;
      const bool diag = is_chunk && qt == kt;  // query i0+col sees key j0+row iff row <= col
      float part[4] = {0.f, 0.f, 0.f, 0.f};
      if (diag)
        sum_tile<true>(v[0], v[1], nlse4, c, row, part);
      else
        sum_tile<false>(v[0], v[1], nlse4, c, 0, part);
      // second half of the query columns; then the S buffer is free
      tmem_ld32(lane_base + sb * 128 + 64, v[0]);
      tmem_ld32(lane_base + sb * 128 + 96, v[1]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar_s_empty0 + 8 * sb);
      if (diag)
        sum_tile<true>(v[0], v[1], nlse4 + 16, c, row - 64, part);
      else
        sum_tile<false>(v[0], v[1], nlse4 + 16, c, 0, part);
      acc += (part[0] + part[1]) + (part[2] + part[3]);
      mbar_arrive(bar_l_empty0 + 8 * sl);
    }
    // combine the groups' sums in a fixed order
    if (grp > 0) red[(grp - 1) * 128 + row] = acc;
    named_bar_sync(1, 128 * L::kGroups);
    if (grp == 0 && ok) {
      float total = acc;
#pragma unroll
      for (int gr = 1; gr < L::kGroups; ++gr) total += red[(gr - 1) * 128 + row];
      const int key = j0 + row;
      if (!H2O_IN_BOUNDS(p.C + p.nq <= p.colsum_ld, p.err)) {
      } else if (is_chunk) {
        if (key < p.nq) out[p.C + key] = total;
      } else if (key < p.n) {
        out[key] = total;
      } else if (key < p.C) {
        out[key] = 0.f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  griddep_launch_dependents();  // the summed weights of this CTA are written
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

template <int D, bool Q8>
static cudaError_t launch_colsum(const AttnMaps& m, const AttnParams& p, cudaStream_t st) {
  using L = ColLayout<D, Q8>;
  static int attr_bits[2] = {0, 0};
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(attn_colsum_kernel<D, Q8>),
                                   L::kAlloc, attr_bits);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cdiv(p.C, 128) + cdiv(p.nq, 128), p.B * p.Hkv);
  cfg.blockDim = dim3(L::kThreads);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attn_colsum_kernel<D, Q8>, m.q, m.kc, m.kn, p);
}

cudaError_t launch_attn_colsum_bf16(int head_dim, const AttnMaps& m, const AttnParams& p,
                                    cudaStream_t st) {
  const bool q8 = p.k_scale != nullptr;  // int8 cache
  if (head_dim == 128) return q8 ? launch_colsum<128, true>(m, p, st) : launch_colsum<128, false>(m, p, st);
  return q8 ? launch_colsum<64, true>(m, p, st) : launch_colsum<64, false>(m, p, st);
}

}  // namespace h2o
