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
// column sum needs no cross-thread reduction.  The key tile, the stationary
// operand, is copied once into TMEM (each thread its own key's row) and read
// from there as the A operand: each MMA then reads only the Q tile from
// shared memory, which otherwise limits the tensor core (two 32 KB operands
// per 128 x 128 x 128 product plus the next Q tile's arrival).  Rows are processed in tiles of
// 128 queries of one head; the sum order is fixed, so results are
// deterministic (no atomics).
//   warp 0      TMA producer: the key tile once, then Q tiles + their lse2
//   warp 1      TMEM allocation; one thread issues the tcgen05.mma, S of row
//               tile u into the 128-column TMEM buffer u % 3
//   warps 2..13 three summing warpgroups; group g takes row tiles u = g, g+3,
//               g+6, ...: one thread per key, all 128 query columns of the
//               tile, read from TMEM in two halves of 64.  A group frees its
//               S buffer as soon as the second half is in registers, so the
//               MMA of its next tile runs while it sums.  Group 0 also copies
//               the key tile into TMEM (columns 384 ..) before the first MMA.
// With the int8 cache (Q8) a cache key tile arrives as int8 codes (TMA, no
// swizzle) and group 0 dequantises each key's row on its way into TMEM
// (q8.cuh).
#include <algorithm>

#include "attn.h"
#include "q8.cuh"
#include "sm100.cuh"

namespace h2o {

template <int D, bool Q8 = false>
struct ColLayout {
  static constexpr int kRegions = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kCodeBytes = Q8 ? 128 * D : 0;  // int8 codes of a cache key tile
  static constexpr int kGroups = 3;                // summing warpgroups
  static constexpr int kQStages = 5;               // Q tiles, released when their MMA completes
  static constexpr int kLseStages = 16;            // row statistics, released by the summing group
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
  static constexpr int kBytes = kCodeOff + kCodeBytes + 8;  // + the key-in-TMEM barrier
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr int kTmemCols = 512;
  static constexpr int kKCol = 128 * kSBufs;       // the key tile, D/2 columns of bf16 pairs
  static_assert(kKCol + D / 2 <= kTmemCols, "TMEM layout");
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

__device__ __forceinline__ uint32_t gl_parity(int u, int stages) {
  return static_cast<uint32_t>((u / stages) & 1);
}

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

// 32 columns: the same arithmetic as sum_tile on one 32-column piece.
template <bool kDiag>
__device__ __forceinline__ void sum_piece(const uint32_t (&v)[32], const float4* nlse4, float c,
                                          int first_col, float (&part)[4]) {
#pragma unroll
  for (int q4 = 0; q4 < 8; ++q4) {
    const float4 nl = nlse4[q4];
    const int col = q4 * 4;
    float x0, x1, x2, x3;
    ffma2(x0, x1, __uint_as_float(v[col]), __uint_as_float(v[col + 1]), c, c, nl.x, nl.y);
    ffma2(x2, x3, __uint_as_float(v[col + 2]), __uint_as_float(v[col + 3]), c, c, nl.z, nl.w);
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
    if (kDiag) {
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
  // the key tile: bar_k completes when its bf16 rows (or, Q8 cache tile, its
  // codes, at kCodeOff) have landed; bar_ktm when group 0 has written it into
  // TMEM
  const bool dequant = Q8 && !is_chunk;
  const uint32_t bar_ktm = sbase + L::kCodeOff + L::kCodeBytes;

  if (threadIdx.x == 0) {
    mbar_init(bar_k, 1);
    mbar_init(bar_ktm, 128);
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
        mbar_arrive_expect_tx(bar_k, L::kCodeBytes);
        tma_load_3d(sbase + L::kCodeOff, &tm_kc, bar_k, 0, j0, b * p.Hkv + g);
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
        // the producer spins too: a suspended wait wakes hundreds of cycles late,
        // and it waits twice per row tile
        if (u >= L::kQStages &&
            !mbar_wait_spin(bar_q_empty0 + 8 * s, ((u / L::kQStages) + 1) & 1, p.err, abort_flag))
          break;
        mbar_arrive_expect_tx(bar_q_full0 + 8 * s, L::kTileBytes);
        for (int r = 0; r < L::kRegions; ++r)
          tma_load_4d(sbase + L::kQOff + s * L::kTileBytes + r * 16384, &tm_q, bar_q_full0 + 8 * s,
                      r * 64, h, qt * 128, b);
        issued_q = u + 1;
        const int sl = u % L::kLseStages;
        if (u >= L::kLseStages &&
            !mbar_wait_spin(bar_l_empty0 + 8 * sl, ((u / L::kLseStages) + 1) & 1, p.err,
                            abort_flag))
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
      mbar_wait_drain(bar_k, 0, p.err);
      for (int u = (issued_q > L::kQStages ? issued_q - L::kQStages : 0); u < issued_q; ++u)
        mbar_wait_drain(bar_q_full0 + 8 * (u % L::kQStages), (u / L::kQStages) & 1, p.err);
      for (int u = (issued_l > L::kLseStages ? issued_l - L::kLseStages : 0); u < issued_l; ++u)
        mbar_wait_drain(bar_l_full0 + 8 * (u % L::kLseStages), (u / L::kLseStages) & 1, p.err);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, false, false);
      const uint64_t q_desc0 = sw128_desc(sbase + L::kQOff, 16, 1024);
      // the issuing thread spins: waking from a suspended wait costs hundreds
      // of cycles on the path that feeds the tensor core
      bool ok = mbar_wait_spin(bar_ktm, 0, p.err, abort_flag);
      for (int u = 0; u < R && ok; ++u) {
        const int s = u % L::kQStages;
        const int sb = u % L::kSBufs;
        ok = mbar_wait_spin(bar_q_full0 + 8 * s, (u / L::kQStages) & 1, p.err, abort_flag);
        if (ok && u >= L::kSBufs)
          ok = mbar_wait_spin(bar_s_empty0 + 8 * sb, ((u / L::kSBufs) + 1) & 1, p.err, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint64_t qd = q_desc0 + ((s * L::kTileBytes) >> 4);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {  // A: the key tile from TMEM, 8 columns per 16 elements
          const uint32_t off = ((ks >> 2) * 16384 + (ks & 3) * 32) >> 4;
          mma_bf16_ts(tmem + sb * 128, tmem + L::kKCol + 8 * ks, qd + off, kIdesc,
                      ks > 0 ? 1u : 0u);
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
    if (grp == 0) {
      // the key tile into TMEM: this thread's key row (j0 + row) as D/2
      // columns of bf16 pairs on its lane, from the 128-byte-swizzled bf16
      // tile (16-byte piece c of region r at piece index c ^ (row & 7)) or,
      // Q8 cache tile, dequantised from its codes and scale
      ok = mbar_wait(bar_k, 0, p.err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        uint32_t w[D / 2];
        if (dequant) {
          const float sc = j0 + row < p.n ? p.k_scale[static_cast<size_t>(bg) * p.C + j0 + row] : 0.f;
#pragma unroll
          for (int i = 0; i < D / 16; ++i) {
            uint32_t piece[8];
            q8_dequant16(*reinterpret_cast<const uint4*>(smem + L::kCodeOff + row * D + 16 * i), sc,
                         piece);
#pragma unroll
            for (int j = 0; j < 8; ++j) w[8 * i + j] = piece[j];
          }
        } else {
#pragma unroll
          for (int c16 = 0; c16 < D / 8; ++c16) {  // 16-byte pieces: 8 elements, 4 columns
            const uint4 v = *reinterpret_cast<const uint4*>(
                smem + L::kKOff + (c16 / 8) * 16384 + row * 128 + (((c16 % 8) ^ (row & 7)) * 16));
            w[4 * c16] = v.x;
            w[4 * c16 + 1] = v.y;
            w[4 * c16 + 2] = v.z;
            w[4 * c16 + 3] = v.w;
          }
        }
#pragma unroll
        for (int c0 = 0; c0 < D / 2; c0 += 32)
          tmem_st32(lane_base + L::kKCol + c0, *reinterpret_cast<uint32_t(*)[32]>(&w[c0]));
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar_ktm);
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

// ---------------------------------------------------------------- persistent variant
//
// One CTA per SM walks a list of work items -- (cache, KV head, key tile), the
// cache tiles holding keys first, then the chunk's key tiles -- taking items
// c, c + grid, c + 2 grid, ...  The pipeline runs across item boundaries: the
// Q and row-statistic rings continue with a global row-tile counter, and the
// next item's key tile is loaded and copied into a second TMEM buffer while
// the current item is summed, so no SM waits for a CTA to start up or drain
// between items.  Two threads (lane 0 of warps 1 and 2) issue the MMAs, the
// row tiles in turn.  Group 0 copies key tiles into TMEM (when the tile has
// landed and its TMEM buffer is free, checked before each of its row tiles).
// Row tile v of an item's sweep goes to S buffer v mod 3 and its summing
// warpgroups (one per buffer, as in the one-CTA-per-tile kernel, or two,
// each taking 64 of the tile's columns), so every key's sum is formed in an
// order fixed by its item, whatever the grid.  Each warpgroup writes its
// partial sums of an item into shared memory and the last to do so for a
// key adds the partials in warpgroup order and writes the summed weight.
// Summing warpgroups per S buffer: 1 (each reads its tile in two halves of
// 64 columns) or 2 (each takes 64 of the tile's columns, twice as many warps
// sharing each SM sub-partition's exponentials, 72 registers a thread).
// Measured on the C 8192 cache: 100.4 us with one, 118.8 with two; on the
// 144-cache stack 17.0 against 20.3 ms.  Also measured and not kept: one
// summing warpgroup per buffer reading the whole tile at once with 152
// registers (warps 0-3 handing theirs over), 106.5 against 105.5 us.
constexpr int kColsumSplit = 1;
// MMA-issuing threads (lane 0 of warps 1 .. kColsumIssuers), taking the row
// tiles in turn.  Each issue of a tile's MMAs returns about when the tensor
// pipe has taken them, so one thread's own waits, commits and bookkeeping
// between tiles leave the pipe idle; a second issuer fills those gaps.
// Measured on the C 8192 cache: 102.4 against 106.5 us with one issuer; on
// the 144-cache stack 18.1 against 18.7 ms.  With two issuers a whole-tile
// read (warps 0-3 handing registers to the summing warpgroups, which free an
// S buffer before summing it) is still no faster: 104.4 us at 160 registers,
// 106.5 at 152 (spills), against 102.4.
constexpr int kColsumIssuers = 2;

template <int D, bool Q8>
struct PColLayout {
  static constexpr int kRegions = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kCodeBytes = Q8 ? 128 * D : 0;
  static constexpr int kGroups = 3;
  static constexpr int kQStages = 4;
  static constexpr int kLseStages = 16;
  static constexpr int kSBufs = kGroups;
  static constexpr int kSplit = kColsumSplit;      // summing warpgroups per S buffer
  static constexpr int kParts = kGroups * kSplit;  // summing warpgroups
  static constexpr int kRedSets = 8;  // items whose partials may be pending at once
  static constexpr int kKOff = 0;                               // bf16 key tile staging
  static constexpr int kCodeOff = kKOff + kTileBytes;           // Q8 codes staging
  static constexpr int kQOff = kCodeOff + kCodeBytes;
  static constexpr int kLseOff = kQOff + kQStages * kTileBytes;
  static constexpr int kRedOff = kLseOff + kLseStages * 512;    // [sets][parts][128] float
  static constexpr int kCntOff = kRedOff + kRedSets * kParts * 128 * 4;   // [sets][128] int
  static constexpr int kDoneOff = kCntOff + kRedSets * 128 * 4;            // [sets][128] int
  static constexpr int kBarOff = kDoneOff + kRedSets * 128 * 4;
  // k_full, k_free, ktm[2], ktm_free[2], q_full[QS], q_empty[QS], l_full[LS],
  // l_empty[LS], s_full[SB], s_empty[SB], drain
  static constexpr int kNumBars = 2 + 2 + 2 + 2 * kQStages + 2 * kLseStages + 2 * kSBufs + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= kMaxDynSmem, "shared-memory layout too large");
  static constexpr int kTmemCols = 512;
  static constexpr int kKCol = 128 * kSBufs;                    // two key buffers of D/2 columns
  static_assert(kKCol + D <= kTmemCols, "TMEM layout");
  static constexpr int kIssuers = kColsumIssuers;  // MMA-issuing warps, 1 .. kIssuers
  static constexpr int kGroupWarp0 = 1 + kIssuers;  // first summing warp
  static constexpr int kThreads = 32 * kGroupWarp0 + 128 * kParts;
};

// Waits until *count >= target (a count that another thread of the CTA
// raises); gives up like mbar_wait_spin.
__device__ __forceinline__ bool wait_count(const volatile int* count, int target, int* err,
                                           volatile int* abort) {
  if (*count >= target) {
    __threadfence_block();
    return true;
  }
  const uint64_t start = global_timer_ns();
  uint32_t n = 0;
  while (*count < target) {
    if ((++n & 255) == 0) {
      if (*abort) return false;
      if (global_timer_ns() - start > kWaitLimitNs) {
        *abort = 1;
        atomicOr(err, kDevErrTimeout);
        return false;
      }
    }
  }
  __threadfence_block();
  return true;
}

// Work item i of the list: key tile `kt` (< NCT: cache keys, else chunk key
// tile kt - NCT) of unit bg.
// The sweep over its R row tiles starts at tile rot and wraps around.
struct ColItem {
  int bg, kt, j0, R, qt_min, span, rot;
  bool is_chunk;
  __device__ __forceinline__ int tile_of(int v) const { return v + rot < R ? v + rot : v + rot - R; }
};

__device__ __forceinline__ ColItem col_item(int i, int BG, int NCT, int NCTC, int NQT, int G) {
  ColItem it;
  const int kt_all = i / BG;
  it.bg = i % BG;
  it.is_chunk = kt_all >= NCT;
  it.kt = it.is_chunk ? kt_all - NCT : kt_all;
  it.j0 = it.kt * 128;
  it.qt_min = it.is_chunk ? it.kt : 0;
  it.span = NQT - it.qt_min;
  it.R = G * it.span;
  const unsigned x = static_cast<unsigned>(it.is_chunk ? NCTC + it.kt : it.kt);
  it.rot = kRotateRows ? static_cast<int>((x * 7u + static_cast<unsigned>(it.bg) * 13u) % it.R) : 0;
  return it;
}

template <int D, bool Q8>
__global__ void __launch_bounds__(PColLayout<D, Q8>::kThreads, 1)
    attn_colsum_persistent(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_kc,
                           const __grid_constant__ CUtensorMap tm_kn, const AttnParams p) {
  using L = PColLayout<D, Q8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int BG = p.B * p.Hkv;
  const int NCT = cdiv(p.n, 128);      // key tiles holding cache keys
  const int NCTC = cdiv(p.C, 128);     // key tiles covering the capacity
  const int NQT = cdiv(p.nq, 128);
  const int items = BG * (NCT + NQT);
  const int first = static_cast<int>(blockIdx.x), stride = static_cast<int>(gridDim.x);

  // slots past the valid ones received no weight (every CTA a share)
  {
    const int empty = p.C - p.n;
    const long long total = static_cast<long long>(BG) * empty;
    for (long long e = static_cast<long long>(first) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<long long>(stride) * blockDim.x) {
      const int bgx = static_cast<int>(e / empty), s = p.n + static_cast<int>(e % empty);
      p.colsum[static_cast<size_t>(bgx) * p.colsum_ld + s] = 0.f;
    }
  }

  const uint32_t bar_k_full = sbase + L::kBarOff;
  const uint32_t bar_k_free = bar_k_full + 8;
  const uint32_t bar_ktm0 = bar_k_free + 8;        // [2]
  const uint32_t bar_ktm_free0 = bar_ktm0 + 16;    // [2]
  const uint32_t bar_q_full0 = bar_ktm_free0 + 16;
  const uint32_t bar_q_empty0 = bar_q_full0 + 8 * L::kQStages;
  const uint32_t bar_l_full0 = bar_q_empty0 + 8 * L::kQStages;
  const uint32_t bar_l_empty0 = bar_l_full0 + 8 * L::kLseStages;
  const uint32_t bar_s_full0 = bar_l_empty0 + 8 * L::kLseStages;
  const uint32_t bar_s_empty0 = bar_s_full0 + 8 * L::kSBufs;
  const uint32_t bar_drain = bar_s_empty0 + 8 * L::kSBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  volatile int* issued = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 8);  // row tiles issued
  float* red = reinterpret_cast<float*>(smem + L::kRedOff);
  int* cnt = reinterpret_cast<int*>(smem + L::kCntOff);     // partials arrived, per set and key
  volatile int* done = reinterpret_cast<volatile int*>(smem + L::kDoneOff);  // uses combined

  if (threadIdx.x == 0) {
    mbar_init(bar_k_full, 1);
    mbar_init(bar_k_free, 128);
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar_ktm0 + 8 * x, 128);
      mbar_init(bar_ktm_free0 + 8 * x, L::kIssuers);
    }
    for (int s = 0; s < L::kQStages; ++s) {
      mbar_init(bar_q_full0 + 8 * s, 1);
      mbar_init(bar_q_empty0 + 8 * s, 1);
    }
    for (int s = 0; s < L::kLseStages; ++s) {
      mbar_init(bar_l_full0 + 8 * s, 1);
      mbar_init(bar_l_empty0 + 8 * s, 128 * L::kSplit);
    }
    for (int s = 0; s < L::kSBufs; ++s) {
      mbar_init(bar_s_full0 + 8 * s, 1);
      mbar_init(bar_s_empty0 + 8 * s, 128 * L::kSplit);
    }
    mbar_init(bar_drain, L::kIssuers);
    *abort_flag = 0;
    *issued = 0;
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < L::kRedSets * 128; i += blockDim.x) {
    cnt[i] = 0;
    done[i] = 0;
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
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int gq = 0, gl = 0, n_items = 0;
      bool ok = true, waited = false;
      for (int i = first; i < items && ok; i += stride, ++n_items) {
        const ColItem it = col_item(i, BG, NCT, NCTC, NQT, p.G);
        const int b = it.bg / p.Hkv, g = it.bg % p.Hkv;
        // the key tile (staging is free once group 0 copied the previous one)
        if (n_items > 0 && !mbar_wait_spin(bar_k_free, (n_items - 1) & 1, p.err, abort_flag)) {
          ok = false;
          break;
        }
        if (Q8 && !it.is_chunk) {
          mbar_arrive_expect_tx(bar_k_full, L::kCodeBytes);
          tma_load_3d(sbase + L::kCodeOff, &tm_kc, bar_k_full, 0, it.j0, b * p.Hkv + g);
        } else {
          mbar_arrive_expect_tx(bar_k_full, L::kTileBytes);
          for (int r = 0; r < L::kRegions; ++r) {
            if (it.is_chunk)
              tma_load_4d(sbase + L::kKOff + r * 16384, &tm_kn, bar_k_full, r * 64, g, it.j0, b);
            else
              tma_load_3d(sbase + L::kKOff + r * 16384, &tm_kc, bar_k_full, r * 64, it.j0,
                          b * p.Hkv + g);
          }
        }
        for (int u = 0; u < it.R; ++u, ++gq, ++gl) {
          const int h = g * p.G + it.tile_of(u) / it.span;
          const int qt = it.qt_min + it.tile_of(u) % it.span;
          const int s = gq % L::kQStages;
          if (gq >= L::kQStages &&
              !mbar_wait_spin(bar_q_empty0 + 8 * s, ((gq / L::kQStages) + 1) & 1, p.err,
                              abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar_q_full0 + 8 * s, L::kTileBytes);
          for (int r = 0; r < L::kRegions; ++r)
            tma_load_4d(sbase + L::kQOff + s * L::kTileBytes + r * 16384, &tm_q,
                        bar_q_full0 + 8 * s, r * 64, h, qt * 128, b);
          const int sl = gl % L::kLseStages;
          if (gl >= L::kLseStages &&
              !mbar_wait_spin(bar_l_empty0 + 8 * sl, ((gl / L::kLseStages) + 1) & 1, p.err,
                              abort_flag)) {
            ok = false;
            break;
          }
          if (!waited) {  // the row statistics come from the preceding forward kernel
            griddep_wait();
            waited = true;
          }
          mbar_arrive_expect_tx(bar_l_full0 + 8 * sl, 512);
          bulk_load(sbase + L::kLseOff + sl * 512,
                    p.nlse2 + (static_cast<size_t>(b) * p.Hq + h) * p.nq_pad + qt * 128, 512,
                    bar_l_full0 + 8 * sl);
        }
      }
      // drain: the copies in flight land before the CTA can exit (the last
      // ring fills and the last key tile)
      if (n_items > 0) mbar_wait_drain(bar_k_full, (n_items - 1) & 1, p.err);
      for (int u = max(0, gq - L::kQStages); u < gq; ++u)
        mbar_wait_drain(bar_q_full0 + 8 * (u % L::kQStages), (u / L::kQStages) & 1, p.err);
      for (int u = max(0, gl - L::kLseStages); u < gl; ++u)
        mbar_wait_drain(bar_l_full0 + 8 * (u % L::kLseStages), (u / L::kLseStages) & 1, p.err);
    }
  } else if (warp <= L::kIssuers) {
    // ------------------------------------------------------------ MMA issuers
    // Issuer `me` takes the row tiles gu with gu % kIssuers == me (a Q stage
    // always with the same issuer) and issues tile gu once tile gu - 1 is
    // issued, so the tiles reach the pipe in order.  That order also makes the
    // parity test of an S buffer's release sound: the buffer's previous use
    // was issued, by either issuer, after the use before it was released.
    // Both issuers commit each key buffer's release.
    static_assert(L::kQStages % L::kIssuers == 0, "a Q stage belongs to one issuer");
    const int me = warp - 1;
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, false, false);
      const uint64_t q_desc0 = sw128_desc(sbase + L::kQOff, 16, 1024);
      int gu = 0, n_items = 0;
      int used0 = 0, used1 = 0, used2 = 0;  // uses of each S buffer before this item
      bool ok = true;
      for (int i = first; i < items && ok; i += stride, ++n_items) {
        const ColItem it = col_item(i, BG, NCT, NCTC, NQT, p.G);
        const int kb = n_items & 1;
        ok = mbar_wait_spin(bar_ktm0 + 8 * kb, (n_items >> 1) & 1, p.err, abort_flag);
        for (int u = 0; u < it.R && ok; ++u, ++gu) {
          if (L::kIssuers > 1 && gu % L::kIssuers != me) continue;
          const int s = gu % L::kQStages;
          const int sb = u % L::kSBufs;  // row tile u of an item: S buffer and group u % 3
          const int j = (sb == 0 ? used0 : sb == 1 ? used1 : used2) + u / L::kSBufs;
          ok = mbar_wait_spin(bar_q_full0 + 8 * s, (gu / L::kQStages) & 1, p.err, abort_flag);
          if (ok && L::kIssuers > 1 && gu > 0) ok = wait_count(issued, gu, p.err, abort_flag);
          if (ok && j >= 1)
            ok = mbar_wait_spin(bar_s_empty0 + 8 * sb, (j - 1) & 1, p.err, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint64_t qd = q_desc0 + ((s * L::kTileBytes) >> 4);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = ((ks >> 2) * 16384 + (ks & 3) * 32) >> 4;
            mma_bf16_ts(tmem + sb * 128, tmem + L::kKCol + kb * (D / 2) + 8 * ks, qd + off,
                        kIdesc, ks > 0 ? 1u : 0u);
          }
          if (L::kIssuers > 1) {
            __threadfence_block();
            *issued = gu + 1;
          }
          mma_commit(bar_s_full0 + 8 * sb);
          mma_commit(bar_q_empty0 + 8 * s);
        }
        mma_commit(bar_ktm_free0 + 8 * kb);  // this key buffer may be rewritten
        used0 += (it.R + 2) / 3;
        used1 += (it.R + 1) / 3;
        used2 += it.R / 3;
      }
      mma_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0, p.err);
    }
  } else {
    // ------------------------------------------------------------ summing groups
    const int quad = warp & 3;
    const int part_id = (warp - L::kGroupWarp0) >> 2;  // summing warpgroup
    const int grp = part_id / L::kSplit;       // row tiles u of an item with u % kGroups == grp
    const int hc = part_id % L::kSplit;        // kSplit 2: its 64 of the buffer's columns
    const int row = quad * 32 + lane;  // key j0 + row of the current item
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float c = p.scale_log2;
    bool ok = true;
    int copied = 0;  // group 0: key tiles copied into TMEM so far (by item count)
    // group 0 copies item k's key tile into TMEM buffer k & 1 (k = copied);
    // blocking: wait until the tile has landed and the buffer's MMAs are done
    auto copy_key_tile = [&](int k, int item_index, bool block) -> bool {
      const ColItem it = col_item(item_index, BG, NCT, NCTC, NQT, p.G);
      const int kb = k & 1;
      bool ready;
      if (block) {
        ready = mbar_wait(bar_k_full, k & 1, p.err, abort_flag);
        if (ready && k >= 2) ready = mbar_wait(bar_ktm_free0 + 8 * kb, ((k - 2) >> 1) & 1, p.err,
                                               abort_flag);
      } else {
        ready = mbar_test_wait(bar_k_full, k & 1) &&
                (k < 2 || mbar_test_wait(bar_ktm_free0 + 8 * kb, ((k - 2) >> 1) & 1));
      }
      ready = __all_sync(0xffffffffu, ready);
      if (!ready) return false;
      tc_fence_after();
      const float sc = (Q8 && !it.is_chunk && it.j0 + row < p.n)
                           ? p.k_scale[static_cast<size_t>(it.bg) * p.C + it.j0 + row] : 0.f;
      // 32 TMEM columns (64 elements) at a time
#pragma unroll
      for (int c0 = 0; c0 < D / 2; c0 += 32) {
        uint32_t w[32];
        if (Q8 && !it.is_chunk) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t piece[8];
            q8_dequant16(*reinterpret_cast<const uint4*>(smem + L::kCodeOff + row * D + 2 * c0 +
                                                         16 * i),
                         sc, piece);
#pragma unroll
            for (int j = 0; j < 8; ++j) w[8 * i + j] = piece[j];
          }
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int c16 = c0 / 4 + q;
            const uint4 v = *reinterpret_cast<const uint4*>(
                smem + L::kKOff + (c16 / 8) * 16384 + row * 128 + (((c16 % 8) ^ (row & 7)) * 16));
            w[4 * q] = v.x;
            w[4 * q + 1] = v.y;
            w[4 * q + 2] = v.z;
            w[4 * q + 3] = v.w;
          }
        }
        tmem_st32(lane_base + L::kKCol + kb * (D / 2) + c0, w);
      }
      mbar_arrive(bar_k_free);  // the staging may take the next key tile
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_ktm0 + 8 * kb);
      return true;
    };
    int gu0 = 0, k = 0;  // first global row tile of the current item; its index
    int used = 0;        // uses of this group's S buffer so far
    for (int i = first; i < items && ok; i += stride, ++k) {
      const ColItem it = col_item(i, BG, NCT, NCTC, NQT, p.G);
      if (part_id == 0 && copied == k) {  // this item's key tile must be in TMEM first
        ok = copy_key_tile(k, i, true);
        if (!ok) break;
        ++copied;
      }
      float acc = 0.f;
      // this group's row tiles of the item, u = grp, grp + 3, ... (global
      // index gu0 + u), so the order of the sums depends on the item alone
      for (int u = grp; u < it.R; u += L::kGroups, ++used) {
        const int gu = gu0 + u;
        if (part_id == 0 && copied == k + 1 && i + stride < items) {  // the next item's key tile, early
          if (copy_key_tile(k + 1, i + stride, false)) ++copied;
        }
        const int sl = gu % L::kLseStages;
        const int sb = grp;
        ok = mbar_wait(bar_s_full0 + 8 * sb, used & 1, p.err, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const int qt = it.qt_min + it.tile_of(u) % it.span;
        const bool diag = it.is_chunk && qt == it.kt;
        float part[4] = {0.f, 0.f, 0.f, 0.f};
        if (L::kSplit == 2) {
          // this warpgroup's 64 columns, 32 at a time; its share of the
          // buffer is free once the second piece is in registers
          uint32_t v[32];
          tmem_ld32(lane_base + sb * 128 + 64 * hc, v);
          tmem_wait_ld();
          ok = mbar_wait(bar_l_full0 + 8 * sl, (gl_parity(gu, L::kLseStages)), p.err, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          const float4* nlse4 = reinterpret_cast<const float4*>(smem + L::kLseOff + sl * 512) + 16 * hc;
          if (diag)
            sum_piece<true>(v, nlse4, c, row - 64 * hc, part);
          else
            sum_piece<false>(v, nlse4, c, 0, part);
          tmem_ld32(lane_base + sb * 128 + 64 * hc + 32, v);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(bar_s_empty0 + 8 * sb);
          if (diag)
            sum_piece<true>(v, nlse4 + 8, c, row - 64 * hc - 32, part);
          else
            sum_piece<false>(v, nlse4 + 8, c, 0, part);
        } else {
          uint32_t v[2][32];
          tmem_ld32(lane_base + sb * 128, v[0]);
          tmem_ld32(lane_base + sb * 128 + 32, v[1]);
          tmem_wait_ld();
          ok = mbar_wait(bar_l_full0 + 8 * sl, (gl_parity(gu, L::kLseStages)), p.err, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          const float4* nlse4 = reinterpret_cast<const float4*>(smem + L::kLseOff + sl * 512);
          if (diag)
            sum_tile<true>(v[0], v[1], nlse4, c, row, part);
          else
            sum_tile<false>(v[0], v[1], nlse4, c, 0, part);
          tmem_ld32(lane_base + sb * 128 + 64, v[0]);
          tmem_ld32(lane_base + sb * 128 + 96, v[1]);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(bar_s_empty0 + 8 * sb);
          if (diag)
            sum_tile<true>(v[0], v[1], nlse4 + 16, c, row - 64, part);
          else
            sum_tile<false>(v[0], v[1], nlse4 + 16, c, 0, part);
        }
        acc += (part[0] + part[1]) + (part[2] + part[3]);
        mbar_arrive(bar_l_empty0 + 8 * sl);
      }
      if (!ok) break;
      // this group's partial of the item (in the set of item k, once the
      // set's previous item is combined); the last summing warpgroup to get
      // here for a key adds the partials in warpgroup order and writes the
      // summed weight
      const int set = k % L::kRedSets;
      const int use = k / L::kRedSets;
      const int slot = set * 128 + row;
      if (done[slot] < use) {
        const uint64_t t0 = global_timer_ns();
        while (done[slot] < use) {
          if (*abort_flag) {
            ok = false;
            break;
          }
          if (global_timer_ns() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicOr(p.err, kDevErrTimeout);
            ok = false;
            break;
          }
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      red[(set * L::kParts + part_id) * 128 + row] = acc;
      __threadfence_block();
      if (atomicAdd(&cnt[slot], 1) == L::kParts * use + L::kParts - 1) {
        __threadfence_block();
        float total = 0.f;
#pragma unroll
        for (int gr = 0; gr < L::kParts; ++gr) total += red[(set * L::kParts + gr) * 128 + row];
        __threadfence_block();
        done[slot] = use + 1;
        float* out = p.colsum + static_cast<size_t>(it.bg) * p.colsum_ld;
        const int key = it.j0 + row;
        if (!H2O_IN_BOUNDS(p.C + p.nq <= p.colsum_ld, p.err)) {
        } else if (it.is_chunk) {
          if (key < p.nq) out[p.C + key] = total;
        } else if (key < p.n) {
          out[key] = total;
        } else if (key < p.C) {
          out[key] = 0.f;
        }
      }
      gu0 += it.R;
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

template <int D, bool Q8>
static cudaError_t launch_colsum_persistent(const AttnMaps& m, const AttnParams& p,
                                           cudaStream_t st) {
  using L = PColLayout<D, Q8>;
  static int attr_bits[2] = {0, 0};
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(attn_colsum_persistent<D, Q8>),
                                   L::kAlloc, attr_bits);
  if (e != cudaSuccess) return e;
  static int sms = 0;  // one CTA per SM
  if (sms == 0) {
    int dev = 0, v = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    sms = v;
  }
  const long long items = static_cast<long long>(p.B) * p.Hkv * (cdiv(p.n, 128) + cdiv(p.nq, 128));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(std::max<long long>(1, std::min<long long>(items, sms))));
  cfg.blockDim = dim3(L::kThreads);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attn_colsum_persistent<D, Q8>, m.q, m.kc, m.kn, p);
}

// The persistent variant (one CTA per SM over a list of key tiles) or one
// CTA per key tile.
constexpr bool kColsumPersistent = true;

cudaError_t launch_attn_colsum_bf16(int head_dim, const AttnMaps& m, const AttnParams& p,
                                    cudaStream_t st) {
  const bool q8 = p.k_scale != nullptr;  // int8 cache
  if (kColsumPersistent) {
    if (head_dim == 128)
      return q8 ? launch_colsum_persistent<128, true>(m, p, st)
                : launch_colsum_persistent<128, false>(m, p, st);
    return q8 ? launch_colsum_persistent<64, true>(m, p, st)
              : launch_colsum_persistent<64, false>(m, p, st);
  }
  if (head_dim == 128) return q8 ? launch_colsum<128, true>(m, p, st) : launch_colsum<128, false>(m, p, st);
  return q8 ? launch_colsum<64, true>(m, p, st) : launch_colsum<64, false>(m, p, st);
}

}  // namespace h2o
