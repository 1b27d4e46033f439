// attn_fwd.cu -- attention forward over [cache slots ++ chunk keys] with
// per-row log-sum-exp, on sm_100a tensor cores (tcgen05, TMEM, TMA).
//
// Computes, for one chunk, O = softmax(scale * Q K^T) V where query i of head h
// sees the n valid cache slots of KV head h / G and the chunk keys j <= i
// ("Learning how to Forget", §1: SDPA over a fixed-size KV cache plus the new
// chunk; FlashInfer-style 1 << N_q << N_k regime named in §2).  It also stores
// the row statistic lse2 = log2(sum_j 2^(x_ij)), x = scale*log2(e)*<q,k>,
// which the column-sum kernel uses to rebuild the normalised probabilities.
//
// One CTA = 128 consecutive queries of one (cache, head).  Warp roles:
//   warp 0      TMA producer: Q once, then K tiles of 128 keys into a ring
//               of 128-byte-swizzled shared-memory slots;
//   warp 10     TMA producer of the V tiles (a second ring);
//   warp 1      allocates TMEM; one thread issues tcgen05.mma:
//                 S(t) = Q K(t)^T   into one of two 128-column TMEM buffers,
//                 O   += P(t) V(t)  into 128 (or 64) TMEM columns;
//   warps 2..9  two threads per query row (= TMEM lane), one per half of the
//               128 keys of a tile (warps 2..5: keys 0..63, warps 6..9: keys
//               64..127): read their half of S(t) from TMEM, mask, exchange
//               the half-row maxima through shared memory, running max with
//               lazy rescaling of O (only when the max grows by more than
//               2^8; each thread rescales its half of the O row), P = 2^(x-m)
//               in bf16 written to a swizzled shared tile for the PV MMA (one
//               128-byte block per half); epilogue O / l on each half row.
#include <cuda_bf16.h>

#include "attn.h"
#include "sm100.cuh"

namespace h2o {

template <int D>
struct FwdLayout {
  static constexpr int kRegions = D / 64;          // 128-byte column blocks of a row
  static constexpr int kTileBytes = 128 * D * 2;   // 128 rows of Q, K or V
  static constexpr int kStages = (D == 128) ? 2 : 3;  // slots per ring (K ring, V ring)
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kTileBytes;
  static constexpr int kVOff = kKOff + kStages * kTileBytes;
  static constexpr int kPOff = kVOff + kStages * kTileBytes;
  static constexpr int kPBytes = 128 * 128 * 2;      // one P tile; two alternate
  static constexpr int kBarOff = kPOff + 2 * kPBytes;
  // q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], s_empty[2],
  // p_full[2], pv_done[2], drain, xchg[2] (half-row exchange, by tile parity)
  static constexpr int kNumBars = 1 + 4 * kStages + 4 + 4 + 1 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kXchgOff = kMiscOff + 16;  // [2 tiles][2 halves][128 rows] float
  static constexpr int kBytes = kXchgOff + 2 * 2 * 128 * 4;
  // room to align the base to 1024 bytes, within the per-CTA maximum
  static constexpr int kAlloc = (kBytes + 1024 < kMaxDynSmem) ? kBytes + 1024 : kMaxDynSmem;
  static_assert(kBytes <= kMaxDynSmem, "shared-memory layout too large");
  static constexpr int kTmemCols = 512;         // S0 | S1 | O
  static constexpr int kOCol = 256;
};

template <int D>
__global__ void __launch_bounds__(352, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_kc,
                    const __grid_constant__ CUtensorMap tm_vc,
                    const __grid_constant__ CUtensorMap tm_kn,
                    const __grid_constant__ CUtensorMap tm_vn, const AttnParams p) {
  using L = FwdLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  if ((smem - smem_raw) + L::kBytes > L::kAlloc) {  // cannot happen with an aligned base
    if (threadIdx.x == 0) atomicOr(p.err, kDevErrSmem);
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int NQT = cdiv(p.nq, 128);
  const int BH = p.B * p.Hq;
  const int bh = blockIdx.x % BH;
  const int qt = NQT - 1 - static_cast<int>(blockIdx.x / BH);  // longest rows first
  const int b = bh / p.Hq;
  const int h = bh % p.Hq;
  const int g = h / p.G;
  const int i0 = qt * 128;
  const int NCT = cdiv(p.n, 128);
  const int T = NCT + qt + 1;  // cache tiles, then chunk tiles 0..qt

  const uint32_t bar_q = sbase + L::kBarOff;
  const uint32_t bar_k_full0 = bar_q + 8;
  const uint32_t bar_k_empty0 = bar_k_full0 + 8 * L::kStages;
  const uint32_t bar_v_full0 = bar_k_empty0 + 8 * L::kStages;
  const uint32_t bar_v_empty0 = bar_v_full0 + 8 * L::kStages;
  const uint32_t bar_s_full0 = bar_v_empty0 + 8 * L::kStages;
  const uint32_t bar_s_empty0 = bar_s_full0 + 16;
  const uint32_t bar_p_full0 = bar_s_empty0 + 16;   // [2]: P(u) written, u & 1
  const uint32_t bar_pv_done0 = bar_p_full0 + 16;   // [2]: PV(u) complete, u & 1
  const uint32_t bar_drain = bar_pv_done0 + 16;
  const uint32_t bar_xchg0 = bar_drain + 8;         // [2]: both halves posted, t & 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar_k_full0 + 8 * s, 1);
      mbar_init(bar_k_empty0 + 8 * s, 1);
      mbar_init(bar_v_full0 + 8 * s, 1);
      mbar_init(bar_v_empty0 + 8 * s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_s_full0 + 8 * s, 1);
      mbar_init(bar_s_empty0 + 8 * s, 256);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_p_full0 + 8 * s, 256);
      mbar_init(bar_pv_done0 + 8 * s, 1);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_xchg0, 256);
    mbar_init(bar_xchg0 + 8, 256);
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

  if (warp == 0 || warp == 10) {
    // ------------------------------------------------------------ producers
    // warp 0 loads Q and the K tiles, warp 10 the V tiles; each ring advances
    // on its own, so K tiles stream ahead of the PV products.
    if (lane == 0) {
      const bool is_v = warp == 10;
      const uint32_t full0 = is_v ? bar_v_full0 : bar_k_full0;
      const uint32_t empty0 = is_v ? bar_v_empty0 : bar_k_empty0;
      const uint32_t ring = sbase + (is_v ? L::kVOff : L::kKOff);
      if (!is_v) {
        mbar_arrive_expect_tx(bar_q, L::kTileBytes);
        for (int r = 0; r < L::kRegions; ++r)
          tma_load_4d(sbase + L::kQOff + r * 16384, &tm_q, bar_q, r * 64, h, i0, b);
      }
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int s = t % L::kStages;
        if (t >= L::kStages &&
            !mbar_wait(empty0 + 8 * s, ((t / L::kStages) + 1) & 1, p.err, abort_flag))
          break;
        const bool chunk = t >= NCT;
        const int j0 = (chunk ? t - NCT : t) * 128;
        const uint32_t dst = ring + s * L::kTileBytes;
        mbar_arrive_expect_tx(full0 + 8 * s, L::kTileBytes);
        for (int r = 0; r < L::kRegions; ++r) {
          if (chunk)
            tma_load_4d(dst + r * 16384, is_v ? &tm_vn : &tm_kn, full0 + 8 * s, r * 64, g, j0, b);
          else
            tma_load_3d(dst + r * 16384, is_v ? &tm_vc : &tm_kc, full0 + 8 * s, r * 64, j0,
                        b * p.Hkv + g);
        }
        issued = t + 1;
      }
      // drain: every issued copy has landed before the CTA can exit
      if (!is_v) mbar_wait_drain(bar_q, 0, p.err);
      for (int t = (issued > L::kStages ? issued - L::kStages : 0); t < issued; ++t)
        mbar_wait_drain(full0 + 8 * (t % L::kStages), (t / L::kStages) & 1, p.err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);
      auto issue_pv = [&](int u) -> bool {
        if (!mbar_wait(bar_p_full0 + 8 * (u & 1), (u >> 1) & 1, p.err, abort_flag)) return false;
        const int s = u % L::kStages;
        if (!mbar_wait(bar_v_full0 + 8 * s, (u / L::kStages) & 1, p.err, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t vbase = sbase + L::kVOff + s * L::kTileBytes;
        const uint32_t pbase = sbase + L::kPOff + (u & 1) * L::kPBytes;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {  // 16 keys per MMA
          const uint64_t a = sw128_desc(pbase + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
          const uint64_t bd = sw128_desc(vbase + ks * 2048, 16384, 1024);
          mma_bf16_ss(tmem + L::kOCol, a, bd, kIdescPV, (u > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(bar_pv_done0 + 8 * (u & 1));
        mma_commit(bar_v_empty0 + 8 * s);
        return true;
      };
      // S(t) = Q K(t)^T into TMEM buffer t & 1
      auto issue_s = [&](int t) -> bool {
        const int s = t % L::kStages;
        if (!mbar_wait(bar_k_full0 + 8 * s, (t / L::kStages) & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t kbase = sbase + L::kKOff + s * L::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {  // 16 head-dim elements per MMA
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_bf16_ss(tmem + (t & 1) * 128, sw128_desc(sbase + L::kQOff + off, 16, 1024),
                      sw128_desc(kbase + off, 16, 1024), kIdescQK, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar_s_full0 + 8 * (t & 1));
        mma_commit(bar_k_empty0 + 8 * s);
        return true;
      };
      // Issue order S(0), S(1), then per tile t: S(t+2) as soon as the softmax
      // has read S(t) out of its buffer, PV(t) as soon as P(t) is written.  The
      // tensor core thus computes the logits two tiles ahead while the softmax
      // runs, instead of queueing S(t) behind PV(t-2).
      bool ok = mbar_wait(bar_q, 0, p.err, abort_flag);
      if (ok) ok = issue_s(0);
      if (ok && T > 1) ok = issue_s(1);
      for (int t = 0; t < T && ok; ++t) {
        if (t + 2 < T) {
          ok = mbar_wait(bar_s_empty0 + 8 * (t & 1), (t >> 1) & 1, p.err, abort_flag);
          if (ok) ok = issue_s(t + 2);
          if (!ok) break;
        }
        ok = issue_pv(t);
      }
      mma_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0, p.err);
    }
  } else {
    // ------------------------------------------------------------ softmax rows
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;      // keys [64*half, 64*half + 64) of each tile
    const int row = quad * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    float* xchg = reinterpret_cast<float*>(smem + L::kXchgOff);  // [2][2][128]
    const float c = p.scale_log2;
    float m_used = -INFINITY;
    float l = 0.f;  // this half's share of the row sum
    bool ok = true;
    uint32_t sv[64];
    for (int t = 0; t < T; ++t) {
      const int sb = t & 1;
      ok = mbar_wait(bar_s_full0 + 8 * sb, (t >> 1) & 1, p.err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      {
        uint32_t(&r0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[0]);
        uint32_t(&r1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[32]);
        const uint32_t sa = lane_base + sb * 128 + half * 64;
        tmem_ld32(sa, r0);
        tmem_ld32(sa + 32, r1);
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(bar_s_empty0 + 8 * sb);

      // visible keys of this half tile for this row (masking is needed only on
      // the partial last cache tile and on the diagonal chunk tile)
      int lim = 64;
      bool masked = false;
      if (t < NCT) {
        const int valid = p.n - t * 128 - half * 64;
        masked = (t == NCT - 1) && valid < 64;
        if (masked) lim = valid;  // may be <= 0: the whole half is masked
      } else if (t - NCT == qt) {
        masked = true;
        lim = row + 1 - half * 64;
      }
      if (masked) {
#pragma unroll
        for (int j = 0; j < 64; ++j)
          if (j >= lim) sv[j] = __float_as_uint(-INFINITY);
      }
      // half-row max: eight independent chains of three-input maxima
      float mx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        mx[e] = fmaxf(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1]));
#pragma unroll
      for (int j = 16; j < 64; j += 16) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          mx[e] = fmax3(mx[e], __uint_as_float(sv[j + 2 * e]), __uint_as_float(sv[j + 2 * e + 1]));
      }
      const float pm = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                             fmaxf(mx[6], mx[7]));
      // exchange half-row maxima (buffer and barrier alternate with the tile parity)
      xchg[(sb * 2 + half) * 128 + row] = pm;
      mbar_arrive(bar_xchg0 + 8 * sb);
      ok = mbar_wait(bar_xchg0 + 8 * sb, (t >> 1) & 1, p.err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const float mt = fmaxf(pm, xchg[(sb * 2 + (half ^ 1)) * 128 + row]) * c;
      const float m_new = fmaxf(m_used, mt);
      const bool need = m_new > m_used + 8.0f;

      // P(t) reuses the buffer PV(t-2) read
      if (t >= 2) {
        ok = mbar_wait(bar_pv_done0 + 8 * (t & 1), ((t >> 1) + 1) & 1, p.err, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      if (__any_sync(0xffffffffu, need)) {
        const float m_target = need ? m_new : m_used;
        if (t > 0) {
          // O must hold PV(t-1) before it is rescaled; each half rescales its columns
          ok = mbar_wait(bar_pv_done0 + 8 * ((t - 1) & 1), ((t - 1) >> 1) & 1, p.err, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          const float alpha = ex2_approx(m_used - m_target);
#pragma unroll
          for (int c0 = 0; c0 < D / 2; c0 += 32) {
            const uint32_t oa = lane_base + L::kOCol + half * (D / 2) + c0;
            uint32_t o[32];
            tmem_ld32(oa, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(oa, o);
          }
          tmem_wait_st();
          l *= alpha;
        }
        m_used = m_target;
      }
      const float msafe = (m_used == -INFINITY) ? 0.f : m_used;
      float ls[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) ls[e] = 0.f;
      uint8_t* prow = smem + L::kPOff + (t & 1) * L::kPBytes + half * 16384 + row * 128;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {  // 16-byte chunks of 8 keys
        float pe[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          pe[e] = ex2_approx(fmaf(__uint_as_float(sv[ch * 8 + e]), c, -msafe));
          ls[e] += pe[e];
        }
        uint4 v;
        v.x = pack_bf16x2(pe[0], pe[1]);
        v.y = pack_bf16x2(pe[2], pe[3]);
        v.z = pack_bf16x2(pe[4], pe[5]);
        v.w = pack_bf16x2(pe[6], pe[7]);
        *reinterpret_cast<uint4*>(prow + ((ch ^ (row & 7)) << 4)) = v;
      }
      l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_p_full0 + 8 * (t & 1));
    }
    // ------------------------------------------------------------ epilogue
    if (ok) {
      ok = mbar_wait(bar_pv_done0 + 8 * ((T - 1) & 1), ((T - 1) >> 1) & 1, p.err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
    }
    // row sum = both halves' shares (same reference max m_used), exchanged in
    // the parity slot the last tile did not use
    if (ok) {
      const int xs = T & 1;
      xchg[(xs * 2 + half) * 128 + row] = l;
      mbar_arrive(bar_xchg0 + 8 * xs);
      ok = mbar_wait(bar_xchg0 + 8 * xs, (T >> 1) & 1, p.err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      const float l_row = l + xchg[((T & 1) * 2 + (half ^ 1)) * 128 + row];
      tc_fence_after();
      const int i = i0 + row;
      const float inv = 1.f / l_row;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) +
                            ((static_cast<size_t>(b) * p.nq + i) * p.Hq + h) * D + half * (D / 2);
#pragma unroll
      for (int c0 = 0; c0 < D / 2; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(lane_base + L::kOCol + half * (D / 2) + c0, o);
        tmem_wait_ld();
        if (i < p.nq) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[q4 * 8 + 0]) * inv, __uint_as_float(o[q4 * 8 + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(o[q4 * 8 + 2]) * inv, __uint_as_float(o[q4 * 8 + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(o[q4 * 8 + 4]) * inv, __uint_as_float(o[q4 * 8 + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(o[q4 * 8 + 6]) * inv, __uint_as_float(o[q4 * 8 + 7]) * inv);
            dst[q4] = v;
          }
        }
      }
      if (half == 0)
        p.lse2[(static_cast<size_t>(b) * p.Hq + h) * p.nq_pad + i] =
            (i < p.nq) ? m_used + __log2f(l_row) : INFINITY;
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

template <int D>
static cudaError_t launch_fwd(const AttnMaps& m, const AttnParams& p, cudaStream_t st) {
  using L = FwdLayout<D>;
  static int attr_bits[2] = {0, 0};
  if (!smem_attr_done(reinterpret_cast<const void*>(attn_fwd_kernel<D>), attr_bits)) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
  }
  const int grid = p.B * p.Hq * cdiv(p.nq, 128);
  attn_fwd_kernel<D><<<grid, 352, L::kAlloc, st>>>(m.q, m.kc, m.vc, m.kn, m.vn, p);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd_bf16(int head_dim, const AttnMaps& m, const AttnParams& p,
                                 cudaStream_t st) {
  return head_dim == 128 ? launch_fwd<128>(m, p, st) : launch_fwd<64>(m, p, st);
}

}  // namespace h2o
