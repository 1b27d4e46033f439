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
//   warp 0      TMA producer: Q once, then K and V tiles of 128 keys into a
//               ring of 128-byte-swizzled shared-memory slots;
//   warp 1      allocates TMEM; one thread issues tcgen05.mma:
//                 S(t) = Q K(t)^T   into one of two 128-column TMEM buffers,
//                 O   += P(t) V(t)  into 128 (or 64) TMEM columns;
//   warps 2..5  one thread per query row (= TMEM lane): read S(t) from TMEM,
//               mask, running max with lazy rescaling of O (only when the max
//               grows by more than 2^8), P = 2^(x - m) in bf16 written to a
//               swizzled shared tile for the PV MMA; epilogue O / l.
#include <cuda_bf16.h>

#include "attn.h"
#include "sm100.cuh"

namespace h2o {

template <int D>
struct FwdLayout {
  static constexpr int kRegions = D / 64;          // 128-byte column blocks of a row
  static constexpr int kTileBytes = 128 * D * 2;   // 128 rows of Q, K or V
  static constexpr int kStages = (D == 128) ? 4 : 6;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = kQOff + kTileBytes;
  static constexpr int kPOff = kKVOff + kStages * kTileBytes;
  static constexpr int kPBytes = 128 * 128 * 2;
  static constexpr int kBarOff = kPOff + kPBytes;
  // q_full, kv_full[S], kv_empty[S], s_full[2], s_empty[2], p_full, pv_done, drain
  static constexpr int kNumBars = 1 + 2 * kStages + 4 + 3;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024 bytes
  static constexpr int kTmemCols = 512;         // S0 | S1 | O
  static constexpr int kOCol = 256;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_kc,
                    const __grid_constant__ CUtensorMap tm_vc,
                    const __grid_constant__ CUtensorMap tm_kn,
                    const __grid_constant__ CUtensorMap tm_vn, const AttnParams p) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
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
  const uint32_t bar_kv_full0 = bar_q + 8;
  const uint32_t bar_kv_empty0 = bar_kv_full0 + 8 * L::kStages;
  const uint32_t bar_s_full0 = bar_kv_empty0 + 8 * L::kStages;
  const uint32_t bar_s_empty0 = bar_s_full0 + 16;
  const uint32_t bar_p_full = bar_s_empty0 + 16;
  const uint32_t bar_pv_done = bar_p_full + 8;
  const uint32_t bar_drain = bar_pv_done + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar_kv_full0 + 8 * s, 1);
      mbar_init(bar_kv_empty0 + 8 * s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_s_full0 + 8 * s, 1);
      mbar_init(bar_s_empty0 + 8 * s, 128);
    }
    mbar_init(bar_p_full, 128);
    mbar_init(bar_pv_done, 1);
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
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;  // K/V ring uses issued so far
      mbar_arrive_expect_tx(bar_q, L::kTileBytes);
      for (int r = 0; r < L::kRegions; ++r)
        tma_load_4d(sbase + L::kQOff + r * 16384, &tm_q, bar_q, r * 64, h, i0, b);
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        const bool chunk = t >= NCT;
        const int j0 = (chunk ? t - NCT : t) * 128;
        for (int w = 0; w < 2; ++w) {
          const int u = 2 * t + w;
          const int s = u % L::kStages;
          if (u >= L::kStages &&
              !mbar_wait(bar_kv_empty0 + 8 * s, ((u / L::kStages) + 1) & 1, p.err, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t dst = sbase + L::kKVOff + s * L::kTileBytes;
          const uint32_t bar = bar_kv_full0 + 8 * s;
          mbar_arrive_expect_tx(bar, L::kTileBytes);
          for (int r = 0; r < L::kRegions; ++r) {
            if (chunk)
              tma_load_4d(dst + r * 16384, w ? &tm_vn : &tm_kn, bar, r * 64, g, j0, b);
            else
              tma_load_3d(dst + r * 16384, w ? &tm_vc : &tm_kc, bar, r * 64, j0, b * p.Hkv + g);
          }
          issued = u + 1;
        }
      }
      // drain: every issued copy has landed before the CTA can exit
      mbar_wait_drain(bar_q, 0, p.err);
      for (int u = (issued > L::kStages ? issued - L::kStages : 0); u < issued; ++u)
        mbar_wait_drain(bar_kv_full0 + 8 * (u % L::kStages), (u / L::kStages) & 1, p.err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);
      auto issue_pv = [&](int u) -> bool {
        if (!mbar_wait(bar_p_full, u & 1, p.err, abort_flag)) return false;
        const int uv = 2 * u + 1;
        const int s = uv % L::kStages;
        if (!mbar_wait(bar_kv_full0 + 8 * s, (uv / L::kStages) & 1, p.err, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t vbase = sbase + L::kKVOff + s * L::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {  // 16 keys per MMA
          const uint64_t a = sw128_desc(sbase + L::kPOff + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
          const uint64_t bd = sw128_desc(vbase + ks * 2048, 16384, 1024);
          mma_bf16_ss(tmem + L::kOCol, a, bd, kIdescPV, (u > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(bar_pv_done);
        mma_commit(bar_kv_empty0 + 8 * s);
        return true;
      };
      bool ok = mbar_wait(bar_q, 0, p.err, abort_flag);
      for (int t = 0; t < T && ok; ++t) {
        const int u = 2 * t;
        const int s = u % L::kStages;
        const int sb = t & 1;
        ok = mbar_wait(bar_kv_full0 + 8 * s, (u / L::kStages) & 1, p.err, abort_flag);
        if (ok && t >= 2) ok = mbar_wait(bar_s_empty0 + 8 * sb, ((t >> 1) + 1) & 1, p.err, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kbase = sbase + L::kKVOff + s * L::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {  // 16 head-dim elements per MMA
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_bf16_ss(tmem + sb * 128, sw128_desc(sbase + L::kQOff + off, 16, 1024),
                      sw128_desc(kbase + off, 16, 1024), kIdescQK, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar_s_full0 + 8 * sb);
        mma_commit(bar_kv_empty0 + 8 * s);
        if (t >= 1) ok = issue_pv(t - 1);
      }
      if (ok) issue_pv(T - 1);
      mma_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0, p.err);
    }
  } else {
    // ------------------------------------------------------------ softmax rows
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float c = p.scale_log2;
    float m_used = -INFINITY;
    float l = 0.f;
    bool ok = true;
    uint32_t sv[128];
    for (int t = 0; t < T; ++t) {
      const int sb = t & 1;
      ok = mbar_wait(bar_s_full0 + 8 * sb, (t >> 1) & 1, p.err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      {
        uint32_t(&r0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[0]);
        uint32_t(&r1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[32]);
        uint32_t(&r2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[64]);
        uint32_t(&r3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[96]);
        const uint32_t sa = lane_base + sb * 128;
        tmem_ld32(sa + 0, r0);
        tmem_ld32(sa + 32, r1);
        tmem_ld32(sa + 64, r2);
        tmem_ld32(sa + 96, r3);
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(bar_s_empty0 + 8 * sb);

      // number of visible keys of this tile for this row
      int lim;
      if (t < NCT) lim = min(128, p.n - t * 128);
      else if (t - NCT == qt) lim = row + 1;
      else lim = 128;
      float mt = -INFINITY;
#pragma unroll
      for (int j = 0; j < 128; ++j) {
        const float x = (j < lim) ? __uint_as_float(sv[j]) * c : -INFINITY;
        sv[j] = __float_as_uint(x);
        mt = fmaxf(mt, x);
      }
      const float m_new = fmaxf(m_used, mt);
      const bool need = m_new > m_used + 8.0f;

      if (t > 0) {
        ok = mbar_wait(bar_pv_done, (t - 1) & 1, p.err, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, need)) {
        const float m_target = need ? m_new : m_used;
        if (t > 0) {
          const float alpha = ex2_approx(m_used - m_target);
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(lane_base + L::kOCol + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(lane_base + L::kOCol + c0, o);
          }
          tmem_wait_st();
          l *= alpha;
        }
        m_used = m_target;
      }
      const float msafe = (m_used == -INFINITY) ? 0.f : m_used;
      float ls = 0.f;
      uint8_t* prow = smem + L::kPOff + row * 128;
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {  // 16-byte chunks of 8 keys
        float pe[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          pe[e] = ex2_approx(__uint_as_float(sv[ch * 8 + e]) - msafe);
          ls += pe[e];
        }
        uint4 v;
        v.x = pack_bf16x2(pe[0], pe[1]);
        v.y = pack_bf16x2(pe[2], pe[3]);
        v.z = pack_bf16x2(pe[4], pe[5]);
        v.w = pack_bf16x2(pe[6], pe[7]);
        const int region = ch >> 3;
        const int cc = ch & 7;
        *reinterpret_cast<uint4*>(prow + region * 16384 + ((cc ^ (row & 7)) << 4)) = v;
      }
      l += ls;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_p_full);
    }
    // ------------------------------------------------------------ epilogue
    if (ok) {
      ok = mbar_wait(bar_pv_done, (T - 1) & 1, p.err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const int i = i0 + row;
      const float inv = 1.f / l;
      __nv_bfloat16* orow =
          reinterpret_cast<__nv_bfloat16*>(p.out) + ((static_cast<size_t>(b) * p.nq + i) * p.Hq + h) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(lane_base + L::kOCol + c0, o);
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
      p.lse2[(static_cast<size_t>(b) * p.Hq + h) * p.nq_pad + i] =
          (i < p.nq) ? m_used + __log2f(l) : INFINITY;
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
  attn_fwd_kernel<D><<<grid, 192, L::kAlloc, st>>>(m.q, m.kc, m.vc, m.kn, m.vn, p);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd_bf16(int head_dim, const AttnMaps& m, const AttnParams& p,
                                 cudaStream_t st) {
  return head_dim == 128 ? launch_fwd<128>(m, p, st) : launch_fwd<64>(m, p, st);
}

}  // namespace h2o
