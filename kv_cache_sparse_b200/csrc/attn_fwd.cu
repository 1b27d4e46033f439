// attn_fwd.cu -- attention forward over [cache slots ++ chunk keys] with
// per-row log-sum-exp, on sm_100a tensor cores (tcgen05, TMEM, TMA).
//
// Computes, for one chunk, O = softmax(scale * Q K^T) V where query i of head h
// sees the n valid cache slots of KV head h / G and the chunk keys j <= i
// ("Learning how to Forget", §1: SDPA over a fixed-size KV cache plus the new
// chunk; FlashInfer-style 1 << N_q << N_k regime named in §2).  It also stores
// the row statistic lse2 = log2(sum_j 2^(x_ij)), x = scale*log2(e)*<q,k>
// (negated), which the column-sum kernel uses to rebuild the normalised
// probabilities.
//
// One CTA = two 128-row query tiles ("A" and "B") of the same KV head --
// normally two heads of one GQA group at the same 128 queries -- that share
// every K and V tile.  Each tile has its own softmax warpgroup, and the two
// groups alternate on the tensor core, so that one group's exponentials run
// while the other group's logits are being read and reduced.
//   warp 0      TMA: both Q tiles, then K(t) and V(t) into two rings of 2 slots
//   warp 1      TMEM allocation; one thread issues tcgen05.mma:
//                 S_X(t) = Q_X K(t)^T  into TMEM columns [128X, 128X+128)
//                 O_X   += P_X(t) V(t) into TMEM columns 256 + 128X, with
//                 P_X(t) read from TMEM (bf16, written over S_X(t))
//   warps 2..3  int8 cache only: dequantisation (below, with warps 4..7 too,
//               the softmax warps then being 8..15); otherwise idle
//   warps 4..7  softmax of tile A, warps 8..11 softmax of tile B: one thread
//               per query row (TMEM lane) reads its 128 logits once, takes
//               the row max, then P = 2^(x - m) (packed f32x2 arithmetic for
//               the scaling and the row sum) as bf16 back into TMEM; lazy
//               rescaling of O (only when the max grows by more than 2^8);
//               epilogue O / l and lse2.
// Ordering: the MMA thread issues PV_X(t) and then S_X(t+1) into the same
// TMEM columns; the commit that signals S_X(t+1) also covers PV_X(t), so the
// softmax that sees S_X(t+1) may rescale O_X and overwrite P_X.
//
// The int8 cache (Q8, q8.cuh): warp 0 brings a cache tile's codes of K and of
// V into one staging buffer each (TMA, no swizzle), and warps 2 to 7
// dequantise them into the same bf16 rings the MMA reads (128-byte swizzle),
// with the row scales; the chunk's own tiles still arrive in bf16 by TMA.
#include <cuda_bf16.h>

#include "attn.h"
#include "q8.cuh"
#include "sm100.cuh"

namespace h2o {

// Pairs of keys (of every 8) whose exponentials run on the FMA pipe
// (exp2_fma2) rather than the special function unit (16 per clock per SM).
// Measured on the headline cache: 0 of 8 157.7 us, 2 of 8 172.7 us, 3 of 8
// 179.2 us -- the tile's softmax chain is bound by latency, not by the
// unit's throughput, and the extra instructions lengthen it.
constexpr int kFwdEmuPairsOf8 = 0;
// Softmax warps spin on the S barrier instead of suspending (a suspended
// warp wakes up later, on the critical chain of its tile).
constexpr bool kFwdSpinS = false;

template <int D, bool Q8 = false>
struct FwdLayout {
  static constexpr int kRegions = D / 64;         // 128-byte column blocks of a row
  static constexpr int kTileBytes = 128 * D * 2;  // 128 rows of Q, K or V
  static constexpr int kKStages = 2;
  static constexpr int kVStages = 2;
  static constexpr int kQOff = 0;  // Q_A, Q_B
  static constexpr int kKOff = kQOff + 2 * kTileBytes;
  static constexpr int kVOff = kKOff + kKStages * kTileBytes;
  // Q8: int8 codes of one K and one V cache tile (128 rows x D bytes each)
  static constexpr int kCodeBytes = Q8 ? 128 * D : 0;
  static constexpr int kK8Off = kVOff + kVStages * kTileBytes;
  static constexpr int kV8Off = kK8Off + kCodeBytes;
  static constexpr int kBarOff = kV8Off + kCodeBytes;
  // q_full, k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], s_full[2], p_full[2],
  // o_done[2], drain; Q8: k8_full, k8_empty, v8_full, v8_empty
  static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 2 + 2 + 2 + 1 + (Q8 ? 4 : 0);
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = (kBytes + 1024 < kMaxDynSmem) ? kBytes + 1024 : kMaxDynSmem;
  static_assert(kBytes <= kMaxDynSmem, "shared-memory layout too large");
  static constexpr int kTmemCols = 512;  // S/P_A | S/P_B | O_A | O_B
  // warpgroup 0: warp 0 TMA, warp 1 MMA, warps 2-3 dequantise (Q8) or idle;
  // Q8: warpgroup 1 dequantises too (six converter warps); then two softmax
  // warpgroups, tiles A and B.  The non-softmax warpgroups give registers
  // back so that the softmax warpgroups hold kSoftmaxRegs each (384 threads:
  // launched with 168 a thread; 512: with 128).
  static constexpr int kSoftWarp0 = Q8 ? 8 : 4;      // first softmax warp
  static constexpr int kConvThreads = 32 * (kSoftWarp0 - 2);
  static constexpr int kThreads = 32 * kSoftWarp0 + 256;
  static constexpr uint32_t kLoadRegs = Q8 ? 56 : 80;
  static constexpr uint32_t kSoftmaxRegs = 200;
  static_assert(32 * kSoftWarp0 * kLoadRegs + 256 * kSoftmaxRegs <=
                    kThreads * ((65536 / kThreads) & ~7),
                "register budget");
};

template <int D, bool Q8>
__global__ void __launch_bounds__(FwdLayout<D, Q8>::kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_kc,
                    const __grid_constant__ CUtensorMap tm_vc,
                    const __grid_constant__ CUtensorMap tm_kn,
                    const __grid_constant__ CUtensorMap tm_vn, const AttnParams p) {
  using L = FwdLayout<D, Q8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  if ((smem - smem_raw) + L::kBytes > L::kAlloc) {  // cannot happen with an aligned base
    if (threadIdx.x == 0) atomicOr(p.err, kDevErrSmem);
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // the column-sum kernel may start setting up on idle SMs; it waits for this
  // grid to complete before it reads the row statistics
  griddep_launch_dependents();

  // ---- work: items (head of the group, query tile) of one (cache, KV head),
  // longest first, taken two at a time
  const int NQT = cdiv(p.nq, 128);
  const int items = p.G * NQT;
  const int BG = p.B * p.Hkv;
  const int bg = blockIdx.x % BG;
  const int pair = blockIdx.x / BG;
  const int b = bg / p.Hkv;
  const int g = bg % p.Hkv;
  const int NCT = cdiv(p.n, 128);
  // tile A = item 2*pair, tile B = item 2*pair + 1 (absent when items is odd)
  const int kA = 2 * pair, kB = 2 * pair + 1;
  const int qtA = NQT - 1 - kA / p.G, hA = g * p.G + kA % p.G;
  const int qtB = kB < items ? NQT - 1 - kB / p.G : 0, hB = g * p.G + kB % p.G;
  const int TA = NCT + qtA + 1;                  // cache tiles, then chunk tiles 0..qt
  const int TB = kB < items ? NCT + qtB + 1 : 0;  // TA >= TB
  const int Tmax = TA;

  const uint32_t bar_q = sbase + L::kBarOff;
  const uint32_t bar_k_full0 = bar_q + 8;
  const uint32_t bar_k_empty0 = bar_k_full0 + 8 * L::kKStages;
  const uint32_t bar_v_full0 = bar_k_empty0 + 8 * L::kKStages;
  const uint32_t bar_v_empty0 = bar_v_full0 + 8 * L::kVStages;
  const uint32_t bar_s_full0 = bar_v_empty0 + 8 * L::kVStages;  // [2]: S_X(t) (and PV_X(t-1)) done
  const uint32_t bar_p_full0 = bar_s_full0 + 16;                // [2]: P_X(t) in TMEM
  const uint32_t bar_o_done0 = bar_p_full0 + 16;                // [2]: last PV_X done
  const uint32_t bar_drain = bar_o_done0 + 16;
  const uint32_t bar_k8_full = bar_drain + 8, bar_k8_empty = bar_drain + 16;  // Q8 only
  const uint32_t bar_v8_full = bar_drain + 24, bar_v8_empty = bar_drain + 32;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < L::kKStages; ++s) {
      mbar_init(bar_k_full0 + 8 * s, 1);
      mbar_init(bar_k_empty0 + 8 * s, 1);
    }
    for (int s = 0; s < L::kVStages; ++s) {
      mbar_init(bar_v_full0 + 8 * s, 1);
      mbar_init(bar_v_empty0 + 8 * s, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar_s_full0 + 8 * x, 1);
      mbar_init(bar_p_full0 + 8 * x, 128);
      mbar_init(bar_o_done0 + 8 * x, 1);
    }
    mbar_init(bar_drain, 1);
    if (Q8) {
      mbar_init(bar_k8_full, 1);
      mbar_init(bar_k8_empty, 1);
      mbar_init(bar_v8_full, 1);
      mbar_init(bar_v8_empty, 1);
    }
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
  if (warp < L::kSoftWarp0) {
  // the TMA / MMA / dequantising warpgroups hand registers to the softmax groups
  warpgroup_reg_dec<L::kLoadRegs>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, (TB > 0 ? 2 : 1) * L::kTileBytes);
      for (int r = 0; r < L::kRegions; ++r)
        tma_load_4d(sbase + L::kQOff + r * 16384, &tm_q, bar_q, r * 64, hA, qtA * 128, b);
      if (TB > 0)
        for (int r = 0; r < L::kRegions; ++r)
          tma_load_4d(sbase + L::kQOff + L::kTileBytes + r * 16384, &tm_q, bar_q, r * 64, hB,
                      qtB * 128, b);
      int issued_k = 0, issued_v = 0, issued8 = 0;
      bool ok = true;
      for (int t = 0; t < Tmax && ok; ++t) {
        const bool chunk = t >= NCT;
        const int j0 = (chunk ? t - NCT : t) * 128;
        if (Q8 && !chunk) {  // the codes of K(t) and V(t) into the staging buffers
          for (int w = 0; w < 2; ++w) {
            const uint32_t full = w ? bar_v8_full : bar_k8_full;
            const uint32_t empty = w ? bar_v8_empty : bar_k8_empty;
            if (t >= 1 && !mbar_wait(empty, (t + 1) & 1, p.err, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(full, L::kCodeBytes);
            tma_load_3d(sbase + (w ? L::kV8Off : L::kK8Off), w ? &tm_vc : &tm_kc, full, 0, j0,
                        b * p.Hkv + g);
          }
          issued8 = t + 1;
          continue;
        }
        for (int w = 0; w < 2; ++w) {  // K(t), then V(t)
          const int NS = w ? L::kVStages : L::kKStages;
          const uint32_t full0 = w ? bar_v_full0 : bar_k_full0;
          const uint32_t empty0 = w ? bar_v_empty0 : bar_k_empty0;
          const int s = t % NS;
          if (t >= NS && !mbar_wait(empty0 + 8 * s, ((t / NS) + 1) & 1, p.err, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t dst = sbase + (w ? L::kVOff : L::kKOff) + s * L::kTileBytes;
          mbar_arrive_expect_tx(full0 + 8 * s, L::kTileBytes);
          for (int r = 0; r < L::kRegions; ++r) {
            if (chunk)
              tma_load_4d(dst + r * 16384, w ? &tm_vn : &tm_kn, full0 + 8 * s, r * 64, g, j0, b);
            else
              tma_load_3d(dst + r * 16384, w ? &tm_vc : &tm_kc, full0 + 8 * s, r * 64, j0,
                          b * p.Hkv + g);
          }
          if (w) issued_v = t + 1; else issued_k = t + 1;
        }
      }
      // drain: every issued copy has landed before the CTA can exit
      mbar_wait_drain(bar_q, 0, p.err);
      if (Q8 && issued8 > 0) {
        mbar_wait_drain(bar_k8_full, (issued8 - 1) & 1, p.err);
        mbar_wait_drain(bar_v8_full, (issued8 - 1) & 1, p.err);
      }
      const int t_tma = Q8 ? NCT : 0;  // Q8: the cache tiles were not copied by TMA
      for (int t = max(t_tma, issued_k - L::kKStages); t < issued_k; ++t)
        mbar_wait_drain(bar_k_full0 + 8 * (t % L::kKStages), (t / L::kKStages) & 1, p.err);
      for (int t = max(t_tma, issued_v - L::kVStages); t < issued_v; ++t)
        mbar_wait_drain(bar_v_full0 + 8 * (t % L::kVStages), (t / L::kVStages) & 1, p.err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);
      auto issue_s = [&](int x, int t) {  // S_X(t) = Q_X K(t)^T
        const uint32_t kbase = sbase + L::kKOff + (t % L::kKStages) * L::kTileBytes;
        const uint32_t qbase = sbase + L::kQOff + x * L::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {  // 16 head-dim elements per MMA
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_bf16_ss(tmem + 128 * x, sw128_desc(qbase + off, 16, 1024),
                      sw128_desc(kbase + off, 16, 1024), kIdescQK, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar_s_full0 + 8 * x);
      };
      auto issue_pv = [&](int x, int t) {  // O_X += P_X(t) V(t), P_X from TMEM
        const uint32_t vbase = sbase + L::kVOff + (t % L::kVStages) * L::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {  // 16 keys per MMA = 8 TMEM columns of P
          mma_bf16_ts(tmem + 256 + 128 * x, tmem + 128 * x + 8 * ks,
                      sw128_desc(vbase + ks * 2048, 16384, 1024), kIdescPV,
                      (t > 0 || ks > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait_spin(bar_q, 0, p.err, abort_flag);
      if (ok) ok = mbar_wait_spin(bar_k_full0, 0, p.err, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        if (TB > 0) issue_s(1, 0);
        mma_commit(bar_k_empty0);
      }
      for (int t = 0; t < Tmax && ok; ++t) {
        ok = mbar_wait_spin(bar_v_full0 + 8 * (t % L::kVStages), (t / L::kVStages) & 1, p.err,
                       abort_flag);
        for (int x = 0; x < 2 && ok; ++x) {
          const int Tx = x ? TB : TA;
          if (t >= Tx) continue;
          ok = mbar_wait_spin(bar_p_full0 + 8 * x, t & 1, p.err, abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_pv(x, t);
          if (t + 1 < Tx) {
            if (x == 0) {  // tile A always needs K(t+1) when tile B does
              const int s1 = (t + 1) % L::kKStages;
              ok = mbar_wait_spin(bar_k_full0 + 8 * s1, ((t + 1) / L::kKStages) & 1, p.err, abort_flag);
              if (!ok) break;
              tc_fence_after();
            }
            issue_s(x, t + 1);
          } else {
            mma_commit(bar_o_done0 + 8 * x);
          }
        }
        if (!ok) break;
        mma_commit(bar_v_empty0 + 8 * (t % L::kVStages));
        if (t + 1 < Tmax) mma_commit(bar_k_empty0 + 8 * ((t + 1) % L::kKStages));
      }
      mma_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0, p.err);
    }
  } else {
    // warps 2 .. kSoftWarp0-1: no role without the int8 cache
    if (Q8) {
    // ------------------------------------------------------------ dequantise (Q8)
    // cache tile t: codes (staging) -> bf16 ring slot t % 2 of K, then of V.
    // 128 x D codes in pieces of 16 (one 16-byte row piece each, consecutive
    // threads on consecutive pieces); each piece becomes two 16-byte chunks of
    // its 128-byte region row, at chunk index ^ (row & 7) (the swizzle).
    constexpr int kPer = D / 16;                    // pieces per row
    constexpr int kNC = L::kConvThreads;
    constexpr int kJobs = (128 * kPer + kNC - 1) / kNC;  // pieces per thread and tile
    const int ct = threadIdx.x - 64;                // 0 .. kNC - 1
    bool ok = true;
    for (int t = 0; t < NCT && ok; ++t) {
      const int j0 = t * 128;
      for (int w = 0; w < 2 && ok; ++w) {
        const float* scale = (w ? p.v_scale : p.k_scale) + static_cast<size_t>(bg) * p.C;
        float sc[kJobs];
#pragma unroll
        for (int k = 0; k < kJobs; ++k) {
          const int r = (ct + kNC * k) / kPer;
          sc[k] = (ct + kNC * k < 128 * kPer && j0 + r < p.n) ? scale[j0 + r] : 0.f;
        }
        const int NS = w ? L::kVStages : L::kKStages;
        const int s = t % NS;
        ok = mbar_wait(w ? bar_v8_full : bar_k8_full, t & 1, p.err, abort_flag);
        if (ok && t >= NS)
          ok = mbar_wait((w ? bar_v_empty0 : bar_k_empty0) + 8 * s, ((t / NS) + 1) & 1, p.err,
                         abort_flag);
        ok = named_bar_and(1, kNC, ok);  // every converter thread takes the same branch
        if (!ok) break;
        const uint8_t* codes = smem + (w ? L::kV8Off : L::kK8Off);
        uint8_t* dst = smem + (w ? L::kVOff : L::kKOff) + s * L::kTileBytes;
#pragma unroll 4
        for (int k = 0; k < kJobs; ++k) {
          const int job = ct + kNC * k;
          if (job >= 128 * kPer) break;
          const int r = job / kPer, i = job % kPer;
          uint32_t wv[8];
          q8_dequant16(*reinterpret_cast<const uint4*>(codes + r * D + 16 * i), sc[k], wv);
          const int e = 16 * i;
          const int reg = e / 64, c16 = (e % 64) / 8;
          uint8_t* rowp = dst + reg * 16384 + r * 128;
          *reinterpret_cast<uint4*>(rowp + ((c16 ^ (r & 7)) * 16)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          *reinterpret_cast<uint4*>(rowp + (((c16 + 1) ^ (r & 7)) * 16)) =
              make_uint4(wv[4], wv[5], wv[6], wv[7]);
        }
        fence_proxy_async_smem();  // the MMA reads the operand through the async proxy
        named_bar_sync(1, kNC);    // all converters are done with the codes and the slot
        if (ct == 0) {
          mbar_arrive((w ? bar_v_full0 : bar_k_full0) + 8 * s);
          mbar_arrive(w ? bar_v8_empty : bar_k8_empty);
        }
      }
    }
    }
  }
  } else {
    // ------------------------------------------------------------ softmax rows
    warpgroup_reg_inc<L::kSoftmaxRegs>();
    const int x = (warp - L::kSoftWarp0) >> 2;  // tile A or B
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int T = x ? TB : TA;
    const int qt = x ? qtB : qtA;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t s_col = lane_base + 128 * x;        // S_X, then P_X over its first 64 columns
    const uint32_t o_col = lane_base + 256 + 128 * x;  // O_X
    const float c = p.scale_log2;
    float m_used = -INFINITY;
    float l = 0.f;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      ok = kFwdSpinS ? mbar_wait_spin(bar_s_full0 + 8 * x, t & 1, p.err, abort_flag)
                     : mbar_wait(bar_s_full0 + 8 * x, t & 1, p.err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // visible keys of this tile for this row (masking is needed only on the
      // partial last cache tile and on the diagonal chunk tile)
      int lim = 128;
      bool masked = false;
      if (t < NCT) {
        masked = (t == NCT - 1) && (p.n - t * 128 < 128);
        if (masked) lim = p.n - t * 128;
      } else if (t - NCT == qt) {
        masked = true;
        lim = row + 1;
      }
      // the tile's 128 logits of this row, read once
      uint32_t v[128];
#pragma unroll
      for (int c0 = 0; c0 < 128; c0 += 32)
        tmem_ld32(s_col + c0, *reinterpret_cast<uint32_t(*)[32]>(&v[c0]));
      tmem_wait_ld();
      if (masked) {
#pragma unroll
        for (int j = 0; j < 128; ++j)
          if (j >= lim) v[j] = __float_as_uint(-INFINITY);
      }
      // row max of the raw logits (scale > 0): eight chains of 3-input maxima
      float mx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        mx[e] = fmaxf(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
#pragma unroll
      for (int j = 16; j < 128; j += 16) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          mx[e] = fmax3(mx[e], __uint_as_float(v[j + 2 * e]), __uint_as_float(v[j + 2 * e + 1]));
      }
      const float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                             fmaxf(mx[6], mx[7])) * c;
      const float m_new = fmaxf(m_used, mt);
      const bool need = m_new > m_used + 8.0f;
      // a warp moves its reference max when one of its rows needs it; O and l
      // are rescaled after P is built (the logits are dead by then)
      const bool rescale = __any_sync(0xffffffffu, need);
      float alpha = 1.f;
      if (rescale) {
        const float m_target = need ? m_new : m_used;
        alpha = ex2_approx(m_used - m_target);
        m_used = m_target;
      }
      const float nm = (m_used == -INFINITY) ? 0.f : -m_used;
      // probabilities (masked logits are -inf and give 0), row sum, bf16 P back
      // into TMEM over the first 64 columns of the S buffer
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
          float x0, x1;
          ffma2(x0, x1, __uint_as_float(v[64 * hh + j]), __uint_as_float(v[64 * hh + j + 1]), c, c,
                nm, nm);
          float p0, p1;
          if (((j >> 1) & 7) < kFwdEmuPairsOf8) {
            exp2_fma2(p0, p1, x0, x1);
            if (masked) {  // the FMA-pipe exp2 floors at 2^-125: masked keys read 0
              p0 = (64 * hh + j < lim) ? p0 : 0.f;
              p1 = (64 * hh + j + 1 < lim) ? p1 : 0.f;
            }
          } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          const int a = (j >> 1) & 1;
          fadd2(ls[2 * a], ls[2 * a + 1], ls[2 * a], ls[2 * a + 1], p0, p1);
          pk[j >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st32(s_col + 32 * hh, pk);  // P columns [32hh, 32hh + 32): keys [64hh, 64hh + 64)
      }
      if (rescale && t > 0) {  // PV_X(t-1) is complete (see above): rescale O_X
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(o_col + c0, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(o_col + c0, o);
        }
      }
      l = l * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p_full0 + 8 * x);
    }
    // ------------------------------------------------------------ epilogue
    if (ok && T > 0) {
      ok = mbar_wait(bar_o_done0 + 8 * x, 0, p.err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        const int i = qt * 128 + row;
        const int h = x ? hB : hA;
        const float inv = 1.f / l;
        __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) +
                              ((static_cast<size_t>(b) * p.nq + i) * p.Hq + h) * D;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(o_col + c0, o);
          tmem_wait_ld();
          if (i < p.nq) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(o[q4 * 8 + 0]) * inv, __uint_as_float(o[q4 * 8 + 1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(o[q4 * 8 + 2]) * inv, __uint_as_float(o[q4 * 8 + 3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(o[q4 * 8 + 4]) * inv, __uint_as_float(o[q4 * 8 + 5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(o[q4 * 8 + 6]) * inv, __uint_as_float(o[q4 * 8 + 7]) * inv);
              dst[q4] = w;
            }
          }
        }
        if (H2O_IN_BOUNDS(i < p.nq_pad && h < p.Hq && b < p.B, p.err))
          p.nlse2[(static_cast<size_t>(b) * p.Hq + h) * p.nq_pad + i] =
              (i < p.nq) ? -(m_used + __log2f(l)) : -INFINITY;
      }
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

template <int D, bool Q8>
static cudaError_t launch_fwd(const AttnMaps& m, const AttnParams& p, cudaStream_t st) {
  using L = FwdLayout<D, Q8>;
  static int attr_bits[2] = {0, 0};
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(attn_fwd_kernel<D, Q8>),
                                   L::kAlloc, attr_bits);
  if (e != cudaSuccess) return e;
  const int pairs = cdiv(p.G * cdiv(p.nq, 128), 2);
  const int grid = p.B * p.Hkv * pairs;
  attn_fwd_kernel<D, Q8><<<grid, L::kThreads, L::kAlloc, st>>>(m.q, m.kc, m.vc, m.kn, m.vn, p);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd_bf16(int head_dim, const AttnMaps& m, const AttnParams& p,
                                 cudaStream_t st) {
  const bool q8 = p.k_scale != nullptr;  // int8 cache
  if (head_dim == 128) return q8 ? launch_fwd<128, true>(m, p, st) : launch_fwd<128, false>(m, p, st);
  return q8 ? launch_fwd<64, true>(m, p, st) : launch_fwd<64, false>(m, p, st);
}

}  // namespace h2o
