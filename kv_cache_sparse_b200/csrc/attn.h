// attn.h -- launchers of the attention kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.h"

namespace h2o {

// TMA descriptors of one call (bf16 path).
struct AttnMaps {
  CUtensorMap q;   // [B, nq, Hq, d]     box (64, 1, 128, 1)
  CUtensorMap kc;  // [B*Hkv, n, d]      box (64, 128, 1)   rows >= n read as zero
  CUtensorMap vc;
  CUtensorMap kn;  // [B, nq, Hkv, d]    box (64, 1, 128, 1) rows >= nq read as zero
  CUtensorMap vn;
};

// TMA descriptors of a backward call: AttnMaps plus dO (layout of q).
struct BwdMaps {
  CUtensorMap q, dout, kc, vc, kn, vn;
};

// Raises the kernel's dynamic shared-memory limit to `bytes` on the current
// device, once per device.  The device's bit in slot_bits is set only after
// cudaFuncSetAttribute succeeded, so a thread that sees it set may launch;
// threads that see it clear all make the (idempotent) call themselves, and
// a failed call is retried by the next launch.
cudaError_t ensure_smem_attr(const void* fn, int bytes, int* slot_bits);

// K1: attention forward + row statistics (tcgen05), head_dim 64 or 128.
cudaError_t launch_attn_fwd_bf16(int head_dim, const AttnMaps& m, const AttnParams& p,
                                 cudaStream_t st);
// K2: summed attention weights per key (tcgen05), head_dim 64 or 128.
cudaError_t launch_attn_colsum_bf16(int head_dim, const AttnMaps& m, const AttnParams& p,
                                    cudaStream_t st);
// fp32 path (FMA): K1 and K2 for float inputs.
cudaError_t launch_attn_f32(int head_dim, const float* q, const float* kc, const float* vc,
                            const float* kn, const float* vn, const AttnParams& p,
                            cudaStream_t st);

// Decode step (n_q = 1, G in {1, 2, 4, 8}): split-KV partials, then the merge,
// summed weights and (if p.evict) the single-token eviction.  esize: bytes per
// cache element -- 2 (bf16), 4 (float), or 1 (int8 codes with per-row scales;
// q, out and the new rows bf16); head_dim 64 or 128.
cudaError_t launch_decode(const DecodeParams& p, int esize, int head_dim, cudaStream_t st);
// Group sizes the decode kernels take (a warp batch holds 32 / G keys).
bool decode_supported(int G);
// Kernel launches per decode step (1: the merge runs in each unit's last CTA).
int decode_launches();

// Backward of the attention (bf16, head_dim 64 or 128): D_i, then dK/dV and
// dQ; out and dout are [B, nq, Hq, d] bf16.
cudaError_t launch_attn_bwd_bf16(int head_dim, const BwdMaps& m, const BwdParams& p,
                                 const void* out, const void* dout, cudaStream_t st);

// Device address of the error word of h2o_attention_static_scratch on the
// current device (null if it cannot be resolved).
int* static_scratch_error_word();

// K3 (with the K/V scatter fused): score update, selection, placement.
cudaError_t launch_evict(const EvictParams& e, int max_chunk, cudaStream_t st);

}  // namespace h2o
