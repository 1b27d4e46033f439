// h2o_api.cu -- host side of the C ABI declared in include/h2o.h.
//
// Validates arguments, lays out the caller's workspace, encodes the TMA
// descriptors of each call and launches the kernels of a step on the
// caller's stream (three; the K/V scatter is fused into K3):
//   K1 attention forward + row statistics   (attn_fwd.cu, tcgen05)
//   K2 summed attention weights per key     (attn_colsum.cu, tcgen05)
//   K3 score update + top-C selection + K/V scatter into the freed slots
//                                           (evict.cu)
// Float32 caches use the fp32 kernels of attn_f32.cu for K1/K2.  A call with
// n_q = 1 (a decode step) runs the two split-KV kernels of decode.cu instead
// when the group has 1, 2, 4 or 8 query heads.  The score-free policies skip
// K2 unless the caller asks for the summed weights.  The backward of the
// attention (attn_bwd.cu) runs on the row statistics K1 left in the
// workspace.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <new>

#include <nvtx3/nvToolsExt.h>

#include "../../include/h2o.h"
#include "attn.h"

using namespace h2o;

struct h2o_cache {
  h2o_config cfg;
  h2o_buffers buf;
  float* k_scale = nullptr;  // int8 cache (Q8): the scales behind the codes of K
  float* v_scale = nullptr;  // and of V, [batch, H_kv, capacity]
  int n = 0;
  int t0 = 0;
  uint64_t launches = 0;
  // workspace carve-up
  int nq_pad = 0;     // row stride of lse2
  int colsum_ld = 0;  // row stride of colsum
  float* lse2 = nullptr;
  float* colsum = nullptr;
  int* plan_slots = nullptr;
  int* plan_tokens = nullptr;
  int* plan_count = nullptr;
  float* dec_logits = nullptr;  // decode: [B*Hkv, G, C + 1]
  float* dec_part = nullptr;    // decode: [B*Hkv, dec_part_ld, G, d + 2]
  int dec_part_ld = 0;
  float* dsum = nullptr;  // backward: -scale * D_i, D_i = <dO_i, O_i>, [B, Hq, nq_pad]
  int fwd_nq = 0;         // n_q of the last attention whose row statistics are
  int fwd_n = -1;         // in the workspace, and the valid slots it saw
  unsigned long long* dec_best = nullptr;  // decode: [B*Hkv, dec_slices_ld]
  int* dec_ticket = nullptr;               // decode: [B*Hkv], zero between steps
  int dec_slices_ld = 0;
  // h2o_chunk_step_host: two staging sets, used by alternate calls, so the
  // copies of one call overlap the kernels of its neighbours.  The copies run
  // on two internal streams (one per direction); events order them with the
  // caller's stream.
  int device = 0;
  uint8_t* stage_q[2] = {nullptr, nullptr};
  uint8_t* stage_kn[2] = {nullptr, nullptr};
  uint8_t* stage_vn[2] = {nullptr, nullptr};
  uint8_t* stage_out[2] = {nullptr, nullptr};
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t ev_in[2] = {nullptr, nullptr};    // inputs of the set uploaded
  cudaEvent_t ev_step[2] = {nullptr, nullptr};  // step that read the set done
  cudaEvent_t ev_out[2] = {nullptr, nullptr};   // output of the set downloaded
  uint64_t host_calls = 0;
  // per-kernel timing (h2o_cache_set_timing)
  bool timing = false;
  cudaEvent_t ev[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
  bool ev_used[5] = {false, false, false, false, false};
};

namespace {

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// NVTX range around the host-side launch of one kernel (or kernel pair), so
// that a profiler's timeline names each part of the step; costs a pointer
// check when no tool is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// bytes per element of q, k_new, v_new and out
size_t esize_of(h2o_dtype t) { return t == H2O_F32 ? 4 : 2; }
// bytes per element of the cache's K and V rows (int8 codes for Q8)
size_t cache_esize(h2o_dtype t) { return t == H2O_F32 ? 4 : (t == H2O_Q8 ? 1 : 2); }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Layout {
  size_t lse, dsum, colsum, slots, tokens, count, dlog, dpart, dbest, dticket, sq[2], skn[2],
      svn[2], sout[2], total;
  int nq_pad, colsum_ld, dpart_ld, dslices_ld;
};

Layout workspace_layout(const h2o_config& c) {
  Layout L{};
  const size_t e = esize_of(c.dtype);
  const size_t BHkv = static_cast<size_t>(c.batch) * c.n_kv_heads;
  L.nq_pad = static_cast<int>(round_up(c.max_chunk, 128));
  L.colsum_ld = static_cast<int>(round_up(static_cast<size_t>(c.capacity) + c.max_chunk, 4));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = round_up(off + bytes, 256);
    return at;
  };
  L.lse = take(static_cast<size_t>(c.batch) * c.n_q_heads * L.nq_pad * 4);
  L.dsum = take(static_cast<size_t>(c.batch) * c.n_q_heads * L.nq_pad * 4);
  L.colsum = take(BHkv * L.colsum_ld * 4);
  L.slots = take(BHkv * c.max_chunk * 4);
  L.tokens = take(BHkv * c.max_chunk * 4);
  L.count = take(BHkv * 4);
  // decode steps (n_q = 1): stored logits and the split-KV partials
  const size_t G = static_cast<size_t>(c.n_q_heads / c.n_kv_heads);
  L.dpart_ld = cdiv(c.capacity + 1, decode_chunk_keys(c.head_dim, static_cast<int>(cache_esize(c.dtype))));
  L.dslices_ld = cdiv(c.capacity + 1, kDecodeSliceKeys);
  const bool dec = decode_supported(static_cast<int>(G));
  L.dlog = take(dec ? BHkv * G * (static_cast<size_t>(c.capacity) + 1) * 4 : 0);
  L.dpart = take(dec ? BHkv * L.dpart_ld * G * (c.head_dim + 2) * 4 : 0);
  L.dbest = take(dec ? BHkv * L.dslices_ld * 8 : 0);
  L.dticket = take(dec ? BHkv * 4 : 0);
  const size_t rows = static_cast<size_t>(c.batch) * c.max_chunk * c.head_dim * e;
  for (int i = 0; i < 2; ++i) {
    L.sq[i] = take(rows * c.n_q_heads);
    L.skn[i] = take(rows * c.n_kv_heads);
    L.svn[i] = take(rows * c.n_kv_heads);
    L.sout[i] = take(rows * c.n_q_heads);
  }
  L.total = off;
  return L;
}

h2o_status check_config(const h2o_config* c) {
  if (!c) return H2O_ERR_INVALID_ARG;
  if (c->dtype != H2O_BF16 && c->dtype != H2O_F32 && c->dtype != H2O_Q8) return H2O_ERR_DTYPE;
  if (c->batch < 1 || c->n_q_heads < 1 || c->n_kv_heads < 1 || c->capacity < 1 ||
      c->max_chunk < 1)
    return H2O_ERR_SHAPE;
  if (c->n_q_heads % c->n_kv_heads != 0) return H2O_ERR_SHAPE;
  if (c->head_dim != 64 && c->head_dim != 128) return H2O_ERR_SHAPE;
  if (c->recent_window < 0 || c->recent_window > c->capacity) return H2O_ERR_SHAPE;
  if (c->policy < H2O_POLICY_H2O || c->policy > H2O_POLICY_SLR) return H2O_ERR_INVALID_ARG;
  if (c->policy == H2O_POLICY_SLR &&
      (c->sink_tokens < 0 || static_cast<long long>(c->sink_tokens) + c->recent_window > c->capacity))
    return H2O_ERR_SHAPE;
  if (static_cast<long long>(c->capacity) + c->max_chunk > kMaxCandidates) return H2O_ERR_SHAPE;
  if (static_cast<long long>(c->batch) * c->n_kv_heads > 65535) return H2O_ERR_SHAPE;
  if (static_cast<long long>(c->batch) * c->n_q_heads * cdiv(c->max_chunk, 128) > (1ll << 31) - 1)
    return H2O_ERR_SHAPE;
  return H2O_OK;
}

// ---------------------------------------------------------------- TMA encoding

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// bf16 tensor of `rank` dims (innermost first), 128-byte swizzled boxes
bool encode_bf16(CUtensorMap* tm, const void* base, int rank, const cuuint64_t* dims,
                 const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [B, nq, H, d] chunk tensors: dims (d, H, nq, B), box (64, 1, 128, 1)
bool encode_chunk(CUtensorMap* tm, const void* base, int B, int nq, int H, int d) {
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)nq, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2,
                                 (cuuint64_t)nq * H * d * 2};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  return encode_bf16(tm, base, 4, dims, strides, box);
}

// [B*Hkv, C, d] cache with only the first n rows visible: dims (d, n, B*Hkv)
bool encode_cache(CUtensorMap* tm, const void* base, int BH, int n, int C, int d) {
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)(n > 0 ? n : 1), (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)C * d * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  return encode_bf16(tm, base, 3, dims, strides, box);
}

// int8 codes of the Q8 cache [B*Hkv, C, d], the first n rows visible: dims
// (d, n, B*Hkv), box (d, 128, 1), no swizzle (the kernels dequantise the tile
// into their 128-byte-swizzled bf16 operand)
bool encode_cache_q8(CUtensorMap* tm, const void* base, int BH, int n, int C, int d) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)(n > 0 ? n : 1), (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)d, (cuuint64_t)C * d};
  const cuuint32_t box[3] = {(cuuint32_t)d, 128, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

h2o_status cuda_status(cudaError_t e) { return e == cudaSuccess ? H2O_OK : H2O_ERR_CUDA; }

// Records timing event i (0: before K1, i: after kernel i) when timing is on.
void mark(h2o_cache* c, int i, cudaStream_t st) {
  if (!c->timing) return;
  if (cudaEventRecord(c->ev[i], st) == cudaSuccess) c->ev_used[i] = true;
}

h2o_status check_step_args(h2o_cache* c, const void* q, const void* kn, const void* vn, int nq,
                           const void* out) {
  if (!c) return H2O_ERR_INVALID_ARG;
  if (nq < 0 || nq > c->cfg.max_chunk) return H2O_ERR_INVALID_ARG;
  if (nq == 0) return H2O_OK;
  if (!q || !kn || !vn || !out) return H2O_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kn, 16) || !aligned(vn, 16) || !aligned(out, 16))
    return H2O_ERR_ALIGN;
  return H2O_OK;
}

AttnParams attn_params(h2o_cache* c, int nq, void* out) {
  const h2o_config& g = c->cfg;
  AttnParams p{};
  p.B = g.batch;
  p.Hq = g.n_q_heads;
  p.Hkv = g.n_kv_heads;
  p.G = g.n_q_heads / g.n_kv_heads;
  p.nq = nq;
  p.n = c->n;
  p.C = g.capacity;
  p.nq_pad = c->nq_pad;
  const float scale = g.softmax_scale > 0.f ? g.softmax_scale : 1.f / sqrtf((float)g.head_dim);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = out;
  p.nlse2 = c->lse2;
  p.colsum = c->colsum;
  p.colsum_ld = c->colsum_ld;
  p.err = c->buf.state + 2;
  p.k_scale = c->k_scale;
  p.v_scale = c->v_scale;
  return p;
}

// K1 + K2 into the workspace (lse2, colsum) and `out`.
// K1 + K2 (K2 only when the summed weights are needed: the H2O policy, or a
// caller asking for them).
h2o_status run_attention(h2o_cache* c, const void* q, const void* kn, const void* vn, int nq,
                         void* out, cudaStream_t st, bool with_colsum = true) {
  const h2o_config& g = c->cfg;
  AttnParams p = attn_params(c, nq, out);
  for (int i = 0; i < 5; ++i) c->ev_used[i] = false;
  mark(c, 0, st);
  if (g.dtype == H2O_F32) {
    NvtxRange r("h2o attention f32 (K1+K2)");
    cudaError_t e = launch_attn_f32(g.head_dim, static_cast<const float*>(q),
                                    static_cast<const float*>(c->buf.k),
                                    static_cast<const float*>(c->buf.v),
                                    static_cast<const float*>(kn), static_cast<const float*>(vn),
                                    p, st);
    c->launches += (c->n < g.capacity) ? 3 : 2;
    mark(c, 1, st);  // the fp32 kernels are reported together as the first part
    mark(c, 2, st);
    return cuda_status(e);
  }
  AttnMaps m;
  const int BH = g.batch * g.n_kv_heads;
  const bool q8 = g.dtype == H2O_Q8;
  auto enc = q8 ? encode_cache_q8 : encode_cache;
  if (!encode_chunk(&m.q, q, g.batch, nq, g.n_q_heads, g.head_dim) ||
      !encode_chunk(&m.kn, kn, g.batch, nq, g.n_kv_heads, g.head_dim) ||
      !encode_chunk(&m.vn, vn, g.batch, nq, g.n_kv_heads, g.head_dim) ||
      !enc(&m.kc, c->buf.k, BH, c->n, g.capacity, g.head_dim) ||
      !enc(&m.vc, c->buf.v, BH, c->n, g.capacity, g.head_dim))
    return H2O_ERR_CUDA;
  cudaError_t e;
  {
    NvtxRange r("h2o K1 attention forward");
    e = launch_attn_fwd_bf16(g.head_dim, m, p, st);
  }
  if (e != cudaSuccess) return H2O_ERR_CUDA;
  c->launches += 1;
  c->fwd_nq = nq;  // the row statistics of this call stay for a backward
  c->fwd_n = c->n;
  mark(c, 1, st);
  if (with_colsum) {
    NvtxRange r("h2o K2 summed weights");
    e = launch_attn_colsum_bf16(g.head_dim, m, p, st);
    if (e != cudaSuccess) return H2O_ERR_CUDA;
    c->launches += 1;
  }
  mark(c, 2, st);
  return H2O_OK;
}

// K3 (selection and the fused K/V scatter) with summed weights `colsum` (row
// stride ld); advances n and t0.
h2o_status run_evict(h2o_cache* c, const float* colsum, int ld, const void* kn, const void* vn,
                     int nq, cudaStream_t st) {
  const h2o_config& g = c->cfg;
  EvictParams e{};
  e.B = g.batch;
  e.Hkv = g.n_kv_heads;
  e.C = g.capacity;
  e.d = g.head_dim;
  e.esize = static_cast<int>(cache_esize(g.dtype));
  e.n = c->n;
  e.t0 = c->t0;
  e.nq = nq;
  e.W = g.recent_window;
  e.colsum = colsum;
  e.colsum_ld = ld;
  e.scores = c->buf.scores;
  e.pos = c->buf.pos;
  e.plan_slots = c->plan_slots;
  e.plan_tokens = c->plan_tokens;
  e.plan_count = c->plan_count;
  e.plan_ld = g.max_chunk;
  e.k_new = kn;
  e.v_new = vn;
  e.k_cache = c->buf.k;
  e.v_cache = c->buf.v;
  e.state = c->buf.state;
  e.policy = g.policy;
  e.sinks = g.sink_tokens;
  e.q8 = g.dtype == H2O_Q8 ? 1 : 0;
  e.k_scale = c->k_scale;
  e.v_scale = c->v_scale;
  if (!c->ev_used[2]) {  // eviction on its own: time it from here
    for (int i = 0; i < 5; ++i) c->ev_used[i] = false;
    mark(c, 2, st);
  }
  cudaError_t err;
  {
    NvtxRange r("h2o K3 score update + selection + scatter");
    err = launch_evict(e, g.max_chunk, st);
  }
  if (err != cudaSuccess) return H2O_ERR_CUDA;
  c->fwd_nq = 0;  // the cache changes: no backward of the earlier attention
  c->launches += 1;
  mark(c, 3, st);
  c->n = c->n + nq < g.capacity ? c->n + nq : g.capacity;
  c->t0 += nq;
  return H2O_OK;
}

bool decode_path(const h2o_cache* c, int nq) {
  return nq == 1 && decode_supported(c->cfg.n_q_heads / c->cfg.n_kv_heads);
}

// The step for one new token per cache (decode.cu): split-KV attention with
// summed weights into the workspace's colsum, and, if evict, the score update
// and placement.  Advances n and t0 when evicting.
h2o_status run_decode(h2o_cache* c, const void* q, const void* kn, const void* vn, void* out,
                      bool evict, cudaStream_t st) {
  const h2o_config& g = c->cfg;
  DecodeParams d{};
  d.B = g.batch;
  d.Hkv = g.n_kv_heads;
  d.G = g.n_q_heads / g.n_kv_heads;
  d.C = g.capacity;
  d.n = c->n;
  d.t0 = c->t0;
  d.W = g.recent_window;
  d.n_chunks = cdiv(c->n + 1, decode_chunk_keys(g.head_dim, static_cast<int>(cache_esize(g.dtype))));
  d.part_ld = c->dec_part_ld;
  d.n_slices = cdiv(c->n + 1, kDecodeSliceKeys);
  d.slices_ld = c->dec_slices_ld;
  d.best = c->dec_best;
  d.ticket = c->dec_ticket;
  // few (cache, KV head) units leave SMs idle: then every merge CTA takes
  // part of O, else only the first of each unit does
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  d.spread_o = g.batch * g.n_kv_heads < sms ? 1 : 0;
  const float scale = g.softmax_scale > 0.f ? g.softmax_scale : 1.f / sqrtf((float)g.head_dim);
  d.scale_log2 = scale * 1.4426950408889634f;
  d.q = q;
  d.k_new = kn;
  d.v_new = vn;
  d.k_cache = c->buf.k;
  d.v_cache = c->buf.v;
  d.out = out;
  d.logits = c->dec_logits;
  d.part = c->dec_part;
  d.colsum = c->colsum;
  d.colsum_ld = c->colsum_ld;
  d.scores = c->buf.scores;
  d.pos = c->buf.pos;
  d.state = c->buf.state;
  d.evict = evict ? 1 : 0;
  d.policy = g.policy;
  d.sinks = g.sink_tokens;
  d.k_scale = c->k_scale;
  d.v_scale = c->v_scale;
  for (int i = 0; i < 5; ++i) c->ev_used[i] = false;
  mark(c, 0, st);
  {
    NvtxRange r("h2o decode step (split-KV attention, merge, eviction)");
    if (launch_decode(d, static_cast<int>(cache_esize(g.dtype)), g.head_dim, st) != cudaSuccess)
      return H2O_ERR_CUDA;
  }
  c->fwd_nq = 0;  // the decode path keeps no row statistics
  c->launches += decode_launches();
  mark(c, 1, st);  // the whole step is reported as the first part
  mark(c, 2, st);
  mark(c, 3, st);
  if (evict) {
    c->n = c->n + 1 < g.capacity ? c->n + 1 : g.capacity;
    c->t0 += 1;
  }
  return H2O_OK;
}

h2o_status copy_colsum(h2o_cache* c, float* dst, int nq, cudaStream_t st) {
  const size_t w = (static_cast<size_t>(c->cfg.capacity) + nq) * sizeof(float);
  return cuda_status(cudaMemcpy2DAsync(dst, w, c->colsum, c->colsum_ld * sizeof(float), w,
                                       static_cast<size_t>(c->cfg.batch) * c->cfg.n_kv_heads,
                                       cudaMemcpyDefault, st));
}

// Creates the two copy streams and the six events of h2o_chunk_step_host on
// the cache's device, on first use.
h2o_status host_streams(h2o_cache* c) {
  if (c->h2d) return H2O_OK;
  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return H2O_ERR_CUDA;
  if (cur != c->device && cudaSetDevice(c->device) != cudaSuccess) return H2O_ERR_CUDA;
  cudaError_t e = cudaStreamCreateWithFlags(&c->h2d, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c->d2h, cudaStreamNonBlocking);
  for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
    e = cudaEventCreateWithFlags(&c->ev_in[i], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_step[i], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_out[i], cudaEventDisableTiming);
  }
  if (cur != c->device) cudaSetDevice(cur);
  return cuda_status(e);
}

}  // namespace

namespace h2o {
cudaError_t ensure_smem_attr(const void* fn, int bytes, int* slot_bits) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool tracked = dev >= 0 && dev < 64;
  const int w = tracked ? dev / 32 : 0, bit = tracked ? 1 << (dev % 32) : 0;
  // handles may be used from different host threads at once: the bit is a
  // fast path published after the attribute is in place (acquire / release)
  if (tracked && (__atomic_load_n(&slot_bits[w], __ATOMIC_ACQUIRE) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && tracked) __atomic_fetch_or(&slot_bits[w], bit, __ATOMIC_RELEASE);
  return e;
}
}  // namespace h2o

extern "C" {

h2o_status h2o_required_bytes(const h2o_config* cfg, h2o_sizes* out) {
  h2o_status s = check_config(cfg);
  if (s != H2O_OK) return s;
  if (!out) return H2O_ERR_INVALID_ARG;
  const size_t slots = static_cast<size_t>(cfg->batch) * cfg->n_kv_heads * cfg->capacity;
  // int8 cache: the codes, then one fp32 scale per row
  out->k_bytes = slots * cfg->head_dim * cache_esize(cfg->dtype) +
                 (cfg->dtype == H2O_Q8 ? slots * sizeof(float) : 0);
  out->v_bytes = out->k_bytes;
  out->scores_bytes = slots * 4;
  out->pos_bytes = slots * 4;
  out->state_bytes = 4 * sizeof(int32_t);
  out->workspace_bytes = workspace_layout(*cfg).total;
  return H2O_OK;
}

h2o_status h2o_cache_create(const h2o_config* cfg, const h2o_buffers* bufs, void* stream,
                            h2o_cache** out) {
  h2o_status s = check_config(cfg);
  if (s != H2O_OK) return s;
  if (!bufs || !out) return H2O_ERR_INVALID_ARG;
  if (!bufs->k || !bufs->v || !bufs->scores || !bufs->pos || !bufs->state || !bufs->workspace)
    return H2O_ERR_INVALID_ARG;
  if (!aligned(bufs->k, 16) || !aligned(bufs->v, 16) || !aligned(bufs->scores, 16) ||
      !aligned(bufs->pos, 16) || !aligned(bufs->state, 16) || !aligned(bufs->workspace, 256))
    return H2O_ERR_ALIGN;
  const Layout L = workspace_layout(*cfg);
  if (bufs->workspace_bytes < L.total) return H2O_ERR_SHAPE;
  if (cfg->dtype != H2O_F32 && !encode_fn()) return H2O_ERR_CUDA;
  h2o_cache* c = new (std::nothrow) h2o_cache();
  if (!c) return H2O_ERR_INVALID_ARG;
  c->cfg = *cfg;
  c->buf = *bufs;
  if (cfg->dtype == H2O_Q8) {
    const size_t codes = static_cast<size_t>(cfg->batch) * cfg->n_kv_heads * cfg->capacity *
                         cfg->head_dim;
    c->k_scale = reinterpret_cast<float*>(static_cast<uint8_t*>(bufs->k) + codes);
    c->v_scale = reinterpret_cast<float*>(static_cast<uint8_t*>(bufs->v) + codes);
  }
  uint8_t* ws = static_cast<uint8_t*>(bufs->workspace);
  c->nq_pad = L.nq_pad;
  c->colsum_ld = L.colsum_ld;
  c->lse2 = reinterpret_cast<float*>(ws + L.lse);
  c->dsum = reinterpret_cast<float*>(ws + L.dsum);
  c->colsum = reinterpret_cast<float*>(ws + L.colsum);
  c->plan_slots = reinterpret_cast<int*>(ws + L.slots);
  c->plan_tokens = reinterpret_cast<int*>(ws + L.tokens);
  c->plan_count = reinterpret_cast<int*>(ws + L.count);
  c->dec_logits = reinterpret_cast<float*>(ws + L.dlog);
  c->dec_part = reinterpret_cast<float*>(ws + L.dpart);
  c->dec_part_ld = L.dpart_ld;
  c->dec_best = reinterpret_cast<unsigned long long*>(ws + L.dbest);
  c->dec_ticket = reinterpret_cast<int*>(ws + L.dticket);
  c->dec_slices_ld = L.dslices_ld;
  for (int i = 0; i < 2; ++i) {
    c->stage_q[i] = ws + L.sq[i];
    c->stage_kn[i] = ws + L.skn[i];
    c->stage_vn[i] = ws + L.svn[i];
    c->stage_out[i] = ws + L.sout[i];
  }
  cudaPointerAttributes pa;
  if (cudaPointerGetAttributes(&pa, bufs->workspace) == cudaSuccess && pa.device >= 0)
    c->device = pa.device;
  else
    cudaGetDevice(&c->device);
  h2o_sizes sz;
  h2o_required_bytes(cfg, &sz);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(bufs->k, 0, sz.k_bytes, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(bufs->v, 0, sz.v_bytes, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(bufs->scores, 0, sz.scores_bytes, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(bufs->pos, 0xFF, sz.pos_bytes, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(bufs->state, 0, sz.state_bytes, st);
  // the decode merge's completion tickets start at zero (each step leaves them so)
  if (e == cudaSuccess && decode_supported(cfg->n_q_heads / cfg->n_kv_heads))
    e = cudaMemsetAsync(ws + L.dticket, 0, static_cast<size_t>(cfg->batch) * cfg->n_kv_heads * 4, st);
  if (e != cudaSuccess) {
    delete c;
    return H2O_ERR_CUDA;
  }
  *out = c;
  return H2O_OK;
}

h2o_status h2o_attention(h2o_cache* c, const void* q, const void* k_new, const void* v_new,
                         int32_t n_q, void* out, float* colsum_out, void* stream) {
  h2o_status s = check_step_args(c, q, k_new, v_new, n_q, out);
  if (s != H2O_OK || n_q == 0) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = decode_path(c, n_q) ? run_decode(c, q, k_new, v_new, out, false, st)
                          : run_attention(c, q, k_new, v_new, n_q, out, st);
  if (s == H2O_OK && colsum_out) s = copy_colsum(c, colsum_out, n_q, st);
  return s;
}

h2o_status h2o_attention_backward(h2o_cache* c, const void* q, const void* k_new,
                                  const void* v_new, int32_t n_q, const void* out,
                                  const void* d_out, float* dq, float* dk_cache, float* dv_cache,
                                  float* dk_new, float* dv_new, void* stream) {
  h2o_status s = check_step_args(c, q, k_new, v_new, n_q, out);
  if (s != H2O_OK || n_q == 0) return s;
  const h2o_config& g = c->cfg;
  if (g.dtype != H2O_BF16) return H2O_ERR_DTYPE;
  if (!d_out || !dq || !dk_cache || !dv_cache || !dk_new || !dv_new) return H2O_ERR_INVALID_ARG;
  if (!aligned(d_out, 16) || !aligned(dq, 16) || !aligned(dk_cache, 16) ||
      !aligned(dv_cache, 16) || !aligned(dk_new, 16) || !aligned(dv_new, 16))
    return H2O_ERR_ALIGN;
  // the row statistics must be those of h2o_attention on this state and n_q
  if (c->fwd_nq != n_q || c->fwd_n != c->n) return H2O_ERR_STATE;
  BwdParams p{};
  p.B = g.batch;
  p.Hq = g.n_q_heads;
  p.Hkv = g.n_kv_heads;
  p.G = g.n_q_heads / g.n_kv_heads;
  p.nq = n_q;
  p.n = c->n;
  p.C = g.capacity;
  p.nq_pad = c->nq_pad;
  p.scale = g.softmax_scale > 0.f ? g.softmax_scale : 1.f / sqrtf((float)g.head_dim);
  p.scale_log2 = p.scale * 1.4426950408889634f;
  p.nlse2 = c->lse2;
  p.dsum = c->dsum;
  p.dq = dq;
  p.dk_cache = dk_cache;
  p.dv_cache = dv_cache;
  p.dk_new = dk_new;
  p.dv_new = dv_new;
  p.err = c->buf.state + 2;
  BwdMaps m;
  const int BH = g.batch * g.n_kv_heads;
  if (!encode_chunk(&m.q, q, g.batch, n_q, g.n_q_heads, g.head_dim) ||
      !encode_chunk(&m.dout, d_out, g.batch, n_q, g.n_q_heads, g.head_dim) ||
      !encode_chunk(&m.kn, k_new, g.batch, n_q, g.n_kv_heads, g.head_dim) ||
      !encode_chunk(&m.vn, v_new, g.batch, n_q, g.n_kv_heads, g.head_dim) ||
      !encode_cache(&m.kc, c->buf.k, BH, c->n, g.capacity, g.head_dim) ||
      !encode_cache(&m.vc, c->buf.v, BH, c->n, g.capacity, g.head_dim))
    return H2O_ERR_CUDA;
  {
    NvtxRange r("h2o attention backward (row dots, dQ, dK/dV)");
    if (launch_attn_bwd_bf16(g.head_dim, m, p, out, d_out, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
      return H2O_ERR_CUDA;
  }
  c->launches += 3;
  return H2O_OK;
}

h2o_status h2o_evict(h2o_cache* c, const float* colsum, const void* k_new, const void* v_new,
                     int32_t n_q, void* stream) {
  if (!c || n_q < 0 || n_q > c->cfg.max_chunk) return H2O_ERR_INVALID_ARG;
  if (n_q == 0) return H2O_OK;
  if (!colsum || !k_new || !v_new) return H2O_ERR_INVALID_ARG;
  if (!aligned(colsum, 4) || !aligned(k_new, 16) || !aligned(v_new, 16)) return H2O_ERR_ALIGN;
  return run_evict(c, colsum, c->cfg.capacity + n_q, k_new, v_new, n_q,
                   static_cast<cudaStream_t>(stream));
}

h2o_status h2o_chunk_step(h2o_cache* c, const void* q, const void* k_new, const void* v_new,
                          int32_t n_q, void* out, float* colsum_out, void* stream) {
  h2o_status s = check_step_args(c, q, k_new, v_new, n_q, out);
  if (s != H2O_OK || n_q == 0) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (decode_path(c, n_q)) {
    // the summed weights are final before the eviction changes the scores
    // and the cache, so they can be copied after it
    s = run_decode(c, q, k_new, v_new, out, true, st);
    if (s == H2O_OK && colsum_out) s = copy_colsum(c, colsum_out, n_q, st);
    return s;
  }
  s = run_attention(c, q, k_new, v_new, n_q, out, st,
                    c->cfg.policy == H2O_POLICY_H2O || colsum_out != nullptr);
  if (s == H2O_OK && colsum_out) s = copy_colsum(c, colsum_out, n_q, st);
  if (s == H2O_OK) s = run_evict(c, c->colsum, c->colsum_ld, k_new, v_new, n_q, st);
  return s;
}

h2o_status h2o_chunk_step_host(h2o_cache* c, const void* q_host, const void* k_new_host,
                               const void* v_new_host, int32_t n_q, void* out_host,
                               float* colsum_out_host, void* stream) {
  if (!c) return H2O_ERR_INVALID_ARG;
  if (n_q < 0 || n_q > c->cfg.max_chunk) return H2O_ERR_INVALID_ARG;
  if (n_q == 0) return H2O_OK;
  if (!q_host || !k_new_host || !v_new_host || !out_host) return H2O_ERR_INVALID_ARG;
  if (host_streams(c) != H2O_OK) return H2O_ERR_CUDA;
  const h2o_config& g = c->cfg;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t rows = static_cast<size_t>(g.batch) * n_q * g.head_dim * esize_of(g.dtype);
  const size_t bq = rows * g.n_q_heads, bkv = rows * g.n_kv_heads;
  const int x = static_cast<int>(c->host_calls & 1);
  // upload into set x once the step two calls back has finished reading it
  cudaError_t e = cudaStreamWaitEvent(c->h2d, c->ev_step[x], 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(c->stage_q[x], q_host, bq, cudaMemcpyHostToDevice, c->h2d);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(c->stage_kn[x], k_new_host, bkv, cudaMemcpyHostToDevice, c->h2d);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(c->stage_vn[x], v_new_host, bkv, cudaMemcpyHostToDevice, c->h2d);
  if (e == cudaSuccess) e = cudaEventRecord(c->ev_in[x], c->h2d);
  // the step waits for its inputs and for the download that last read out[x]
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, c->ev_in[x], 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, c->ev_out[x], 0);
  if (e != cudaSuccess) return H2O_ERR_CUDA;
  h2o_status s = h2o_chunk_step(c, c->stage_q[x], c->stage_kn[x], c->stage_vn[x], n_q,
                                c->stage_out[x], colsum_out_host, stream);
  if (s != H2O_OK) return s;
  e = cudaEventRecord(c->ev_step[x], st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(c->d2h, c->ev_step[x], 0);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(out_host, c->stage_out[x], bq, cudaMemcpyDeviceToHost, c->d2h);
  if (e == cudaSuccess) e = cudaEventRecord(c->ev_out[x], c->d2h);
  if (e != cudaSuccess) return H2O_ERR_CUDA;
  ++c->host_calls;
  return H2O_OK;
}

h2o_status h2o_cache_host_join(h2o_cache* c, void* stream) {
  if (!c) return H2O_ERR_INVALID_ARG;
  if (c->host_calls == 0) return H2O_OK;
  // the download stream is in order: its latest event covers every earlier call
  const int last = static_cast<int>((c->host_calls - 1) & 1);
  return cuda_status(cudaStreamWaitEvent(static_cast<cudaStream_t>(stream), c->ev_out[last], 0));
}

h2o_status h2o_cache_read(const h2o_cache* c, void* k, void* v, float* scores, int32_t* pos,
                          int32_t* n_t0, void* stream) {
  if (!c) return H2O_ERR_INVALID_ARG;
  h2o_sizes sz;
  h2o_required_bytes(&c->cfg, &sz);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (k) e = cudaMemcpyAsync(k, c->buf.k, sz.k_bytes, cudaMemcpyDefault, st);
  if (e == cudaSuccess && v) e = cudaMemcpyAsync(v, c->buf.v, sz.v_bytes, cudaMemcpyDefault, st);
  if (e == cudaSuccess && scores)
    e = cudaMemcpyAsync(scores, c->buf.scores, sz.scores_bytes, cudaMemcpyDefault, st);
  if (e == cudaSuccess && pos)
    e = cudaMemcpyAsync(pos, c->buf.pos, sz.pos_bytes, cudaMemcpyDefault, st);
  if (n_t0) {
    n_t0[0] = c->n;
    n_t0[1] = c->t0;
  }
  return cuda_status(e);
}

h2o_status h2o_cache_write(h2o_cache* c, const void* k, const void* v, const float* scores,
                           const int32_t* pos, const int32_t* n_t0, void* stream) {
  if (!c || !k || !v || !scores || !pos || !n_t0) return H2O_ERR_INVALID_ARG;
  if (n_t0[0] < 0 || n_t0[0] > c->cfg.capacity || n_t0[1] < n_t0[0]) return H2O_ERR_INVALID_ARG;
  h2o_sizes sz;
  h2o_required_bytes(&c->cfg, &sz);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(c->buf.k, k, sz.k_bytes, cudaMemcpyDefault, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(c->buf.v, v, sz.v_bytes, cudaMemcpyDefault, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(c->buf.scores, scores, sz.scores_bytes, cudaMemcpyDefault, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(c->buf.pos, pos, sz.pos_bytes, cudaMemcpyDefault, st);
  static int32_t fresh[4];
  fresh[0] = n_t0[0];
  fresh[1] = n_t0[1];
  fresh[2] = 0;
  fresh[3] = 0;
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(c->buf.state, fresh, sizeof(fresh), cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return H2O_ERR_CUDA;
  c->n = n_t0[0];
  c->t0 = n_t0[1];
  c->fwd_nq = 0;
  return H2O_OK;
}

h2o_status h2o_cache_check(h2o_cache* c, void* stream) {
  if (!c) return H2O_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return H2O_ERR_CUDA;
  int32_t word = 0;
  if (cudaMemcpy(&word, c->buf.state + 2, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return H2O_ERR_CUDA;
  if (word & kDevErrTimeout) return H2O_ERR_TIMEOUT;
  if (word & (kDevErrPlan | kDevErrSmem | kDevErrBounds)) return H2O_ERR_STATE;
  return H2O_OK;
}

h2o_status h2o_cache_info(const h2o_cache* c, int32_t* n, int32_t* t0, uint64_t* launches) {
  if (!c) return H2O_ERR_INVALID_ARG;
  if (n) *n = c->n;
  if (t0) *t0 = c->t0;
  if (launches) *launches = c->launches;
  return H2O_OK;
}

h2o_status h2o_cache_set_timing(h2o_cache* c, int enable) {
  if (!c) return H2O_ERR_INVALID_ARG;
  if (enable && !c->ev[0]) {
    for (int i = 0; i < 5; ++i)
      if (cudaEventCreate(&c->ev[i]) != cudaSuccess) return H2O_ERR_CUDA;
  }
  c->timing = enable != 0;
  for (int i = 0; i < 5; ++i) c->ev_used[i] = false;
  return H2O_OK;
}

h2o_status h2o_cache_kernel_ms(h2o_cache* c, float* ms4) {
  if (!c || !ms4) return H2O_ERR_INVALID_ARG;
  for (int i = 0; i < 4; ++i) ms4[i] = 0.f;
  int last = -1;
  for (int i = 4; i >= 0 && last < 0; --i)
    if (c->ev_used[i]) last = i;
  if (last < 0) return H2O_OK;
  if (cudaEventSynchronize(c->ev[last]) != cudaSuccess) return H2O_ERR_CUDA;
  for (int k = 0; k < 4; ++k) {
    if (c->ev_used[k] && c->ev_used[k + 1]) {
      float ms = 0.f;
      if (cudaEventElapsedTime(&ms, c->ev[k], c->ev[k + 1]) != cudaSuccess) return H2O_ERR_CUDA;
      ms4[k] = ms;
    }
  }
  return H2O_OK;
}

void h2o_cache_destroy(h2o_cache* c) {
  if (!c) return;
  for (int i = 0; i < 5; ++i)
    if (c->ev[i]) cudaEventDestroy(c->ev[i]);
  // copies still in flight write caller memory: let them finish first
  if (c->h2d) cudaStreamSynchronize(c->h2d);
  if (c->d2h) cudaStreamSynchronize(c->d2h);
  for (int i = 0; i < 2; ++i) {
    if (c->ev_in[i]) cudaEventDestroy(c->ev_in[i]);
    if (c->ev_step[i]) cudaEventDestroy(c->ev_step[i]);
    if (c->ev_out[i]) cudaEventDestroy(c->ev_out[i]);
  }
  if (c->h2d) cudaStreamDestroy(c->h2d);
  if (c->d2h) cudaStreamDestroy(c->d2h);
  delete c;
}

const char* h2o_status_string(h2o_status s) {
  switch (s) {
    case H2O_OK: return "ok";
    case H2O_ERR_INVALID_ARG: return "invalid argument";
    case H2O_ERR_SHAPE: return "unsupported shape or buffer too small";
    case H2O_ERR_DTYPE: return "unsupported dtype";
    case H2O_ERR_ALIGN: return "misaligned pointer";
    case H2O_ERR_CUDA: return "CUDA runtime error";
    case H2O_ERR_TIMEOUT: return "device wait timed out";
    case H2O_ERR_STATE: return "inconsistent eviction plan";
  }
  return "unknown status";
}

}  // extern "C"
