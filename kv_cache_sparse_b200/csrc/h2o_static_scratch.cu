// h2o_static_scratch.cu -- attention with summed weights for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or hand this library a workspace):
// engines and plugin hosts that own the whole device-memory budget and give
// a plugin only its inputs and outputs, and serving loops that must not
// allocate once they run, since an allocation can block on the device and
// can fail when the host framework has reserved or fragmented the memory.
// h2o_attention_static_scratch serves them.  It runs the same two kernels as
// h2o_attention (attention forward, then the per-key summed weights), but the
// one piece of scratch they share -- the per-row log-sum-exp written by the
// first kernel and read by the second -- lives in the file-scope device
// array below instead of a caller workspace.
//
// The array is part of the library image: every GPU on which the library is
// loaded holds it (kStaticScratchRows floats, 16 MiB) until the process
// exits.  Every call on a device uses the same array and it keeps the last
// call's contents.  Nothing in it has to start at zero: the first kernel of
// a call writes every row the second kernel of that call reads.  Calls whose
// work overlaps on the GPU (two streams, or two host threads) race on it.  A
// second static word records an expired bounded wait: each call clears it
// first (cudaMemsetAsync on its device address, which allocates nothing) and
// h2o_static_scratch_check reports it.
#include <math.h>

#include <atomic>
#include <mutex>

#include "../../include/h2o.h"
#include "attn.h"

namespace {

using namespace h2o;

// Rows of the static scratch: one float per (cache, query head, query row
// padded to a multiple of 128).
constexpr long long kStaticScratchRows = 4ll << 20;

static __device__ __align__(256) float g_row_lse2[kStaticScratchRows];
// Where the kernels latch an expired bounded wait (they never leave one
// pending); this entry point has no cache state word to put it in.  Each
// call clears it first; h2o_static_scratch_check reads it.
static __device__ int g_wait_error;

constexpr int kMaxDevices = 64;
// device addresses of g_row_lse2 and g_wait_error, per device; published
// (release) only once both are known, so a reader that sees them non-null
// (acquire) may use them
std::atomic<float*> g_scratch_addr[kMaxDevices];
std::atomic<int*> g_error_addr[kMaxDevices];
std::mutex g_setup_mutex;

// Resolves the arrays' device addresses on the current device, once per
// device.  Host code must not pass `g_row_lse2` itself to a kernel: on the
// host that name is only a stand-in for the symbol, not a device address.
h2o_status scratch_address(float** out, int** err) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return H2O_ERR_CUDA;
  float* a = g_scratch_addr[dev].load(std::memory_order_acquire);
  int* w = g_error_addr[dev].load(std::memory_order_acquire);
  if (a == nullptr || w == nullptr) {
    // first use on this device: one thread looks the addresses up
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    a = g_scratch_addr[dev].load(std::memory_order_relaxed);
    w = g_error_addr[dev].load(std::memory_order_relaxed);
    if (a == nullptr || w == nullptr) {
      void* p = nullptr;
      void* e = nullptr;
      if (cudaGetSymbolAddress(&p, g_row_lse2) != cudaSuccess || p == nullptr) return H2O_ERR_CUDA;
      if (cudaGetSymbolAddress(&e, g_wait_error) != cudaSuccess || e == nullptr) return H2O_ERR_CUDA;
      a = static_cast<float*>(p);
      w = static_cast<int*>(e);
      g_error_addr[dev].store(w, std::memory_order_release);
      g_scratch_addr[dev].store(a, std::memory_order_release);
    }
  }
  *out = a;
  *err = w;
  return H2O_OK;
}

typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                             const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                             const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                             CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encoder() {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  }
  return fn;
}

// 128-byte-swizzled bf16 map; boxes of 64 elements x 128 rows
bool make_map(CUtensorMap* tm, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides) {
  EncodeFn fn = encoder();
  if (!fn) return false;
  const cuuint32_t box4[4] = {64, 1, 128, 1};
  const cuuint32_t box3[3] = {64, 128, 1};
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
            rank == 4 ? box4 : box3, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

extern "C" H2O_API h2o_status h2o_attention_static_scratch(
    const h2o_config* cfg, const void* k_cache, const void* v_cache, int32_t n, const void* q,
    const void* k_new, const void* v_new, int32_t n_q, void* out, float* colsum_out,
    void* stream) {
  if (!cfg) return H2O_ERR_INVALID_ARG;
  const h2o_config& g = *cfg;
  if (g.dtype != H2O_BF16 && g.dtype != H2O_F32) return H2O_ERR_DTYPE;
  if (g.batch < 1 || g.n_q_heads < 1 || g.n_kv_heads < 1 || g.capacity < 1 || g.max_chunk < 1 ||
      g.n_q_heads % g.n_kv_heads != 0 || (g.head_dim != 64 && g.head_dim != 128) ||
      static_cast<long long>(g.batch) * g.n_kv_heads > 65535)
    return H2O_ERR_SHAPE;
  if (n_q < 0 || n_q > g.max_chunk || n < 0 || n > g.capacity) return H2O_ERR_INVALID_ARG;
  if (n_q == 0) return H2O_OK;
  if (!k_cache || !v_cache || !q || !k_new || !v_new || !out || !colsum_out)
    return H2O_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(q) || !aligned16(k_new) ||
      !aligned16(v_new) || !aligned16(out) || (reinterpret_cast<uintptr_t>(colsum_out) & 3))
    return H2O_ERR_ALIGN;
  const int nq_pad = cdiv(n_q, 128) * 128;
  if (static_cast<long long>(g.batch) * g.n_q_heads * nq_pad > kStaticScratchRows)
    return H2O_ERR_SHAPE;  // more query rows than the static scratch holds

  float* lse2 = nullptr;
  int* err = nullptr;
  h2o_status s = scratch_address(&lse2, &err);
  if (s != H2O_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // this call's kernels latch a timeout into a clean word
  if (cudaMemsetAsync(err, 0, sizeof(int), st) != cudaSuccess) return H2O_ERR_CUDA;

  AttnParams p{};
  p.B = g.batch;
  p.Hq = g.n_q_heads;
  p.Hkv = g.n_kv_heads;
  p.G = g.n_q_heads / g.n_kv_heads;
  p.nq = n_q;
  p.n = n;
  p.C = g.capacity;
  p.nq_pad = nq_pad;
  const float scale = g.softmax_scale > 0.f ? g.softmax_scale : 1.f / sqrtf((float)g.head_dim);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = out;
  p.nlse2 = lse2;  // holds minus the row log-sum-exp
  p.colsum = colsum_out;  // written in place: [batch, H_kv, capacity + n_q]
  p.colsum_ld = g.capacity + n_q;
  p.err = err;
  p.k_scale = nullptr;  // bf16 / fp32 cache (this entry point takes no int8 cache)
  p.v_scale = nullptr;

  if (g.dtype == H2O_F32) {
    cudaError_t e = launch_attn_f32(g.head_dim, static_cast<const float*>(q),
                                    static_cast<const float*>(k_cache),
                                    static_cast<const float*>(v_cache),
                                    static_cast<const float*>(k_new),
                                    static_cast<const float*>(v_new), p, st);
    return e == cudaSuccess ? H2O_OK : H2O_ERR_CUDA;
  }
  const int d = g.head_dim;
  const cuuint64_t qd[4] = {(cuuint64_t)d, (cuuint64_t)g.n_q_heads, (cuuint64_t)n_q,
                            (cuuint64_t)g.batch};
  const cuuint64_t qs[3] = {(cuuint64_t)d * 2, (cuuint64_t)g.n_q_heads * d * 2,
                            (cuuint64_t)n_q * g.n_q_heads * d * 2};
  const cuuint64_t kd[4] = {(cuuint64_t)d, (cuuint64_t)g.n_kv_heads, (cuuint64_t)n_q,
                            (cuuint64_t)g.batch};
  const cuuint64_t ks[3] = {(cuuint64_t)d * 2, (cuuint64_t)g.n_kv_heads * d * 2,
                            (cuuint64_t)n_q * g.n_kv_heads * d * 2};
  const cuuint64_t cd[3] = {(cuuint64_t)d, (cuuint64_t)(n > 0 ? n : 1),
                            (cuuint64_t)g.batch * g.n_kv_heads};
  const cuuint64_t cs[2] = {(cuuint64_t)d * 2, (cuuint64_t)g.capacity * d * 2};
  AttnMaps m;
  if (!make_map(&m.q, q, 4, qd, qs) || !make_map(&m.kn, k_new, 4, kd, ks) ||
      !make_map(&m.vn, v_new, 4, kd, ks) || !make_map(&m.kc, k_cache, 3, cd, cs) ||
      !make_map(&m.vc, v_cache, 3, cd, cs))
    return H2O_ERR_CUDA;
  if (launch_attn_fwd_bf16(d, m, p, st) != cudaSuccess) return H2O_ERR_CUDA;
  if (launch_attn_colsum_bf16(d, m, p, st) != cudaSuccess) return H2O_ERR_CUDA;
  return H2O_OK;
}

namespace h2o {
// The static entry point's error word on the current device (null when its
// address cannot be resolved); the failure-path self-test latches into it.
int* static_scratch_error_word() {
  float* a = nullptr;
  int* w = nullptr;
  return scratch_address(&a, &w) == H2O_OK ? w : nullptr;
}
}  // namespace h2o

extern "C" H2O_API h2o_status h2o_static_scratch_check(void* stream) {
  float* a = nullptr;
  int* w = nullptr;
  h2o_status s = scratch_address(&a, &w);
  if (s != H2O_OK) return s;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return H2O_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, w, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return H2O_ERR_CUDA;
  if (word & h2o::kDevErrTimeout) return H2O_ERR_TIMEOUT;
  if (word & ~h2o::kDevErrTimeout) return H2O_ERR_STATE;
  return H2O_OK;
}
