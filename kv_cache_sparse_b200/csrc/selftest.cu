// selftest.cu -- diagnostic entry point h2o_selftest_wait_timeout: one warp
// waits, with the kernels' bounded wait, on an mbarrier nothing arrives at;
// the wait gives up after the given limit, latches the timeout bit and the
// kernel returns (no trap, no hang).  Without a word of the caller's, the bit
// goes to the word h2o_static_scratch_check reports.  h2o_selftest_exp2
// evaluates the kernels' FMA-pipe exp2 (exp2_fma2) on given inputs, so that
// it can be checked against the library exp2f.
#include "../../include/h2o.h"
#include "attn.h"
#include "sm100.cuh"

namespace {

__global__ void wait_timeout_probe(int* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = h2o::smem_u32(&bar);
  if (threadIdx.x == 0) {
    h2o::mbar_init(b, 1);
    abort_flag = 0;
    h2o::fence_barrier_init();
  }
  __syncthreads();
  // phase 0 of a fresh barrier never completes: nothing arrives
  h2o::mbar_wait_until(b, 0, err, &abort_flag, limit_ns);
}

__global__ void exp2_fma_probe(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
  float ya, yb;
  h2o::exp2_fma2(ya, yb, a, b);
  y[i] = ya;
  if (i + 1 < n) y[i + 1] = yb;
}

}  // namespace

extern "C" H2O_API h2o_status h2o_selftest_exp2(const float* x, float* y, int32_t n,
                                                void* stream) {
  if (!x || !y || n < 0) return H2O_ERR_INVALID_ARG;
  if (n == 0) return H2O_OK;
  const int pairs = (n + 1) / 2;
  exp2_fma_probe<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? H2O_OK : H2O_ERR_CUDA;
}

extern "C" H2O_API h2o_status h2o_selftest_wait_timeout(int32_t* err_word, uint32_t limit_us,
                                                        void* stream) {
  if (limit_us == 0 || limit_us > 2000000) return H2O_ERR_INVALID_ARG;
  // no word given: the static-scratch entry point's word on this device
  if (!err_word) err_word = h2o::static_scratch_error_word();
  if (!err_word) return H2O_ERR_CUDA;
  wait_timeout_probe<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      err_word, static_cast<uint64_t>(limit_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? H2O_OK : H2O_ERR_CUDA;
}
