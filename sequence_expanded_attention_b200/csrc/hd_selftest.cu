// hd_selftest.cu -- self-checks of two device building blocks, callable
// through the C ABI so that tests can run them on the GPU:
//   hd_selftest_ex2      the FMA-pipe exp2 (ex2_poly) and MUFU ex2.approx on
//                        caller-given inputs, for comparison with a reference;
//   hd_selftest_timeout  a bounded mbarrier wait on a barrier that nothing
//                        ever arrives on: it must give up after the given
//                        number of clocks and report HD_DEV_TIMEOUT, leaving
//                        the context usable (the kernels' failure path).
#include "../../include/hd.h"
#include "hd_kernels.cuh"

namespace {

__global__ void ex2_kernel(const float *__restrict__ x, float *__restrict__ y_poly,
                           float *__restrict__ y_mufu, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    y_poly[i] = hd::ex2_poly(x[i]);
    y_mufu[i] = hd::ex2_approx(x[i]);
  }
}

__global__ void timeout_kernel(int32_t *status, long long limit_clocks) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    hd::mbar_init(&bar, 1);
    hd::fence_barrier_init();
  }
  __syncthreads();
  // Nothing arrives on `bar`: phase 0 never completes.
  if (!hd::mbar_wait_limit(&bar, 0, limit_clocks)) hd::report(status, hd::kDevTimeout);
}

}  // namespace

extern "C" {

hd_status hd_selftest_ex2(const float *x, float *y_poly, float *y_mufu, int64_t n, void *stream) {
  if (n < 0 || (n > 0 && (!x || !y_poly || !y_mufu))) return HD_ERR_INVALID_ARG;
  if (n == 0) return HD_OK;
  const int threads = 256;
  const int64_t blocks = (n + threads - 1) / threads;
  if (blocks > 0x7fffffffLL) return HD_ERR_INVALID_ARG;
  ex2_kernel<<<(unsigned)blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(x, y_poly,
                                                                                 y_mufu, n);
  return cudaGetLastError() == cudaSuccess ? HD_OK : HD_ERR_CUDA;
}

hd_status hd_selftest_timeout(int32_t *dev_status, long long limit_clocks, void *stream) {
  if (!dev_status || limit_clocks < 0 || limit_clocks > (1LL << 31)) return HD_ERR_INVALID_ARG;
  timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev_status, limit_clocks);
  return cudaGetLastError() == cudaSuccess ? HD_OK : HD_ERR_CUDA;
}

}  // extern "C"
