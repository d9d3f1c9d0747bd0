// Diagnostics behind the C ABI: the runtime limit of the kernels' bounded waits, a probe kernel
// whose wait nothing completes (to exercise the timeout path without touching real work), and an
// evaluator of the forward's FMA-pipe exponential so that its error can be measured directly.

#include "common.cuh"
#include "host.h"

namespace gpt {

gpt_status wait_limit_set_diag(long long cycles) { return set_wait_limit_here(cycles); }

// One thread initialises an mbarrier that expects one arrival, which never comes, and waits on it
// through the same bounded wait the GEMM and attention kernels use: the wait runs out after the
// limit in force, records GPT_ERR_DEVICE_TIMEOUT in *status and the kernel returns.
__global__ void wait_probe_kernel(int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status);
  __syncthreads();
}

__global__ void exp2_poly2_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    float p0, p1;
    exp2_poly2(p0, p1, x[i], x[i + 1]);
    y[i] = p0;
    y[i + 1] = p1;
  } else if (i < n) {
    float p0, p1;
    exp2_poly2(p0, p1, x[i], x[i]);
    y[i] = p0;
  }
}

}  // namespace gpt

extern "C" {

gpt_status gpt_set_wait_limit(long long cycles) {
  int sms = 0;
  GPT_TRY(gpt::device_info(&sms));
  GPT_TRY(gpt::wait_limit_set_gemm(cycles));
  GPT_TRY(gpt::wait_limit_set_attention(cycles));
  GPT_TRY(gpt::wait_limit_set_diag(cycles));
  return GPT_OK;
}

gpt_status gpt_debug_wait_probe(int* status, void* stream) {
  if (!status) return GPT_ERR_INVALID_ARG;
  int sms = 0;
  GPT_TRY(gpt::device_info(&sms));
  gpt::wait_probe_kernel<<<1, 32, 0, gpt::as_stream(stream)>>>(status);
  gpt::count_launch();
  GPT_CUDA_TRY(cudaGetLastError());
  return GPT_OK;
}

gpt_status gpt_debug_exp2_poly2(const float* x, float* y, int n, void* stream) {
  if (!x || !y || n <= 0) return GPT_ERR_INVALID_ARG;
  int sms = 0;
  GPT_TRY(gpt::device_info(&sms));
  const int pairs = (n + 1) / 2;
  gpt::exp2_poly2_kernel<<<(pairs + 255) / 256, 256, 0, gpt::as_stream(stream)>>>(x, y, n);
  gpt::count_launch();
  GPT_CUDA_TRY(cudaGetLastError());
  return GPT_OK;
}

}  // extern "C"
