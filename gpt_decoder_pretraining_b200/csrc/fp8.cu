// Per-tensor e4m3 quantisation for the 8-bit GEMM (the FP8 matrix products of the d24 speedrun,
// "supa beginna nanochat", and of the alpha-nanochat-d24 run).
//
//   amax = max |x|;  scale = 448 / amax (1 when amax = 0);  q = e4m3(x·scale);  dq = amax / 448
//
// 448 is the largest finite e4m3 value.  x·scale is one fp32 multiply and e4m3(·) rounds to nearest
// even with saturation to ±448 (cvt.rn.satfinite), so every code is decided in fp32.  The GEMM
// multiplies its accumulator by dq_a·dq_b.  The maximum is order-independent, so the result is
// deterministic.

#include "common.cuh"
#include "host.h"

namespace gpt {

namespace {

__global__ void __launch_bounds__(256) amax_bf16_kernel(const uint16_t* __restrict__ x, long long n,
                                                        unsigned int* __restrict__ amax_bits) {
  float m = 0.f;
  const long long n8 = n / 8;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const uint4 v = reinterpret_cast<const uint4*>(x)[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) m = fmaxf(m, fmaxf(fabsf(bf_lo(w[e])), fabsf(bf_hi(w[e]))));
  }
  for (long long i = 8 * n8 + (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    m = fmaxf(m, fabsf(bf2f(x[i])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  // non-negative floats order like their bit patterns
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

__device__ __forceinline__ float amax_to_scale(unsigned int bits) {
  const float amax = __uint_as_float(bits);
  return amax > 0.f ? 448.f / amax : 1.f;
}

__global__ void __launch_bounds__(256) quantize_e4m3_kernel(const uint16_t* __restrict__ x, long long n,
                                                            const unsigned int* __restrict__ amax_bits,
                                                            uint8_t* __restrict__ q,
                                                            float* __restrict__ dq) {
  const float amax = __uint_as_float(*amax_bits);
  const float scale = amax_to_scale(*amax_bits);
  if (blockIdx.x == 0 && threadIdx.x == 0) *dq = amax > 0.f ? amax / 448.f : 1.f;
  const long long n8 = n / 8;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const uint4 v = reinterpret_cast<const uint4*>(x)[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint16_t p0, p1;
      const float a0 = bf_lo(w[2 * h]) * scale, a1 = bf_hi(w[2 * h]) * scale;
      const float a2 = bf_lo(w[2 * h + 1]) * scale, a3 = bf_hi(w[2 * h + 1]) * scale;
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(p0) : "f"(a1), "f"(a0));
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(p1) : "f"(a3), "f"(a2));
      out[h] = (uint32_t)p0 | ((uint32_t)p1 << 16);
    }
    reinterpret_cast<uint2*>(q)[i] = make_uint2(out[0], out[1]);
  }
  for (long long i = 8 * n8 + (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    uint16_t p;
    const float a = bf2f(x[i]) * scale;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(p) : "f"(0.f), "f"(a));
    q[i] = (uint8_t)(p & 0xFF);
  }
}

}  // namespace

gpt_status quantize_e4m3(const void* x, long long n, void* q, float* dq, unsigned int* amax_scratch,
                         cudaStream_t s) {
  if (!x || !q || !dq || !amax_scratch || n <= 0) return GPT_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(q) & 7))
    return GPT_ERR_UNSUPPORTED_SHAPE;
  int sms = 0;
  GPT_TRY(device_info(&sms));
  GPT_CUDA_TRY(cudaMemsetAsync(amax_scratch, 0, sizeof(unsigned int), s));
  const long long want = (n / 8 + 255) / 256 + 1;
  const int grid = (int)std::max<long long>(1, std::min<long long>(want, (long long)sms * 8));
  amax_bf16_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const uint16_t*>(x), n, amax_scratch);
  count_launch();
  GPT_CUDA_TRY(cudaGetLastError());
  quantize_e4m3_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const uint16_t*>(x), n, amax_scratch,
                                            reinterpret_cast<uint8_t*>(q), dq);
  count_launch();
  GPT_CUDA_TRY(cudaGetLastError());
  return GPT_OK;
}

}  // namespace gpt

extern "C" gpt_status gpt_quantize_e4m3(const void* x, long long n, void* q, float* dq,
                                        unsigned int* amax_scratch, void* stream) {
  return gpt::quantize_e4m3(x, n, q, dq, amax_scratch, gpt::as_stream(stream));
}
