// The lambda re-parameterisation, lambda = exp(lq1 . lk1) - exp(lq2 . lk2) + lambda_init
// (page "Differential Transformer: Canceling Context Noise with Differential
// Attention", section "Cancelling Context Noise Through Attention Map
// Subtraction"; peer review "Differential Transformer", Summary, Eq. 2).
// One warp: two strided fp32 dot products, a shuffle reduction, two expf.
#include "internal.h"

namespace diffattn {

__global__ void __launch_bounds__(32) lambda_kernel(const float* __restrict__ lq1, const float* __restrict__ lk1,
                                                    const float* __restrict__ lq2, const float* __restrict__ lk2,
                                                    int d, float lambda_init, float* __restrict__ out) {
  float a = 0.f, b = 0.f;
  for (int i = threadIdx.x; i < d; i += 32) {
    a = fmaf(lq1[i], lk1[i], a);
    b = fmaf(lq2[i], lk2[i], b);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, off);
    b += __shfl_xor_sync(0xffffffffu, b, off);
  }
  if (threadIdx.x == 0) *out = expf(a) - expf(b) + lambda_init;
}

cudaError_t launch_lambda(const float* lq1, const float* lk1, const float* lq2, const float* lk2, int d,
                          float lambda_init, float* out, cudaStream_t stream) {
  lambda_kernel<<<1, 32, 0, stream>>>(lq1, lk1, lq2, lk2, d, lambda_init, out);
  return cudaGetLastError();
}

}  // namespace diffattn
