// lambda_v1.cu -- the V1 lambda re-parameterisation on the GPU.
//
// "Differential Attention (V2)" lesson, "The differential concept": one scalar per head pair,
//   lambda = exp(lq1 . lk1) - exp(lq2 . lk2) + lambda_init,
// lambda_init a small positive number such as 0.8; the value may be negative. One warp per
// pair forms both dot products (fp32, shuffle reduction), evaluates the accurate expf and
// writes the value to every requested row, so it can feed the per-token lambda argument of
// the prefill and decode entry points.

#include "internal.h"

namespace da2 {

__global__ void __launch_bounds__(128)
lambda_v1_kernel(const float* __restrict__ lq1, const float* __restrict__ lk1, const float* __restrict__ lq2,
                 const float* __restrict__ lk2, float lambda_init, int n_pairs, int d, int rows,
                 float* __restrict__ out) {
  const int p = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (p >= n_pairs) return;
  float d1 = 0.f, d2 = 0.f;
  const size_t base = static_cast<size_t>(p) * d;
  for (int i = lane; i < d; i += 32) {
    d1 = fmaf(__ldg(lq1 + base + i), __ldg(lk1 + base + i), d1);
    d2 = fmaf(__ldg(lq2 + base + i), __ldg(lk2 + base + i), d2);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    d1 += __shfl_xor_sync(0xffffffffu, d1, off);
    d2 += __shfl_xor_sync(0xffffffffu, d2, off);
  }
  const float lam = expf(d1) - expf(d2) + lambda_init;
  for (int r = lane; r < rows; r += 32) out[static_cast<size_t>(r) * n_pairs + p] = lam;
}

cudaError_t launch_lambda_v1(const float* lq1, const float* lk1, const float* lq2, const float* lk2,
                             float lambda_init, int n_pairs, int d, int rows, float* out, cudaStream_t stream) {
  const int blocks = (n_pairs * 32 + 127) / 128;
  lambda_v1_kernel<<<blocks, 128, 0, stream>>>(lq1, lk1, lq2, lk2, lambda_init, n_pairs, d, rows, out);
  return cudaGetLastError();
}

}  // namespace da2
