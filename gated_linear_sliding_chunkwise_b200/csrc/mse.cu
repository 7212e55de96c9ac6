// Stage-1 attention-approximation loss for the portable path (English
// gist.science summary, section 2.B "Stage 1"; Chinese summary, section
// 2.2): the mean squared error between the layer's output o and the
// teacher's attention output y, and its gradient 2 (o - y) / n.  The
// tensor-core forward computes the same quantities in its epilogue.
#include "common.cuh"
#include "lizard_internal.h"

namespace lz {
namespace {

template <typename T>
__global__ void __launch_bounds__(256) mse_kernel(const T *o, const T *y, T *dout, float *loss, size_t n,
                                                  float grad_scale, float loss_scale) {
  __shared__ float red[8];
  float acc = 0.f;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const float d = to_f32(o[i]) - to_f32(y[i]);
    acc = fmaf(d, d, acc);
    dout[i] = from_f32<T>(d * grad_scale);
  }
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += red[w];
    atomicAdd(loss, t * loss_scale);
  }
}

}  // namespace

cudaError_t launch_mse(const void *o, const void *target, void *dout, float *loss, size_t n, bool bf16,
                       cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const float gs = (float)(2.0 / (double)n), ls = (float)(1.0 / (double)n);
  const size_t want = (n + 255) / 256;
  const int grid = (int)(want < 148 * 8 ? want : 148 * 8);
  if (bf16)
    mse_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(o),
                                                   static_cast<const __nv_bfloat16 *>(target),
                                                   static_cast<__nv_bfloat16 *>(dout), loss, n, gs, ls);
  else
    mse_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float *>(o), static_cast<const float *>(target),
                                           static_cast<float *>(dout), loss, n, gs, ls);
  return cudaGetLastError();
}

}  // namespace lz
