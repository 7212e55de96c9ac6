// Sequence parallelism: the small kernels that join segment summaries.
//
// The GLA recurrence S_t = diag(exp a_t) S_{t-1} + phi_k(k_t) v_t^T (English
// gist.science summary, section 2.A "State Update") is affine in its start
// state; over a segment with summed log-decay R and end state U from a zero
// start, a start state S ends as diag(exp R) S + U.  Each segment's (U, R)
// comes from the state pass; these kernels form R on the portable path and
// chain the gathered summaries into one segment's start state.
#include "common.cuh"
#include "lizard_internal.h"

namespace lz {
namespace {

// R[bh][i] = sum_t a[bh][t][i]: thread = key dimension (coalesced across the
// block), one block per sequence, accumulated in fp64.
__global__ void __launch_bounds__(128) decay_sum_kernel(const float *a, float *R, int L, int D) {
  const int bh = blockIdx.x, i = threadIdx.x;
  if (i >= D) return;
  const float *src = a + (size_t)bh * L * D + i;
  double s = 0.0;
  for (int t = 0; t < L; ++t) s += (double)src[(size_t)t * D];
  R[(size_t)bh * D + i] = (float)s;
}

// out[bh] = S_rank with S_0 = state_in (or 0), S_{j+1} = diag(exp R_j) S_j + U_j.
// One thread per state element: grid (BH, D*D / 256); element e of the
// D x D state is row i = e / D (key dimension), column e % D.
__global__ void __launch_bounds__(256) chain_states_kernel(const float *U, const float *R, const float *state_in,
                                                           float *out, int BH, int D, int rank) {
  const int bh = blockIdx.x;
  const int e = blockIdx.y * 256 + threadIdx.x;
  const int i = e / D;
  const size_t DD = (size_t)D * D;
  float s = state_in ? state_in[bh * DD + e] : 0.f;
  for (int j = 0; j < rank; ++j) {
    const size_t sj = (size_t)j * BH + bh;
    s = fmaf(expf(R[sj * D + i]), s, U[sj * DD + e]);
  }
  out[bh * DD + e] = s;
}

}  // namespace

cudaError_t launch_decay_sum(const float *a, float *R, int BH, int L, int D, cudaStream_t s) {
  if (D > 128) return cudaErrorInvalidValue;
  decay_sum_kernel<<<BH, 128, 0, s>>>(a, R, L, D);
  return cudaGetLastError();
}

cudaError_t launch_chain_states(const float *U, const float *R, const float *state_in, float *out, int BH, int D,
                                int rank, cudaStream_t s) {
  if ((D * D) % 256 != 0) return cudaErrorInvalidValue;
  chain_states_kernel<<<dim3(BH, D * D / 256), 256, 0, s>>>(U, R, state_in, out, BH, D, rank);
  return cudaGetLastError();
}

}  // namespace lz
