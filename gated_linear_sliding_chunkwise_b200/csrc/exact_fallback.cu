// Exact fallback of the tensor-core backward for sequences whose cumulative
// log-decay spans more than the tensor-core kernels' exponent range inside
// one 128-token tile (the low-precision underflow that the log-space gate
// absorption is about: Chinese gist.science summary, section 2.3; English
// summary, section 2.C).  (The forward handles such sequences inside its
// own kernel: tc_fwd.cu, exact_gla_sequence.)
//
// The tensor-core kernels absorb the decay of a tile as exp(b - r) and
// exp(r - b) around one reference point r per tile.  When, in some key
// dimension, the tile's log-decay spread exceeds kMaxSpread, those factors
// leave the bf16 / fp32 exponent range.  The gate prep marks such sequences;
// here they get slots (up to kFallbackSlots per call), and the portable
// kernels -- whose chunked products use the element-wise exp(b_t - b_j),
// exact for any decay -- rerun their GLA backward, one grid slot per marked
// sequence: dphi_q, dphi_k (fp32, in the slot's arrays, which the feature-map
// pass reads for these sequences), dv_gla, da and dstate_in into the arrays
// the tensor-core kernels use, then dg from da at the end.  A marked
// sequence beyond the last slot keeps the tensor-core result and sets the
// RANGE bit of the status word.
#include "common.cuh"
#include "lizard_internal.h"

namespace lz {
namespace {

__global__ void __launch_bounds__(256) assign_slots_kernel(const uint32_t *flags, int *slot_of, int *seq_of_slot,
                                                           int BH, int K, uint32_t *status) {
  __shared__ int s_cnt;
  if (threadIdx.x == 0) s_cnt = 0;
  for (int k = threadIdx.x; k < K; k += blockDim.x) seq_of_slot[k] = -1;
  __syncthreads();
  for (int bh = threadIdx.x; bh < BH; bh += blockDim.x) {
    int slot = -1;
    if (flags[bh]) {
      const int k = atomicAdd(&s_cnt, 1);
      if (k < K) {
        slot = k;
        seq_of_slot[k] = bh;
      } else {
        atomicOr(status, 2u);   // no slot left: this sequence keeps the inexact result
      }
    }
    slot_of[bh] = slot;
  }
}

// dg from da for every occupied slot: per key dimension dg = da sigmoid(-g) /
// tau; with the scalar gate, dg_t = sum_i da_t[i] sigmoid(-g_t) / tau (one
// warp per token).
template <typename T>
__global__ void __launch_bounds__(256) slot_dg_kernel(float *dg, const float *da, const T *g, const int *seq_of_slot,
                                                      int L, int D, float inv_tau, int scalar_gate) {
  const int bh = seq_of_slot[blockIdx.y];
  if (bh < 0) return;
  const float *a = da + (size_t)bh * L * D;
  if (!scalar_gate) {
    const size_t n = (size_t)L * D;
    const T *gs = g + (size_t)bh * n;
    float *out = dg + (size_t)bh * n;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x)
      out[e] = a[e] * dlogsigmoid(to_f32(gs[e])) * inv_tau;
    return;
  }
  const int lane = threadIdx.x & 31;
  const int warps = (int)(gridDim.x * blockDim.x) >> 5;
  for (int t = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5); t < L; t += warps) {
    float s = 0.f;
    for (int i = lane; i < D; i += 32) s += a[(size_t)t * D + i];
    s = warp_sum(s);
    if (lane == 0) dg[(size_t)bh * L + t] = s * dlogsigmoid(to_f32(g[(size_t)bh * L + t])) * inv_tau;
  }
}

}  // namespace

cudaError_t launch_assign_slots(const uint32_t *flags, int *slot_of, int *seq_of_slot, int BH, int K,
                                uint32_t *status, cudaStream_t s) {
  assign_slots_kernel<<<1, 256, 0, s>>>(flags, slot_of, seq_of_slot, BH, K, status);
  return cudaGetLastError();
}

cudaError_t launch_slot_dg(float *dg, const float *da, const void *g, const int *seq_of_slot, int K, int L, int D,
                           float inv_tau, bool scalar_gate, bool bf16, cudaStream_t s) {
  const size_t per_seq = (size_t)L * D;
  const dim3 grid((unsigned)((per_seq + 255) / 256 < 64 ? (per_seq + 255) / 256 : 64), K);
  if (bf16)
    slot_dg_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(dg, da, static_cast<const __nv_bfloat16 *>(g), seq_of_slot, L, D,
                                                       inv_tau, scalar_gate ? 1 : 0);
  else
    slot_dg_kernel<float><<<grid, 256, 0, s>>>(dg, da, static_cast<const float *>(g), seq_of_slot, L, D, inv_tau,
                                               scalar_gate ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace lz
