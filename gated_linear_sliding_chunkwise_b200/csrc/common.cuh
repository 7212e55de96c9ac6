// Shared device helpers for the Lizard kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define LZ_DEV __device__ __forceinline__

namespace lz {

// Activation storage types.  Every kernel computes in fp32.
template <typename T> LZ_DEV float to_f32(T x);
template <> LZ_DEV float to_f32<float>(float x) { return x; }
template <> LZ_DEV float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> LZ_DEV T from_f32(float x);
template <> LZ_DEV float from_f32<float>(float x) { return x; }
template <> LZ_DEV __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// log of the gate: logsigmoid(g) / tau, in the overflow-free form
// min(g, 0) - log(1 + exp(-|g|)).
LZ_DEV float log_decay(float g, float inv_tau) {
  return (fminf(g, 0.f) - log1pf(expf(-fabsf(g)))) * inv_tau;
}

// d logsigmoid(g) / dg = sigmoid(-g) = 1 / (1 + exp(g)).
LZ_DEV float dlogsigmoid(float g) { return 1.f / (1.f + expf(g)); }

LZ_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
LZ_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
LZ_DEV int warp_min_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Largest exponent spread (in natural-log units) inside one chunk for which
// the log-space absorption Qt = phi_q exp(b - r), Kt = phi_k exp(r - b)
// stays inside the fp32/bf16 exponent range with margin.  Chunks whose
// cumulative decay exceeds it take the per-element exact path instead.
constexpr float kMaxSpread = 64.f;
constexpr float kMaxSpreadExp = 6.2351490808e27f;   // exp(kMaxSpread)

// Sentinel for "no valid logit yet" in online softmax (finite, so that
// exp(m_old - m_new) never forms inf - inf).
constexpr float kNegBig = -1.0e30f;

}  // namespace lz
