// Single-token decode step: constant-size GLA state plus a ring-buffer
// window (English gist.science summary, section 2.A "State Update"; the
// fixed-size KV cache of the Chinese summary, section 2.1).
//
// One CTA per (batch, head), 256 threads.  The step is bound by HBM: the
// fp32 state S[dk][dv] is read once and written once, the window caches are
// read once.  The state loads are issued first (16-byte vectors, a warp
// covers one 512-byte row) so they are in flight while the gate and the
// feature maps are computed; the update S <- diag(gamma) S + phi_k v^T and
// the read-out o = S^T phi_q happen in the same pass over the registers.
#include "common.cuh"
#include "lizard_internal.h"

namespace lz {

// Load 8 consecutive activations as fp32 (one 16-byte vector for bf16).
LZ_DEV void load8(const __nv_bfloat16 *p, float *o) {
  const uint4 u = *reinterpret_cast<const uint4 *>(p);
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    o[2 * i] = f.x;
    o[2 * i + 1] = f.y;
  }
}
LZ_DEV void load8(const float *p, float *o) {
  const float4 a = *reinterpret_cast<const float4 *>(p);
  const float4 b = *reinterpret_cast<const float4 *>(p + 4);
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
  o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}

template <typename T, int D>
__global__ void __launch_bounds__(256) decode_kernel(DecodeArgs p) {
  constexpr int F = D / 2;
  constexpr int CG = D / 4;            // float4 column groups of a state row
  constexpr int RG = 256 / CG;         // row groups
  constexpr int RPG = D / RG;          // rows per thread
  constexpr int VG = D / 8;            // 8-wide column groups of a value row
  constexpr int EG = 256 / VG;         // entry groups for the value sum
  constexpr int PARTS = 256 / D;       // split of the feature-map dot products
  __shared__ float xq[D], xk[D], xv[D], gam[D], phq[D], phk[D];
  __shared__ float zpart[PARTS][D];
  __shared__ float red[EG > RG ? EG : RG][D];
  __shared__ float ogla[D];
  __shared__ float stat[4];
  extern __shared__ float logits[];    // [window + M]
  const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const T *qs = static_cast<const T *>(p.q) + (size_t)bh * D;
  const T *ks = static_cast<const T *>(p.k) + (size_t)bh * D;
  const T *vs = static_cast<const T *>(p.v) + (size_t)bh * D;
  const T *gs = static_cast<const T *>(p.g) + (size_t)bh * D;
  float *S = p.state + (size_t)bh * D * D;

  // 1. state loads in flight first
  const int cg = tid % CG, rg = tid / CG;
  float4 sreg[RPG];
#pragma unroll
  for (int r = 0; r < RPG; ++r)
    sreg[r] = *reinterpret_cast<const float4 *>(S + (size_t)(rg * RPG + r) * D + cg * 4);

  // 2. token, gate
  if (tid < D) {
    xq[tid] = to_f32(qs[tid]);
    xk[tid] = to_f32(ks[tid]);
    xv[tid] = to_f32(vs[tid]);
    gam[tid] = expf(log_decay(to_f32(gs[tid]), p.inv_tau));
  }
  __syncthreads();

  // 3. feature maps phi(x) = [softmax(x W), softmax(-x W)]
  {
    const int o = tid % D, part = tid / D;
    const int map = o / F, f = o % F;
    const float *W = map == 0 ? p.wq : p.wk;
    const float *x = map == 0 ? xq : xk;
    float z = 0.f;
    if (W) {
      const float *Wh = W + (size_t)h * D * F;
      const int i0 = part * (D / PARTS);
#pragma unroll 8
      for (int i = i0; i < i0 + D / PARTS; ++i) z = fmaf(x[i], Wh[(size_t)i * F + f], z);
    }
    zpart[part][o] = z;
  }
  __syncthreads();
  if (warp < 2) {
    const int map = warp;
    const float *W = map == 0 ? p.wq : p.wk;
    float *out = map == 0 ? phq : phk;
    const float *x = map == 0 ? xq : xk;
    if (!W) {
      for (int i = lane; i < D; i += 32) out[i] = x[i];
    } else {
      constexpr int ZJ = F / 32;
      float z[ZJ];
      float mx = kNegBig, mn = -kNegBig;
#pragma unroll
      for (int j = 0; j < ZJ; ++j) {
        float acc = 0.f;
#pragma unroll
        for (int pp = 0; pp < PARTS; ++pp) acc += zpart[pp][map * F + lane + 32 * j];
        z[j] = acc;
        mx = fmaxf(mx, acc);
        mn = fminf(mn, acc);
      }
      mx = warp_max(mx);
      mn = -warp_max(-mn);
      float sp = 0.f, sn = 0.f, ep[ZJ], en[ZJ];
#pragma unroll
      for (int j = 0; j < ZJ; ++j) {
        ep[j] = expf(z[j] - mx);
        en[j] = expf(mn - z[j]);
        sp += ep[j];
        sn += en[j];
      }
      sp = 1.f / warp_sum(sp);
      sn = 1.f / warp_sum(sn);
#pragma unroll
      for (int j = 0; j < ZJ; ++j) {
        out[lane + 32 * j] = ep[j] * sp;
        out[F + lane + 32 * j] = en[j] * sn;
      }
    }
  }
  __syncthreads();

  // 4. one pass over the state: update, store, read out
  {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 v4 = make_float4(xv[cg * 4], xv[cg * 4 + 1], xv[cg * 4 + 2], xv[cg * 4 + 3]);
#pragma unroll
    for (int r = 0; r < RPG; ++r) {
      const int i = rg * RPG + r;
      const float gi = gam[i], ki = phk[i], qi = phq[i];
      float4 s = sreg[r];
      s.x = fmaf(gi, s.x, ki * v4.x);
      s.y = fmaf(gi, s.y, ki * v4.y);
      s.z = fmaf(gi, s.z, ki * v4.z);
      s.w = fmaf(gi, s.w, ki * v4.w);
      *reinterpret_cast<float4 *>(S + (size_t)i * D + cg * 4) = s;
      acc.x = fmaf(qi, s.x, acc.x);
      acc.y = fmaf(qi, s.y, acc.y);
      acc.z = fmaf(qi, s.z, acc.z);
      acc.w = fmaf(qi, s.w, acc.w);
    }
    red[rg][cg * 4] = acc.x;
    red[rg][cg * 4 + 1] = acc.y;
    red[rg][cg * 4 + 2] = acc.z;
    red[rg][cg * 4 + 3] = acc.w;
  }
  __syncthreads();
  if (tid < D) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < RG; ++r) s += red[r][tid];
    ogla[tid] = s;
  }

  // 5. anchor window: slots [0, n) of the ring plus the meta tokens
  const long long pos = p.pos[b];
  const int W = p.window;
  const int slot = (int)(pos % W);
  const int n = (int)(pos + 1 < (long long)W ? pos + 1 : W);
  const int ntot = n + p.M;
  const T *kc = static_cast<const T *>(p.k_cache) + (size_t)bh * W * D;
  const T *vc = static_cast<const T *>(p.v_cache) + (size_t)bh * W * D;
  for (int j = warp; j < ntot; j += 8) {
    float dot = 0.f;
    if (j < n) {
      const T *kr = j == slot ? ks : kc + (size_t)j * D;
      for (int i = lane; i < D; i += 32) dot = fmaf(xq[i], to_f32(kr[i]), dot);
    } else {
      const float *mk = p.meta_k + ((size_t)h * p.M + (j - n)) * D;
      for (int i = lane; i < D; i += 32) dot = fmaf(xq[i], mk[i], dot);
    }
    dot = warp_sum(dot);
    if (lane == 0) logits[j] = dot * p.scale;
  }
  __syncthreads();
  if (warp == 0) {
    float mx = kNegBig;
    for (int j = lane; j < ntot; j += 32) mx = fmaxf(mx, logits[j]);
    mx = warp_max(mx);
    float sum = 0.f;
    for (int j = lane; j < ntot; j += 32) {
      const float e = expf(logits[j] - mx);
      logits[j] = e;
      sum += e;
    }
    sum = warp_sum(sum);
    if (lane == 0) stat[0] = 1.f / sum;
  }
  __syncthreads();
  {
    const int vg = tid % VG, eg = tid / VG;
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.f;
    for (int j = eg; j < ntot; j += EG) {
      const float pj = logits[j];
      float vv[8];
      if (j < n) {
        load8((j == slot ? vs : vc + (size_t)j * D) + vg * 8, vv);
      } else if (p.meta_v) {
        const float *mv = p.meta_v + ((size_t)h * p.M + (j - n)) * D + vg * 8;
#pragma unroll
        for (int c = 0; c < 8; ++c) vv[c] = mv[c];
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) vv[c] = 0.f;
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = fmaf(pj, vv[c], acc[c]);
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) red[eg][vg * 8 + c] = acc[c];
  }
  __syncthreads();
  if (tid < D) {
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < EG; ++e) s += red[e][tid];
    const float alpha = p.alpha ? p.alpha[h] : 1.f;
    T *os = static_cast<T *>(p.o) + (size_t)bh * D;
    os[tid] = from_f32<T>(ogla[tid] + alpha * s * stat[0]);
    // 6. the new token enters the ring (the slot is read from the inputs above)
    T *kcw = static_cast<T *>(p.k_cache) + ((size_t)bh * W + slot) * D;
    T *vcw = static_cast<T *>(p.v_cache) + ((size_t)bh * W + slot) * D;
    kcw[tid] = ks[tid];
    vcw[tid] = vs[tid];
  }
}

__global__ void advance_pos_kernel(int64_t *pos, int B) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) pos[b] += 1;
}

template <typename T, int D>
static cudaError_t launch_decode_t(const DecodeArgs &a, int B, int64_t *pos, cudaStream_t s) {
  const size_t smem = (size_t)(a.window + a.M) * sizeof(float);
  auto k = decode_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<B * a.H, 256, smem, s>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  advance_pos_kernel<<<(B + 127) / 128, 128, 0, s>>>(pos, B);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a, int B, int D, bool bf16, int64_t *pos, cudaStream_t s) {
  if (bf16) return D == 128 ? launch_decode_t<__nv_bfloat16, 128>(a, B, pos, s) : launch_decode_t<__nv_bfloat16, 64>(a, B, pos, s);
  return D == 128 ? launch_decode_t<float, 128>(a, B, pos, s) : launch_decode_t<float, 64>(a, B, pos, s);
}

}  // namespace lz
