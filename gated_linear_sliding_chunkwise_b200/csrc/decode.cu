// Single-token decode step: constant-size GLA state plus a ring-buffer
// window (English gist.science summary, section 2.A "State Update"; the
// fixed-size KV cache of the Chinese summary, section 2.1).
//
// One CTA per (batch, head), 256 threads.  The step is bound by HBM: the
// fp32 state S[dk][dv] is read and written once (2/3 of the bytes) and the
// window caches are read once.  Every long-latency load is issued at the
// start so the CTA pays about one memory latency:
//   - the state goes straight to registers (16-byte vectors, one warp per
//     512-byte row),
//   - the first block of up to 128 window slots (keys and values) is copied
//     to shared memory with cp.async,
//   - the feature-map weights (L2-resident, shared by the batch) are read
//     as 16-byte vectors, all in flight together.
// The state update S <- diag(gamma) S + phi_k v^T and the read-out
// o = S^T phi_q happen in the same pass over the registers.
#include "common.cuh"
#include "lizard_internal.h"

namespace lz {

constexpr int kDecWB = 128;   // window slots staged in shared memory per block

LZ_DEV void cp_async16(void *smem, const void *gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
LZ_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
LZ_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// 8 consecutive activations as fp32 (one 16-byte vector for bf16).
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

// Stage window slots [j0, j0 + nb) of both caches into shared memory.
template <typename T, int D>
LZ_DEV void stage_window(T *Ks, T *Vs, const T *kc, const T *vc, int j0, int nb, int tid) {
  constexpr int VPR = D * (int)sizeof(T) / 16;   // 16-byte vectors per row
  for (int e = tid; e < nb * VPR; e += 256) {
    const int r = e / VPR, c = e % VPR;
    cp_async16(reinterpret_cast<char *>(Ks + (size_t)r * D) + c * 16,
               reinterpret_cast<const char *>(kc + (size_t)(j0 + r) * D) + c * 16);
    cp_async16(reinterpret_cast<char *>(Vs + (size_t)r * D) + c * 16,
               reinterpret_cast<const char *>(vc + (size_t)(j0 + r) * D) + c * 16);
  }
  cp_async_commit();
}

template <typename T, int D>
__global__ void __launch_bounds__(256, 2) decode_kernel(DecodeArgs p) {
  constexpr int F = D / 2;
  constexpr int CG = D / 4;            // float4 column groups of a state row
  constexpr int RG = 256 / CG;         // row groups
  constexpr int RPG = D / RG;          // state rows per thread
  constexpr int VG = D / 8;            // 8-wide column groups of a value row
  constexpr int EG = 256 / VG;         // slot groups for the value sum
  constexpr int FG = F / 4;            // float4 feature groups of a W row
  constexpr int IP = 128 / FG;         // parts of the dk range per map
  constexpr int IPL = D / IP;          // dk rows per part
  __shared__ float xq[D], xk[D], xv[D], gam[D], phq[D], phk[D];
  __shared__ float zpart[2][IP][F];
  __shared__ float red[EG > RG ? EG : RG][D];
  __shared__ float ogla[D];
  __shared__ float wred[2][8];
  extern __shared__ __align__(16) unsigned char dyn[];
  T *Ks = reinterpret_cast<T *>(dyn);                 // [kDecWB][D]
  T *Vs = Ks + kDecWB * D;                             // [kDecWB][D]
  float *logits = reinterpret_cast<float *>(Vs + kDecWB * D);   // [window + M]

  const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const T *qs = static_cast<const T *>(p.q) + (size_t)bh * D;
  const T *ks = static_cast<const T *>(p.k) + (size_t)bh * D;
  const T *vs = static_cast<const T *>(p.v) + (size_t)bh * D;
  const T *gs = static_cast<const T *>(p.g) + (size_t)bh * D;
  float *S = p.state + (size_t)bh * D * D;
  const long long pos = p.pos[b];
  const int W = p.window;
  const int slot = (int)(pos % W);
  const int n = (int)(pos + 1 < (long long)W ? pos + 1 : W);
  const int ntot = n + p.M;
  const T *kc = static_cast<const T *>(p.k_cache) + (size_t)bh * W * D;
  const T *vc = static_cast<const T *>(p.v_cache) + (size_t)bh * W * D;

  // 1. everything long-latency in flight: window block 0, state, token
  const int nb0 = min(n, kDecWB);
  stage_window<T, D>(Ks, Vs, kc, vc, 0, nb0, tid);
  const int cg = tid % CG, rg = tid / CG;
  float4 sreg[RPG];
#pragma unroll
  for (int r = 0; r < RPG; ++r)
    sreg[r] = *reinterpret_cast<const float4 *>(S + (size_t)(rg * RPG + r) * D + cg * 4);
  if (tid < D) {
    xq[tid] = to_f32(qs[tid]);
    xk[tid] = to_f32(ks[tid]);
    xv[tid] = to_f32(vs[tid]);
    gam[tid] = expf(log_decay(to_f32(gs[tid]), p.inv_tau));
  }
  __syncthreads();

  // 2. feature maps phi(x) = [softmax(x W), softmax(-x W)]: thread = (map,
  //    4 features, IPL rows of W), all W vectors loaded before use
  {
    const int map = tid >> 7, r = tid & 127, fg = r % FG, ip = r / FG;
    const float *Wm = map == 0 ? p.wq : p.wk;
    const float *x = map == 0 ? xq : xk;
    float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    if (Wm) {
      const float *Wh = Wm + (size_t)h * D * F + (size_t)(ip * IPL) * F + fg * 4;
      constexpr int BATCH = IPL < 4 ? IPL : 4;   // bounds live registers next to the state
#pragma unroll
      for (int i0 = 0; i0 < IPL; i0 += BATCH) {
        float4 wv[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) wv[i] = *reinterpret_cast<const float4 *>(Wh + (size_t)(i0 + i) * F);
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          const float xi = x[ip * IPL + i0 + i];
          z.x = fmaf(xi, wv[i].x, z.x);
          z.y = fmaf(xi, wv[i].y, z.y);
          z.z = fmaf(xi, wv[i].z, z.z);
          z.w = fmaf(xi, wv[i].w, z.w);
        }
      }
    }
    zpart[map][ip][fg * 4] = z.x;
    zpart[map][ip][fg * 4 + 1] = z.y;
    zpart[map][ip][fg * 4 + 2] = z.z;
    zpart[map][ip][fg * 4 + 3] = z.w;
  }
  __syncthreads();
  if (warp < 2) {
    const int map = warp;
    const float *Wm = map == 0 ? p.wq : p.wk;
    float *out = map == 0 ? phq : phk;
    const float *x = map == 0 ? xq : xk;
    if (!Wm) {
      for (int i = lane; i < D; i += 32) out[i] = x[i];
    } else {
      constexpr int ZJ = F / 32;
      float z[ZJ];
      float mx = kNegBig, mn = -kNegBig;
#pragma unroll
      for (int j = 0; j < ZJ; ++j) {
        float acc = 0.f;
#pragma unroll
        for (int pp = 0; pp < IP; ++pp) acc += zpart[map][pp][lane + 32 * j];
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

  // 3. one pass over the state: update, store, read out
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

  // 4. anchor logits: one slot per thread, 16-byte loads from shared memory
  const T *newk = ks;
  for (int j0 = 0; j0 < n; j0 += kDecWB) {
    const int nb = min(kDecWB, n - j0);
    if (j0 > 0) {
      __syncthreads();
      stage_window<T, D>(Ks, Vs, kc, vc, j0, nb, tid);
    }
    cp_async_wait_all();
    __syncthreads();
    for (int jj = tid; jj < nb; jj += 256) {
      const int j = j0 + jj;
      const T *kr = j == slot ? newk : Ks + (size_t)jj * D;
      float dot = 0.f;
      // start each slot at a different 16-byte column so that a warp's
      // shared-memory reads spread over the banks
#pragma unroll
      for (int c0 = 0; c0 < D / 8; ++c0) {
        const int c = (c0 + jj) % (D / 8);
        float kv[8];
        load8(kr + c * 8, kv);
#pragma unroll
        for (int u = 0; u < 8; ++u) dot = fmaf(xq[c * 8 + u], kv[u], dot);
      }
      logits[j] = dot * p.scale;
    }
  }
  for (int m = tid; m < p.M; m += 256) {
    const float *mk = p.meta_k + ((size_t)h * p.M + m) * D;
    float dot = 0.f;
    for (int i = 0; i < D; ++i) dot = fmaf(xq[i], mk[i], dot);
    logits[n + m] = dot * p.scale;
  }
  __syncthreads();
  // softmax over the ntot logits (block-wide max and sum)
  {
    float mx = kNegBig;
    for (int j = tid; j < ntot; j += 256) mx = fmaxf(mx, logits[j]);
    mx = warp_max(mx);
    if (lane == 0) wred[0][warp] = mx;
    __syncthreads();
    mx = wred[0][0];
#pragma unroll
    for (int w = 1; w < 8; ++w) mx = fmaxf(mx, wred[0][w]);
    float sum = 0.f;
    for (int j = tid; j < ntot; j += 256) {
      const float e = expf(logits[j] - mx);
      logits[j] = e;
      sum += e;
    }
    sum = warp_sum(sum);
    if (lane == 0) wred[1][warp] = sum;
  }
  __syncthreads();
  float inv_sum = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) inv_sum += wred[1][w];
  inv_sum = 1.f / inv_sum;

  // 5. o_swa = sum_j p_j v_j (+ meta values)
  const int vg = tid % VG, eg = tid / VG;
  float acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;
  for (int j0 = 0; j0 < n; j0 += kDecWB) {
    const int nb = min(kDecWB, n - j0);
    if (j0 > 0 || n > kDecWB) {   // the staged block is not the one needed
      __syncthreads();
      stage_window<T, D>(Ks, Vs, kc, vc, j0, nb, tid);
      cp_async_wait_all();
      __syncthreads();
    }
    for (int jj = eg; jj < nb; jj += EG) {
      const int j = j0 + jj;
      float vv[8];
      load8((j == slot ? vs : Vs + (size_t)jj * D) + vg * 8, vv);
      const float pj = logits[j];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = fmaf(pj, vv[c], acc[c]);
    }
  }
  if (p.meta_v) {
    for (int m = eg; m < p.M; m += EG) {
      const float pj = logits[n + m];
      const float *mv = p.meta_v + ((size_t)h * p.M + m) * D + vg * 8;
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = fmaf(pj, mv[c], acc[c]);
    }
  }
  __syncthreads();
#pragma unroll
  for (int c = 0; c < 8; ++c) red[eg][vg * 8 + c] = acc[c];
  __syncthreads();
  if (tid < D) {
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < EG; ++e) s += red[e][tid];
    const float alpha = p.alpha ? p.alpha[h] : 1.f;
    T *os = static_cast<T *>(p.o) + (size_t)bh * D;
    os[tid] = from_f32<T>(ogla[tid] + alpha * s * inv_sum);
    // 6. the new token enters the ring (its slot was read from the inputs)
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
  const size_t smem = 2 * (size_t)kDecWB * D * sizeof(T) + (size_t)(a.window + a.M) * sizeof(float);
  auto k = decode_kernel<T, D>;
  // The attribute is per device; set it when this device has not yet seen a
  // launch this large (decode is called once per generated token).
  static size_t configured[64] = {};
  int dev = 0;
  cudaError_t e0 = cudaGetDevice(&dev);
  if (e0 != cudaSuccess) return e0;
  if (dev < 0 || dev >= 64 || smem > configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = smem;
  }
  k<<<B * a.H, 256, smem, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  advance_pos_kernel<<<(B + 127) / 128, 128, 0, s>>>(pos, B);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a, int B, int D, bool bf16, int64_t *pos, cudaStream_t s) {
  if (bf16) return D == 128 ? launch_decode_t<__nv_bfloat16, 128>(a, B, pos, s) : launch_decode_t<__nv_bfloat16, 64>(a, B, pos, s);
  return D == 128 ? launch_decode_t<float, 128>(a, B, pos, s) : launch_decode_t<float, 64>(a, B, pos, s);
}

}  // namespace lz
