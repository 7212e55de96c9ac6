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
#include <atomic>

#include "common.cuh"
#include "lizard_internal.h"

namespace lz {

constexpr int kDecWB = 128;   // window slots staged in shared memory per block

__global__ void advance_pos_kernel(int64_t *pos, int B) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) pos[b] += 1;
}

// The pos increment folded into the step: every CTA arrives on a counter
// once it has read all the pos values it uses (one thread per CTA, after a
// barrier behind those reads); the last to arrive adds 1 to every pos and
// resets the counter.  Launches take their counter from a ring of
// kPosSlots, so steps in flight on different streams do not share one.
constexpr int kPosSlots = 64;
__device__ unsigned int g_pos_arrivals[kPosSlots];

LZ_DEV void pos_arrive(const DecodeArgs &p) {
  if (!p.pos_inc) return;
  __threadfence();
  const unsigned int ctas = gridDim.x * gridDim.y * gridDim.z;
  if (atomicAdd(&g_pos_arrivals[p.pos_slot], 1u) == ctas - 1) {
    g_pos_arrivals[p.pos_slot] = 0u;
    for (int b = 0; b < p.pos_B; ++b) p.pos_inc[b] += 1;
  }
}

int next_pos_slot() {
  static std::atomic<unsigned int> ctr{0};
  return (int)(ctr.fetch_add(1u) % kPosSlots);
}

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
  const T *gs = static_cast<const T *>(p.g) + (size_t)bh * (p.scalar_gate ? 1 : D);
  float *S = p.state + (size_t)bh * D * D;
  const long long pos = p.pos[b];
  if (p.pos_inc) {   // every thread has read pos: this CTA arrives
    __syncthreads();
    if (tid == 0) pos_arrive(p);
  }
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
    gam[tid] = expf(log_decay(to_f32(gs[p.scalar_gate ? 0 : tid]), p.inv_tau));
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


// ------------------------------------------------------------------------
// Streaming decode (bf16, d = 128, window <= 128, M <= 16): a persistent
// kernel, one CTA per SM.  The (batch, head) pairs are taken in head-major
// order, a contiguous run per CTA, so a CTA keeps the feature-map weights and
// meta tokens of its current head in shared memory.  Each pair is four
// chunks of at most 32 KB -- the key window (with the new token's q, k, v, g
// riding along), state rows 0..63, state rows 64..127, the value window --
// that a producer warp copies into a ring of shared-memory slots with bulk
// copies (cp.async.bulk, completion on an mbarrier), up to kStreamSlots
// chunks ahead of the consumers, so HBM keeps streaming while the CTA
// computes.  The updated state goes back with 16-byte stores straight from
// registers.
namespace {

constexpr int kStreamSlots = 4;
constexpr uint32_t kChunkBytes = 32768;
constexpr int SD = 128, SF = 64;
constexpr int kMaxRunPairs = 64;                  // pairs whose (n, slot) are precomputed
constexpr size_t kRingOff = 0;
constexpr size_t kWOff = kStreamSlots * (size_t)kChunkBytes;   // W_q | W_k, fp32 [128][64] each
constexpr size_t kTokOff = kWOff + 2 * SD * SF * 4;           // [q, k, v, g][128] bf16 (slot 0's token)
constexpr size_t kMetaOff = kTokOff + 4 * SD * 2;   // meta_k | meta_v, fp32 [M][128]

__device__ uint32_t g_decode_status;   // bit 1: a bounded wait gave up

LZ_DEV uint32_t s_addr(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
LZ_DEV void s_mbar_init(uint64_t *bar) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(s_addr(bar)) : "memory");
}
LZ_DEV void s_mbar_expect(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(s_addr(bar)), "r"(bytes) : "memory");
}
LZ_DEV bool s_mbar_wait(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < (1u << 22); ++i) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(s_addr(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}
LZ_DEV void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(s_addr(dst)),
      "l"(src), "r"(bytes), "r"(s_addr(bar))
      : "memory");
}

struct PairInfo {
  int bh, h, n, slot;
};

// Pair k of this CTA's run (head-major order: q -> head q / B, batch q % B).
LZ_DEV PairInfo pair_info(const DecodeArgs &p, int B, int first, int k, const int *s_n, const int *s_slot) {
  PairInfo r;
  const int q = first + k, h = q / B, b = q % B;
  r.bh = b * p.H + h;
  r.h = h;
  if (k < kMaxRunPairs) {
    r.n = s_n[k];
    r.slot = s_slot[k];
  } else {
    const long long pos = p.pos[b];
    r.n = (int)(pos + 1 < (long long)p.window ? pos + 1 : p.window);
    r.slot = (int)(pos % p.window);
  }
  return r;
}

// Thread roles: warps 0..7 consume (256 threads), warp 8 produces (one lane
// walks the chunk sequence, waits until a slot is released -- `empty`
// mbarrier, one arrival per reading warp -- and refills it), warps 9..12
// prepare (128 threads): for each pair, as soon as its key chunk and token
// have landed, they form phi_q, phi_k, the decay gamma and the meta logits
// into a two-entry record ring, so that the consumers of the pair before
// are not held up by that work.  Consumers meet on named barrier 1, the
// prep warps on named barrier 2, only where data flows between them.
constexpr int kConsumers = 256;
constexpr int kPrep = 128;
constexpr int kDecThreads = kConsumers + 32 + kPrep;
LZ_DEV void s_mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(s_addr(bar)) : "memory");
}
LZ_DEV void s_mbar_init_n(uint64_t *bar, uint32_t n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(s_addr(bar)), "r"(n) : "memory");
}
LZ_DEV void consumers_sync() { asm volatile("bar.sync 1, %0;\n" ::"n"(kConsumers) : "memory"); }
LZ_DEV void prep_sync() { asm volatile("bar.sync 2, %0;\n" ::"n"(kPrep) : "memory"); }
// Barrier over the prep warps that also returns whether any of them passed true.
LZ_DEV bool prep_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 2, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kPrep)
      : "memory");
  return r != 0;
}
// Barrier over the consumers that also returns whether any of them passed true.
LZ_DEV bool consumers_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kConsumers)
      : "memory");
  return r != 0;
}

struct PairRec {                 // what the prep warps hand to the consumers for one pair
  float phq[SD], phk[SD], gam[SD], ml[16];
  float lg[SD];                  // window logits (scaled), slots 0 .. n - 1
  float xk[SD], xv[SD];          // the new token's k and v
};

__global__ void __launch_bounds__(kDecThreads, 1) decode_stream_kernel(const __grid_constant__ DecodeArgs p, int B, int run) {
  extern __shared__ __align__(1024) unsigned char dsm[];
  unsigned char *ring = dsm + kRingOff;
  float *Wq = reinterpret_cast<float *>(dsm + kWOff), *Wk = Wq + SD * SF;
  __nv_bfloat16 *tokring = reinterpret_cast<__nv_bfloat16 *>(dsm + kTokOff);
  float *mk_s = reinterpret_cast<float *>(dsm + kMetaOff), *mv_s = mk_s + p.M * SD;
  __shared__ uint64_t full[kStreamSlots], empty[kStreamSlots];
  __shared__ uint64_t wfull, wempty, rfull[2], rempty[2];
  __shared__ PairRec rec[2];
  __shared__ __align__(16) float zpart[8][SD];       // read-out partials per row group
  __shared__ float prob[128 + 16];
  __shared__ float red[8][SD];
  __shared__ float s_wmax[8], s_wsum[9];             // per-warp softmax maxima and sums (+ the meta sum)
  __shared__ float p_red[4][2];                      // prep: per-warp maxima, then sums
  __shared__ int s_n[kMaxRunPairs], s_slot[kMaxRunPairs];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BH = B * p.H;
  const int first = blockIdx.x * run;
  const int npairs = max(0, min(run, BH - first));
  const int nchunks = 4 * npairs;
  for (int k = tid; k < npairs && k < kMaxRunPairs; k += blockDim.x) {
    const long long pos = p.pos[(first + k) % B];
    s_n[k] = (int)(pos + 1 < (long long)p.window ? pos + 1 : p.window);
    s_slot[k] = (int)(pos % p.window);
  }
  if (tid == 0) {
    // slot 0 always holds a key chunk and its token (4 chunks per pair, 4
    // slots): only the prep warps read it
    for (int i = 0; i < kStreamSlots; ++i) {
      s_mbar_init_n(&full[i], 1);
      s_mbar_init_n(&empty[i], i == 0 ? kPrep / 32 : kConsumers / 32);
    }
    s_mbar_init_n(&wfull, 1);
    s_mbar_init_n(&wempty, kConsumers / 32 + kPrep / 32);
    for (int i = 0; i < 2; ++i) {
      s_mbar_init_n(&rfull[i], kPrep / 32);
      s_mbar_init_n(&rempty[i], kConsumers / 32);
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncthreads();
  // with the increment folded in, every pair's (n, slot) was read above
  if (tid == 0) pos_arrive(p);

  if (warp == kConsumers / 32) {
    // ------------------------------------------------------- producer ---
    if (lane == 0) {
      int prev_head = -1, nh = 0;
      bool ok = true;
      for (int c = 0; c < nchunks && ok; ++c) {
        const PairInfo pi = pair_info(p, B, first, c >> 2, s_n, s_slot);
        const int kind = c & 3, sl = c % kStreamSlots;
        if (kind == 0 && pi.h != prev_head) {
          // weights and meta tokens of the next head, once every reader is
          // done with the current ones
          if (nh > 0) ok = s_mbar_wait(&wempty, (uint32_t)(nh - 1) & 1u);
          if (!ok) break;
          const uint32_t wb = (p.wq ? SD * SF * 4 : 0) + (p.wk ? SD * SF * 4 : 0);
          const uint32_t mb = (uint32_t)p.M * SD * 4 * (p.meta_v ? 2 : 1);
          s_mbar_expect(&wfull, wb + mb);
          if (p.wq) bulk_load(Wq, p.wq + (size_t)pi.h * SD * SF, SD * SF * 4, &wfull);
          if (p.wk) bulk_load(Wk, p.wk + (size_t)pi.h * SD * SF, SD * SF * 4, &wfull);
          if (p.M > 0) bulk_load(mk_s, p.meta_k + (size_t)pi.h * p.M * SD, p.M * SD * 4, &wfull);
          if (p.M > 0 && p.meta_v) bulk_load(mv_s, p.meta_v + (size_t)pi.h * p.M * SD, p.M * SD * 4, &wfull);
          prev_head = pi.h;
          ++nh;
        }
        if (c >= kStreamSlots) ok = s_mbar_wait(&empty[sl], (uint32_t)(c / kStreamSlots - 1) & 1u);
        if (!ok) break;
        uint64_t *bar = &full[sl];
        unsigned char *dst = ring + (size_t)sl * kChunkBytes;
        if (kind == 0 || kind == 3) {
          const uint32_t bytes = (uint32_t)pi.n * SD * 2;
          const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(kind == 0 ? p.k_cache : p.v_cache) +
                                     (size_t)pi.bh * p.window * SD;
          // the new token's q, k, v and (per-dimension) g ride along with kind 0;
          // a scalar gate is a single value that the prep warps read directly
          const int ntok = p.scalar_gate ? 3 : 4;
          s_mbar_expect(bar, bytes + (kind == 0 ? (uint32_t)ntok * SD * 2 : 0));
          bulk_load(dst, src, bytes, bar);
          if (kind == 0) {
            __nv_bfloat16 *tk = tokring;   // the key chunk is always slot 0
            const void *srcs[4] = {p.q, p.k, p.v, p.g};
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (u < ntok)
                bulk_load(tk + u * SD, static_cast<const __nv_bfloat16 *>(srcs[u]) + (size_t)pi.bh * SD, SD * 2,
                          bar);
          }
        } else {
          s_mbar_expect(bar, kChunkBytes);
          bulk_load(dst, p.state + (size_t)pi.bh * SD * SD + (size_t)(kind - 1) * 64 * SD, kChunkBytes, bar);
        }
      }
      if (!ok) atomicOr(&g_decode_status, 1u);
    }
    return;
  }

  if (warp > kConsumers / 32) {
    // ----------------------------------------------------------- prep ---
    const int pt = tid - (kConsumers + 32), pw = pt >> 5;
    const __nv_bfloat16 *tk = tokring;   // slot 0
    int cur_head = -1, nh = 0;
    for (int k = 0; k < npairs; ++k) {
      const PairInfo pi = pair_info(p, B, first, k, s_n, s_slot);
      bool ok = s_mbar_wait(&full[0], (uint32_t)k & 1u);
      if (pi.h != cur_head) {
        ok &= s_mbar_wait(&wfull, (uint32_t)nh & 1u);
        ++nh;
        cur_head = pi.h;
      }
      if (k >= 2) ok &= s_mbar_wait(&rempty[k & 1], (uint32_t)((k >> 1) - 1) & 1u);
      if (prep_any(!ok)) {   // all prep warps stop together; the consumers time out on the record
        atomicOr(&g_decode_status, 1u);
        return;
      }
      PairRec &R = rec[k & 1];
      // the new token's k, v for the consumers, and the window logits
      // s q . k_j: thread = slot j (the slot being replaced takes the new key)
      R.xk[pt] = __bfloat162float(tk[SD + pt]);
      R.xv[pt] = __bfloat162float(tk[2 * SD + pt]);
      if (pt < pi.n) {
        const __nv_bfloat16 *kr = pt == pi.slot ? tk + SD : reinterpret_cast<const __nv_bfloat16 *>(ring) + (size_t)pt * SD;
        float d0 = 0.f, d1 = 0.f;
#pragma unroll 4
        for (int c0 = 0; c0 < 16; ++c0) {
          const int cc = (c0 + pt) & 15;   // spread a warp's reads over the banks
          float kv[8], q8[8];
          load8(kr + cc * 8, kv);
          load8(tk + cc * 8, q8);
#pragma unroll
          for (int u = 0; u < 8; u += 2) {
            d0 = fmaf(q8[u], kv[u], d0);
            d1 = fmaf(q8[u + 1], kv[u + 1], d1);
          }
        }
        R.lg[pt] = (d0 + d1) * p.scale;
      }
      const __nv_bfloat16 gv = p.scalar_gate ? static_cast<const __nv_bfloat16 *>(p.g)[pi.bh] : tk[3 * SD + pt];
      R.gam[pt] = expf(log_decay(__bfloat162float(gv), p.inv_tau));
      // z = x W: thread = (map, feature); 4 partial sums over the 128 rows
      const int map = pt >> 6, f = pt & 63;
      const __nv_bfloat16 *x = tk + map * SD;
      const float *W = map == 0 ? Wq : Wk;
      const bool has_w = map == 0 ? p.wq != nullptr : p.wk != nullptr;
      float z = 0.f;
      if (has_w) {
        float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int i = 0; i < SD; ++i) a4[i & 3] = fmaf(__bfloat162float(x[i]), W[i * SF + f], a4[i & 3]);
        z = (a4[0] + a4[1]) + (a4[2] + a4[3]);
      }
      // phi = [softmax(z), softmax(-z)] over the 64 features of this map
      // (two warps per map meet through p_red)
      float mx = warp_max(z), mn = warp_max(-z);
      if (lane == 0) { p_red[pw][0] = mx; p_red[pw][1] = mn; }
      prep_sync();
      mx = fmaxf(p_red[pw][0], p_red[pw ^ 1][0]);
      mn = fmaxf(p_red[pw][1], p_red[pw ^ 1][1]);
      const float ep = expf(z - mx), en = expf(-z - mn);
      const float sp = warp_sum(ep), sn = warp_sum(en);
      prep_sync();
      if (lane == 0) { p_red[pw][0] = sp; p_red[pw][1] = sn; }
      prep_sync();
      const float isp = 1.f / (p_red[pw][0] + p_red[pw ^ 1][0]);
      const float isn = 1.f / (p_red[pw][1] + p_red[pw ^ 1][1]);
      float *ph = map == 0 ? R.phq : R.phk;
      if (has_w) {
        ph[f] = ep * isp;
        ph[SF + f] = en * isn;
      } else {   // identity map
        ph[f] = __bfloat162float(x[f]);
        ph[SF + f] = __bfloat162float(x[SF + f]);
      }
      // meta logits: thread = (meta token m, 16 dimensions), 8 lanes per token
      {
        const int m = pt >> 3, part = pt & 7;
        float d = 0.f;
        if (m < p.M) {
#pragma unroll
          for (int i = 0; i < 16; ++i) d = fmaf(__bfloat162float(tk[part * 16 + i]), mk_s[m * SD + part * 16 + i], d);
        }
        d += __shfl_xor_sync(0xffffffffu, d, 4);
        d += __shfl_xor_sync(0xffffffffu, d, 2);
        d += __shfl_xor_sync(0xffffffffu, d, 1);
        if (m < p.M && part == 0) R.ml[m] = d * p.scale;
      }
      __syncwarp();
      if (lane == 0) {
        s_mbar_arrive(&rfull[k & 1]);
        s_mbar_arrive(&empty[0]);   // the token and the weights are read
        if (k + 1 >= npairs || pair_info(p, B, first, k + 1, s_n, s_slot).h != pi.h) s_mbar_arrive(&wempty);
      }
      prep_sync();   // p_red is reused by the next pair
    }
    return;
  }

  // ---------------------------------------------------------- consumers ---
  const int cg = tid & 31, rg = tid >> 5;   // state: float4 column group, row group (8 rows)
  const int vg = tid & 15, eg = tid >> 4;   // values: 8 columns, slot group
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float inv_l = 0.f, alpha_h = 1.f;   // this pair's 1 / softmax sum; this head's alpha
  int cur_head = -1, nh = 0;
  bool failed = false;
  int c_stop = nchunks;
  PairInfo pi{0, 0, 0, 0};
  for (int c = 0; c < nchunks; ++c) {
    const int kind = c & 3, sl = c % kStreamSlots, kp = c >> 2;
    const unsigned char *chunk = ring + (size_t)sl * kChunkBytes;
    bool new_head = false;
    if (kind == 0) {
      pi = pair_info(p, B, first, kp, s_n, s_slot);
      new_head = pi.h != cur_head;
      acc = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // the key chunk (slot 0) is read by the prep warps only: the consumers
    // start a pair on its record
    bool ok = kind == 0 ? s_mbar_wait(&rfull[kp & 1], (uint32_t)(kp >> 1) & 1u)
                        : s_mbar_wait(&full[sl], (uint32_t)(c / kStreamSlots) & 1u);
    if (new_head) {
      ok &= s_mbar_wait(&wfull, (uint32_t)nh & 1u);   // meta values
      ++nh;
      cur_head = pi.h;
      alpha_h = p.alpha ? p.alpha[pi.h] : 1.f;
    }
    if (!ok) {
      atomicOr(&g_decode_status, 1u);
      failed = true;
    }
    // A failed (bounded) wait inside a pair only leaves stale slot data; the
    // consumers decide together, at the next pair, to stop.  The vote is
    // also the barrier that ends the previous pair's read-out.
    if (kind == 0 && consumers_any(failed)) {
      c_stop = c;
      break;
    }
    const int n = pi.n, slot = pi.slot, h = pi.h, bh = pi.bh;
    const PairRec &R = rec[kp & 1];
    if (kind == 0) {
      // softmax over the n window logits (from the prep warps) and the M
      // meta logits, spread over the consumer warps: warp maxima, then one
      // exp per slot and warp sums
      const int j = tid >> 1, half = tid & 1;
      const float lj = j < n ? R.lg[j] : kNegBig;
      {
        const float wm = warp_max(lj);
        if (lane == 0) s_wmax[warp] = wm;
      }
      consumers_sync();
      float mx = kNegBig;
#pragma unroll
      for (int w = 0; w < 8; ++w) mx = fmaxf(mx, s_wmax[w]);
      for (int m = 0; m < p.M; ++m) mx = fmaxf(mx, R.ml[m]);
      {
        const float e = j < n ? expf(lj - mx) : 0.f;
        if (j < n && half == 0) prob[j] = e;
        const float ws = warp_sum(half == 0 ? e : 0.f);
        if (lane == 0) s_wsum[warp] = ws;
        if (warp == 0) {   // the meta tokens
          const float em = lane < p.M ? expf(R.ml[lane] - mx) : 0.f;
          if (lane < p.M) prob[n + lane] = em;
          const float ms = warp_sum(em);
          if (lane == 0) s_wsum[8] = ms;
        }
      }
      consumers_sync();   // the probabilities are ready
      {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < 9; ++w) sum += s_wsum[w];
        inv_l = 1.f / sum;
      }
    } else if (kind == 1 || kind == 2) {
      // ---- state rows (kind - 1) * 64 .. + 63: update, store, read out
      const float4 v4 = make_float4(R.xv[cg * 4], R.xv[cg * 4 + 1], R.xv[cg * 4 + 2], R.xv[cg * 4 + 3]);
      float *S = p.state + (size_t)bh * SD * SD;
      float4 sv[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) sv[r] = *reinterpret_cast<const float4 *>(chunk + (size_t)(rg * 8 + r) * SD * 4 + cg * 16);
      __syncwarp();
      if (lane == 0) s_mbar_arrive(&empty[sl]);
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int i = (kind - 1) * 64 + rg * 8 + r;
        const float gi = R.gam[i], ki = R.phk[i], qi = R.phq[i];
        float4 s = sv[r];
        s.x = fmaf(gi, s.x, ki * v4.x);
        s.y = fmaf(gi, s.y, ki * v4.y);
        s.z = fmaf(gi, s.z, ki * v4.z);
        s.w = fmaf(gi, s.w, ki * v4.w);
        *reinterpret_cast<float4 *>(S + (size_t)i * SD + cg * 4) = s;
        acc.x = fmaf(qi, s.x, acc.x);
        acc.y = fmaf(qi, s.y, acc.y);
        acc.z = fmaf(qi, s.z, acc.z);
        acc.w = fmaf(qi, s.w, acc.w);
      }
    } else {
      // ---- o_swa = sum_j p_j v_j (+ meta values); the replaced slot takes
      //      the new value; then o = o_gla + alpha o_swa / l
      float a8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) a8[u] = 0.f;
      for (int j = eg; j < n; j += 16) {
        float vv[8];
        if (j == slot) {
#pragma unroll
          for (int u = 0; u < 8; ++u) vv[u] = R.xv[vg * 8 + u];
        } else {
          load8(reinterpret_cast<const __nv_bfloat16 *>(chunk) + (size_t)j * SD + vg * 8, vv);
        }
        const float pj = prob[j];
#pragma unroll
        for (int u = 0; u < 8; ++u) a8[u] = fmaf(pj, vv[u], a8[u]);
      }
      __syncwarp();
      if (lane == 0) s_mbar_arrive(&empty[sl]);
      if (p.meta_v)
        for (int m = eg; m < p.M; m += 16) {
          const float pj = prob[n + m];
#pragma unroll
          for (int u = 0; u < 8; ++u) a8[u] = fmaf(pj, mv_s[m * SD + vg * 8 + u], a8[u]);
        }
      __syncwarp();
      if (lane == 0 && (kp + 1 >= npairs || pair_info(p, B, first, kp + 1, s_n, s_slot).h != h))
        s_mbar_arrive(&wempty);   // last pair of this head: its meta values are read
#pragma unroll
      for (int u = 0; u < 8; ++u) a8[u] += __shfl_xor_sync(0xffffffffu, a8[u], 16);
      if (lane < 16)
#pragma unroll
        for (int u = 0; u < 8; ++u) red[warp][vg * 8 + u] = a8[u];
      // the read-out partials of the two state chunks, per row group
      *reinterpret_cast<float4 *>(&zpart[rg][cg * 4]) = acc;
      consumers_sync();
      if (tid < SD) {
        float so = 0.f, sg = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) so += red[w][tid];
#pragma unroll
        for (int r = 0; r < 8; ++r) sg += zpart[r][tid];
        static_cast<__nv_bfloat16 *>(p.o)[(size_t)bh * SD + tid] = __float2bfloat16_rn(sg + alpha_h * so * inv_l);
        // the new token enters the ring (both windows were read above); the
        // fp32 copies hold it exactly (bf16 -> fp32 -> bf16 is lossless)
        const size_t cw = ((size_t)bh * p.window + slot) * SD + tid;
        static_cast<__nv_bfloat16 *>(p.k_cache)[cw] = __float2bfloat16_rn(R.xk[tid]);
        static_cast<__nv_bfloat16 *>(p.v_cache)[cw] = __float2bfloat16_rn(R.xv[tid]);
      }
      // the record of this pair is no longer read (the next pair's softmax
      // starts on a consumer barrier, after every read above)
      __syncwarp();
      if (lane == 0) s_mbar_arrive(&rempty[kp & 1]);
    }
  }
  if (c_stop < nchunks && tid == 0) {
    // stopped after a failed wait: let the copies the producer may still have
    // in flight (chunks c_stop .. c_stop + slots - 1, and a weight copy) land
    // before the shared memory goes away; every wait is bounded
    for (int c = c_stop; c < c_stop + kStreamSlots && c < nchunks; ++c)
      s_mbar_wait(&full[c % kStreamSlots], (uint32_t)(c / kStreamSlots) & 1u);
    s_mbar_wait(&wfull, (uint32_t)nh & 1u);
  }
}

}  // namespace

bool decode_stream_supported(int D, bool bf16, int window, int M) {
  return bf16 && D == SD && window <= 128 && M <= 16;
}

cudaError_t launch_decode_stream(const DecodeArgs &a, int B, int64_t *pos, cudaStream_t s) {
  const size_t smem = kMetaOff + 2 * (size_t)16 * SD * 4;   // room for M <= 16 meta keys and values
  static int sms[64] = {};
  static bool configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(decode_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int BH = B * a.H;
  const int run = (BH + sms[dev] - 1) / sms[dev];   // pairs per CTA
  const int grid = (BH + run - 1) / run;
  // The increment rides on the step when every CTA reads its pos values at
  // its start (runs of at most kMaxRunPairs pairs); else a second kernel.
  DecodeArgs d = a;
  const bool fold = run <= kMaxRunPairs;
  d.pos_inc = fold ? pos : nullptr;
  d.pos_slot = fold ? next_pos_slot() : 0;
  d.pos_B = B;
  decode_stream_kernel<<<grid, kDecThreads, smem, s>>>(d, B, run);
  e = cudaGetLastError();
  if (e != cudaSuccess || fold) return e;
  advance_pos_kernel<<<(B + 127) / 128, 128, 0, s>>>(pos, B);
  return cudaGetLastError();
}

// Window caches from a prefix: slot s of sequence (b, h) receives the last
// prefix token t < L with t mod W == s (zeros when no token reached it);
// pos[b] = L.  Thread = one 16-byte vector of a slot's key and value rows.
__global__ void prefill_cache_kernel(const uint4 *k, const uint4 *v, uint4 *kc, uint4 *vc, int64_t *pos, int L,
                                     int W, int vec_k, int vec_v, int H) {
  const int s = blockIdx.x, bh = blockIdx.y;
  const int t = s < L ? s + W * ((L - 1 - s) / W) : -1;
  for (int e = threadIdx.x; e < vec_k + vec_v; e += blockDim.x) {
    const bool isk = e < vec_k;
    const int u = isk ? e : e - vec_k, vec = isk ? vec_k : vec_v;
    const uint4 *src = isk ? k : v;
    uint4 *dst = isk ? kc : vc;
    dst[((size_t)bh * W + s) * vec + u] = t >= 0 ? src[((size_t)bh * L + t) * vec + u] : make_uint4(0u, 0u, 0u, 0u);
  }
  if (s == 0 && threadIdx.x == 0 && bh % H == 0) pos[bh / H] = L;
}

cudaError_t launch_prefill_cache(const void *k, const void *v, void *kc, void *vc, int64_t *pos, int B, int H,
                                 int L, int W, size_t row_bytes_k, size_t row_bytes_v, cudaStream_t s) {
  prefill_cache_kernel<<<dim3(W, B * H), 128, 0, s>>>(
      static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), static_cast<uint4 *>(kc),
      static_cast<uint4 *>(vc), pos, L, W, (int)(row_bytes_k / 16), (int)(row_bytes_v / 16), H);
  return cudaGetLastError();
}

int decode_stream_status_take() {
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_decode_status, sizeof(v)) != cudaSuccess) return -1;
  if (v) {
    const uint32_t z = 0;
    if (cudaMemcpyToSymbol(g_decode_status, &z, sizeof(z)) != cudaSuccess) return -1;
  }
  return (int)v;
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
  DecodeArgs d = a;   // the pos increment rides on the step
  d.pos_inc = pos;
  d.pos_slot = next_pos_slot();
  d.pos_B = B;
  k<<<B * a.H, 256, smem, s>>>(d);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a, int B, int D, bool bf16, int64_t *pos, cudaStream_t s) {
  if (bf16) return D == 128 ? launch_decode_t<__nv_bfloat16, 128>(a, B, pos, s) : launch_decode_t<__nv_bfloat16, 64>(a, B, pos, s);
  return D == 128 ? launch_decode_t<float, 128>(a, B, pos, s) : launch_decode_t<float, 64>(a, B, pos, s);
}

}  // namespace lz
