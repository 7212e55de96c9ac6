// Portable fp32 (CUDA-core) forward of the Lizard hybrid layer.
//
// Three kernels:
//   prep_kernel    a = logsigmoid(g)/tau, phi_q(q), phi_k(k)        per token
//   gla_fwd_simt   chunkwise GLA with the cumulative gate absorbed  per (b,h)
//   swa_mix_simt   window + meta softmax (online) and the mix       per (b,h,64 queries)
//
// GLA branch (English gist.science summary, section 2.A "State Update"),
// computed chunkwise with the gate in log space (Chinese summary, section
// 2.3 "hardware-aware algorithm"): inside a chunk, b_t is the inclusive
// cumulative log-decay and r = b at the chunk's last token;
//   Qt = phi_q exp(b - r), Kt = phi_k exp(r - b)
//   o  = (Qt exp(r)) S_prev + tril(Qt Kt^T) V
//   S  = diag(exp r) S_prev + Kt^T V
// Because phi >= 0 every term of Qt Kt^T is a positive product, so fp32
// rounding is relative per term.  A chunk whose spread b_0 - r exceeds
// kMaxSpread computes tril(...) element by element with exp(b_t - b_j).
#include "common.cuh"
#include "lizard_internal.h"

namespace lz {

constexpr int kPrepTok = 64;   // tokens per prep CTA
constexpr int kFwdC = 64;      // GLA chunk (forward)
constexpr int kSwaQ = 64;      // queries per anchor-branch CTA
constexpr int kSwaK = 64;      // keys per anchor-branch block

// ---------------------------------------------------------------- prep ----
// One warp per token.  Lane l holds x[l + 32 j]; z_f for f = l + 32 jj.
template <typename T, int D>
__global__ void __launch_bounds__(256) prep_kernel(PrepArgs p) {
  constexpr int F = D / 2;
  constexpr int XJ = D / 32;   // x values per lane
  constexpr int ZJ = F / 32;   // z values per lane
  extern __shared__ float sm[];
  float* Wq = sm;              // [D][F]
  float* Wk = sm + D * F;      // [D][F]
  int bh = blockIdx.y;
  const int sb = blockIdx.y;          // scratch row: the grid slot
  if (p.seq_of_slot) {
    bh = p.seq_of_slot[sb];
    if (bh < 0) return;
  }
  const int h = bh % p.H;
  const int t0 = blockIdx.x * kPrepTok;
  const bool has_wq = p.wq != nullptr, has_wk = p.wk != nullptr;
  if (has_wq)
    for (int i = threadIdx.x; i < D * F; i += blockDim.x) Wq[i] = p.wq[(size_t)h * D * F + i];
  if (has_wk)
    for (int i = threadIdx.x; i < D * F; i += blockDim.x) Wk[i] = p.wk[(size_t)h * D * F + i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* qs = static_cast<const T*>(p.q);
  const T* ks = static_cast<const T*>(p.k);
  const T* gs = static_cast<const T*>(p.g);
  for (int tt = warp; tt < kPrepTok; tt += 8) {
    const int t = t0 + tt;
    if (t >= p.L) break;
    const size_t row = ((size_t)bh * p.L + t) * D;    // inputs
    const size_t srow = ((size_t)sb * p.L + t) * D;   // scratch outputs
    // scalar gate: one logit per token and head, the same decay for every dimension
    const float a_tok = p.scalar_gate ? log_decay(to_f32(gs[(size_t)bh * p.L + t]), p.inv_tau) : 0.f;
#pragma unroll
    for (int j = 0; j < XJ; ++j) {
      const int i = lane + 32 * j;
      p.a[srow + i] = p.scalar_gate ? a_tok : log_decay(to_f32(gs[row + i]), p.inv_tau);
    }
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const T* xs = which == 0 ? qs : ks;
      float* out = which == 0 ? p.phq : p.phk;
      const bool has_w = which == 0 ? has_wq : has_wk;
      const float* W = which == 0 ? Wq : Wk;
      float xr[XJ];
#pragma unroll
      for (int j = 0; j < XJ; ++j) xr[j] = to_f32(xs[row + lane + 32 * j]);
      if (!has_w) {
#pragma unroll
        for (int j = 0; j < XJ; ++j) out[srow + lane + 32 * j] = xr[j];
        continue;
      }
      float z[ZJ];
#pragma unroll
      for (int jj = 0; jj < ZJ; ++jj) z[jj] = 0.f;
#pragma unroll
      for (int j = 0; j < XJ; ++j) {
        for (int il = 0; il < 32; ++il) {
          const float xi = __shfl_sync(0xffffffffu, xr[j], il);
          const float* wrow = W + (j * 32 + il) * F;
#pragma unroll
          for (int jj = 0; jj < ZJ; ++jj) z[jj] = fmaf(xi, wrow[lane + 32 * jj], z[jj]);
        }
      }
      // softmax(z) and softmax(-z) over the F features.
      float mx = kNegBig, mn = -kNegBig;
#pragma unroll
      for (int jj = 0; jj < ZJ; ++jj) { mx = fmaxf(mx, z[jj]); mn = fminf(mn, z[jj]); }
      mx = warp_max(mx);
      mn = -warp_max(-mn);
      float ep[ZJ], en[ZJ], sp = 0.f, sn = 0.f;
#pragma unroll
      for (int jj = 0; jj < ZJ; ++jj) {
        ep[jj] = expf(z[jj] - mx);
        en[jj] = expf(mn - z[jj]);
        sp += ep[jj];
        sn += en[jj];
      }
      sp = warp_sum(sp);
      sn = warp_sum(sn);
      const float ip = 1.f / sp, in_ = 1.f / sn;
#pragma unroll
      for (int jj = 0; jj < ZJ; ++jj) {
        out[srow + lane + 32 * jj] = ep[jj] * ip;
        out[srow + F + lane + 32 * jj] = en[jj] * in_;
      }
    }
  }
}

// ------------------------------------------------------------ GLA fwd -----
template <typename T, int D>
__global__ void __launch_bounds__(256) gla_fwd_simt(GlaFwdArgs p) {
  constexpr int C = kFwdC;
  constexpr int VT = D / 16;          // output columns per thread (O tile)
  constexpr int ST = D / 16;          // state tile edge per thread
  extern __shared__ float sm[];
  float* S = sm;                      // [D][D] state (row = key feature)
  float* P1 = S + D * D;              // [C][D] phi_q -> Qt
  float* P2 = P1 + C * D;             // [C][D] phi_k -> Kt
  float* P3 = P2 + C * D;             // [C][D] a -> b (cumulative)
  float* Vs = P3 + C * D;             // [C][D]
  float* A = Vs + C * D;              // [C][C]
  float* dec = A + C * C;             // [D] exp(r): state decay over the chunk
  float* eq = dec + D;                // [D] multiplier turning P1 into phi_q exp(b)
  const int bh = blockIdx.x;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const T* vsrc = static_cast<const T*>(p.v);
  for (int i = tid; i < D * D; i += 256)
    S[i] = p.state_in ? p.state_in[(size_t)bh * D * D + i] : 0.f;
  __syncthreads();
  for (int c0 = 0; c0 < p.L; c0 += C) {
    const int n = min(C, p.L - c0);
    const size_t base = ((size_t)bh * p.L + c0) * D;
    for (int e = tid; e < C * D; e += 256) {
      const int t = e / D;
      const bool ok = t < n;
      P1[e] = ok ? p.phq[base + e] : 0.f;
      P2[e] = ok ? p.phk[base + e] : 0.f;
      P3[e] = ok ? p.a[base + e] : 0.f;
      Vs[e] = ok ? to_f32(vsrc[base + e]) : 0.f;
    }
    __syncthreads();
    float spread = 0.f;
    if (tid < D) {
      float run = 0.f;
      for (int t = 0; t < C; ++t) { run += P3[t * D + tid]; P3[t * D + tid] = run; }
      dec[tid] = expf(run);
      spread = P3[tid] - run;
    }
    const bool exact = __syncthreads_or(spread > kMaxSpread) != 0;
    if (exact) {
      // Per-element decay exp(b_t - b_j) for every pair j <= t.
      for (int e = tid; e < C * C; e += 256) {
        const int t = e / C, j = e % C;
        float acc = 0.f;
        if (j <= t)
          for (int i = 0; i < D; ++i)
            acc += P1[t * D + i] * P2[j * D + i] * expf(P3[t * D + i] - P3[j * D + i]);
        A[e] = acc;
      }
      __syncthreads();
    }
    for (int e = tid; e < C * D; e += 256) {
      const int i = e % D;
      const float b = P3[e], r = P3[(C - 1) * D + i];
      P1[e] *= exact ? expf(b) : expf(b - r);
      P2[e] *= expf(r - b);
    }
    if (tid < D) eq[tid] = exact ? 1.f : dec[tid];
    __syncthreads();
    if (!exact) {
      for (int e = tid; e < C * C; e += 256) {
        const int t = e / C, j = e % C;
        float acc = 0.f;
        if (j <= t) {
#pragma unroll 8
          for (int i = 0; i < D; ++i) acc = fmaf(P1[t * D + i], P2[j * D + i], acc);
        }
        A[e] = acc;
      }
      __syncthreads();
    }
    // O = (P1 * eq) S + A V ; thread owns rows ty*4..+3, cols tx*VT..+VT-1.
    {
      float acc[4][VT];
#pragma unroll
      for (int a_ = 0; a_ < 4; ++a_)
#pragma unroll
        for (int c = 0; c < VT; ++c) acc[a_][c] = 0.f;
      for (int i = 0; i < D; ++i) {
        const float e_ = eq[i];
        float qv[4];
#pragma unroll
        for (int a_ = 0; a_ < 4; ++a_) qv[a_] = P1[(ty * 4 + a_) * D + i] * e_;
#pragma unroll
        for (int c = 0; c < VT; ++c) {
          const float s = S[i * D + tx * VT + c];
#pragma unroll
          for (int a_ = 0; a_ < 4; ++a_) acc[a_][c] = fmaf(qv[a_], s, acc[a_][c]);
        }
      }
      for (int j = 0; j < C; ++j) {
        float av[4];
#pragma unroll
        for (int a_ = 0; a_ < 4; ++a_) av[a_] = A[(ty * 4 + a_) * C + j];
#pragma unroll
        for (int c = 0; c < VT; ++c) {
          const float vv = Vs[j * D + tx * VT + c];
#pragma unroll
          for (int a_ = 0; a_ < 4; ++a_) acc[a_][c] = fmaf(av[a_], vv, acc[a_][c]);
        }
      }
#pragma unroll
      for (int a_ = 0; a_ < 4; ++a_) {
        const int t = ty * 4 + a_;
        if (t < n)
#pragma unroll
          for (int c = 0; c < VT; ++c) p.o_gla[base + t * D + tx * VT + c] = acc[a_][c];
      }
    }
    __syncthreads();
    // S = diag(exp r) S + Kt^T V ; thread owns rows ty*ST.., cols tx*ST..
    {
      float acc[ST][ST];
#pragma unroll
      for (int a_ = 0; a_ < ST; ++a_)
#pragma unroll
        for (int c = 0; c < ST; ++c) acc[a_][c] = S[(ty * ST + a_) * D + tx * ST + c] * dec[ty * ST + a_];
      for (int j = 0; j < C; ++j) {
        float kv[ST];
#pragma unroll
        for (int a_ = 0; a_ < ST; ++a_) kv[a_] = P2[j * D + ty * ST + a_];
#pragma unroll
        for (int c = 0; c < ST; ++c) {
          const float vv = Vs[j * D + tx * ST + c];
#pragma unroll
          for (int a_ = 0; a_ < ST; ++a_) acc[a_][c] = fmaf(kv[a_], vv, acc[a_][c]);
        }
      }
      __syncthreads();
#pragma unroll
      for (int a_ = 0; a_ < ST; ++a_)
#pragma unroll
        for (int c = 0; c < ST; ++c) S[(ty * ST + a_) * D + tx * ST + c] = acc[a_][c];
    }
    __syncthreads();
  }
  if (p.state_out)
    for (int i = tid; i < D * D; i += 256) p.state_out[(size_t)bh * D * D + i] = S[i];
}

// ------------------------------------------------------- anchor + mix -----
// Online softmax over blocks of 64 keys; the meta tokens form the first
// block.  Thread (ty, tx) owns query rows ty*4..+3 and value columns
// tx*VT..+VT-1 of the accumulator.  Keys j < 0 come from the prefix (row
// P + j of k_prefix / v_prefix), when there is one.
template <typename T, int D>
__global__ void __launch_bounds__(256) swa_mix_simt(SwaMixArgs p) {
  constexpr int VT = D / 16;
  constexpr int KP = kSwaK + 1;       // padded logit row
  extern __shared__ float sm[];
  float* Q = sm;                      // [64][D]
  float* Kb = Q + kSwaQ * D;          // [64][D]
  float* Vb = Kb + kSwaK * D;         // [64][D]
  float* P = Vb + kSwaK * D;          // [64][KP]
  float* mrow = P + kSwaQ * KP;       // [64]
  float* lrow = mrow + kSwaQ;         // [64]
  float* crow = lrow + kSwaQ;         // [64]
  const int bh = blockIdx.y, h = bh % p.H;
  const int t0 = blockIdx.x * kSwaQ;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int warp = tid >> 5, lane = tid & 31;
  const T* qs = static_cast<const T*>(p.q);
  const T* ks = static_cast<const T*>(p.k);
  const T* vs = static_cast<const T*>(p.v);
  const T* kps = static_cast<const T*>(p.k_prefix);
  const T* vps = static_cast<const T*>(p.v_prefix);
  T* os = static_cast<T*>(p.o);
  const size_t base = (size_t)bh * p.L * D;
  const float alpha = p.alpha ? p.alpha[h] : 1.f;
  const int nq = min(kSwaQ, p.L - t0);

  float acc[4][VT];
#pragma unroll
  for (int a_ = 0; a_ < 4; ++a_)
#pragma unroll
    for (int c = 0; c < VT; ++c) acc[a_][c] = 0.f;

  if (p.branch != 1) {  // anchor branch present
    for (int e = tid; e < kSwaQ * D; e += 256) {
      const int t = e / D;
      Q[e] = t < nq ? to_f32(qs[base + (size_t)t0 * D + e]) : 0.f;
    }
    if (tid < kSwaQ) { mrow[tid] = kNegBig; lrow[tid] = 0.f; }
    const int kstart = max(-p.P, t0 - p.window + 1);
    const int kend = min(p.L, t0 + nq);   // exclusive
    const int nblk = (kend - kstart + kSwaK - 1) / kSwaK + (p.M > 0 ? 1 : 0);
    for (int blk = 0; blk < nblk; ++blk) {
      const bool meta = p.M > 0 && blk == 0;
      const int ks0 = kstart + (blk - (p.M > 0 ? 1 : 0)) * kSwaK;
      __syncthreads();
      for (int e = tid; e < kSwaK * D; e += 256) {
        const int jj = e / D, i = e % D;
        float kv = 0.f, vv = 0.f;
        if (meta) {
          if (jj < p.M) {
            kv = p.meta_k[((size_t)h * p.M + jj) * D + i];
            vv = p.meta_v ? p.meta_v[((size_t)h * p.M + jj) * D + i] : 0.f;
          }
        } else {
          const int j = ks0 + jj;
          if (j < kend && j >= 0) {
            kv = to_f32(ks[base + (size_t)j * D + i]);
            vv = to_f32(vs[base + (size_t)j * D + i]);
          } else if (j < kend) {   // -P <= j < 0
            const size_t pr = ((size_t)bh * p.P + (p.P + j)) * D + i;
            kv = to_f32(kps[pr]);
            vv = to_f32(vps[pr]);
          }
        }
        Kb[e] = kv;
        Vb[e] = vv;
      }
      __syncthreads();
      // logits for rows ty*4.., keys tx*4..
      {
        float s[4][4];
#pragma unroll
        for (int a_ = 0; a_ < 4; ++a_)
#pragma unroll
          for (int c = 0; c < 4; ++c) s[a_][c] = 0.f;
        for (int i = 0; i < D; ++i) {
          float qv[4], kv[4];
#pragma unroll
          for (int a_ = 0; a_ < 4; ++a_) qv[a_] = Q[(ty * 4 + a_) * D + i];
#pragma unroll
          for (int c = 0; c < 4; ++c) kv[c] = Kb[(tx * 4 + c) * D + i];
#pragma unroll
          for (int a_ = 0; a_ < 4; ++a_)
#pragma unroll
            for (int c = 0; c < 4; ++c) s[a_][c] = fmaf(qv[a_], kv[c], s[a_][c]);
        }
#pragma unroll
        for (int a_ = 0; a_ < 4; ++a_) {
          const int t = t0 + ty * 4 + a_;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int jj = tx * 4 + c;
            bool ok;
            if (meta) ok = jj < p.M;
            else {
              const int j = ks0 + jj;
              ok = j < kend && j <= t && j > t - p.window;
            }
            ok = ok && (ty * 4 + a_) < nq;
            P[(ty * 4 + a_) * KP + jj] = ok ? s[a_][c] * p.scale : kNegBig;
          }
        }
      }
      __syncthreads();
      // online softmax update, one warp per 8 rows
      for (int rr = warp; rr < kSwaQ; rr += 8) {
        const float s0 = P[rr * KP + lane], s1 = P[rr * KP + lane + 32];
        const float mo = mrow[rr];
        const float mn = fmaxf(mo, warp_max(fmaxf(s0, s1)));
        const float p0 = s0 > 0.5f * kNegBig ? expf(s0 - mn) : 0.f;
        const float p1 = s1 > 0.5f * kNegBig ? expf(s1 - mn) : 0.f;
        P[rr * KP + lane] = p0;
        P[rr * KP + lane + 32] = p1;
        const float sum = warp_sum(p0 + p1);
        if (lane == 0) {
          const float corr = expf(mo - mn);
          crow[rr] = corr;
          lrow[rr] = lrow[rr] * corr + sum;
          mrow[rr] = mn;
        }
      }
      __syncthreads();
#pragma unroll
      for (int a_ = 0; a_ < 4; ++a_) {
        const float corr = crow[ty * 4 + a_];
#pragma unroll
        for (int c = 0; c < VT; ++c) acc[a_][c] *= corr;
      }
      for (int jj = 0; jj < kSwaK; ++jj) {
        float pv[4];
#pragma unroll
        for (int a_ = 0; a_ < 4; ++a_) pv[a_] = P[(ty * 4 + a_) * KP + jj];
#pragma unroll
        for (int c = 0; c < VT; ++c) {
          const float vv = Vb[jj * D + tx * VT + c];
#pragma unroll
          for (int a_ = 0; a_ < 4; ++a_) acc[a_][c] = fmaf(pv[a_], vv, acc[a_][c]);
        }
      }
    }
    __syncthreads();
  }
  // epilogue: o = o_gla + alpha * o_swa
#pragma unroll
  for (int a_ = 0; a_ < 4; ++a_) {
    const int tt = ty * 4 + a_;
    if (tt >= nq) continue;
    const size_t row = base + (size_t)(t0 + tt) * D;
    float inv_l = 0.f;
    if (p.branch != 1) inv_l = 1.f / lrow[tt];
#pragma unroll
    for (int c = 0; c < VT; ++c) {
      const int col = tx * VT + c;
      float out = p.branch != 2 ? p.o_gla[row + col] : 0.f;
      if (p.branch != 1) out += alpha * acc[a_][c] * inv_l;
      os[row + col] = from_f32<T>(out);
    }
    if (p.lse && p.branch != 1 && tx == 0)
      p.lse[(size_t)bh * p.L + t0 + tt] = mrow[tt] + logf(lrow[tt]);
  }
}

// ------------------------------------------------------------ launchers ---
template <typename T, int D>
static cudaError_t launch_prep_t(const PrepArgs& a, int BH, cudaStream_t s) {
  const size_t smem = 2 * (size_t)D * (D / 2) * sizeof(float);
  auto k = prep_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.L + kPrepTok - 1) / kPrepTok, BH);
  k<<<grid, 256, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_prep(const PrepArgs& a, int BH, int D, bool bf16, cudaStream_t s) {
  if (a.L == 0) return cudaSuccess;
  if (bf16) return D == 128 ? launch_prep_t<__nv_bfloat16, 128>(a, BH, s) : launch_prep_t<__nv_bfloat16, 64>(a, BH, s);
  return D == 128 ? launch_prep_t<float, 128>(a, BH, s) : launch_prep_t<float, 64>(a, BH, s);
}

template <typename T, int D>
static cudaError_t launch_gla_fwd_t(const GlaFwdArgs& a, int BH, cudaStream_t s) {
  const size_t smem = ((size_t)D * D + 4 * (size_t)kFwdC * D + kFwdC * kFwdC + 2 * D) * sizeof(float);
  auto k = gla_fwd_simt<T, D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<BH, 256, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gla_fwd_simt(const GlaFwdArgs& a, int BH, int D, bool bf16, cudaStream_t s) {
  if (bf16) return D == 128 ? launch_gla_fwd_t<__nv_bfloat16, 128>(a, BH, s) : launch_gla_fwd_t<__nv_bfloat16, 64>(a, BH, s);
  return D == 128 ? launch_gla_fwd_t<float, 128>(a, BH, s) : launch_gla_fwd_t<float, 64>(a, BH, s);
}

template <typename T, int D>
static cudaError_t launch_swa_mix_t(const SwaMixArgs& a, int BH, cudaStream_t s) {
  const size_t smem = ((size_t)kSwaQ * D + 2 * (size_t)kSwaK * D + kSwaQ * (kSwaK + 1) + 3 * kSwaQ) * sizeof(float);
  auto k = swa_mix_simt<T, D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.L + kSwaQ - 1) / kSwaQ, BH);
  k<<<grid, 256, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_swa_mix_simt(const SwaMixArgs& a, int BH, int D, bool bf16, cudaStream_t s) {
  if (a.L == 0) return cudaSuccess;
  if (bf16) return D == 128 ? launch_swa_mix_t<__nv_bfloat16, 128>(a, BH, s) : launch_swa_mix_t<__nv_bfloat16, 64>(a, BH, s);
  return D == 128 ? launch_swa_mix_t<float, 128>(a, BH, s) : launch_swa_mix_t<float, 64>(a, BH, s);
}

}  // namespace lz
