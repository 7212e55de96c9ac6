// Portable fp32 (CUDA-core) backward of the Lizard hybrid layer.
//
//   gla_states_simt   forward state pass, keeps S at the start of every chunk
//   gla_bwd_simt      reverse chunk scan carrying dS            per (b,h)
//   swa_bwd_q         anchor-branch dq, meta-token and alpha grads per (b,h,64 queries)
//   swa_bwd_kv        anchor-branch dk, dv                      per (b,h,64 keys)
//   finish_bwd        feature-map backward, gate chain rule, final sums
//
// GLA gradients per chunk (b_t the in-chunk cumulative log-decay, r = b at
// the chunk's last token, Qt = phi_q exp(b - r), Kt = phi_k exp(r - b),
// A = tril(Qt Kt^T), dA = tril(dO V^T), dS the gradient into the chunk's end
// state):
//   dv      = A^T dO + Kt dS
//   dphi_q  = exp(b - r) (dA Kt) + exp(b) (dO S_prev^T)
//   dphi_k  = exp(r - b) (dA^T Qt + V dS^T)
//   dS_prev = diag(exp r) dS + (phi_q exp(b))^T dO
// and the log-decay gradient is the reverse cumulative sum, over the whole
// sequence, of phi_q dphi_q - phi_k dphi_k.
#include "common.cuh"
#include "lizard_internal.h"

namespace lz {

constexpr int kSwaT = 64;    // queries / keys per anchor-branch tile
constexpr int kFinTok = 256; // tokens per finishing CTA
constexpr int kFinSub = 32;  // tokens per finishing sub-tile

// --------------------------------------------------------- state pass -----
template <typename T, int D>
__global__ void __launch_bounds__(256) gla_states_simt(GlaStatesArgs p) {
  constexpr int C = kBwdC;
  constexpr int ST = D / 16;
  extern __shared__ float sm[];
  float *S = sm;                  // [D][D]
  float *Kb = S + D * D;          // [C][D]
  float *Bb = Kb + C * D;         // [C][D]
  float *Vb = Bb + C * D;         // [C][D]
  float *dec = Vb + C * D;        // [D]
  int bh = blockIdx.x;
  const int sb = blockIdx.x;   // scratch row: the grid slot
  if (p.seq_of_slot) {
    bh = p.seq_of_slot[sb];
    if (bh < 0) return;
  }
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const T *vsrc = static_cast<const T *>(p.v);
  const int nch = (p.L + C - 1) / C;
  for (int i = tid; i < D * D; i += 256) S[i] = p.state_in ? p.state_in[(size_t)bh * D * D + i] : 0.f;
  __syncthreads();
  for (int c = 0; c < nch; ++c) {
    const int c0 = c * C, n = min(C, p.L - c0);
    float *dst = p.sprev + ((size_t)sb * nch + c) * D * D;
    for (int i = tid; i < D * D; i += 256) dst[i] = S[i];
    const size_t base = ((size_t)sb * p.L + c0) * D;    // scratch
    const size_t ibase = ((size_t)bh * p.L + c0) * D;   // inputs
    for (int e = tid; e < C * D; e += 256) {
      const bool ok = e / D < n;
      Kb[e] = ok ? p.phk[base + e] : 0.f;
      Bb[e] = ok ? p.a[base + e] : 0.f;
      Vb[e] = ok ? to_f32(vsrc[ibase + e]) : 0.f;
    }
    __syncthreads();
    if (tid < D) {
      float run = 0.f;
      for (int t = 0; t < C; ++t) { run += Bb[t * D + tid]; Bb[t * D + tid] = run; }
      dec[tid] = expf(run);
    }
    __syncthreads();
    // Kt = phi_k exp(r - b) <= phi_k: safe for any decay.
    for (int e = tid; e < C * D; e += 256) Kb[e] *= expf(Bb[(C - 1) * D + e % D] - Bb[e]);
    __syncthreads();
    float acc[ST][ST];
#pragma unroll
    for (int a_ = 0; a_ < ST; ++a_)
#pragma unroll
      for (int c_ = 0; c_ < ST; ++c_) acc[a_][c_] = S[(ty * ST + a_) * D + tx * ST + c_] * dec[ty * ST + a_];
    for (int j = 0; j < C; ++j) {
#pragma unroll
      for (int a_ = 0; a_ < ST; ++a_) {
        const float kv = Kb[j * D + ty * ST + a_];
#pragma unroll
        for (int c_ = 0; c_ < ST; ++c_) acc[a_][c_] = fmaf(kv, Vb[j * D + tx * ST + c_], acc[a_][c_]);
      }
    }
    __syncthreads();
#pragma unroll
    for (int a_ = 0; a_ < ST; ++a_)
#pragma unroll
      for (int c_ = 0; c_ < ST; ++c_) S[(ty * ST + a_) * D + tx * ST + c_] = acc[a_][c_];
    __syncthreads();
  }
  // S = S_L: with an incoming final-state gradient G, every token's log-decay
  // gradient also carries sum_v G[i][v] S_L[i][v] (S_L scales with the total
  // log-decay of dimension i)
  if (p.kap && tid < D) {
    const float *G = p.dstate_out + ((size_t)bh * D + tid) * D;
    float s = 0.f;
    for (int v = 0; v < D; ++v) s = fmaf(G[v], S[tid * D + v], s);
    p.kap[(size_t)sb * D + tid] = s;
  }
}

// ------------------------------------------------------ GLA reverse scan --
template <typename T, int D>
__global__ void __launch_bounds__(256) gla_bwd_simt(GlaBwdArgs p) {
  constexpr int C = kBwdC;
  constexpr int SP = D + 1;            // padded row of the two state tiles
  constexpr int IT = D / 16;           // i per thread in (t, i) tiles (t: 2 per thread)
  constexpr int ST = D / 16;
  extern __shared__ float sm[];
  float *dS = sm;                      // [D][SP] gradient into the current chunk's end state
  float *Sp = dS + D * SP;             // [D][SP] state at the chunk start; reused for dB
  float *Qb = Sp + D * SP;             // [C][D]
  float *Kb = Qb + C * D;              // [C][D]
  float *Bb = Kb + C * D;              // [C][D]
  float *Vb = Bb + C * D;              // [C][D]
  float *Ob = Vb + C * D;              // [C][D]
  float *A = Ob + C * D;               // [C][C]
  float *dA = A + C * C;               // [C][C]
  float *dec = dA + C * C;             // [D]
  int bh = blockIdx.x;
  const int sb = blockIdx.x;   // scratch row: the grid slot
  if (p.seq_of_slot) {
    bh = p.seq_of_slot[sb];
    if (bh < 0) return;
  }
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const T *vsrc = static_cast<const T *>(p.v);
  const T *osrc = static_cast<const T *>(p.dout);
  const int nch = (p.L + C - 1) / C;
  // dS starts as the gradient flowing into the final state (zero when unused)
  for (int i = tid; i < D * SP; i += 256)
    dS[i] = (p.dstate_out && i % SP < D) ? p.dstate_out[(size_t)bh * D * D + (i / SP) * D + i % SP] : 0.f;
  // reverse running sum of dB (thread i < D), from the final state's share
  float carry = (p.kap && tid < D) ? p.kap[(size_t)sb * D + tid] : 0.f;
  __syncthreads();
  for (int c = nch - 1; c >= 0; --c) {
    const int c0 = c * C, n = min(C, p.L - c0);
    const size_t sbase = ((size_t)sb * p.L + c0) * D;   // scratch
    const size_t base = ((size_t)bh * p.L + c0) * D;    // inputs and outputs
    const float *sp_src = p.sprev + ((size_t)sb * nch + c) * D * D;
    for (int e = tid; e < D * D; e += 256) Sp[(e / D) * SP + e % D] = sp_src[e];
    for (int e = tid; e < C * D; e += 256) {
      const bool ok = e / D < n;
      Qb[e] = ok ? p.phq[sbase + e] : 0.f;
      Kb[e] = ok ? p.phk[sbase + e] : 0.f;
      Bb[e] = ok ? p.a[sbase + e] : 0.f;
      Vb[e] = ok ? to_f32(vsrc[base + e]) : 0.f;
      Ob[e] = ok ? to_f32(osrc[base + e]) : 0.f;
    }
    __syncthreads();
    float spread = 0.f;
    if (tid < D) {
      float run = 0.f;
      for (int t = 0; t < C; ++t) { run += Bb[t * D + tid]; Bb[t * D + tid] = run; }
      dec[tid] = expf(run);
      spread = Bb[tid] - run;
    }
    const bool exact = __syncthreads_or(spread > kMaxSpread) != 0;
    // dA = tril(dO V^T); in the exact path also A from the raw features.
    for (int e = tid; e < C * C; e += 256) {
      const int t = e / C, j = e % C;
      float acc = 0.f, aa = 0.f;
      if (j <= t) {
        for (int v = 0; v < D; ++v) acc = fmaf(Ob[t * D + v], Vb[j * D + v], acc);
        if (exact)
          for (int i = 0; i < D; ++i)
            aa += Qb[t * D + i] * Kb[j * D + i] * expf(Bb[t * D + i] - Bb[j * D + i]);
      }
      dA[e] = acc;
      if (exact) A[e] = aa;
    }
    __syncthreads();
    if (!exact) {
      for (int e = tid; e < C * D; e += 256) {
        const float b = Bb[e], r = Bb[(C - 1) * D + e % D];
        Qb[e] *= expf(b - r);
        Kb[e] *= expf(r - b);
      }
      __syncthreads();
      for (int e = tid; e < C * C; e += 256) {
        const int t = e / C, j = e % C;
        float acc = 0.f;
        if (j <= t)
          for (int i = 0; i < D; ++i) acc = fmaf(Qb[t * D + i], Kb[j * D + i], acc);
        A[e] = acc;
      }
      __syncthreads();
    }
    // Intra-chunk parts of dphi_q (Xq) and dphi_k (Xk), and phi * X (Yq, Yk),
    // for rows t = ty*2 + {0,1} and features i = tx + 16 * {0..IT-1}.
    float Xq[2][IT], Yq[2][IT], Xk[2][IT], Yk[2][IT];
#pragma unroll
    for (int a_ = 0; a_ < 2; ++a_) {
      const int t = ty * 2 + a_;
#pragma unroll
      for (int u = 0; u < IT; ++u) {
        const int i = tx + 16 * u;
        const float bt = Bb[t * D + i], r = Bb[(C - 1) * D + i];
        float sq = 0.f, sk = 0.f;
        if (!exact) {
          for (int j = 0; j < C; ++j) {
            sq = fmaf(dA[t * C + j], Kb[j * D + i], sq);   // (dA Kt)[t][i]
            sk = fmaf(dA[j * C + t], Qb[j * D + i], sk);   // (dA^T Qt)[t][i]
          }
          Xq[a_][u] = expf(bt - r) * sq;
          Yq[a_][u] = Qb[t * D + i] * sq;
          Xk[a_][u] = expf(r - bt) * sk;
          Yk[a_][u] = Kb[t * D + i] * sk;
        } else {
          for (int j = 0; j <= t; ++j) sq += dA[t * C + j] * Kb[j * D + i] * expf(bt - Bb[j * D + i]);
          for (int j = t; j < C; ++j) sk += dA[j * C + t] * Qb[j * D + i] * expf(Bb[j * D + i] - bt);
          Xq[a_][u] = sq;
          Yq[a_][u] = Qb[t * D + i] * sq;
          Xk[a_][u] = sk;
          Yk[a_][u] = Kb[t * D + i] * sk;
        }
      }
    }
    __syncthreads();
    // Qb <- phi_q exp(b); Kb <- phi_k exp(r - b)
    for (int e = tid; e < C * D; e += 256) {
      const float b = Bb[e], r = Bb[(C - 1) * D + e % D];
      if (exact) {
        Qb[e] *= expf(b);
        Kb[e] *= expf(r - b);
      } else {
        Qb[e] *= expf(r);
      }
    }
    __syncthreads();
    float dB[2][IT];
#pragma unroll
    for (int a_ = 0; a_ < 2; ++a_) {
      const int t = ty * 2 + a_;
#pragma unroll
      for (int u = 0; u < IT; ++u) {
        const int i = tx + 16 * u;
        float U = 0.f, W = 0.f;
        for (int v = 0; v < D; ++v) {
          U = fmaf(Ob[t * D + v], Sp[i * SP + v], U);   // (dO S_prev^T)[t][i]
          W = fmaf(Vb[t * D + v], dS[i * SP + v], W);   // (V dS^T)[t][i]
        }
        const float bt = Bb[t * D + i], r = Bb[(C - 1) * D + i];
        const float dq_ = Xq[a_][u] + expf(bt) * U;
        const float ek = expf(r - bt);
        const float dk_ = Xk[a_][u] + ek * W;
        dB[a_][u] = Yq[a_][u] + Qb[t * D + i] * U - Yk[a_][u] - Kb[t * D + i] * W;
        if (t < n) {   // in slot mode (exact fallback) dphi go to the slot's fp32 arrays
          const size_t o = (p.seq_of_slot ? sbase : base) + t * D + i;
          p.dphq[o] = dq_;
          p.dphk[o] = dk_;
        }
      }
    }
    __syncthreads();
#pragma unroll
    for (int a_ = 0; a_ < 2; ++a_)
#pragma unroll
      for (int u = 0; u < IT; ++u) Sp[(ty * 2 + a_) * SP + tx + 16 * u] = dB[a_][u];
    // dv = A^T dO + Kbar dS (rows j = ty*2.., columns tx + 16 u)
#pragma unroll
    for (int a_ = 0; a_ < 2; ++a_) {
      const int j = ty * 2 + a_;
#pragma unroll
      for (int u = 0; u < IT; ++u) {
        const int v = tx + 16 * u;
        float acc = 0.f;
        for (int t = j; t < C; ++t) acc = fmaf(A[t * C + j], Ob[t * D + v], acc);
        for (int i = 0; i < D; ++i) acc = fmaf(Kb[j * D + i], dS[i * SP + v], acc);
        if (j < n) p.dv_gla[base + j * D + v] = acc;
      }
    }
    __syncthreads();
    // dS <- diag(exp r) dS + (phi_q exp b)^T dO ; thread owns rows ty*ST.., cols tx*ST..
    {
      float acc[ST][ST];
#pragma unroll
      for (int a_ = 0; a_ < ST; ++a_)
#pragma unroll
        for (int c_ = 0; c_ < ST; ++c_) acc[a_][c_] = dS[(ty * ST + a_) * SP + tx * ST + c_] * dec[ty * ST + a_];
      for (int t = 0; t < C; ++t) {
#pragma unroll
        for (int a_ = 0; a_ < ST; ++a_) {
          const float qv = Qb[t * D + ty * ST + a_];
#pragma unroll
          for (int c_ = 0; c_ < ST; ++c_) acc[a_][c_] = fmaf(qv, Ob[t * D + tx * ST + c_], acc[a_][c_]);
        }
      }
#pragma unroll
      for (int a_ = 0; a_ < ST; ++a_)
#pragma unroll
        for (int c_ = 0; c_ < ST; ++c_) dS[(ty * ST + a_) * SP + tx * ST + c_] = acc[a_][c_];
    }
    // da: reverse cumulative sum of dB, carried across chunks
    if (tid < D) {
      for (int t = C - 1; t >= 0; --t) {
        carry += Sp[t * SP + tid];
        if (t < n) p.da[base + t * D + tid] = carry;
      }
    }
    __syncthreads();
  }
  if (p.dstate_in)
    for (int e = tid; e < D * D; e += 256) p.dstate_in[(size_t)bh * D * D + e] = dS[(e / D) * SP + e % D];
}

// ------------------------------------------------- anchor branch: dq -----
// Three passes over the key blocks of one 64-query tile (meta block first):
// (1) row max / normaliser, (2) o_swa and D = dO_swa . o_swa, (3) dq and the
// meta-token gradients.  dO_swa = alpha_h dout; G holds the raw dout.
template <typename T, int D>
__global__ void __launch_bounds__(256) swa_bwd_q(SwaBwdQArgs p) {
  constexpr int VT = D / 16;
  constexpr int KP = kSwaT + 1;
  extern __shared__ float sm[];
  float *Q = sm;                       // [64][D]
  float *G = Q + kSwaT * D;            // [64][D] dO_swa
  float *Kb = G + kSwaT * D;           // [64][D]
  float *Vb = Kb + kSwaT * D;          // [64][D]
  float *P = Vb + kSwaT * D;           // [64][KP]
  float *mrow = P + kSwaT * KP;        // [64]
  float *lrow = mrow + kSwaT;          // [64]
  float *Drow = lrow + kSwaT;          // [64]
  float *redbuf = Drow + kSwaT;        // [8]
  float *PM = redbuf + 8;              // [64][16] meta-token probabilities
  const int bh = blockIdx.y, h = bh % p.H, t0 = blockIdx.x * kSwaT;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4, warp = tid >> 5, lane = tid & 31;
  const T *qs = static_cast<const T *>(p.q);
  const T *ks = static_cast<const T *>(p.k);
  const T *vs = static_cast<const T *>(p.v);
  const T *gs = static_cast<const T *>(p.dout);
  const size_t base = (size_t)bh * p.L * D;
  const float alpha = p.alpha ? p.alpha[h] : 1.f;
  const int nq = min(kSwaT, p.L - t0);
  for (int e = tid; e < kSwaT * D; e += 256) {
    const bool ok = e / D < nq;
    Q[e] = ok ? to_f32(qs[base + (size_t)t0 * D + e]) : 0.f;
    G[e] = ok ? to_f32(gs[base + (size_t)t0 * D + e]) : 0.f;   // raw dout
  }
  if (tid < kSwaT) { mrow[tid] = kNegBig; lrow[tid] = 0.f; }
  // keys j < 0 come from the prefix (row P + j of k_prefix / v_prefix)
  const int kstart = max(-p.P, t0 - p.window + 1);
  const int kend = t0 + nq;
  const int hasm = p.M > 0 ? 1 : 0;
  const int nblk = (kend - kstart + kSwaT - 1) / kSwaT + hasm;
  const T *kps = static_cast<const T *>(p.k_prefix);
  const T *vps = static_cast<const T *>(p.v_prefix);

  auto load_block = [&](int blk, bool &meta, int &ks0) {
    meta = hasm && blk == 0;
    ks0 = kstart + (blk - hasm) * kSwaT;
    for (int e = tid; e < kSwaT * D; e += 256) {
      const int jj = e / D, i = e % D;
      float kv = 0.f, vv = 0.f;
      if (meta) {
        if (jj < p.M) {
          kv = p.meta_k[((size_t)h * p.M + jj) * D + i];
          vv = p.meta_v ? p.meta_v[((size_t)h * p.M + jj) * D + i] : 0.f;
        }
      } else if (ks0 + jj < kend && ks0 + jj >= 0) {
        kv = to_f32(ks[base + (size_t)(ks0 + jj) * D + i]);
        vv = to_f32(vs[base + (size_t)(ks0 + jj) * D + i]);
      } else if (ks0 + jj < kend) {   // -P <= j < 0
        const size_t pr = ((size_t)bh * p.P + (p.P + ks0 + jj)) * D + i;
        kv = to_f32(kps[pr]);
        vv = to_f32(vps[pr]);
      }
      Kb[e] = kv;
      Vb[e] = vv;
    }
  };
  // masked, scaled logits of rows ty*4.., keys tx*4.. into P
  auto logits = [&](bool meta, int ks0) {
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
      const int tt = ty * 4 + a_, t = t0 + tt;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int jj = tx * 4 + c;
        bool ok = meta ? jj < p.M : (ks0 + jj < kend && ks0 + jj <= t && ks0 + jj > t - p.window);
        ok = ok && tt < nq;
        P[tt * KP + jj] = ok ? s[a_][c] * p.scale : kNegBig;
      }
    }
  };

  // pass 1: statistics
  for (int blk = 0; blk < nblk; ++blk) {
    bool meta; int ks0;
    __syncthreads();
    load_block(blk, meta, ks0);
    __syncthreads();
    logits(meta, ks0);
    __syncthreads();
    for (int rr = warp; rr < kSwaT; rr += 8) {
      const float s0 = P[rr * KP + lane], s1 = P[rr * KP + lane + 32];
      const float mo = mrow[rr];
      const float mn = fmaxf(mo, warp_max(fmaxf(s0, s1)));
      const float e0 = s0 > 0.5f * kNegBig ? expf(s0 - mn) : 0.f;
      const float e1 = s1 > 0.5f * kNegBig ? expf(s1 - mn) : 0.f;
      const float sum = warp_sum(e0 + e1);
      if (lane == 0) { lrow[rr] = lrow[rr] * expf(mo - mn) + sum; mrow[rr] = mn; }
    }
  }
  __syncthreads();
  if (tid < kSwaT) {
    const float lse = tid < nq ? mrow[tid] + logf(lrow[tid]) : 0.f;
    mrow[tid] = lse;  // mrow now holds the log-normaliser
    if (tid < nq) p.lse[(size_t)bh * p.L + t0 + tid] = lse;
  }
  // pass 2: o_swa (registers), then D
  float acc[4][VT];
#pragma unroll
  for (int a_ = 0; a_ < 4; ++a_)
#pragma unroll
    for (int c = 0; c < VT; ++c) acc[a_][c] = 0.f;
  for (int blk = 0; blk < nblk; ++blk) {
    bool meta; int ks0;
    __syncthreads();
    load_block(blk, meta, ks0);
    __syncthreads();
    logits(meta, ks0);
    __syncthreads();
    for (int e = tid; e < kSwaT * kSwaT; e += 256) {
      const int tt = e / kSwaT, jj = e % kSwaT;
      const float s = P[tt * KP + jj];
      P[tt * KP + jj] = s > 0.5f * kNegBig ? expf(s - mrow[tt]) : 0.f;
    }
    __syncthreads();
    for (int jj = 0; jj < kSwaT; ++jj) {
#pragma unroll
      for (int a_ = 0; a_ < 4; ++a_) {
        const float pv = P[(ty * 4 + a_) * KP + jj];
#pragma unroll
        for (int c = 0; c < VT; ++c) acc[a_][c] = fmaf(pv, Vb[jj * D + tx * VT + c], acc[a_][c]);
      }
    }
  }
  // D_t = alpha sum_v dout o_swa ; dalpha_h += sum_t sum_v dout o_swa
  float dsum = 0.f;
#pragma unroll
  for (int a_ = 0; a_ < 4; ++a_) {
    float part = 0.f;
#pragma unroll
    for (int c = 0; c < VT; ++c) part = fmaf(G[(ty * 4 + a_) * D + tx * VT + c], acc[a_][c], part);
    // reduce over the 16 tx lanes (lanes tx..tx+15 share ty within a warp half)
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (tx == 0) {
      Drow[ty * 4 + a_] = alpha * part;
      if (ty * 4 + a_ < nq) dsum += part;
    }
  }
  __syncthreads();
  if (tid < nq) p.Dterm[(size_t)bh * p.L + t0 + tid] = Drow[tid];
  if (p.dalpha) {
    // tx == 0 threads hold partial sums: gather per warp then one atomic
    float w = warp_sum(dsum);
    if (lane == 0) redbuf[warp] = w;
    __syncthreads();
    if (tid == 0) {
      float s = 0.f;
      for (int i = 0; i < 8; ++i) s += redbuf[i];
      atomicAdd(p.dalpha + h, s);
    }
  }
  // pass 3: ds = p (dp - D); dq = scale ds K; meta grads
  float dq[4][VT];
#pragma unroll
  for (int a_ = 0; a_ < 4; ++a_)
#pragma unroll
    for (int c = 0; c < VT; ++c) dq[a_][c] = 0.f;
  for (int blk = 0; blk < nblk; ++blk) {
    bool meta; int ks0;
    __syncthreads();
    load_block(blk, meta, ks0);
    __syncthreads();
    logits(meta, ks0);
    __syncthreads();
    // ds in place of P, rows ty*4.., keys tx*4..
    {
      float dp[4][4];
#pragma unroll
      for (int a_ = 0; a_ < 4; ++a_)
#pragma unroll
        for (int c = 0; c < 4; ++c) dp[a_][c] = 0.f;
      for (int v = 0; v < D; ++v) {
        float gv[4], vv[4];
#pragma unroll
        for (int a_ = 0; a_ < 4; ++a_) gv[a_] = G[(ty * 4 + a_) * D + v];
#pragma unroll
        for (int c = 0; c < 4; ++c) vv[c] = Vb[(tx * 4 + c) * D + v];
#pragma unroll
        for (int a_ = 0; a_ < 4; ++a_)
#pragma unroll
          for (int c = 0; c < 4; ++c) dp[a_][c] = fmaf(gv[a_], vv[c], dp[a_][c]);
      }
#pragma unroll
      for (int a_ = 0; a_ < 4; ++a_) {
        const int tt = ty * 4 + a_;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int jj = tx * 4 + c;
          const float s = P[tt * KP + jj];
          const float pr = s > 0.5f * kNegBig ? expf(s - mrow[tt]) : 0.f;
          if (meta && jj < 16) PM[tt * 16 + jj] = pr;
          P[tt * KP + jj] = pr * (alpha * dp[a_][c] - Drow[tt]);
        }
      }
    }
    __syncthreads();
    for (int jj = 0; jj < kSwaT; ++jj) {
#pragma unroll
      for (int a_ = 0; a_ < 4; ++a_) {
        const float dsv = P[(ty * 4 + a_) * KP + jj];
#pragma unroll
        for (int c = 0; c < VT; ++c) dq[a_][c] = fmaf(dsv, Kb[jj * D + tx * VT + c], dq[a_][c]);
      }
    }
    if (meta) {
      // dmeta_k[m] += scale sum_t ds[t][m] q_t ; dmeta_v[m] += sum_t p[t][m] dO_t
      for (int e = tid; e < p.M * D; e += 256) {
        const int m = e / D, i = e % D;
        float gk = 0.f, gv = 0.f;
        for (int tt = 0; tt < nq; ++tt) {
          gk = fmaf(P[tt * KP + m], Q[tt * D + i], gk);
          gv = fmaf(PM[tt * 16 + m], G[tt * D + i], gv);
        }
        if (p.dmeta_k) atomicAdd(p.dmeta_k + ((size_t)h * p.M + m) * D + i, gk * p.scale);
        if (p.dmeta_v) atomicAdd(p.dmeta_v + ((size_t)h * p.M + m) * D + i, alpha * gv);
      }
    }
  }
#pragma unroll
  for (int a_ = 0; a_ < 4; ++a_) {
    const int tt = ty * 4 + a_;
    if (tt < nq)
#pragma unroll
      for (int c = 0; c < VT; ++c) p.dq_swa[base + (size_t)(t0 + tt) * D + tx * VT + c] = dq[a_][c] * p.scale;
  }
}

// --------------------------------------------- anchor branch: dk, dv -----
// Key tile [j0, j0+64); the queries that see it are [j0, j0+63+window).
// With a key/value prefix of P tokens, the first ceil(P/64) tiles cover the
// prefix keys -P .. -1 (j0 < 0; their gradients go to dk_prefix / dv_prefix).
template <typename T, int D>
__global__ void __launch_bounds__(256) swa_bwd_kv(SwaBwdKVArgs p) {
  constexpr int VT = D / 16;
  constexpr int KP = kSwaT + 1;
  extern __shared__ float sm[];
  float *Kt = sm;                      // [64][D] this tile's keys
  float *Vt = Kt + kSwaT * D;          // [64][D]
  float *Qb = Vt + kSwaT * D;          // [64][D]
  float *Gb = Qb + kSwaT * D;          // [64][D] dO_swa
  float *P = Gb + kSwaT * D;           // [64 q][KP]
  float *dSm = P + kSwaT * KP;         // [64 q][KP]
  float *lse = dSm + kSwaT * KP;       // [64]
  float *Dq = lse + kSwaT;             // [64]
  const int npre = (p.P + kSwaT - 1) / kSwaT;
  const int bh = blockIdx.y, h = bh % p.H, j0 = ((int)blockIdx.x - npre) * kSwaT;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const T *qs = static_cast<const T *>(p.q);
  const T *ks = static_cast<const T *>(p.k);
  const T *vs = static_cast<const T *>(p.v);
  const T *gs = static_cast<const T *>(p.dout);
  const T *kps = static_cast<const T *>(p.k_prefix);
  const T *vps = static_cast<const T *>(p.v_prefix);
  const size_t base = (size_t)bh * p.L * D;
  const float alpha = p.alpha ? p.alpha[h] : 1.f;
  const int nk = min(kSwaT, p.L - j0);
  const int jlo = -p.P;                 // the first key there is
  for (int e = tid; e < kSwaT * D; e += 256) {
    const int j = j0 + e / D, i = e % D;
    float kv = 0.f, vv = 0.f;
    if (j >= 0 && e / D < nk) {
      kv = to_f32(ks[base + (size_t)j * D + i]);
      vv = to_f32(vs[base + (size_t)j * D + i]);
    } else if (j < 0 && j >= jlo) {
      const size_t pr = ((size_t)bh * p.P + (p.P + j)) * D + i;
      kv = to_f32(kps[pr]);
      vv = to_f32(vps[pr]);
    }
    Kt[e] = kv;
    Vt[e] = vv;
  }
  float dk[4][VT], dv[4][VT];
#pragma unroll
  for (int a_ = 0; a_ < 4; ++a_)
#pragma unroll
    for (int c = 0; c < VT; ++c) { dk[a_][c] = 0.f; dv[a_][c] = 0.f; }
  const int qend = min(p.L, j0 + nk - 1 + p.window);   // exclusive
  for (int q0 = max(j0, 0); q0 < qend; q0 += kSwaT) {
    const int nq = min(kSwaT, qend - q0);
    __syncthreads();
    for (int e = tid; e < kSwaT * D; e += 256) {
      const bool ok = e / D < nq;
      Qb[e] = ok ? to_f32(qs[base + (size_t)q0 * D + e]) : 0.f;
      Gb[e] = ok ? alpha * to_f32(gs[base + (size_t)q0 * D + e]) : 0.f;
    }
    if (tid < kSwaT) {
      lse[tid] = tid < nq ? p.lse[(size_t)bh * p.L + q0 + tid] : 0.f;
      Dq[tid] = tid < nq ? p.Dterm[(size_t)bh * p.L + q0 + tid] : 0.f;
    }
    __syncthreads();
    // rows = queries ty*4.., cols = keys tx*4..
    {
      float s[4][4], dp[4][4];
#pragma unroll
      for (int a_ = 0; a_ < 4; ++a_)
#pragma unroll
        for (int c = 0; c < 4; ++c) { s[a_][c] = 0.f; dp[a_][c] = 0.f; }
      for (int i = 0; i < D; ++i) {
        float qv[4], kv[4], gv[4], vv[4];
#pragma unroll
        for (int a_ = 0; a_ < 4; ++a_) { qv[a_] = Qb[(ty * 4 + a_) * D + i]; gv[a_] = Gb[(ty * 4 + a_) * D + i]; }
#pragma unroll
        for (int c = 0; c < 4; ++c) { kv[c] = Kt[(tx * 4 + c) * D + i]; vv[c] = Vt[(tx * 4 + c) * D + i]; }
#pragma unroll
        for (int a_ = 0; a_ < 4; ++a_)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            s[a_][c] = fmaf(qv[a_], kv[c], s[a_][c]);
            dp[a_][c] = fmaf(gv[a_], vv[c], dp[a_][c]);
          }
      }
#pragma unroll
      for (int a_ = 0; a_ < 4; ++a_) {
        const int tq = ty * 4 + a_, t = q0 + tq;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int jj = tx * 4 + c, j = j0 + jj;
          const bool ok = tq < nq && jj < nk && j >= jlo && j <= t && j > t - p.window;
          const float pr = ok ? expf(s[a_][c] * p.scale - lse[tq]) : 0.f;
          P[tq * KP + jj] = pr;
          dSm[tq * KP + jj] = pr * (dp[a_][c] - Dq[tq]);
        }
      }
    }
    __syncthreads();
    // dk[j] += scale sum_t ds[t][j] q_t ; dv[j] += sum_t p[t][j] dO_t  (rows = keys ty*4..)
    for (int tq = 0; tq < kSwaT; ++tq) {
#pragma unroll
      for (int a_ = 0; a_ < 4; ++a_) {
        const float dsv = dSm[tq * KP + ty * 4 + a_];
        const float pv = P[tq * KP + ty * 4 + a_];
#pragma unroll
        for (int c = 0; c < VT; ++c) {
          dk[a_][c] = fmaf(dsv, Qb[tq * D + tx * VT + c], dk[a_][c]);
          dv[a_][c] = fmaf(pv, Gb[tq * D + tx * VT + c], dv[a_][c]);
        }
      }
    }
  }
#pragma unroll
  for (int a_ = 0; a_ < 4; ++a_) {
    const int jj = ty * 4 + a_, j = j0 + jj;
    if (j >= 0 && jj < nk) {
#pragma unroll
      for (int c = 0; c < VT; ++c) {
        p.dk_swa[base + (size_t)j * D + tx * VT + c] = dk[a_][c] * p.scale;
        p.dv_swa[base + (size_t)j * D + tx * VT + c] = dv[a_][c];
      }
    } else if (j < 0 && j >= jlo) {   // a prefix key: its final gradient (anchor part only)
      T *dkp = static_cast<T *>(p.dk_prefix), *dvp = static_cast<T *>(p.dv_prefix);
      const size_t pr = ((size_t)bh * p.P + (p.P + j)) * D;
#pragma unroll
      for (int c = 0; c < VT; ++c) {
        dkp[pr + tx * VT + c] = from_f32<T>(dk[a_][c] * p.scale);
        dvp[pr + tx * VT + c] = from_f32<T>(dv[a_][c]);
      }
    }
  }
}

// ------------------------------------------------------------- finish -----
// Per token: dx = phi-backward(x, W, dphi) + anchor part, dv = sum of both
// branches, dg = da * sigmoid(-g) / tau.  dW = sum_t x_t dz_t^T accumulated
// per CTA in registers (thread owns W entries tid + 256 u) and added to the
// output with one atomic per entry per CTA.
template <typename T, int D>
__global__ void __launch_bounds__(256) finish_bwd(FinishBwdArgs p) {
  constexpr int F = D / 2;
  constexpr int WP = F + 1;                 // padded W row
  constexpr int XJ = D / 32, ZJ = F / 32;
  constexpr int WPT = D * F / 256;          // W entries per thread
  extern __shared__ float sm[];
  float *Ws[2] = {sm, sm + D * WP};         // [D][WP] each
  float *Xs[2] = {sm + 2 * D * WP, sm + 2 * D * WP + kFinSub * D};             // [sub][D]
  float *Zs[2] = {sm + 2 * D * WP + 2 * kFinSub * D,
                  sm + 2 * D * WP + 2 * kFinSub * D + kFinSub * F};           // [sub][F]
  const int bh = blockIdx.y, h = bh % p.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float *Wg[2] = {p.wq, p.wk};
  for (int m = 0; m < 2; ++m)
    if (Wg[m])
      for (int e = tid; e < D * F; e += 256) Ws[m][(e / F) * WP + e % F] = Wg[m][(size_t)h * D * F + e];
  float dW[2][WPT];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int u = 0; u < WPT; ++u) dW[m][u] = 0.f;
  const T *xsrc[2] = {static_cast<const T *>(p.q), static_cast<const T *>(p.k)};
  const float *dph[2] = {p.dphq, p.dphk};
  const float *dsw[2] = {p.dq_swa, p.dk_swa};
  T *dst[2] = {static_cast<T *>(p.dq), static_cast<T *>(p.dk)};
  const T *gsrc = static_cast<const T *>(p.g);
  T *dvdst = static_cast<T *>(p.dv);
  const int tbeg = blockIdx.x * kFinTok;
  const int tlim = min(p.L, tbeg + kFinTok);
  __syncthreads();
  for (int s0 = tbeg; s0 < tlim; s0 += kFinSub) {
    for (int tt = warp; tt < kFinSub; tt += 8) {
      const int t = s0 + tt;
      const bool live = t < tlim;
      const size_t row = ((size_t)bh * p.L + (live ? t : 0)) * D;
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        float xr[XJ], gr[XJ];
#pragma unroll
        for (int j = 0; j < XJ; ++j) {
          xr[j] = live ? to_f32(xsrc[m][row + lane + 32 * j]) : 0.f;
          gr[j] = (live && dph[m]) ? dph[m][row + lane + 32 * j] : 0.f;
        }
        float dx[XJ];
#pragma unroll
        for (int j = 0; j < XJ; ++j) dx[j] = 0.f;
        if (Wg[m] && dph[m]) {
          float z[ZJ];
#pragma unroll
          for (int jj = 0; jj < ZJ; ++jj) z[jj] = 0.f;
#pragma unroll
          for (int j = 0; j < XJ; ++j)
            for (int il = 0; il < 32; ++il) {
              const float xi = __shfl_sync(0xffffffffu, xr[j], il);
              const float *wrow = Ws[m] + (j * 32 + il) * WP;
#pragma unroll
              for (int jj = 0; jj < ZJ; ++jj) z[jj] = fmaf(xi, wrow[lane + 32 * jj], z[jj]);
            }
          float mx = kNegBig, mn = -kNegBig;
#pragma unroll
          for (int jj = 0; jj < ZJ; ++jj) { mx = fmaxf(mx, z[jj]); mn = fminf(mn, z[jj]); }
          mx = warp_max(mx);
          mn = -warp_max(-mn);
          float pp[ZJ], pn[ZJ], sp = 0.f, sn = 0.f;
#pragma unroll
          for (int jj = 0; jj < ZJ; ++jj) {
            pp[jj] = expf(z[jj] - mx); sp += pp[jj];
            pn[jj] = expf(mn - z[jj]); sn += pn[jj];
          }
          sp = 1.f / warp_sum(sp);
          sn = 1.f / warp_sum(sn);
          // dphi halves: feature f sits at x-lane (f % 32) word (f / 32)
          float dpv[ZJ], dnv[ZJ], ip = 0.f, in_ = 0.f;
#pragma unroll
          for (int jj = 0; jj < ZJ; ++jj) {
            pp[jj] *= sp; pn[jj] *= sn;
            dpv[jj] = gr[jj];            // f = lane + 32 jj  (< F)
            dnv[jj] = gr[jj + ZJ];       // F + f
            ip += dpv[jj] * pp[jj];
            in_ += dnv[jj] * pn[jj];
          }
          ip = warp_sum(ip);
          in_ = warp_sum(in_);
          float dz[ZJ];
#pragma unroll
          for (int jj = 0; jj < ZJ; ++jj) dz[jj] = pp[jj] * (dpv[jj] - ip) - pn[jj] * (dnv[jj] - in_);
          // dx[i] = sum_f dz[f] W[i][f]
#pragma unroll
          for (int jj = 0; jj < ZJ; ++jj)
            for (int fl = 0; fl < 32; ++fl) {
              const float dzf = __shfl_sync(0xffffffffu, dz[jj], fl);
              const int f = jj * 32 + fl;
#pragma unroll
              for (int j = 0; j < XJ; ++j) dx[j] = fmaf(dzf, Ws[m][(lane + 32 * j) * WP + f], dx[j]);
            }
#pragma unroll
          for (int jj = 0; jj < ZJ; ++jj) Zs[m][tt * F + lane + 32 * jj] = live ? dz[jj] : 0.f;
#pragma unroll
          for (int j = 0; j < XJ; ++j) Xs[m][tt * D + lane + 32 * j] = xr[j];
        } else {
#pragma unroll
          for (int j = 0; j < XJ; ++j) dx[j] = gr[j];   // identity map (or branch off)
        }
        if (live) {
#pragma unroll
          for (int j = 0; j < XJ; ++j) {
            const int i = lane + 32 * j;
            float tot = dx[j];
            if (dsw[m]) tot += dsw[m][row + i];
            dst[m][row + i] = from_f32<T>(tot);
          }
        }
      }
      if (live) {
#pragma unroll
        for (int j = 0; j < XJ; ++j) {
          const int i = lane + 32 * j;
          float dvv = 0.f;
          if (p.dv_gla) dvv += p.dv_gla[row + i];
          if (p.dv_swa) dvv += p.dv_swa[row + i];
          dvdst[row + i] = from_f32<T>(dvv);
          if (p.write_dg && !p.scalar_gate) {
            float dg = 0.f;
            if (p.da) dg = p.da[row + i] * dlogsigmoid(to_f32(gsrc[row + i])) * p.inv_tau;
            p.dg[row + i] = dg;
          }
        }
      }
      if (p.write_dg && p.scalar_gate) {   // one logit feeds every dimension: sum over them
        float s = 0.f;
        if (live && p.da)
#pragma unroll
          for (int j = 0; j < XJ; ++j) s += p.da[row + lane + 32 * j];
        s = warp_sum(s);
        if (live && lane == 0) {
          const size_t gi = (size_t)bh * p.L + t;
          p.dg[gi] = p.da ? s * dlogsigmoid(to_f32(gsrc[gi])) * p.inv_tau : 0.f;
        }
      }
    }
    __syncthreads();
    // dW += X^T dZ over this sub-tile (entry e = tid + 256 u: i = e / F, f = e % F)
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      if (!(Wg[m] && dph[m])) continue;
#pragma unroll
      for (int u = 0; u < WPT; ++u) {
        const int e = tid + 256 * u, i = e / F, f = e % F;
        float acc = dW[m][u];
        for (int tt = 0; tt < kFinSub; ++tt) acc = fmaf(Xs[m][tt * D + i], Zs[m][tt * F + f], acc);
        dW[m][u] = acc;
      }
    }
    __syncthreads();
  }
  float *dWg[2] = {p.dwq, p.dwk};
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    if (!(Wg[m] && dph[m] && dWg[m])) continue;
#pragma unroll
    for (int u = 0; u < WPT; ++u) atomicAdd(dWg[m] + (size_t)h * D * F + tid + 256 * u, dW[m][u]);
  }
}

// ------------------------------------------------------------ launchers ---
template <typename K>
static cudaError_t prep_launch(K k, size_t smem) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

#define LZ_DISPATCH(fn, ...)                                                   \
  (bf16 ? (D == 128 ? fn<__nv_bfloat16, 128>(__VA_ARGS__) : fn<__nv_bfloat16, 64>(__VA_ARGS__)) \
        : (D == 128 ? fn<float, 128>(__VA_ARGS__) : fn<float, 64>(__VA_ARGS__)))

template <typename T, int D>
static cudaError_t states_t(const GlaStatesArgs &a, int BH, cudaStream_t s) {
  const size_t smem = ((size_t)D * D + 3 * (size_t)kBwdC * D + D) * sizeof(float);
  cudaError_t e = prep_launch(gla_states_simt<T, D>, smem);
  if (e != cudaSuccess) return e;
  gla_states_simt<T, D><<<BH, 256, smem, s>>>(a);
  return cudaGetLastError();
}
cudaError_t launch_gla_states(const GlaStatesArgs &a, int BH, int D, bool bf16, cudaStream_t s) {
  if (a.L == 0) return cudaSuccess;
  return LZ_DISPATCH(states_t, a, BH, s);
}

template <typename T, int D>
static cudaError_t glabwd_t(const GlaBwdArgs &a, int BH, cudaStream_t s) {
  const size_t smem = (2 * (size_t)D * (D + 1) + 5 * (size_t)kBwdC * D + 2 * kBwdC * kBwdC + D) * sizeof(float);
  cudaError_t e = prep_launch(gla_bwd_simt<T, D>, smem);
  if (e != cudaSuccess) return e;
  gla_bwd_simt<T, D><<<BH, 256, smem, s>>>(a);
  return cudaGetLastError();
}
cudaError_t launch_gla_bwd_simt(const GlaBwdArgs &a, int BH, int D, bool bf16, cudaStream_t s) {
  return LZ_DISPATCH(glabwd_t, a, BH, s);
}

template <typename T, int D>
static cudaError_t swaq_t(const SwaBwdQArgs &a, int BH, cudaStream_t s) {
  const size_t smem = (4 * (size_t)kSwaT * D + kSwaT * (kSwaT + 1) + 3 * kSwaT + 8 + kSwaT * 16) * sizeof(float);
  cudaError_t e = prep_launch(swa_bwd_q<T, D>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.L + kSwaT - 1) / kSwaT, BH);
  swa_bwd_q<T, D><<<grid, 256, smem, s>>>(a);
  return cudaGetLastError();
}
cudaError_t launch_swa_bwd_q(const SwaBwdQArgs &a, int BH, int D, bool bf16, cudaStream_t s) {
  if (a.L == 0) return cudaSuccess;
  return LZ_DISPATCH(swaq_t, a, BH, s);
}

template <typename T, int D>
static cudaError_t swakv_t(const SwaBwdKVArgs &a, int BH, cudaStream_t s) {
  const size_t smem = (4 * (size_t)kSwaT * D + 2 * kSwaT * (kSwaT + 1) + 2 * kSwaT) * sizeof(float);
  cudaError_t e = prep_launch(swa_bwd_kv<T, D>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.P + kSwaT - 1) / kSwaT + (a.L + kSwaT - 1) / kSwaT, BH);
  swa_bwd_kv<T, D><<<grid, 256, smem, s>>>(a);
  return cudaGetLastError();
}
cudaError_t launch_swa_bwd_kv(const SwaBwdKVArgs &a, int BH, int D, bool bf16, cudaStream_t s) {
  if (a.L == 0) return cudaSuccess;
  return LZ_DISPATCH(swakv_t, a, BH, s);
}

template <typename T, int D>
static cudaError_t finish_t(const FinishBwdArgs &a, int BH, cudaStream_t s) {
  const size_t smem = (2 * (size_t)D * (D / 2 + 1) + 2 * (size_t)kFinSub * D + 2 * (size_t)kFinSub * (D / 2)) * sizeof(float);
  cudaError_t e = prep_launch(finish_bwd<T, D>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.L + kFinTok - 1) / kFinTok, BH);
  finish_bwd<T, D><<<grid, 256, smem, s>>>(a);
  return cudaGetLastError();
}
cudaError_t launch_finish_bwd(const FinishBwdArgs &a, int BH, int D, bool bf16, cudaStream_t s) {
  if (a.L == 0) return cudaSuccess;
  return LZ_DISPATCH(finish_t, a, BH, s);
}

}  // namespace lz
