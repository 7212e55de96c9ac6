// Tensor-core (tcgen05 / TMEM / TMA) forward of the Lizard hybrid layer,
// bf16 activations, dk = dv = 128, window <= 128, M <= 16.
//
// One CTA (128 threads, one TMEM lane per thread) walks one (batch, head)
// sequence in tiles of T = 128 tokens, i.e. two 64-token chunks per tile with
// the cumulative gate absorbed once per tile.  Per tile:
//
//   TMA     X_q, X_k, V, G (gate logits) of the tile and K of the previous
//           tile, 128-byte swizzled; later V of the previous tile.
//   MMA 1   L  = X_q [K_prev ; X_k]^T            (window logits, 128 x 256)
//           Zq = X_q W_q, Zk = X_k W_k           (feature-map projections)
//   gates   thread = key dimension i, tokens in reverse:
//             acc_t = sum_{s>t} -a_s,  E_t = exp(acc_t) = exp(b_t - r)
//           written as bf16 over G; exp(r) = exp(-acc_{-1}) decays the state.
//   rows    thread = token t:
//             anchor softmax over the 256 logits (band mask) and the M meta
//             logits -> P^ = exp(l - max), unnormalised, into TMEM;
//             phi_q, phi_k from Zq, Zk; Qt = phi_q E l/alpha (TMEM),
//             Kt = phi_k / E (shared memory);
//           thread = key dimension i: S' = diag(exp r) S in TMEM, and its
//           bf16 copy in shared memory.
//   MMA 2   A  = Qt Kt^T
//   rows    A^ = tril(A) (TMEM; l/alpha comes in through Qt)
//   MMA 3   O  = Qt S' + A^ V + P^ [V_prev ; V];   S = S' + Kt^T V
//   store   o = O alpha/l + (alpha/l) sum_m p_m mv_m
//
// Scaling the GLA operands by l/alpha lets one accumulator hold both
// branches: o = o_gla + alpha o_swa = (alpha/l) (o_gla l/alpha + P^ V).
// (English gist.science summary, section 2.A: state update, anchor window
// attention with meta tokens, final mix; Chinese summary, section 2.3: gate
// absorbed into q and k in log space so the core runs as bf16 GEMMs.)
//
// Long sequences with few (batch, head) pairs are split into segments so
// that every SM has a sequence slice: a state pass (the same kernel in
// mode 1: gates, phi_k, state update only) gives each segment's local end
// state and total log-decay, a combine kernel chains them into each
// segment's start state, and the full pass runs all segments in parallel.
//
// A tile whose in-tile log-decay spread exceeds kMaxSpread in some key
// dimension sets the RANGE bit of the workspace status word (the portable
// path computes such inputs exactly).  Every mbarrier wait is bounded; a
// wait that gives up sets the TIMEOUT bit and the CTA stops, frees its TMEM
// and returns.
#include "common.cuh"
#include "lizard_internal.h"
#include "tc_common.cuh"
#include "tc_host.h"

namespace lz {
namespace {

using namespace tc;

constexpr int T = 128;             // tokens per tile
constexpr int D = 128;             // dk = dv
constexpr int F = D / 2;           // feature-map width per half
constexpr uint32_t REG = kReg;     // one 64-column swizzled region of a 128-row tile
constexpr uint32_t TILE = kTile;   // a 128 x 128 bf16 tile
constexpr int MAXM = 16;
constexpr int NTHREADS = 256;     // two warpgroups

// shared-memory regions (offsets from the 1024-aligned base)
constexpr uint32_t R_XQ = 0;            // X_q, then S' (bf16, MN-major)
constexpr uint32_t R_XK = 1 * TILE;     // X_k, then Kt
constexpr uint32_t R_KP = 2 * TILE;     // K of the previous tile
constexpr uint32_t R_V = 3 * TILE;      // V
constexpr uint32_t R_G = 4 * TILE;      // G, then E, then V of the previous tile
constexpr uint32_t R_WQ = 5 * TILE;     // W_q bf16, [dk rows][64 features], MN-major
constexpr uint32_t R_WK = 5 * TILE + REG;
constexpr uint32_t SMEM_TILES = 5 * TILE + 2 * REG;
constexpr size_t SMEM_BYTES = SMEM_TILES + 1024;   // + alignment slack

// TMEM columns
constexpr uint32_t C_S = 0, C_O = 128, C_ZQ = 128, C_ZK = 192, C_A = 128;
constexpr uint32_t C_L = 256, C_P = 256, C_QT = 384, C_AH = 448;

constexpr uint32_t ST_TIMEOUT = 1u, ST_RANGE = 2u;

struct Params {
  CUtensorMap mq, mk, mv, mg;
  const float *wq, *wk, *meta_k, *meta_v, *alpha, *state_in;
  __nv_bfloat16 *o;
  float *state_out, *lse;
  uint32_t *status;
  const float *seg_start;   // [BH][nseg][D][D] start state of each segment (nseg > 1)
  float *seg_state;         // mode 1: [BH][nseg][D][D] local end state (zero start)
  float *seg_decay;         // mode 1: [BH][nseg][D] summed log-decay of the segment
  __nv_bfloat16 *snap;      // mode 1 with nseg == 1: [BH][ntiles][D][D] bf16 S' of every tile
  int H, L, M, window, branch;
  int mode;                 // 0: full forward, 1: state pass
  int nseg, tiles_per_seg;
  float inv_tau, scale;
};


__device__ __forceinline__ void issue_tile_loads(const Params &p, unsigned char *sm, uint64_t *bar, int bh,
                                                 int t0, bool full) {
  mbar_expect_tx(bar, (full ? 5 : 3) * TILE);
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    if (full) {
      tma_load_3d(sm + R_XQ + r * REG, &p.mq, bar, 64 * r, t0, bh);
      tma_load_3d(sm + R_KP + r * REG, &p.mk, bar, 64 * r, t0 - T, bh);
    }
    tma_load_3d(sm + R_XK + r * REG, &p.mk, bar, 64 * r, t0, bh);
    tma_load_3d(sm + R_V + r * REG, &p.mv, bar, 64 * r, t0, bh);
    tma_load_3d(sm + R_G + r * REG, &p.mg, bar, 64 * r, t0, bh);
  }
}

// Gates, thread = key dimension i: in-tile suffix sums of the log-decay,
// E_t = exp(sum_{s>t} -a_s) = exp(b_t - r) written as bf16 over the gate
// logits, exp(r) (the tile's decay) into s_dec[i].  16 tokens per step; the
// next step's logits are read before this step's factors are written.
// Returns the largest exponent of E in this dimension (its value at t = 0).
__device__ __forceinline__ float gates_by_dim(unsigned char *sm, int i, int t0, int L, float inv_tau,
                                              float *s_dec) {
  unsigned char *gcol = sm + R_G + (i >> 6) * REG;
  const int ci = i & 63;
  float acc = 0.f, spread = 0.f, gn[16];
#pragma unroll
  for (int u = 0; u < 16; ++u)
    gn[u] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(gcol + sw128_offset(T - 16 + u, ci)));
#pragma unroll 1
  for (int tb = T - 16; tb >= 0; tb -= 16) {
    float a[16], pre[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) a[u] = (t0 + tb + u < L) ? log_decay_fast(gn[u], inv_tau) : 0.f;
    if (tb > 0) {
#pragma unroll
      for (int u = 0; u < 16; ++u)
        gn[u] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(gcol + sw128_offset(tb - 16 + u, ci)));
    }
#pragma unroll
    for (int u = 15; u >= 0; --u) { pre[u] = acc; acc -= a[u]; }
#pragma unroll
    for (int u = 0; u < 16; ++u)
      *reinterpret_cast<__nv_bfloat16 *>(gcol + sw128_offset(tb + u, ci)) = __float2bfloat16_rn(__expf(pre[u]));
    spread = pre[0];
  }
  s_dec[i] = __expf(-acc);
  return spread;
}

// Qt for dimensions 64 h .. 64 h + 63: phi_q E gscale, bf16 pairs into TMEM.
__device__ __forceinline__ void qt_half(unsigned char *sm, uint32_t tl, int row, int h, float gscale) {
  float ph[F];
  const float s = feature_half(tl + C_ZQ, h, ph) * gscale;
#pragma unroll
  for (int c16 = 0; c16 < 4; ++c16) {     // 16 dims = 8 TMEM columns
    float e16[16];
    unpack8(*chunk_ptr(sm, R_G, row, 8 * h + 2 * c16), e16);
    unpack8(*chunk_ptr(sm, R_G, row, 8 * h + 2 * c16 + 1), e16 + 8);
    uint32_t r8[8];
#pragma unroll
    for (int u = 0; u < 16; u += 2)
      r8[u / 2] = pack_bf16(ph[16 * c16 + u] * e16[u] * s, ph[16 * c16 + u + 1] * e16[u + 1] * s);
    tmem_st8(tl + C_QT + 32 * h + 8 * c16, r8);
  }
}

// Kt for dimensions 64 h .. 64 h + 63: phi_k / E, bf16 into shared memory
// over X_k.  E comes as bf16 from the gate region (full pass) or as fp32
// from TMEM (state pass).
__device__ __forceinline__ void kt_half(unsigned char *sm, uint32_t tl, int row, int h, bool e_in_tmem) {
  float ph[F];
  const float s = feature_half(tl + C_ZK, h, ph);
#pragma unroll
  for (int c16 = 0; c16 < 4; ++c16) {
    float e16[16], k16[16];
    if (e_in_tmem) {
      tmem_ld16(tl + C_L + 64 * h + 16 * c16, e16);
    } else {
      unpack8(*chunk_ptr(sm, R_G, row, 8 * h + 2 * c16), e16);
      unpack8(*chunk_ptr(sm, R_G, row, 8 * h + 2 * c16 + 1), e16 + 8);
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) k16[u] = __fdividef(ph[16 * c16 + u] * s, e16[u]);
    *chunk_ptr(sm, R_XK, row, 8 * h + 2 * c16) = pack8(k16);
    *chunk_ptr(sm, R_XK, row, 8 * h + 2 * c16 + 1) = pack8(k16 + 8);
  }
}

// Named barriers between the two warpgroups (id 0 is __syncthreads).
constexpr int BAR_E = 1;       // gate factors E written (group 1 -> group 0)
constexpr int BAR_G = 2;       // row scales of the anchor softmax written (group 0 -> group 1)
constexpr int BAR_DECAY = 3;   // + group: the row-wise decay scan inside one group

__global__ void __launch_bounds__(NTHREADS, 1) tc_fwd_kernel(const __grid_constant__ Params p) {
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(16) float s_mk[MAXM][D];
  __shared__ __align__(16) float s_mv[MAXM][D];
  __shared__ float s_ml[MAXM][T];     // meta logits, then their mixing weights, per row
  __shared__ float s_dec[D];
  __shared__ float s_gscale[T], s_oscale[T];
  __shared__ float s_wtot[2][4][16];
  __shared__ uint64_t bar_tma, bar_vp, bar_m1, bar_m2, bar_m3;
  __shared__ uint32_t s_tmem;
  __shared__ int s_fail;

  const int tid = threadIdx.x, warp = tid >> 5;
  const int wg = tid >> 7;                             // warpgroup
  const int row = tid & 127;                           // TMEM lane == tile row
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const int bh = blockIdx.x, h = bh % p.H, seg = blockIdx.y;
  const float alpha = p.alpha ? p.alpha[h] : 1.f;
  const bool full = p.mode == 0;
  const bool gla = p.branch != 2, swa = full && p.branch != 1;
  const uint32_t sbase = smem_u32(sm);

  if (warp == 0) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_tma, 1);
    mbar_init(&bar_vp, 1);
    mbar_init(&bar_m1, 1);
    mbar_init(&bar_m2, 1);
    mbar_init(&bar_m3, 1);
    fence_barrier_init();
    s_fail = 0;
  }
  // feature-map weights -> bf16, MN-major [dk row][feature]; group 0 W_q, group 1 W_k
  {
    const int i = row;
    const float *W = wg == 0 ? p.wq : p.wk;
    const uint32_t reg = wg == 0 ? R_WQ : R_WK;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float f[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) f[u] = W ? W[((size_t)h * D + i) * F + c * 8 + u] : 0.f;
      *reinterpret_cast<uint4 *>(sm + reg + sw128_offset(i, c * 8)) = pack8(f);
    }
  }
  for (int e = tid; e < MAXM * D; e += NTHREADS) {
    const int m = e / D;
    s_mk[m][e % D] = m < p.M ? p.meta_k[(size_t)h * p.M * D + e] : 0.f;
    s_mv[m][e % D] = (m < p.M && p.meta_v) ? p.meta_v[(size_t)h * p.M * D + e] : 0.f;
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s_tmem;
  const uint32_t tl = tb + lane_off;

  // initial state -> TMEM columns [0, 128), lane = key dimension; each
  // group writes one half of the columns
  {
    const float *src = nullptr;
    if (full && p.nseg > 1) src = p.seg_start + (((size_t)bh * p.nseg + seg) * D + row) * D;
    else if (full && p.state_in) src = p.state_in + ((size_t)bh * D + row) * D;
    else if (p.snap && p.state_in) src = p.state_in + ((size_t)bh * D + row) * D;
#pragma unroll
    for (int c = 64 * wg; c < 64 * wg + 64; c += 8) {
      uint32_t r[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) r[u] = __float_as_uint(src ? src[c + u] : 0.f);
      tmem_st8(tl + C_S + c, r);
    }
    tmem_st_wait();
  }

  const int ntiles_all = (p.L + T - 1) / T;
  const int cbeg = seg * p.tiles_per_seg;
  const int cend = min(ntiles_all, cbeg + p.tiles_per_seg);
  uint32_t *err = p.status;
  float tot_decay = 0.f;                      // state pass: summed log-decay of the dimension this thread owns
  if (tid == 0 && cbeg < cend) issue_tile_loads(p, sm, &bar_tma, bh, cbeg * T, full);
  const uint32_t id_128 = idesc_bf16(128, 128, 0, 0);
  const uint32_t id_z = idesc_bf16(128, 64, 0, 1);
  const uint32_t id_mn = idesc_bf16(128, 128, 0, 1);
  const uint32_t id_st = idesc_bf16(128, 128, 1, 1);

  for (int c = cbeg; c < cend; ++c) {
    const uint32_t par = (c - cbeg) & 1;
    const int t0 = c * T;
    const int tq = t0 + row;                  // this thread's query token
    const bool qvalid = tq < p.L;

    // ---------------------------------------------------------- MMA 1 ---
    bool ok = mbar_wait(&bar_tma, par, err, ST_TIMEOUT);
    if (__syncthreads_or(!ok)) { s_fail = 1; break; }
    if (tid == 0) {
      tc_fence_after();
      const uint32_t xq = sbase + R_XQ, xk = sbase + R_XK, kp = sbase + R_KP;
      if (swa) {
        for (int s = 0; s < 8; ++s) mma_ss(tb + C_L, desc_k(xq, s), desc_k(kp, s), id_128, s > 0);
        for (int s = 0; s < 8; ++s) mma_ss(tb + C_L + 128, desc_k(xq, s), desc_k(xk, s), id_128, s > 0);
      }
      if (full)
        for (int s = 0; s < 8; ++s) mma_ss(tb + C_ZQ, desc_k(xq, s), desc_mn(sbase + R_WQ, s), id_z, s > 0);
      for (int s = 0; s < 8; ++s) mma_ss(tb + C_ZK, desc_k(xk, s), desc_mn(sbase + R_WK, s), id_z, s > 0);
      mma_commit(&bar_m1);
    }

    if (full && wg == 1) {
      // ------------------------------- group 1: gates, then phi half 1 ---
      const float spread = gates_by_dim(sm, row, t0, p.L, p.inv_tau, s_dec);
      if (spread > kMaxSpread && gla) atomicOr(err, ST_RANGE);
      bar_arrive(BAR_E, NTHREADS);
      ok &= mbar_wait(&bar_m1, par, err, ST_TIMEOUT);
      tc_fence_after();
      kt_half(sm, tl, row, 1, false);
      bar_sync(BAR_G, NTHREADS);
      qt_half(sm, tl, row, 1, s_gscale[row]);
    } else if (full) {
      // ---------------------- group 0: anchor softmax, then phi half 0 ---
      ok &= mbar_wait(&bar_m1, par, err, ST_TIMEOUT);
      tc_fence_after();
      float lsum = 1.f, mx = 0.f;                 // row normaliser and max (scaled logits)
      if (swa) {
        // meta logits q . mk_m (scaled) into s_ml, four meta tokens per pass
        for (int m0 = 0; m0 < p.M; m0 += 4) {
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
          for (int ch = 0; ch < 16; ++ch) {
            float q8[8];
            unpack8(*chunk_ptr(sm, R_XQ, row, ch), q8);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float4 a = *reinterpret_cast<const float4 *>(&s_mk[m0 + k][ch * 8]);
              const float4 b = *reinterpret_cast<const float4 *>(&s_mk[m0 + k][ch * 8 + 4]);
              acc[2 * k] = fmaf(q8[0], a.x, fmaf(q8[1], a.y, fmaf(q8[2], a.z, fmaf(q8[3], a.w, acc[2 * k]))));
              acc[2 * k + 1] = fmaf(q8[4], b.x, fmaf(q8[5], b.y, fmaf(q8[6], b.z, fmaf(q8[7], b.w, acc[2 * k + 1]))));
            }
          }
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (m0 + k < p.M) s_ml[m0 + k][row] = (acc[2 * k] + acc[2 * k + 1]) * p.scale;
        }
        mx = kNegBig;
        for (int m = 0; m < p.M; ++m) mx = fmaxf(mx, s_ml[m][row]);
        // Logit column cl holds key t0 - T + cl.  Row r sees columns
        // [r + T + 1 - window, r + T] (and keys >= 0), so warp w4 only
        // visits 32-column chunks w4 + (T + 1 - window) / 32 .. w4 + 4, and
        // only the first and last of those need the band mask.
        const int w4 = warp & 3;
        const int cbase = t0 - T;
        const int lo_c = max(tq - p.window + 1, 0) - cbase, hi_c = tq - cbase;
        int ch_lo = (32 * w4 + T + 1 - p.window) >> 5;
        if (cbase < 0) ch_lo = max(ch_lo, 4);
        const int ch_hi = w4 + 4;
        const int in_lo = 32 * w4 + 31 + T + 1 - p.window;   // interior chunk: 32 ch >= in_lo
        for (int ch = ch_lo; ch <= ch_hi; ++ch) {
          float v[32];
          tmem_ld32(tl + C_L + ch * 32, v);
          float m4[4] = {kNegBig, kNegBig, kNegBig, kNegBig};
          if (32 * ch >= in_lo && 32 * ch + 31 <= 32 * w4 + T && 32 * ch + cbase >= 0) {
#pragma unroll
            for (int u = 0; u < 32; ++u) m4[u & 3] = fmaxf(m4[u & 3], v[u]);
          } else {
#pragma unroll
            for (int u = 0; u < 32; ++u) {
              const int cl = 32 * ch + u;
              if (cl >= lo_c && cl <= hi_c) m4[u & 3] = fmaxf(m4[u & 3], v[u]);
            }
          }
          const float cm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
          if (cm > kNegBig) mx = fmaxf(mx, cm * p.scale);
        }
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
        for (int ch = ch_lo; ch <= ch_hi; ++ch) {
          float v[32];
          tmem_ld32(tl + C_L + ch * 32, v);
          const bool inner = 32 * ch >= in_lo && 32 * ch + 31 <= 32 * w4 + T && 32 * ch + cbase >= 0;
          uint32_t pk[16];
#pragma unroll
          for (int u = 0; u < 32; u += 2) {
            float e0 = __expf(fmaf(v[u], p.scale, -mx));
            float e1 = __expf(fmaf(v[u + 1], p.scale, -mx));
            if (!inner) {
              const int cl = 32 * ch + u;
              e0 = (cl >= lo_c && cl <= hi_c) ? e0 : 0.f;
              e1 = (cl + 1 >= lo_c && cl + 1 <= hi_c) ? e1 : 0.f;
            }
            s4[(u >> 1) & 3] += e0 + e1;
            pk[u / 2] = alpha != 0.f ? pack_bf16(e0, e1) : 0u;
          }
          tmem_st8(tl + C_P + ch * 16, pk);
          tmem_st8(tl + C_P + ch * 16 + 8, pk + 8);
        }
        // chunks outside the band: P = 0 (written after the band's logits
        // were read, since P column 16 ch overlays logit chunk ch / 2)
        {
          uint32_t zero[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
          for (int ch = 0; ch < 8; ++ch) {
            if (ch >= ch_lo && ch <= ch_hi) continue;
            tmem_st8(tl + C_P + ch * 16, zero);
            tmem_st8(tl + C_P + ch * 16 + 8, zero);
          }
        }
        float sm_meta = 0.f;
        for (int m = 0; m < p.M; ++m) {
          const float e = __expf(s_ml[m][row] - mx);
          sm_meta += e;
          s_ml[m][row] = e;
        }
        lsum = ((s4[0] + s4[1]) + (s4[2] + s4[3])) + sm_meta;
        if (!qvalid) lsum = 1.f;
        if (qvalid && p.lse) p.lse[(size_t)bh * p.L + tq] = mx + logf(lsum);
      }
      // GLA operands carry l/alpha so that one accumulator holds both terms
      const bool mixed = swa && alpha != 0.f;
      const float gscale = mixed ? lsum / alpha : 1.f;
      s_gscale[row] = gscale;
      s_oscale[row] = mixed ? alpha / lsum : 1.f;
      if (swa) {
        const float mscale = mixed ? alpha / lsum : 0.f;   // meta-value weight per exp
        for (int m = 0; m < p.M; ++m) s_ml[m][row] *= mscale;
      }
      bar_arrive(BAR_G, NTHREADS);
      bar_sync(BAR_E, NTHREADS);
      qt_half(sm, tl, row, 0, gscale);
      kt_half(sm, tl, row, 0, false);
    } else {
      // ------------- state pass: fp32 decay factors, phi_k half per group ---
      for (int c16 = 4 * wg; c16 < 4 * wg + 4; ++c16) {
        float E[16], tot[16];
        row_decay16(sm + R_G, row, c16, qvalid, p.inv_tau, s_wtot[wg], E, tot, BAR_DECAY + wg);
        uint32_t r[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) r[u] = __float_as_uint(E[u]);
        tmem_st8(tl + C_L + c16 * 16, r);
#pragma unroll
        for (int u = 0; u < 8; ++u) r[u] = __float_as_uint(E[8 + u]);
        tmem_st8(tl + C_L + c16 * 16 + 8, r);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          if (row == c16 * 16 + u) {   // the dimension this thread owns
            s_dec[row] = __expf(-tot[u]);   // exp(r)
            tot_decay -= tot[u];             // r, the tile's log-decay
          }
          if (row == 0 && E[u] > kMaxSpreadExp && gla) atomicOr(err, ST_RANGE);
        }
      }
      tmem_st_wait();
      ok &= mbar_wait(&bar_m1, par, err, ST_TIMEOUT);
      tc_fence_after();
      kt_half(sm, tl, row, wg, true);
    }
    tmem_st_wait();
    fence_proxy_async();
    tc_fence_before();
    if (__syncthreads_or(!ok)) { s_fail = 1; break; }

    // ---------------------------------------------------------- MMA 2 ---
    if (tid == 0) {
      tc_fence_after();
      if (gla && full)
        for (int s = 0; s < 8; ++s) mma_ts(tb + C_A, tb + C_QT + s * 8, desc_k(sbase + R_XK, s), id_128, s > 0);
      mma_commit(&bar_m2);
      // V of the previous tile into the G region (E has been consumed)
      mbar_expect_tx(&bar_vp, swa ? TILE : 0);
      if (swa) {
        tma_load_3d(sm + R_G, &p.mv, &bar_vp, 0, t0 - T, bh);
        tma_load_3d(sm + R_G + REG, &p.mv, &bar_vp, 64, t0 - T, bh);
      }
    }

    // -------------- state rescale (thread = dimension, column half per group) ---
    if (gla) {
      tc_fence_after();
      const int i = row;
      const float dec = s_dec[i];
      for (int c16 = 4 * wg; c16 < 4 * wg + 4; ++c16) {
        float v[16];
        tmem_ld16(tl + C_S + c16 * 16, v);
        uint32_t r[8];
#pragma unroll
        for (int u = 0; u < 16; ++u) v[u] *= dec;
#pragma unroll
        for (int u = 0; u < 8; ++u) r[u] = __float_as_uint(v[u]);
        tmem_st8(tl + C_S + c16 * 16, r);
#pragma unroll
        for (int u = 0; u < 8; ++u) r[u] = __float_as_uint(v[8 + u]);
        tmem_st8(tl + C_S + c16 * 16 + 8, r);
        if (full) {   // bf16 copy S'[i][v], MN-major: rows = i (K of the O = Qt S' product)
          *chunk_ptr(sm, R_XQ, i, 2 * c16) = pack8(v);
          *chunk_ptr(sm, R_XQ, i, 2 * c16 + 1) = pack8(v + 8);
        } else if (p.snap) {   // the backward's copy of S', row-major [i][v]
          uint4 *dst = reinterpret_cast<uint4 *>(p.snap + (((size_t)bh * ntiles_all + c) * D + i) * D + c16 * 16);
          dst[0] = pack8(v);
          dst[1] = pack8(v + 8);
        }
      }
    }
    ok = mbar_wait(&bar_m2, par, err, ST_TIMEOUT);
    tc_fence_after();

    // ---------------------- masked intra A (column half per group) ---
    if (gla && full) {
      for (int c16 = 4 * wg; c16 < 4 * wg + 4; ++c16) {
        float v[16];
        tmem_ld16(tl + C_A + c16 * 16, v);
        uint32_t r[8];
#pragma unroll
        for (int u = 0; u < 16; u += 2) {
          const int j = c16 * 16 + u;        // tile-local key index
          // A = Qt Kt^T already carries l/alpha through Qt
          const float a0 = (j <= row) ? v[u] : 0.f;
          const float a1 = (j + 1 <= row) ? v[u + 1] : 0.f;
          r[u / 2] = pack_bf16(a0, a1);
        }
        tmem_st8(tl + C_AH + c16 * 8, r);
      }
    }
    tmem_st_wait();
    fence_proxy_async();
    tc_fence_before();
    ok &= mbar_wait(&bar_vp, par, err, ST_TIMEOUT);
    if (__syncthreads_or(!ok)) { s_fail = 1; break; }

    // ---------------------------------------------------------- MMA 3 ---
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sp = sbase + R_XQ, v = sbase + R_V, vp = sbase + R_G, kt = sbase + R_XK;
      uint32_t accum = 0;
      if (gla && full) {
        for (int s = 0; s < 8; ++s) { mma_ts(tb + C_O, tb + C_QT + s * 8, desc_mn(sp, s), id_mn, accum); accum = 1; }
        for (int s = 0; s < 8; ++s) mma_ts(tb + C_O, tb + C_AH + s * 8, desc_mn(v, s), id_mn, 1);
      }
      if (swa) {
        for (int s = 0; s < 8; ++s) { mma_ts(tb + C_O, tb + C_P + s * 8, desc_mn(vp, s), id_mn, accum); accum = 1; }
        for (int s = 0; s < 8; ++s) mma_ts(tb + C_O, tb + C_P + 64 + s * 8, desc_mn(v, s), id_mn, 1);
      }
      if (gla)
        for (int s = 0; s < 8; ++s) mma_ss(tb + C_S, desc_mn(kt, s), desc_mn(v, s), id_st, 1);
      mma_commit(&bar_m3);
    }
    ok = mbar_wait(&bar_m3, par, err, ST_TIMEOUT);
    if (__syncthreads_or(!ok)) { s_fail = 1; break; }
    tc_fence_after();
    if (tid == 0 && c + 1 < cend) issue_tile_loads(p, sm, &bar_tma, bh, t0 + T, full);

    // ---------------------------- epilogue (column half per group) ---
    if (full) {
      // tcgen05.ld is warp-collective: every lane loads, valid rows store
      __nv_bfloat16 *orow = p.o + ((size_t)bh * p.L + (qvalid ? tq : 0)) * D;
      const float oscale = s_oscale[row];
      for (int c16 = 4 * wg; c16 < 4 * wg + 4; ++c16) {
        float v[16];
        tmem_ld16(tl + C_O + c16 * 16, v);
#pragma unroll
        for (int u = 0; u < 16; ++u) v[u] *= oscale;
        if (swa && p.meta_v) {
          for (int m = 0; m < p.M; ++m) {
            const float w = s_ml[m][row];
            const float4 *mv = reinterpret_cast<const float4 *>(&s_mv[m][c16 * 16]);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const float4 x = mv[q4];
              v[4 * q4] = fmaf(w, x.x, v[4 * q4]);
              v[4 * q4 + 1] = fmaf(w, x.y, v[4 * q4 + 1]);
              v[4 * q4 + 2] = fmaf(w, x.z, v[4 * q4 + 2]);
              v[4 * q4 + 3] = fmaf(w, x.w, v[4 * q4 + 3]);
            }
          }
        }
        if (qvalid) {
          uint4 *dst = reinterpret_cast<uint4 *>(orow + c16 * 16);
          dst[0] = pack8(v);
          dst[1] = pack8(v + 8);
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  }

  float *sdst = nullptr;
  if (full && p.state_out && gla && seg == p.nseg - 1) sdst = p.state_out + ((size_t)bh * D + row) * D;
  if (!full && p.seg_state) {
    sdst = p.seg_state + (((size_t)bh * p.nseg + seg) * D + row) * D;
    if ((row >> 6) == wg) p.seg_decay[((size_t)bh * p.nseg + seg) * D + row] = tot_decay;
  }
  if (!s_fail && sdst) {
    tc_fence_after();
    for (int c16 = 4 * wg; c16 < 4 * wg + 4; ++c16) {
      float v[16];
      tmem_ld16(tl + C_S + c16 * 16, v);
#pragma unroll
      for (int u = 0; u < 16; u += 4)
        *reinterpret_cast<float4 *>(sdst + c16 * 16 + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
    }
  }
  if (s_fail && tid == 0) {
    // let whatever was issued drain before the shared memory is released
    mbar_wait(&bar_tma, 0, nullptr, 0, 1u << 16);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 512);
}

// Start state of every segment: S_0 = state_in (or 0),
// S_{s+1} = diag(exp(decay_s)) S_s + local_s.
__global__ void __launch_bounds__(256) seg_combine_kernel(const float *seg_state, const float *seg_decay,
                                                          const float *state_in, float *seg_start, int nseg) {
  const int bh = blockIdx.x;
  for (int e = threadIdx.x; e < D * D; e += 256) {
    const int i = e / D;
    float sv = state_in ? state_in[(size_t)bh * D * D + e] : 0.f;
    seg_start[((size_t)bh * nseg) * D * D + e] = sv;
    for (int sg = 1; sg < nseg; ++sg) {
      const size_t prev = (size_t)bh * nseg + sg - 1;
      sv = expf(seg_decay[prev * D + i]) * sv + seg_state[prev * D * D + e];
      seg_start[((size_t)bh * nseg + sg) * D * D + e] = sv;
    }
  }
}

}  // namespace

bool tc_fwd_supported(int dk, int dv, int window, int M, bool bf16) {
  return bf16 && dk == D && dv == D && window <= T && M <= MAXM;
}

// Segments per sequence: enough (batch, head, segment) CTAs to cover the
// 148 SMs once, each segment at least two tiles long.
void tc_fwd_segments(int BH, int L, int *nseg, int *tiles_per_seg) {
  const int ntiles = (L + T - 1) / T;
  int n = BH >= 120 ? 1 : 148 / (BH > 0 ? BH : 1);
  n = n < ntiles / 2 ? n : ntiles / 2;
  if (n < 1) n = 1;
  const int tps = (ntiles + n - 1) / n;
  *tiles_per_seg = tps > 0 ? tps : 1;
  *nseg = tps > 0 ? (ntiles + tps - 1) / tps : 1;
}

size_t tc_fwd_workspace_bytes(int BH, int L) {
  int nseg, tps;
  tc_fwd_segments(BH, L, &nseg, &tps);
  if (nseg <= 1) return 0;
  return (size_t)BH * nseg * (2 * (size_t)D * D + D) * sizeof(float);
}

int tc_fwd_stage_count(int BH, int L) {
  int nseg, tps;
  tc_fwd_segments(BH, L, &nseg, &tps);
  return nseg > 1 ? 3 : 1;
}

// Forward state pass over whole sequences that keeps, for every 128-token
// tile, the bf16 state at the tile's start already decayed by the tile's
// gates, S' = diag(exp r) S (the backward's input).
cudaError_t launch_tc_state_snapshots(const TcFwdArgs &a, void *snap, cudaStream_t s) {
  Params p;
  memset(&p, 0, sizeof(p));
  const uint64_t rows = (uint64_t)a.L;
  if (!make_map_bf16_3d(&p.mq, a.q, D, rows, a.BH, T) || !make_map_bf16_3d(&p.mk, a.k, D, rows, a.BH, T) ||
      !make_map_bf16_3d(&p.mv, a.v, D, rows, a.BH, T) || !make_map_bf16_3d(&p.mg, a.g, D, rows, a.BH, T))
    return cudaErrorInvalidValue;
  p.wq = a.wq;
  p.wk = a.wk;
  p.meta_k = a.meta_k;
  p.meta_v = a.meta_v;
  p.alpha = a.alpha;
  p.state_in = a.state_in;
  p.status = a.status;
  p.snap = static_cast<__nv_bfloat16 *>(snap);
  p.H = a.H;
  p.L = a.L;
  p.M = a.M;
  p.window = a.window;
  p.branch = 0;
  p.mode = 1;
  p.nseg = 1;
  p.tiles_per_seg = (a.L + T - 1) / T;
  p.inv_tau = a.inv_tau;
  p.scale = a.scale;
  // the state pass starts from state_in when there is one
  p.seg_start = a.state_in;
  p.seg_state = nullptr;
  p.seg_decay = nullptr;
  cudaError_t e = cudaFuncSetAttribute(tc_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  tc_fwd_kernel<<<dim3(a.BH, 1), NTHREADS, SMEM_BYTES, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_tc_fwd(const TcFwdArgs &a, int stage, cudaStream_t s) {
  int nseg, tps;
  tc_fwd_segments(a.BH, a.L, &nseg, &tps);
  float *seg_state = static_cast<float *>(a.seg_ws);
  float *seg_start = seg_state ? seg_state + (size_t)a.BH * nseg * D * D : nullptr;
  float *seg_decay = seg_start ? seg_start + (size_t)a.BH * nseg * D * D : nullptr;
  if (nseg > 1 && stage == 1) {
    seg_combine_kernel<<<a.BH, 256, 0, s>>>(seg_state, seg_decay, a.state_in, seg_start, nseg);
    return cudaGetLastError();
  }
  Params p;
  memset(&p, 0, sizeof(p));
  const uint64_t rows = (uint64_t)a.L;
  if (!make_map_bf16_3d(&p.mq, a.q, D, rows, a.BH, T) || !make_map_bf16_3d(&p.mk, a.k, D, rows, a.BH, T) ||
      !make_map_bf16_3d(&p.mv, a.v, D, rows, a.BH, T) ||
      !make_map_bf16_3d(&p.mg, a.g ? a.g : a.q, D, rows, a.BH, T))   // g unused without the GLA branch
    return cudaErrorInvalidValue;
  p.wq = a.wq;
  p.wk = a.wk;
  p.meta_k = a.meta_k;
  p.meta_v = a.meta_v;
  p.alpha = a.alpha;
  p.state_in = a.state_in;
  p.o = static_cast<__nv_bfloat16 *>(a.o);
  p.state_out = a.state_out;
  p.lse = a.lse;
  p.status = a.status;
  p.seg_start = seg_start;
  p.seg_state = seg_state;
  p.seg_decay = seg_decay;
  p.H = a.H;
  p.L = a.L;
  p.M = a.M;
  p.window = a.window;
  p.branch = a.branch;
  p.nseg = nseg;
  p.tiles_per_seg = tps;
  p.inv_tau = a.inv_tau;
  p.scale = a.scale;
  static size_t configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || configured[dev] < SMEM_BYTES) {
    e = cudaFuncSetAttribute(tc_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = SMEM_BYTES;
  }
  if (nseg > 1 && stage == 0) {          // state pass over every segment but the last
    p.mode = 1;
    tc_fwd_kernel<<<dim3(a.BH, nseg - 1), NTHREADS, SMEM_BYTES, s>>>(p);
  } else {                               // full pass
    p.mode = 0;
    tc_fwd_kernel<<<dim3(a.BH, nseg), NTHREADS, SMEM_BYTES, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace lz
