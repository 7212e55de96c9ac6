// Tensor-core (tcgen05 / TMEM / TMA) backward of the GLA branch, bf16,
// dk = dv = 128, 128-token tiles (English gist.science summary, section
// 2.A "State Update"; the gate absorbed into q and k in log space as the
// Chinese summary, section 2.3, describes).
//
// Per tile, with E = exp(b - r) (b the in-tile cumulative log-decay, r its
// value at the tile's end), Qt = phi_q E, Kt = phi_k / E, S' = diag(exp r) S
// the tile's start state decayed over the tile, and dS the gradient into the
// tile's end state:
//   dA   = tril(dO V^T)                       (query x key)
//   GQ   = dO S'^T + dA Kt                    dphi_q = E GQ
//   GK   = dA^T Qt + V dS^T                   dphi_k = GK / E
//   dv   = tril(Qt Kt^T)^T dO + Kt dS
//   dB   = Qt GQ - Kt GK  (gradient of b; its reverse cumulative sum over the
//          sequence is the log-decay gradient)
//   dS_prev = diag(exp r) (dS + Qt^T dO)
//
// The decay factors E (fp32) and the tiles' log-decays r come precomputed
// from launch_gate_prep.
//
// Qt and Kt enter the GK and GQ products as bf16 pairs hi + lo.  At small
// feature-map weights phi is close to uniform, so dphi carries a large
// component shared by all features that the feature-map backward removes
// again; one bf16 rounding of Qt or Kt would leave errors of a few percent
// of what remains in dW_k and dW_q.
//
// tc_gla_dstates_kernel  reverse pass per sequence: dS of every tile (bf16
//                        copies) and the gradient of the initial state.
// tc_gla_bwd_tile_kernel the formulas above per 128-token tile, given the
//                        S' and dS copies; one persistent CTA per SM walks a
//                        contiguous run of (sequence, tile) items.  dB and dv
//                        go out in fp32; dphi_q and dphi_k in bf16, each
//                        half-row shifted by its first value (the feature
//                        map's softmax backward ignores a constant per half,
//                        and the shift takes out the part all features share).
// gate_grad_kernel       reverse cumulative sum of dB -> gate-logit gradient.
#include "common.cuh"
#include "lizard_internal.h"
#include "tc_common.cuh"
#include "tc_host.h"

namespace lz {
namespace {

using namespace tc;

constexpr int T = 128;
constexpr int D = 128;
constexpr int F = D / 2;
constexpr uint32_t TILE = kTile;
constexpr uint32_t REG = kReg;
constexpr uint32_t ST_TIMEOUT = 1u, ST_RANGE = 2u;

struct DsParams {
  CUtensorMap mq, mo;
  CUtensorMap me;              // fp32 decay factors (loads)
  const float *wq;
  const float *e32, *gate_r;   // fp32 decay factors [BH*L][D] and tile log-decays [BH][ntiles][D]
  __nv_bfloat16 *snap;      // [BH][ntiles][D][D] dS - 1 dS[0] at each tile's end (bf16)
  float *snap_r0;           // [BH][ntiles][D] row 0 of that dS (fp32)
  float *dstate_in;         // [BH][D][D] or null
  const float *dstate_out;  // [BH][D][D] gradient into the final state, or null (zero)
  uint32_t *status;
  int H, L;
  float inv_tau;
};

struct TileParams {
  CUtensorMap mq, mk, mv, mo, msp, mds;       // msp / mds: [BH*ntiles][D][D] snapshots
  CUtensorMap mw;                             // [H*2][D][F] bf16 feature-map weights (W_q, W_k per head)
  CUtensorMap mdq, mdk;                       // bf16 outputs dphi_q, dphi_k, row halves centred (TMA stores)
  CUtensorMap mdb, mdv;                       // fp32 outputs dB, dv (TMA stores)
  CUtensorMap me;                             // fp32 decay factors (loads)
  const float *e32;            // fp32 decay factors [BH*L][D]
  const float *sp_r0, *ds_r0;  // [BH*ntiles][D] row 0 of S' and of dS (the copies hold the rest)
  float *colsum;               // [BH*ntiles][D] column sums of dB per tile (out)
  uint32_t *status;
  int H, L, ntiles, BH;
  float inv_tau;
};


__device__ __forceinline__ void stage_weights(unsigned char *dst, const float *W, int h, int row) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float f[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) f[u] = W ? W[((size_t)h * D + row) * F + c * 8 + u] : 0.f;
    *reinterpret_cast<uint4 *>(dst + sw128_offset(row, c * 8)) = pack8(f);
  }
}

// ------------------------------------------------------ reverse dS pass ---
// Two warpgroups (256 threads): thread = tile row / state row `row` of its
// group; the groups take halves of the key dimensions (E, phi_q) and of the
// state's columns (copy and rescale).
constexpr int NT_DS = 256;
__global__ void __launch_bounds__(NT_DS, 1) tc_gla_dstates_kernel(const __grid_constant__ DsParams p) {
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  __shared__ float s_dec[D];
  __shared__ __align__(16) float s_row0[D];   // row 0 of dS, taken out of the bf16 copy
  __shared__ __align__(16) float s_rt[D];     // the tile's log-decays r (arrive with its loads)
  __shared__ uint64_t bar_tma, bar_m1, bar_m2;
  __shared__ uint32_t s_tmem;
  // Qt (hi) over X_q, the remainder Qt - bf16(Qt) in R_QL, dO, W_q, the
  // tile's fp32 decay factors E (four 32-column boxes)
  constexpr uint32_t R_XQ = 0, R_QL = TILE, R_O = 2 * TILE, R_W = 3 * TILE, R_E = 3 * TILE + TILE / 2;
  constexpr uint32_t C_S = 0, C_Z = 128;
  const int tid = threadIdx.x, warp = tid >> 5, wg = tid >> 7, row = tid & 127;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const int bh = blockIdx.x, h = bh % p.H;
  const uint32_t sbase = smem_u32(sm);
  const int ntiles = (p.L + T - 1) / T;
  if (warp == 0) { tmem_alloc(&s_tmem, 512); tmem_relinquish(); }
  if (tid == 0) {
    mbar_init(&bar_tma, 1);
    mbar_init(&bar_m1, 1);
    mbar_init(&bar_m2, 1);
    fence_barrier_init();
  }
  if (wg == 0) stage_weights(sm + R_W, p.wq, h, row);
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s_tmem, tl = tb + lane_off;
  {   // dS starts as the gradient flowing into the last tile's end state (the
      // final state): dstate_out, or zero; lane = key dimension, column half per group
    const float *src = p.dstate_out ? p.dstate_out + ((size_t)bh * D + row) * D : nullptr;
    for (int c = 64 * wg; c < 64 * wg + 64; c += 8) {
      uint32_t z[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) z[u] = __float_as_uint(src ? src[c + u] : 0.f);
      tmem_st8(tl + C_S + c, z);
    }
    tmem_st_wait();
  }
  const uint32_t id_z = idesc_bf16(128, 64, 0, 1);
  const uint32_t id_st = idesc_bf16(128, 128, 1, 1);
  // Tile c's loads in two parts: E and r (their places are free once Qt is
  // formed, so they go out before the dS product), then X_q and dO (free
  // once the product is done).  The barrier expects all of them at once.
  auto loads = [&](int c, bool e_r, bool xq_o) {
    if (e_r) {
      mbar_expect_tx(&bar_tma, 4 * TILE + D * 4);
      bulk_load_1d(s_rt, p.gate_r + ((size_t)bh * ntiles + c) * D, D * 4, &bar_tma);
      for (int bx = 0; bx < 4; ++bx) tma_load_3d(sm + R_E + bx * 16384, &p.me, &bar_tma, 32 * bx, c * T, bh);
    }
    if (xq_o)
      for (int r = 0; r < 2; ++r) {
        tma_load_3d(sm + R_XQ + r * REG, &p.mq, &bar_tma, 64 * r, c * T, bh);
        tma_load_3d(sm + R_O + r * REG, &p.mo, &bar_tma, 64 * r, c * T, bh);
      }
  };
  // thread 0: parity and tile of a load batch issued and not yet waited for
  // (pend -1: none), and whether its X_q / dO half is still to be issued
  int pend = -1, pend_c = 0;
  bool half = false;
  if (tid == 0 && ntiles > 0) {
    loads(ntiles - 1, true, true);
    pend = 0;
  }
  bool fail = false;
  for (int c = ntiles - 1; c >= 0; --c) {
    const uint32_t par = (ntiles - 1 - c) & 1;
    bool ok = mbar_wait(&bar_tma, par, p.status, ST_TIMEOUT);
    if (__syncthreads_or(!ok)) { fail = true; break; }
    pend = -1;
    if (tid == 0) {
      tc_fence_after();
      for (int s = 0; s < 8; ++s) mma_ss(tb + C_Z, desc_k(sbase + R_XQ, s), desc_mn(sbase + R_W, s), id_z, s > 0);
      mma_commit(&bar_m1);
    }
    // copy of dS (the gradient into this tile's end state), column half per
    // group, as dS - 1 dS[0] in bf16 with row 0 in fp32 (the rows share a
    // large common part that a plain bf16 copy would round element by element)
    {
      const size_t tile = (size_t)bh * ntiles + c;
      if ((warp & 3) == 0) {   // the warps holding TMEM lane 0: row 0 to shared memory
        for (int ch = 2 * wg; ch < 2 * wg + 2; ++ch) {
          float v[32];
          tmem_ld32(tl + C_S + ch * 32, v);
          if (row == 0)
#pragma unroll
            for (int u = 0; u < 32; ++u) s_row0[ch * 32 + u] = v[u];
        }
      }
      __syncthreads();
      __nv_bfloat16 *dst = p.snap + (tile * D + row) * D;
      for (int ch = 2 * wg; ch < 2 * wg + 2; ++ch) {
        float v[32];
        tmem_ld32(tl + C_S + ch * 32, v);
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] -= s_row0[ch * 32 + u];
#pragma unroll
        for (int u = 0; u < 32; u += 8) *reinterpret_cast<uint4 *>(dst + ch * 32 + u) = pack8(v + u);
      }
      if (tid < D) p.snap_r0[tile * D + tid] = s_row0[tid];
    }
    // the tile's decay exp(r)
    if (wg == 0) s_dec[row] = __expf(s_rt[row]);
    ok = mbar_wait(&bar_m1, par, p.status, ST_TIMEOUT);
    tc_fence_after();
    {   // Qt = phi_q E into shared memory over X_q (row = token), dimension half per group
      float ph[F];
      const float sc = feature_half(tl + C_Z, wg, ph);
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        float q16[16];
#pragma unroll
        for (int u = 0; u < 16; u += 4) {   // E of dimensions 64 wg + 16 c16 + u .. (zero past L)
          const float4 E = *f32_stage_ptr(sm + R_E, row, 64 * wg + 16 * c16 + u);
          q16[u] = ph[16 * c16 + u] * sc * E.x;
          q16[u + 1] = ph[16 * c16 + u + 1] * sc * E.y;
          q16[u + 2] = ph[16 * c16 + u + 2] * sc * E.z;
          q16[u + 3] = ph[16 * c16 + u + 3] * sc * E.w;
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint4 hi, lo;
          split8(q16 + 8 * hh, hi, lo);
          *chunk_ptr(sm, R_XQ, row, 8 * wg + 2 * c16 + hh) = hi;
          *chunk_ptr(sm, R_QL, row, 8 * wg + 2 * c16 + hh) = lo;
        }
      }
    }
    fence_proxy_async();
    tc_fence_before();
    if (__syncthreads_or(!ok)) { fail = true; break; }
    if (tid == 0) {   // dS += (Qt hi + lo)^T dO
      tc_fence_after();
      for (int s = 0; s < 8; ++s) mma_ss(tb + C_S, desc_mn(sbase + R_XQ, s), desc_mn(sbase + R_O, s), id_st, 1);
      for (int s = 0; s < 8; ++s) mma_ss(tb + C_S, desc_mn(sbase + R_QL, s), desc_mn(sbase + R_O, s), id_st, 1);
      mma_commit(&bar_m2);
      if (c > 0) {   // E and r were read before the barrier above
        loads(c - 1, true, false);
        pend = (int)(par ^ 1u);
        pend_c = c - 1;
        half = true;
      }
    }
    ok = mbar_wait(&bar_m2, par, p.status, ST_TIMEOUT);
    if (__syncthreads_or(!ok)) { fail = true; break; }
    tc_fence_after();
    if (tid == 0 && c > 0) {
      loads(c - 1, false, true);
      half = false;
    }
    {   // dS_prev = diag(exp r) (dS + Qt^T dO), column half per group
      const float dec = s_dec[row];
      for (int ch = 4 * wg; ch < 4 * wg + 4; ++ch) {
        float v[16];
        tmem_ld16(tl + C_S + ch * 16, v);
        uint32_t r[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) r[u] = __float_as_uint(v[u] * dec);
        tmem_st8(tl + C_S + ch * 16, r);
#pragma unroll
        for (int u = 0; u < 8; ++u) r[u] = __float_as_uint(v[8 + u] * dec);
        tmem_st8(tl + C_S + ch * 16 + 8, r);
      }
      tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
  }
  if (fail && tid == 0 && pend >= 0) {
    // let the loads already issued land before the shared memory is released
    // (a half-issued batch is completed first, so the barrier's wait can end)
    if (half) loads(pend_c, false, true);
    mbar_wait(&bar_tma, (uint32_t)pend, nullptr, 0, 1u << 16);
  }
  if (!fail && p.dstate_in) {
    tc_fence_after();
    float *dst = p.dstate_in + ((size_t)bh * D + row) * D;
    for (int ch = 2 * wg; ch < 2 * wg + 2; ++ch) {
      float v[32];
      tmem_ld32(tl + C_S + ch * 32, v);
#pragma unroll
      for (int u = 0; u < 32; u += 4)
        *reinterpret_cast<float4 *>(dst + ch * 32 + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 512);
}

// ------------------------------------------------------------ per tile ----
// Two warpgroups (256 threads): each thread owns tile row `row` (TMEM lane)
// in its group; the groups split the row work by columns (dimension halves
// for E, phi, dphi and dB; one mask each for dA and dA^T).
constexpr int NT_TILE = 256;
__global__ void __launch_bounds__(NT_TILE, 1) tc_gla_bwd_tile_kernel(const __grid_constant__ TileParams p) {
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bars[9];
  __shared__ uint32_t s_tmem;
  // Per row: dO . S'[0], V . dS[0], sum_i Kt[i] -- the rank-one parts of GQ,
  // GK and dv that the copies (S' - 1 S'[0], dS - 1 dS[0]) leave out.  Before
  // the sums are formed, and again once they are read, the same storage holds
  // the row-0 vectors S'[0] (floats 0..127) and dS[0] (128..255), which every
  // row reads.
  __shared__ __align__(16) float s_r1[3][T];
  float *s_row0 = &s_r1[0][0];
  // X_q -> Qt (hi), X_k -> Kt (hi), V, dO, [W_q | W_k] -> S' -> dS, Qt (lo), Kt (lo)
  constexpr uint32_t R_XQ = 0, R_XK = TILE, R_V = 2 * TILE, R_O = 3 * TILE, R_W = 4 * TILE, R_QL = 5 * TILE,
                     R_KL = 6 * TILE;
  // TMEM, in order of use:
  //   dA [128,256) dA^T [256,384) Zq [384,448) Zk [448,512)
  //   dA^ [0,64) dA^T^ [64,128) ; GQ [256,384) (its dO S'^T part while the
  //   rows form Qt and Kt) ; E (fp32, while Qt and Kt are formed) [128,256)
  //   A^T [384,512) ; A^T^ (bf16) [128,192) ; GK [384,512) ; DV [0,128)
  constexpr uint32_t C_DAH = 0, C_DATH = 64, C_DV = 0, C_DA = 128, C_E = 128, C_ATH = 128, C_DAT = 256,
                     C_AT = 384, C_GQ = 256, C_ZQ = 384, C_ZK = 448, C_GK = 384;
  const int tid = threadIdx.x, warp = tid >> 5, wg = tid >> 7, row = tid & 127;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t sbase = smem_u32(sm);
  // Persistent: CTA b walks the contiguous run [w0, w1) of (sequence, tile)
  // items, item w = tile w % ntiles of sequence w / ntiles.  The next item's
  // inputs go out as this item frees their places: the weights once the last
  // products are done, V and dO once the dB store has read its staging, X_q
  // and X_k after the dphi stores, the decay factors after the dv store.
  const int nwork = p.ntiles * p.BH;
  const int w0 = (int)((long long)blockIdx.x * nwork / gridDim.x);
  const int w1 = (int)((long long)(blockIdx.x + 1) * nwork / gridDim.x);
  // part 0: weights (arms the barrier), 1: X_q, 2: V, dO, 3: X_k
  auto item_loads = [&](int w, int part) {
    const int lbh = w / p.ntiles, lt0 = (w % p.ntiles) * T;
    if (part == 0) mbar_expect_tx(&bars[0], 5 * TILE);
    for (int r = 0; r < 2; ++r) {
      if (part == 0) tma_load_3d(sm + R_W + r * REG, &p.mw, &bars[0], 0, 0, 2 * (lbh % p.H) + r);
      if (part == 1) tma_load_3d(sm + R_XQ + r * REG, &p.mq, &bars[0], 64 * r, lt0, lbh);
      if (part == 3) tma_load_3d(sm + R_XK + r * REG, &p.mk, &bars[0], 64 * r, lt0, lbh);
      if (part == 2) {
        tma_load_3d(sm + R_V + r * REG, &p.mv, &bars[0], 64 * r, lt0, lbh);
        tma_load_3d(sm + R_O + r * REG, &p.mo, &bars[0], 64 * r, lt0, lbh);
      }
    }
  };
  // the fp32 decay factors of item w, four 32-column boxes: dimensions 0..63
  // over Qt lo, 64..127 over Kt lo (free from the item's end until its
  // rows have moved them to TMEM); rows past L read as zero
  auto e_tma = [&](int w) {
    const int lbh = w / p.ntiles, lt0 = (w % p.ntiles) * T;
    mbar_expect_tx(&bars[8], 2 * TILE);
    for (int bx = 0; bx < 4; ++bx)
      tma_load_3d(sm + (bx < 2 ? R_QL : R_KL) + (bx & 1) * 16384, &p.me, &bars[8], 32 * bx, lt0, lbh);
  };
  if (warp == 0) { tmem_alloc(&s_tmem, 512); tmem_relinquish(); }
  if (tid == 0) {
    for (int i = 0; i < 9; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
    if (w0 < w1) {
      item_loads(w0, 0);
      item_loads(w0, 1);
      item_loads(w0, 2);
      item_loads(w0, 3);
      e_tma(w0);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s_tmem, tl = tb + lane_off;
  const uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
  const uint32_t id_mn = idesc_bf16(128, 128, 0, 1);
  const uint32_t id_z = idesc_bf16(128, 64, 0, 1);
  // copies in flight when a wait gives up (tid 0's view): the parity of an
  // armed phase of bars[0] and of bars[8], and whether the S' / dS loads of
  // this item are out
  int pend0 = w0 < w1 ? 0 : -1, pend_e = w0 < w1 ? 0 : -1;
  bool pend_sp = false, pend_ds = false;
  bool ok = true;
  uint32_t par = 0;
  for (int w = w0, itn = 0; w < w1; ++w, ++itn) {
  par = (uint32_t)itn & 1u;
  const int bh = w / p.ntiles, c = w % p.ntiles, t0 = c * T, tq = t0 + row;
  const bool valid = tq < p.L;
  const int snap_idx = w;   // == bh * ntiles + c
  const bool more = w + 1 < w1;
  float r1[3];   // this half's dO . S'[0], V . dS[0], sum Kt
  if (tid < 64) {   // the row-0 vectors, while the tile arrives
    const float *src = tid < 32 ? p.sp_r0 + (size_t)snap_idx * D + 4 * tid : p.ds_r0 + (size_t)snap_idx * D + 4 * (tid - 32);
    *reinterpret_cast<float4 *>(s_row0 + 4 * tid) = __ldg(reinterpret_cast<const float4 *>(src));
  }
  ok = mbar_wait(&bars[0], par, p.status, ST_TIMEOUT);
  if (__syncthreads_or(!ok)) { ok = false; goto done; }
  pend0 = -1;
  // 1. dA = dO V^T, dA^T = V dO^T, Zq = X_q W_q, Zk = X_k W_k
  if (tid == 0) {
    tc_fence_after();
    for (int s = 0; s < 8; ++s) mma_ss(tb + C_DA, desc_k(sbase + R_O, s), desc_k(sbase + R_V, s), id_kk, s > 0);
    for (int s = 0; s < 8; ++s) mma_ss(tb + C_DAT, desc_k(sbase + R_V, s), desc_k(sbase + R_O, s), id_kk, s > 0);
    for (int s = 0; s < 8; ++s) mma_ss(tb + C_ZQ, desc_k(sbase + R_XQ, s), desc_mn(sbase + R_W, s), id_z, s > 0);
    for (int s = 0; s < 8; ++s) mma_ss(tb + C_ZK, desc_k(sbase + R_XK, s), desc_mn(sbase + R_W + REG, s), id_z, s > 0);
    mma_commit(&bars[1]);
  }
  ok = mbar_wait(&bars[1], par, p.status, ST_TIMEOUT);
  if (__syncthreads_or(!ok)) { ok = false; goto done; }
  tc_fence_after();
  if (tid == 0) {   // the weights are consumed: S' goes into their place
    pend_sp = true;
    mbar_expect_tx(&bars[2], TILE);
    tma_load_3d(sm + R_W, &p.msp, &bars[2], 0, 0, snap_idx);
    tma_load_3d(sm + R_W + REG, &p.msp, &bars[2], 64, 0, snap_idx);
  }
  // 2. group 0: masked dA (row = query, key j <= row); group 1: masked dA^T
  //    (row = key, query j >= row); packed bf16 into [0,128)
  {
    const uint32_t src = wg == 0 ? C_DA : C_DAT, dst = wg == 0 ? C_DAH : C_DATH;
#pragma unroll 1
    for (int c2 = 0; c2 < 2; ++c2) {
      float dav[2][32];
      tmem_ld32x2(tl + src + c2 * 64, tl + src + c2 * 64 + 32, dav[0], dav[1]);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int ch = 2 * c2 + h;
        const float *v = dav[h];
        uint32_t a[16];
#pragma unroll
        for (int u = 0; u < 32; u += 2) {
          const int j = ch * 32 + u;
          const bool k0 = wg == 0 ? j <= row : j >= row, k1 = wg == 0 ? j + 1 <= row : j + 1 >= row;
          a[u / 2] = pack_bf16(k0 ? v[u] : 0.f, k1 ? v[u + 1] : 0.f);
        }
        tmem_st8(tl + dst + ch * 16, a);
        tmem_st8(tl + dst + ch * 16 + 8, a + 8);
      }
    }
  }
  tmem_st_wait();
  tc_fence_before();
  __syncthreads();   // dA read out before E overwrites its columns
  tc_fence_after();
  // 3a. GQ = dO S'^T (the columns of dA^T are spent): it runs while the rows
  //     form Qt and Kt, and once it is done the dS copy can take S's place
  bool t0ok = true;   // tid 0: its own waits below succeeded
  if (tid == 0) {
    t0ok = mbar_wait(&bars[2], par, p.status, ST_TIMEOUT);
    if (t0ok) {
      pend_sp = false;
      tc_fence_after();
      for (int s = 0; s < 8; ++s) mma_ss(tb + C_GQ, desc_k(sbase + R_O, s), desc_k(sbase + R_W, s), id_kk, s > 0);
      mma_commit(&bars[4]);
    }
  }
  //    E in fp32 (dimensions 64 wg .., from shared memory) into TMEM, then
  //    Qt = phi_q E and Kt = phi_k / E for the same dimensions (rows past L:
  //    Kt = 0), each as a bf16 pair hi + lo
  ok = mbar_wait(&bars[8], par, p.status, ST_TIMEOUT);
  if (__syncthreads_or(!ok)) { ok = false; goto done; }
  pend_e = -1;
  {
    const unsigned char *es = sm + (wg == 0 ? R_QL : R_KL);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float4 a = *f32_stage_ptr(const_cast<unsigned char *>(es), row, 8 * u);
      const float4 b = *f32_stage_ptr(const_cast<unsigned char *>(es), row, 8 * u + 4);
      const uint32_t r8[8] = {__float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(a.z), __float_as_uint(a.w),
                              __float_as_uint(b.x), __float_as_uint(b.y), __float_as_uint(b.z), __float_as_uint(b.w)};
      tmem_st8(tl + C_E + 64 * wg + 8 * u, r8);
    }
  }
  tmem_st_wait();
  __syncthreads();   // E read out of Qt lo | Kt lo before they are written
  r1[0] = r1[1] = r1[2] = 0.f;
  {
    const float *ms = s_row0 + 64 * wg, *md = s_row0 + D + 64 * wg;
#pragma unroll 2
    for (int ch = 0; ch < 8; ++ch) {
      float o8[8], v8[8];
      unpack8(*chunk_ptr(sm, R_O, row, 8 * wg + ch), o8);
      unpack8(*chunk_ptr(sm, R_V, row, 8 * wg + ch), v8);
      const float4 a0 = *reinterpret_cast<const float4 *>(ms + 8 * ch),
                   a1 = *reinterpret_cast<const float4 *>(ms + 8 * ch + 4);
      const float4 b0 = *reinterpret_cast<const float4 *>(md + 8 * ch),
                   b1 = *reinterpret_cast<const float4 *>(md + 8 * ch + 4);
      r1[0] += o8[0] * a0.x + o8[1] * a0.y + o8[2] * a0.z + o8[3] * a0.w + o8[4] * a1.x + o8[5] * a1.y +
               o8[6] * a1.z + o8[7] * a1.w;
      r1[1] += v8[0] * b0.x + v8[1] * b0.y + v8[2] * b0.z + v8[3] * b0.w + v8[4] * b1.x + v8[5] * b1.y +
               v8[6] * b1.z + v8[7] * b1.w;
    }
  }
#pragma unroll 1
  for (int m = 0; m < 2; ++m) {
    float ph[F];
    const float s = feature_half(tl + (m == 0 ? C_ZQ : C_ZK), wg, ph);
    const uint32_t reg = m == 0 ? R_XQ : R_XK, reg_lo = m == 0 ? R_QL : R_KL;
#pragma unroll
    for (int c16 = 0; c16 < 4; ++c16) {
      float E[16], x16[16];
      tmem_ld16(tl + C_E + 64 * wg + 16 * c16, E);
#pragma unroll
      for (int u = 0; u < 16; ++u)
        x16[u] = m == 0 ? ph[16 * c16 + u] * s * E[u] : (valid ? __fdividef(ph[16 * c16 + u] * s, E[u]) : 0.f);
      if (m == 1)
#pragma unroll
        for (int u = 0; u < 16; ++u) r1[2] += x16[u];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint4 hi, lo;
        split8(x16 + 8 * hh, hi, lo);
        *chunk_ptr(sm, reg, row, 8 * wg + 2 * c16 + hh) = hi;
        *chunk_ptr(sm, reg_lo, row, 8 * wg + 2 * c16 + hh) = lo;
      }
    }
  }
  fence_proxy_async();
  tc_fence_before();
  // every row is done with the row-0 vectors (s_r1 takes the sums) and with Zq, Zk
  if (__syncthreads_or(!t0ok)) { ok = false; goto done; }
  if (wg == 1)
#pragma unroll
    for (int k = 0; k < 3; ++k) s_r1[k][row] = r1[k];
  // 3b. A^T = Kt Qt^T (rows = keys) over Zq, Zk; the dS copy replaces S'
  if (tid == 0) {
    tc_fence_after();
    for (int s = 0; s < 8; ++s) mma_ss(tb + C_AT, desc_k(sbase + R_XK, s), desc_k(sbase + R_XQ, s), id_kk, s > 0);
    mma_commit(&bars[3]);
    t0ok = mbar_wait(&bars[4], par, p.status, ST_TIMEOUT);
    if (t0ok) {
      pend_ds = true;
      mbar_expect_tx(&bars[6], TILE);
      tma_load_3d(sm + R_W, &p.mds, &bars[6], 0, 0, snap_idx);
      tma_load_3d(sm + R_W + REG, &p.mds, &bars[6], 64, 0, snap_idx);
    }
  }
  ok = mbar_wait(&bars[3], par, p.status, ST_TIMEOUT);
  if (__syncthreads_or(!ok || !t0ok)) { ok = false; goto done; }
  if (wg == 0)   // the two halves' sums meet; read after the next barrier
#pragma unroll
    for (int k = 0; k < 3; ++k) s_r1[k][row] += r1[k];
  tc_fence_after();
  //    A^T^ = A^T masked to queries j >= key row, packed bf16 into TMEM over
  //    the spent E columns, 64 query columns per group
  float atv[2][32];
  tmem_ld32x2(tl + C_AT + 64 * wg, tl + C_AT + 64 * wg + 32, atv[0], atv[1]);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int ch = 2 * wg + h;
    const float *v = atv[h];
    uint32_t a[16];
#pragma unroll
    for (int u = 0; u < 32; u += 2) {
      const int j = ch * 32 + u;
      a[u / 2] = pack_bf16(j >= row ? v[u] : 0.f, j + 1 >= row ? v[u + 1] : 0.f);
    }
    tmem_st8(tl + C_ATH + ch * 16, a);
    tmem_st8(tl + C_ATH + ch * 16 + 8, a + 8);
  }
  tmem_st_wait();
  tc_fence_before();
  __syncthreads();   // A^T read out before GK overwrites its columns
  // 4a. GQ += dA^ (Kt hi + lo) ;  GK = dA^T^ (Qt hi + lo)
  if (tid == 0) {
    tc_fence_after();
    for (int s = 0; s < 8; ++s) mma_ts(tb + C_GQ, tb + C_DAH + s * 8, desc_mn(sbase + R_XK, s), id_mn, 1);
    for (int s = 0; s < 8; ++s) mma_ts(tb + C_GQ, tb + C_DAH + s * 8, desc_mn(sbase + R_KL, s), id_mn, 1);
    for (int s = 0; s < 8; ++s) mma_ts(tb + C_GK, tb + C_DATH + s * 8, desc_mn(sbase + R_XQ, s), id_mn, s > 0);
    for (int s = 0; s < 8; ++s) mma_ts(tb + C_GK, tb + C_DATH + s * 8, desc_mn(sbase + R_QL, s), id_mn, 1);
    mma_commit(&bars[5]);
  }
  ok = mbar_wait(&bars[5], par, p.status, ST_TIMEOUT);
  ok &= mbar_wait(&bars[6], par, p.status, ST_TIMEOUT);
  if (__syncthreads_or(!ok)) { ok = false; goto done; }
  pend_ds = false;
  // 4b. GK += V dS^T ;  DV = A^T^ dO + Kt dS
  if (tid == 0) {
    tc_fence_after();
    for (int s = 0; s < 8; ++s) mma_ss(tb + C_GK, desc_k(sbase + R_V, s), desc_k(sbase + R_W, s), id_kk, 1);
    for (int s = 0; s < 8; ++s) mma_ts(tb + C_DV, tb + C_ATH + s * 8, desc_mn(sbase + R_O, s), id_mn, s > 0);
    for (int s = 0; s < 8; ++s) mma_ss(tb + C_DV, desc_k(sbase + R_XK, s), desc_mn(sbase + R_W, s), id_mn, 1);
    mma_commit(&bars[7]);
  }
  {
    // 5. rows, dimension half per group, staged as fp32 tiles in the spent
    //    regions and written with TMA stores (rows past L are clipped by the
    //    maps): dB = Qt GQ - Kt GK (Qt, Kt as hi + lo, so that dB matches the
    //    products) over V | dO; then dphi_q = E GQ (bf16) over Qt hi and
    //    dphi_k = GK / E over Kt hi; then dv over Qt lo | Kt lo.  E (fp32) is
    //    read again from global memory, its loads in flight while the last
    //    products run.
    float4 e4[16];
    const float *er = p.e32 + ((size_t)bh * p.L + (valid ? tq : 0)) * D + 64 * wg;
#pragma unroll
    for (int u = 0; u < 16; ++u)
      e4[u] = valid ? *reinterpret_cast<const float4 *>(er + 4 * u) : make_float4(1.f, 1.f, 1.f, 1.f);
    // dS[0] for the dv pass, back into shared memory once the sums are read
    const float4 ds0 = tid < 32 ? __ldg(reinterpret_cast<const float4 *>(p.ds_r0 + (size_t)snap_idx * D + 4 * tid))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
    ok = mbar_wait(&bars[7], par, p.status, ST_TIMEOUT);
    if (__syncthreads_or(!ok)) { ok = false; goto done; }
    tc_fence_after();
    if (tid == 0 && more) {   // the products are done with the weights' place: the next item's weights
      pend0 = (int)(par ^ 1u);
      item_loads(w + 1, 0);
    }
    unsigned char *st0 = sm + R_V;
    // rank-one parts of GQ and GK left out of the S' and dS copies
    const float cq = s_r1[0][row], ck = s_r1[1][row], kap = s_r1[2][row];
#pragma unroll 1
    for (int c16 = 4 * wg; c16 < 4 * wg + 4; ++c16) {
      float gq[16], gk[16], q16[16], k16[16], lo[16];
      tmem_ld16x2(tl + C_GQ + c16 * 16, tl + C_GK + c16 * 16, gq, gk);
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        gq[u] += cq;
        gk[u] += ck;
      }

      unpack8(*chunk_ptr(sm, R_XQ, row, 2 * c16), q16);
      unpack8(*chunk_ptr(sm, R_XQ, row, 2 * c16 + 1), q16 + 8);
      unpack8(*chunk_ptr(sm, R_QL, row, 2 * c16), lo);
      unpack8(*chunk_ptr(sm, R_QL, row, 2 * c16 + 1), lo + 8);
#pragma unroll
      for (int u = 0; u < 16; ++u) q16[u] += lo[u];
      unpack8(*chunk_ptr(sm, R_XK, row, 2 * c16), k16);
      unpack8(*chunk_ptr(sm, R_XK, row, 2 * c16 + 1), k16 + 8);
      unpack8(*chunk_ptr(sm, R_KL, row, 2 * c16), lo);
      unpack8(*chunk_ptr(sm, R_KL, row, 2 * c16 + 1), lo + 8);
#pragma unroll
      for (int u = 0; u < 16; ++u) k16[u] += lo[u];
#pragma unroll
      for (int u = 0; u < 16; u += 4)
        *f32_stage_ptr(st0, row, c16 * 16 + u) =
            make_float4(q16[u] * gq[u] - k16[u] * gk[u], q16[u + 1] * gq[u + 1] - k16[u + 1] * gk[u + 1],
                        q16[u + 2] * gq[u + 2] - k16[u + 2] * gk[u + 2], q16[u + 3] * gq[u + 3] - k16[u + 3] * gk[u + 3]);
    }
    fence_proxy_async();
    __syncthreads();   // also: every Qt / Kt read is done before their regions are reused
    if (tid == 0) {
      for (int bx = 0; bx < 4; ++bx) tma_store_3d(&p.mdb, st0 + bx * 16384, 32 * bx, t0, bh);
      bulk_commit();
    }
    if (tid < 32) *reinterpret_cast<float4 *>(s_row0 + D + 4 * tid) = ds0;   // read after two barriers
    {   // the tile's column sums of dB (the gate gradient's carry from later
        // tiles): thread = column, half the rows per group, into the free
        // s_r1[0] | s_r1[2] (read after the next barrier)
      const int c = tid & 127, b = c >> 5, jj = (c & 31) >> 2;
      const unsigned char *col = st0 + b * 16384 + (c & 3) * 4;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int r = 64 * wg; r < 64 * wg + 64; ++r)
        acc[r & 3] += *reinterpret_cast<const float *>(col + r * 128 + ((jj ^ (r & 7)) << 4));
      s_r1[2 * wg][c] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    }
    // dphi_q - c_q (bf16) over Qt hi, dphi_k - c_k over Kt hi, one 32 KB
    // swizzled bf16 tile each, c the half-row's first value: a constant added
    // to one half of a row leaves the feature map's softmax backward
    // unchanged, so the finish pass reads them as they are, and taking out
    // the part all features share keeps the per-feature differences that the
    // backward uses at full bf16 precision
    float mq = 0.f, mk = 0.f;
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
      const int c16 = 4 * wg + k4;
      float gq[16], gk[16];
      tmem_ld16x2(tl + C_GQ + c16 * 16, tl + C_GK + c16 * 16, gq, gk);
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        gq[u] += cq;
        gk[u] += ck;
      }
      if (k4 == 0) {
        mq = e4[0].x * gq[0];
        mk = __fdividef(gk[0], e4[0].x);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 E = e4[4 * k4 + u];
        gq[4 * u] = E.x * gq[4 * u] - mq;
        gq[4 * u + 1] = E.y * gq[4 * u + 1] - mq;
        gq[4 * u + 2] = E.z * gq[4 * u + 2] - mq;
        gq[4 * u + 3] = E.w * gq[4 * u + 3] - mq;
        gk[4 * u] = __fdividef(gk[4 * u], E.x) - mk;
        gk[4 * u + 1] = __fdividef(gk[4 * u + 1], E.y) - mk;
        gk[4 * u + 2] = __fdividef(gk[4 * u + 2], E.z) - mk;
        gk[4 * u + 3] = __fdividef(gk[4 * u + 3], E.w) - mk;
      }
      *chunk_ptr(sm, R_XQ, row, 2 * c16) = pack8(gq);
      *chunk_ptr(sm, R_XQ, row, 2 * c16 + 1) = pack8(gq + 8);
      *chunk_ptr(sm, R_XK, row, 2 * c16) = pack8(gk);
      *chunk_ptr(sm, R_XK, row, 2 * c16 + 1) = pack8(gk + 8);
    }
    fence_proxy_async();
    __syncthreads();
    if (tid == 0) {
      for (int r = 0; r < 2; ++r) {
        tma_store_3d(&p.mdq, sm + R_XQ + r * REG, 64 * r, t0, bh);
        tma_store_3d(&p.mdk, sm + R_XK + r * REG, 64 * r, t0, bh);
      }
      bulk_commit();
    }
    if (tid < D) p.colsum[(size_t)w * D + tid] = s_r1[0][tid] + s_r1[2][tid];
    // dv, staged in the spent Qt lo | Kt lo regions (group wg's two 32-column
    // boxes in one of them), so that it need not wait for the dB store
    const float *md = s_row0 + D;
    unsigned char *st_dv = sm + (wg == 0 ? R_QL : R_KL);
    float dvv[2][32];
    tmem_ld32x2(tl + C_DV + 64 * wg, tl + C_DV + 64 * wg + 32, dvv[0], dvv[1]);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int ch = 2 * wg + h;
      const float *dv = dvv[h];
#pragma unroll
      for (int u = 0; u < 32; u += 4) {   // + (sum_i Kt[i]) dS[0]
        const float4 m4 = *reinterpret_cast<const float4 *>(md + ch * 32 + u);
        *f32_stage_ptr(st_dv, row, h * 32 + u) = make_float4(fmaf(kap, m4.x, dv[u]), fmaf(kap, m4.y, dv[u + 1]),
                                                             fmaf(kap, m4.z, dv[u + 2]), fmaf(kap, m4.w, dv[u + 3]));
      }
    }
    fence_proxy_async();
    __syncthreads();
    if (tid == 0) {
      for (int bx = 0; bx < 4; ++bx)
        tma_store_3d(&p.mdv, sm + (bx < 2 ? R_QL : R_KL) + (bx & 1) * 16384, 32 * bx, t0, bh);
      bulk_commit();
      if (more) {   // the next item's tiles, each as soon as its place has been read out
        bulk_wait_read_n<2>();   // dB out of V | dO
        item_loads(w + 1, 2);
        bulk_wait_read_n<1>();   // dphi out of Qt hi | Kt hi
        item_loads(w + 1, 1);
        item_loads(w + 1, 3);
        bulk_wait_read();        // dv out of Qt lo | Kt lo
        pend_e = (int)(par ^ 1u);
        e_tma(w + 1);            // over Qt lo | Kt lo, both read out by now
      }
    }
  }
  tc_fence_before();
  __syncthreads();   // this item's TMEM and shared-memory reads are done
  }
done:
  if (tid == 0) {
    bulk_wait_all();   // this CTA's stores are complete (and have read their staging)
    if (!ok) {         // a wait gave up: let the copies still in flight land first
      if (pend0 >= 0) mbar_wait(&bars[0], (uint32_t)pend0, nullptr, 0, 1u << 16);
      if (pend_e >= 0) mbar_wait(&bars[8], (uint32_t)pend_e, nullptr, 0, 1u << 16);
      if (pend_sp) mbar_wait(&bars[2], par, nullptr, 0, 1u << 16);
      if (pend_ds) mbar_wait(&bars[6], par, nullptr, 0, 1u << 16);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(s_tmem, 512);
}

// ------------------------------------------------------- gate gradient ----
// dg_t = dlogsigmoid(g_t) / tau * sum_{s >= t} dB_s, per (sequence, key
// dimension), in one pass over dB: the tile kernel leaves each tile's column
// sums of dB, so the part of the sum beyond a tile (plus the final state's
// share) is known before the tile is walked.  One CTA per (sequence, 64
// dimensions): warp w walks tiles w, w + 8, ... backwards (lane = two
// dimensions, eight token rows in flight).
constexpr int kGateWarps = 8;
__global__ void __launch_bounds__(256) gate_grad_kernel(const float *__restrict__ dB,
                                                       const __nv_bfloat16 *__restrict__ g, float *__restrict__ dg,
                                                       int L, float inv_tau, const float *kap, const float *colsum) {
  // lane = two adjacent dimensions: a warp reads whole 128-byte lines of g
  // (32 dimensions per lane left half lines) and 256-byte rows of dB and dg
  const int bh = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int i = blockIdx.y * 64 + 2 * lane;
  const int ntiles = (L + T - 1) / T;
  const size_t base = (size_t)bh * L * D + i;
  const float *cs = colsum + (size_t)bh * ntiles * D + i;
  // the sum starts with the final state's share (an incoming final-state gradient)
  float2 k0 = make_float2(0.f, 0.f);
  if (kap) {
    const float2 a = *reinterpret_cast<const float2 *>(kap + (size_t)bh * 2 * D + i);
    const float2 b = *reinterpret_cast<const float2 *>(kap + ((size_t)bh * 2 + 1) * D + i);
    k0 = make_float2(a.x + b.x, a.y + b.y);
  }
  for (int c = warp; c < ntiles; c += kGateWarps) {
    float2 later[4] = {k0, make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    for (int c2 = c + 1; c2 < ntiles; ++c2) {
      const float2 v = *reinterpret_cast<const float2 *>(cs + (size_t)c2 * D);
      later[c2 & 3].x += v.x;
      later[c2 & 3].y += v.y;
    }
    float cx = (later[0].x + later[1].x) + (later[2].x + later[3].x);
    float cy = (later[0].y + later[1].y) + (later[2].y + later[3].y);
    const int ta = c * T, tz = min(L, ta + T);
    int t = tz - 1;
    for (; t - 7 >= ta; t -= 8) {
      float2 b[8], gv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        b[u] = *reinterpret_cast<const float2 *>(dB + base + (size_t)(t - u) * D);
        gv[u] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(g + base + (size_t)(t - u) * D));
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        cx += b[u].x;
        cy += b[u].y;
        *reinterpret_cast<float2 *>(dg + base + (size_t)(t - u) * D) =
            make_float2(cx * dlogsigmoid(gv[u].x) * inv_tau, cy * dlogsigmoid(gv[u].y) * inv_tau);
      }
    }
    for (; t >= ta; --t) {
      const float2 b = *reinterpret_cast<const float2 *>(dB + base + (size_t)t * D);
      const float2 gv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(g + base + (size_t)t * D));
      cx += b.x;
      cy += b.y;
      *reinterpret_cast<float2 *>(dg + base + (size_t)t * D) =
          make_float2(cx * dlogsigmoid(gv.x) * inv_tau, cy * dlogsigmoid(gv.y) * inv_tau);
    }
  }
}

constexpr int kGateSeg = 8;   // token segments (one per warp) of the scalar-gate kernel

// Scalar gate (one logit per token and head, shared by every key dimension):
// dg_t = dlogsigmoid(g_t) / tau * sum_{s >= t} sum_i dB_s[i].  One CTA per
// sequence; warp w owns token segment w of 8.  Pass 1: each warp reduces
// its rows over the 128 dimensions (lane = 4 dimensions, one float4 each,
// 8 rows in flight) and parks the row sums in dg; pass 2 walks the segment
// backwards 32 rows at a time with a warp-wide suffix scan, starting from
// the later segments' totals.
__global__ void __launch_bounds__(256) gate_grad_scalar_kernel(const float *dB, const __nv_bfloat16 *g, float *dg,
                                                              int L, float inv_tau, const float *kap) {
  __shared__ float s_tot[kGateSeg];
  const int bh = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = (L + kGateSeg - 1) / kGateSeg;
  const int ta = min(L, warp * seg), tz = min(L, ta + seg);
  const float *src = dB + (size_t)bh * L * D + lane * 4;
  float *dst = dg + (size_t)bh * L;
  float total = 0.f;
  for (int t = ta; t < tz; t += 8) {
    float r[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      r[u] = 0.f;
      if (t + u < tz) {
        const float4 x = *reinterpret_cast<const float4 *>(src + (size_t)(t + u) * D);
        r[u] = (x.x + x.y) + (x.z + x.w);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int u = 0; u < 8; ++u) r[u] += __shfl_xor_sync(0xffffffffu, r[u], o);
    if (lane < 8 && t + lane < tz) {
      float mine = r[0];
#pragma unroll
      for (int u = 1; u < 8; ++u) mine = lane == u ? r[u] : mine;
      dst[t + lane] = mine;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) total += t + u < tz ? r[u] : 0.f;
  }
  if (lane == 0) s_tot[warp] = total;
  __syncthreads();   // also orders each warp's parked row sums before pass 2
  float carry = 0.f;   // starts with the final state's share, summed over the dimensions
  if (kap) {
    const float *k2 = kap + (size_t)bh * 2 * D;
#pragma unroll
    for (int u = 0; u < 8; ++u) carry += k2[lane * 8 + u];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) carry += __shfl_xor_sync(0xffffffffu, carry, o);
  }
  for (int w = warp + 1; w < kGateSeg; ++w) carry += s_tot[w];
  for (int hi = tz - 1; hi >= ta; hi -= 32) {
    const int t = hi - lane;                   // lane 0 takes the latest row
    const bool in = t >= ta;
    float x = in ? dst[t] : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {         // suffix sum toward lane 0
      const float y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (in) dst[t] = (carry + x) * dlogsigmoid(__bfloat162float(g[(size_t)bh * L + t])) * inv_tau;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
}

// bf16 copies of the feature-map weights, [H][2][D][F] (W_q then W_k of
// each head), for the tile kernel's TMA loads.
__global__ void __launch_bounds__(256) weights_bf16_kernel(const float *wq, const float *wk,
                                                          __nv_bfloat16 *out) {
  const int hm = blockIdx.x, h = hm >> 1;
  const float *W = ((hm & 1) ? wk : wq) + (size_t)h * D * F;
  __nv_bfloat16 *o = out + (size_t)hm * D * F;
  for (int e = threadIdx.x * 4; e < D * F; e += 256 * 4) {
    const float4 x = *reinterpret_cast<const float4 *>(W + e);
    *reinterpret_cast<__nv_bfloat162 *>(o + e) = __floats2bfloat162_rn(x.x, x.y);
    *reinterpret_cast<__nv_bfloat162 *>(o + e + 2) = __floats2bfloat162_rn(x.z, x.w);
  }
}

constexpr size_t DS_SMEM = 5 * TILE + TILE / 2 + 1024;
constexpr size_t TILE_SMEM = 7 * TILE + 1024;

}  // namespace

// One copy region: [BH][ntiles][D][D] bf16 (each tile's matrix minus its
// row 0), then [BH][ntiles][D] fp32 (row 0).
size_t tc_gla_bwd_weights_bytes(int H) { return (size_t)H * 2 * D * F * sizeof(__nv_bfloat16); }

cudaError_t launch_weights_bf16(const float *wq, const float *wk, void *out, int H, cudaStream_t s) {
  weights_bf16_kernel<<<2 * H, 256, 0, s>>>(wq, wk, static_cast<__nv_bfloat16 *>(out));
  return cudaGetLastError();
}

namespace {
// The final state's share of the log-decay gradient from a final state the
// forward kept: kap[bh][h][i] = sum over column half h of G[i][v] S_L[i][v]
// (G the incoming final-state gradient); thread = (half, key dimension).
__global__ void __launch_bounds__(256) state_share_kernel(const float *S, const float *G, float *kap) {
  const int bh = blockIdx.x, i = threadIdx.x & 127, h = threadIdx.x >> 7;
  const float4 *s4 = reinterpret_cast<const float4 *>(S + ((size_t)bh * D + i) * D + 64 * h);
  const float4 *g4 = reinterpret_cast<const float4 *>(G + ((size_t)bh * D + i) * D + 64 * h);
  float part = 0.f;
#pragma unroll 4
  for (int u = 0; u < 16; ++u) {
    const float4 a = s4[u], b = g4[u];
    part = fmaf(b.x, a.x, part);
    part = fmaf(b.y, a.y, part);
    part = fmaf(b.z, a.z, part);
    part = fmaf(b.w, a.w, part);
  }
  kap[((size_t)bh * 2 + h) * D + i] = part;
}
}  // namespace

cudaError_t launch_state_share(const float *S, const float *G, float *kap, int BH, cudaStream_t s) {
  state_share_kernel<<<BH, 256, 0, s>>>(S, G, kap);
  return cudaGetLastError();
}

size_t tc_gla_bwd_snapshot_bytes(int BH, int L) {
  const size_t n = (size_t)BH * ((L + T - 1) / T);
  return n * D * D * sizeof(__nv_bfloat16) + n * D * sizeof(float);
}
static const float *snapshot_row0(const void *snap, int BH, int L) {
  return reinterpret_cast<const float *>(static_cast<const __nv_bfloat16 *>(snap) +
                                         (size_t)BH * ((L + T - 1) / T) * D * D);
}

// The GLA tile kernel's speed depends on where the driver places its code,
// which follows the order in which kernels are first touched: setting its
// attribute before any other kernel of the library is used puts it first,
// whatever the sizes of the kernels that run before it.
cudaError_t tc_gla_bwd_preload() {
  return cudaFuncSetAttribute(tc_gla_bwd_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TILE_SMEM);
}

cudaError_t launch_tc_gla_bwd(const TcGlaBwdArgs &a, int stage, cudaStream_t s) {
  const int ntiles = (a.L + T - 1) / T;
  const uint64_t rows = (uint64_t)a.L;
  if (stage == 0) {   // reverse dS pass
    DsParams p;
    memset(&p, 0, sizeof(p));
    if (!make_map_bf16_3d(&p.mq, a.q, D, rows, a.BH, T) || !make_map_bf16_3d(&p.mo, a.dout, D, rows, a.BH, T) ||
        !make_map_f32_3d(&p.me, a.e32, D, rows, a.BH, T))
      return cudaErrorInvalidValue;
    p.wq = a.wq;
    p.e32 = a.e32;
    p.gate_r = a.gate_r;
    p.snap = static_cast<__nv_bfloat16 *>(a.snap_ds);
    p.snap_r0 = const_cast<float *>(snapshot_row0(a.snap_ds, a.BH, a.L));
    p.dstate_in = a.dstate_in;
    p.dstate_out = a.dstate_out;
    p.status = a.status;
    p.H = a.H;
    p.L = a.L;
    p.inv_tau = a.inv_tau;
    cudaError_t e = cudaFuncSetAttribute(tc_gla_dstates_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DS_SMEM);
    if (e != cudaSuccess) return e;
    tc_gla_dstates_kernel<<<a.BH, NT_DS, DS_SMEM, s>>>(p);
    return cudaGetLastError();
  }
  if (stage == 1) {   // per-tile gradients
    TileParams p;
    memset(&p, 0, sizeof(p));
    if (!make_map_bf16_3d(&p.mq, a.q, D, rows, a.BH, T) || !make_map_bf16_3d(&p.mk, a.k, D, rows, a.BH, T) ||
        !make_map_bf16_3d(&p.mv, a.v, D, rows, a.BH, T) || !make_map_bf16_3d(&p.mo, a.dout, D, rows, a.BH, T) ||
        !make_map_bf16_3d(&p.msp, a.snap_s, D, D, (uint64_t)a.BH * ntiles, T) ||
        !make_map_bf16_3d(&p.mw, a.w16, F, D, (uint64_t)a.H * 2, T) ||
        !make_map_bf16_3d(&p.mds, a.snap_ds, D, D, (uint64_t)a.BH * ntiles, T) ||
        !make_map_bf16_3d(&p.mdq, a.dphq, D, rows, a.BH, T) || !make_map_bf16_3d(&p.mdk, a.dphk, D, rows, a.BH, T) ||
        !make_map_f32_3d(&p.mdb, a.dB, D, rows, a.BH, T) || !make_map_f32_3d(&p.mdv, a.dv, D, rows, a.BH, T) ||
        !make_map_f32_3d(&p.me, a.e32, D, rows, a.BH, T))
      return cudaErrorInvalidValue;
    p.colsum = a.colsum;
    p.e32 = a.e32;
    p.sp_r0 = snapshot_row0(a.snap_s, a.BH, a.L);
    p.ds_r0 = snapshot_row0(a.snap_ds, a.BH, a.L);

    p.status = a.status;
    p.H = a.H;
    p.L = a.L;
    p.ntiles = ntiles;
    p.BH = a.BH;
    p.inv_tau = a.inv_tau;
    cudaError_t e = cudaFuncSetAttribute(tc_gla_bwd_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TILE_SMEM);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int nwork = ntiles * a.BH;   // one persistent CTA per SM over contiguous runs of tiles
    tc_gla_bwd_tile_kernel<<<nwork < sms ? nwork : sms, NT_TILE, TILE_SMEM, s>>>(p);
    return cudaGetLastError();
  }
  if (a.scalar_gate)
    gate_grad_scalar_kernel<<<a.BH, 256, 0, s>>>(a.dB, static_cast<const __nv_bfloat16 *>(a.g), a.dg, a.L,
                                                 a.inv_tau, a.kap);
  else
    gate_grad_kernel<<<dim3(a.BH, D / 64), 256, 0, s>>>(a.dB, static_cast<const __nv_bfloat16 *>(a.g), a.dg, a.L,
                                                        a.inv_tau, a.kap, a.colsum);
  return cudaGetLastError();
}

}  // namespace lz
