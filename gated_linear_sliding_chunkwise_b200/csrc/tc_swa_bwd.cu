// Tensor-core (tcgen05 / TMEM / TMA) backward of the anchor branch: sliding
// window softmax with meta-token sinks (English gist.science summary,
// section 2.A "Anchor Window Attention"), bf16, d = 128, window <= 128.
//
// Softmax backward for query t with weights p over its window keys and the
// meta tokens, dO_swa = alpha dout:
//   D_t = dO_swa . o_swa_t,   dS = p (dO_swa . value - D_t)
//   dq_t = scale sum dS key,  dkey += scale dS q_t,  dvalue += p dO_swa
//
// tc_swa_bwd_q_kernel   one CTA per (sequence, 128-query tile): logits and
//                       softmax again, o_swa = P V for D, dP, dS, dq; writes
//                       dq, the log-normaliser and D, and adds the tile's
//                       terms of the meta-token gradients
//                       (dmeta_k += scale sum_t dS_meta[t] q_t,
//                       dmeta_v += alpha sum_t p_meta[t] dout_t).
// tc_swa_bwd_kv_kernel  one CTA per (sequence, 128-key block): the two query
//                       tiles that see the block; dK and dV accumulate in TMEM.
//
// A key/value prefix of P <= window tokens before token 0 (a segment of a
// longer sequence) enters the first query tile's band as its previous keys
// and values, and adds one key block per sequence (keys -128 .. -1, of which
// -P .. -1 exist) whose gradients go to dk_prefix / dv_prefix.
//
// Every mbarrier wait is bounded; a wait that gives up sets the TIMEOUT bit
// of the status word and the CTA leaves after freeing its TMEM.
#include "common.cuh"
#include "lizard_internal.h"
#include "tc_common.cuh"
#include "tc_host.h"

namespace lz {
namespace {

using namespace tc;

constexpr int T = 128;
constexpr int D = 128;
constexpr int MAXM = 16;
constexpr uint32_t TILE = kTile;
constexpr size_t SMEM_BYTES = 6 * TILE + 1024;
constexpr uint32_t ST_TIMEOUT = 1u;

struct QParams {
  CUtensorMap mq, mk, mv, mo;
  CUtensorMap mkp, mvp;       // key / value prefix [BH][P][D] (P > 0 only)
  CUtensorMap mdq;            // fp32 dq output (TMA stores)
  CUtensorMap mxq, mdqo;      // fused: bf16 GLA part dx_q (load), bf16 final dq (store)
  const float *meta_k, *meta_v, *alpha;
  float *dq, *lse, *Dterm, *dalpha;
  float *dmeta_k, *dmeta_v;   // meta-token gradients [H][M][D], accumulated (null: not wanted)
  const float *lse_in;        // the forward's softmax normalisers (null: formed here, into lse)
  uint32_t *status;
  int H, L, M, window;
  float scale;
  int fused;
  int BH;
  int P;
};

struct KVParams {
  CUtensorMap mq, mk, mv, mo;
  CUtensorMap mkp, mvp;       // key / value prefix [BH][P][D] (P > 0 only)
  CUtensorMap mdk, mdv;       // fp32 dk, dv outputs (TMA stores)
  CUtensorMap mxk, mdvg;      // fused: bf16 GLA part dx_k, fp32 GLA dv (loads)
  CUtensorMap mdko, mdvo;     // fused: bf16 final dk, dv (stores)
  const float *alpha, *lse, *Dterm;
  float *dk, *dv;
  __nv_bfloat16 *dk_prefix, *dv_prefix;   // [BH][P][D] (P > 0 only)
  uint32_t *status;
  int H, L, window;
  float scale;
  int fused;
  int BH;
  int P;
};

__device__ __forceinline__ void setup_cta(uint32_t *tmem_slot, uint64_t *bars, int nbars, int tid) {
  if ((tid >> 5) == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < nbars; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
  }
}

// ------------------------------------------------------------- dq pass ----
// Two warpgroups (256 threads): thread = query row `row` of its group.  The
// groups split the band's logit chunks (alternate chunks), the columns of O'
// and dq', and the meta dot products (group 0 q . mk, group 1 dO . mv);
// row sums and maxima meet in shared memory.
constexpr int NT_Q = 256;

// Meta-token gradient terms of one 128-row tile, for this warp's 32 columns
// n0 .. n0 + 31: acc[m][n] += sum_r W[m][r] X[r][n] over the tile's rows r
// (tokens), X the swizzled bf16 tile at region xreg, W the per-row meta
// weights as bf16 hi + lo planes [MAXM][ld] (rows m >= M read as zero).
// Warp-level mma.sync m16n8k16: A = W (16 meta rows x 16 tokens per step),
// B = X (16 tokens x 8 columns, read transposed by ldmatrix.trans), four
// n-tiles of 8 columns; acc[j] is n-tile j's C fragment (rows g and g + 8,
// columns 2t, 2t + 1 with g = lane / 4, t = lane % 4).  W enters as hi + lo,
// so the sums keep about 16 bits of each weight.
__device__ __forceinline__ void meta_grad_mma(const unsigned char *sm, uint32_t xreg, const __nv_bfloat16 *whi,
                                              const __nv_bfloat16 *wlo, int ld, int n0, int M, int lane,
                                              float (&acc)[4][4]) {
  const int g = lane >> 2, t = lane & 3;
  const bool r0 = g < M, r1 = g + 8 < M;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int k0 = 16 * ks;
    uint32_t ah[4], al[4];
    const int e0 = g * ld + k0 + 2 * t, e1 = (g + 8) * ld + k0 + 2 * t;
    ah[0] = r0 ? *reinterpret_cast<const uint32_t *>(whi + e0) : 0u;
    ah[1] = r1 ? *reinterpret_cast<const uint32_t *>(whi + e1) : 0u;
    ah[2] = r0 ? *reinterpret_cast<const uint32_t *>(whi + e0 + 8) : 0u;
    ah[3] = r1 ? *reinterpret_cast<const uint32_t *>(whi + e1 + 8) : 0u;
    al[0] = r0 ? *reinterpret_cast<const uint32_t *>(wlo + e0) : 0u;
    al[1] = r1 ? *reinterpret_cast<const uint32_t *>(wlo + e1) : 0u;
    al[2] = r0 ? *reinterpret_cast<const uint32_t *>(wlo + e0 + 8) : 0u;
    al[3] = r1 ? *reinterpret_cast<const uint32_t *>(wlo + e1 + 8) : 0u;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      // matrices: rows k0 .. k0 + 7 | k0 + 8 .. k0 + 15 of columns c .. c + 7,
      // then the same of columns c + 8 .. c + 15 (c = n0 + 16 j)
      const int r = k0 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int col = n0 + 16 * j + ((lane >> 4) & 1) * 8;
      const uint32_t addr = smem_u32(sm + xreg + (col >> 6) * kReg + sw128_offset(r, col & 63));
      uint32_t b[4];
      asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
                   : "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3])
                   : "r"(addr));
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float *c = acc[2 * j + u];
#pragma unroll
        for (int hl = 0; hl < 2; ++hl) {
          const uint32_t *a = hl ? al : ah;
          asm volatile(
              "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
              "{%0, %1, %2, %3};\n"
              : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
              : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[2 * u]), "r"(b[2 * u + 1]));
        }
      }
    }
  }
}

__global__ void __launch_bounds__(NT_Q, 1) tc_swa_bwd_q_kernel(const __grid_constant__ QParams p) {
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(16) float s_mk[MAXM][D];
  __shared__ __align__(16) float s_mv[MAXM][D];
  __shared__ float s_x[MAXM][T];        // dO . mv_m per row, later the meta dS per row
  __shared__ float s_pmax[2][T], s_psum[2][T], s_dpart[2][T];
  __shared__ float s_red[4];
  __shared__ uint64_t bars[7];
  __shared__ uint32_t s_tmem;
  // regions: Q, dO, K_prev, K, V_prev, V
  constexpr uint32_t R_Q = 0, R_O = TILE, R_KP = 2 * TILE, R_K = 3 * TILE, R_VP = 4 * TILE, R_V = 5 * TILE;
  // TMEM: logits [0,256) then P^ [0,128), dP' [256,512) (issued with the
  // logits), dS [128,256), dq' [0,128)
  constexpr uint32_t C_L = 0, C_P = 0, C_DP = 256, C_DS = 128, C_DQ = 0;
  // The meta weights of the meta-token gradients (per row: the meta dS for
  // dmeta_k, the meta probabilities for dmeta_v), bf16 hi + lo planes
  // [2][2][MAXM][MW_LD], in the V_prev region: only dP' reads V_prev, and
  // the next item's tiles arrive there after the dq' product.
  constexpr uint32_t R_MW = R_VP;
  constexpr int MW_LD = T + 8;   // padded rows: conflict-free fragment loads

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wg = tid >> 7, row = tid & 127;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t sbase = smem_u32(sm);
  uint64_t *bar_tma = &bars[0], *bar_m = &bars[1], *bar_late = &bars[6];
  setup_cta(&s_tmem, bars, 7, tid);
  // Persistent: CTA b walks the contiguous run [w0, w1) of (sequence, tile)
  // items, the tiles of a sequence in order; the meta tokens are staged again
  // only when the head changes, and the next item's tiles are loaded as soon
  // as this item's shared memory is free.
  const int ntiles = (p.L + T - 1) / T, nwork = ntiles * p.BH;
  const int w0 = (int)((long long)blockIdx.x * nwork / gridDim.x);
  const int w1 = (int)((long long)(blockIdx.x + 1) * nwork / gridDim.x);
  // Tile loads of item w, in two parts: `early` = the regions free once the
  // dq' product has run (all but V when the GLA part arrives in V, all but
  // Q | dO when dq is staged there), on bar_tma; `late` = the rest, after
  // the store, on bar_late.  With the GLA part in V, only the last product
  // (dO V^T) waits for the late tile.
  auto tile_loads = [&](int w, bool early, bool late) {
    const int lbh = w / ntiles, lt0 = (w % ntiles) * T;
    if (early) mbar_expect_tx(bar_tma, (p.fused ? 5 : 4) * TILE);
    if (late) mbar_expect_tx(bar_late, (p.fused ? 1 : 2) * TILE);
    const bool qo_early = p.fused != 0, v_early = p.fused == 0;
    for (int r = 0; r < 2; ++r) {
      if (qo_early ? early : late) {
        uint64_t *b = qo_early ? bar_tma : bar_late;
        tma_load_3d(sm + R_Q + r * kReg, &p.mq, b, 64 * r, lt0, lbh);
        tma_load_3d(sm + R_O + r * kReg, &p.mo, b, 64 * r, lt0, lbh);
      }
      if (early) {
        // keys and values of the previous tile; before token 0, the prefix
        // (its rows before the first prefix token read as zero)
        if (lt0 == 0 && p.P > 0) {
          tma_load_3d(sm + R_KP + r * kReg, &p.mkp, bar_tma, 64 * r, p.P - T, lbh);
          tma_load_3d(sm + R_VP + r * kReg, &p.mvp, bar_tma, 64 * r, p.P - T, lbh);
        } else {
          tma_load_3d(sm + R_KP + r * kReg, &p.mk, bar_tma, 64 * r, lt0 - T, lbh);
          tma_load_3d(sm + R_VP + r * kReg, &p.mv, bar_tma, 64 * r, lt0 - T, lbh);
        }
        tma_load_3d(sm + R_K + r * kReg, &p.mk, bar_tma, 64 * r, lt0, lbh);
      }
      if (v_early ? early : late) tma_load_3d(sm + R_V + r * kReg, &p.mv, v_early ? bar_tma : bar_late, 64 * r, lt0, lbh);
    }
  };
  if (tid == 0 && w0 < w1) tile_loads(w0, true, true);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s_tmem, tl = tb + lane_off;
  const uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
  const uint32_t id_mn = idesc_bf16(128, 128, 0, 1);
  const int m_rows = (p.M + 3) / 4 * 4;   // meta rows read (groups of four; zero past M)
  // meta-token gradients: group 0 dmeta_k (rows of Q), group 1 dmeta_v (rows
  // of dO), each warp 32 columns; summed over the CTA's items of one head in
  // registers, added to memory when the head changes
  const bool mgrad = p.M > 0 && (wg == 0 ? p.dmeta_k != nullptr : p.dmeta_v != nullptr);
  const bool mw_write = p.M > 0 && (p.dmeta_k != nullptr || p.dmeta_v != nullptr);
  float macc[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int u = 0; u < 4; ++u) macc[j][u] = 0.f;
  int cur_h = -1;
  bool ok = true;
  for (int w = w0, it = 0; w < w1; ++w, ++it) {
  const uint32_t par = (uint32_t)it & 1u;
  const int bh = w / ntiles, h = bh % p.H, t0 = (w % ntiles) * T, tq = t0 + row;
  const bool qvalid = tq < p.L;
  const float alpha = p.alpha ? p.alpha[h] : 1.f;
  if (h != cur_h) {
    cur_h = h;
    for (int e = tid; e < m_rows * D; e += NT_Q) {
      const int m = e / D;
      s_mk[m][e % D] = m < p.M ? p.meta_k[(size_t)h * p.M * D + e] : 0.f;
      s_mv[m][e % D] = (m < p.M && p.meta_v) ? p.meta_v[(size_t)h * p.M * D + e] : 0.f;
    }
    __syncthreads();
  }
  ok = mbar_wait(bar_tma, par, p.status, ST_TIMEOUT);
  if (!p.fused) ok = ok && mbar_wait(bar_late, par, p.status, ST_TIMEOUT);   // Q and dO come late
  if (__syncthreads_or(!ok)) goto done;

  // 1. logits L = Q [K_prev ; K]^T and dP' = dO [V_prev ; V]^T (with the GLA
  //    part in V, dO V^T once V has arrived, after the meta dot products)
  bool v_ok = true;
  if (tid == 0) {
    tc_fence_after();
    for (int s = 0; s < 8; ++s) mma_ss(tb + C_L, desc_k(sbase + R_Q, s), desc_k(sbase + R_KP, s), id_kk, s > 0);
    for (int s = 0; s < 8; ++s) mma_ss(tb + C_L + 128, desc_k(sbase + R_Q, s), desc_k(sbase + R_K, s), id_kk, s > 0);
    for (int s = 0; s < 8; ++s) mma_ss(tb + C_DP, desc_k(sbase + R_O, s), desc_k(sbase + R_VP, s), id_kk, s > 0);
    if (!p.fused) {
      for (int s = 0; s < 8; ++s) mma_ss(tb + C_DP + 128, desc_k(sbase + R_O, s), desc_k(sbase + R_V, s), id_kk, s > 0);
      mma_commit(bar_m);
    }
  }
  {
    const float lse_row = (p.lse_in && qvalid) ? p.lse_in[(size_t)bh * p.L + tq] : 0.f;
    // meta dot products while the MMAs run, by mma.sync over each warp's 32
    // rows, every lane getting its own row's: group 0 q . mk_m (kept in
    // registers), group 1 dO . mv_m (to shared memory)
    float ml[MAXM], em[MAXM], dom[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) { ml[m] = 0.f; em[m] = 0.f; dom[m] = 0.f; }
    if (p.M > 0) {
      rowdots_mma<true>(sm, wg == 0 ? R_Q : R_O, 32 * (warp & 3), wg == 0 ? s_mk : s_mv, p.M, nullptr, lane, ml);
      if (wg == 1)
#pragma unroll
        for (int m = 0; m < MAXM; ++m)
          if (m < p.M) s_x[m][row] = ml[m];
    }
    if (p.fused && tid == 0) {
      v_ok = mbar_wait(bar_late, par, p.status, ST_TIMEOUT);
      tc_fence_after();
      if (v_ok)
        for (int s = 0; s < 8; ++s) mma_ss(tb + C_DP + 128, desc_k(sbase + R_O, s), desc_k(sbase + R_V, s), id_kk, s > 0);
      mma_commit(bar_m);   // also when V never came: the products issued above complete
    }
    ok = mbar_wait(bar_m, par, p.status, ST_TIMEOUT) && v_ok;
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();
    if (p.fused && tid == 0) {   // the GLA part of dq into the V region (only dP' read V)
      mbar_expect_tx(&bars[5], TILE);
      tma_load_3d(sm + R_V, &p.mxq, &bars[5], 0, t0, bh);
      tma_load_3d(sm + R_V + kReg, &p.mxq, &bars[5], 64, t0, bh);
    }
    float mx = kNegBig;
    if (wg == 0) {
#pragma unroll
      for (int m = 0; m < MAXM; ++m)
        if (m < p.M) {
          dom[m] = s_x[m][row];
          ml[m] *= p.scale;
          mx = fmaxf(mx, ml[m]);
        }
    }
    // With the forward's normaliser lse = log sum exp of the row's scaled
    // logits, P = exp(l - lse) directly: no max pass, and P^ below is P.
    const bool given = p.lse_in != nullptr;

    // 2. softmax over the band (see the forward): logit column cl holds key
    //    t0 - T + cl; warp w4 visits chunks ch_lo .. ch_hi, group 1 the
    //    chunks ch_lo, ch_lo + 2, ... and group 0 (which also has the meta
    //    terms) the others
    //    (keys >= -P, P the prefix length)
    const int w4 = warp & 3, cbase = t0 - T;
    const int lo_c = max(tq - p.window + 1, -p.P) - cbase, hi_c = tq - cbase;
    int ch_lo = (32 * w4 + T + 1 - p.window) >> 5;
    if (cbase < 0) ch_lo = max(ch_lo, (T - p.P) >> 5);
    const int ch_hi = w4 + 4;
    const int in_lo = 32 * w4 + 31 + T + 1 - p.window;
    // an odd band's last chunk is halved: group 1 its first 16 columns,
    // group 0 the other 16 (as in the forward)
    const bool split = ((ch_hi - ch_lo) & 1) == 0;
    const int full_hi = split ? ch_hi - 1 : ch_hi;
    const int hcol = 32 * ch_hi + 16 * (1 - wg);
    const bool hinner = hcol >= in_lo && hcol + 15 <= 32 * w4 + T && hcol + cbase >= -p.P;
    const int lo_h = hinner ? -1 : lo_c - hcol, hi_h = hinner ? 16 : hi_c - hcol;   // the half's exponent mask
    if (given) {
      mx = lse_row;
    } else {
    if (split) {
      float v[16];
      tmem_ld16(tl + C_L + hcol, v);
      float m4[4] = {kNegBig, kNegBig, kNegBig, kNegBig};
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (hinner || (hcol + u >= lo_c && hcol + u <= hi_c)) m4[u & 3] = fmaxf(m4[u & 3], v[u]);
      const float cm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      if (cm > kNegBig) mx = fmaxf(mx, cm * p.scale);
    }
    for (int ch = ch_lo + 1 - wg; ch <= full_hi; ch += 2) {
      float v[32];
      tmem_ld32(tl + C_L + ch * 32, v);
      float m4[4] = {kNegBig, kNegBig, kNegBig, kNegBig};
      if (32 * ch >= in_lo && 32 * ch + 31 <= 32 * w4 + T && 32 * ch + cbase >= -p.P) {
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
    s_pmax[wg][row] = mx;
    bar_sync(1, NT_Q);
    mx = fmaxf(s_pmax[0][row], s_pmax[1][row]);
    }
    //    P^ = exp(l - max) of this group's chunks, held in registers until
    //    both groups have read their logits (P^ overlays logit chunks 0 .. 3)
    //    and, for D = dO_swa . o_swa = alpha (sum_j P^_j dP'_j + sum_m e_m
    //    dO . mv_m) / l, the sums of P^ dP' over the same chunks
    uint32_t pk[2][16], pkh[8];
    float s4[4] = {0.f, 0.f, 0.f, 0.f}, d4[4] = {0.f, 0.f, 0.f, 0.f};
    if (split) {
      float v[16], dp[16];
      tmem_ld16(tl + C_L + hcol, v);
      tmem_ld16(tl + C_DP + hcol, dp);
#pragma unroll
      for (int u = 0; u < 16; u += 2) {
        float e0 = __expf(fmaf(v[u], p.scale, -mx));
        float e1 = __expf(fmaf(v[u + 1], p.scale, -mx));
        e0 = (u >= lo_h && u <= hi_h) ? e0 : 0.f;
        e1 = (u + 1 >= lo_h && u + 1 <= hi_h) ? e1 : 0.f;
        s4[(u >> 1) & 3] += e0 + e1;
        d4[(u >> 1) & 3] = fmaf(e0, dp[u], fmaf(e1, dp[u + 1], d4[(u >> 1) & 3]));
        pkh[u / 2] = pack_bf16(e0, e1);
      }
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int ch = ch_lo + 1 - wg + 2 * k;
      if (ch > full_hi) continue;
      float v[32], dp[32];
      tmem_ld32(tl + C_L + ch * 32, v);
      tmem_ld32(tl + C_DP + ch * 32, dp);
      const bool inner = 32 * ch >= in_lo && 32 * ch + 31 <= 32 * w4 + T && 32 * ch + cbase >= -p.P;
      // one masked copy of the loop (interior chunks: bounds that pass every column)
      const int lo_e = inner ? -1 : lo_c - 32 * ch, hi_e = inner ? 32 : hi_c - 32 * ch;
#pragma unroll
      for (int u = 0; u < 32; u += 2) {
        float e0 = __expf(fmaf(v[u], p.scale, -mx));
        float e1 = __expf(fmaf(v[u + 1], p.scale, -mx));
        e0 = (u >= lo_e && u <= hi_e) ? e0 : 0.f;
        e1 = (u + 1 >= lo_e && u + 1 <= hi_e) ? e1 : 0.f;
        s4[(u >> 1) & 3] += e0 + e1;
        d4[(u >> 1) & 3] = fmaf(e0, dp[u], fmaf(e1, dp[u + 1], d4[(u >> 1) & 3]));
        pk[k][u / 2] = pack_bf16(e0, e1);
      }
    }
    float psum = (s4[0] + s4[1]) + (s4[2] + s4[3]);
    float dpart = (d4[0] + d4[1]) + (d4[2] + d4[3]);
    if (wg == 0) {
#pragma unroll
      for (int m = 0; m < MAXM; ++m)
        if (m < p.M) {
          em[m] = __expf(ml[m] - mx);
          psum += em[m];
          dpart = fmaf(em[m], dom[m], dpart);
        }
    }
    s_psum[wg][row] = psum;
    s_dpart[wg][row] = dpart;
    bar_sync(2, NT_Q);
    const float lsum = s_psum[0][row] + s_psum[1][row];
    const float inv_l = given ? 1.f : 1.f / lsum;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int ch = ch_lo + 1 - wg + 2 * k;
      if (ch > full_hi) continue;
      tmem_st8(tl + C_P + ch * 16, pk[k]);
      tmem_st8(tl + C_P + ch * 16 + 8, pk[k] + 8);
    }
    if (split) tmem_st8(tl + C_P + ch_hi * 16 + 8 * (1 - wg), pkh);
    {
      uint32_t zero[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      for (int ch = wg; ch < 8; ch += 2) {
        if (ch >= ch_lo && ch <= ch_hi) continue;
        tmem_st8(tl + C_P + ch * 16, zero);
        tmem_st8(tl + C_P + ch * 16 + 8, zero);
      }
    }
    if (wg == 0 && qvalid && !given) p.lse[(size_t)bh * p.L + tq] = mx + logf(lsum);
    tmem_st_wait();
    // 3. D (dO_swa . o_swa) from the two groups' sums
    float dal = (s_dpart[0][row] + s_dpart[1][row]) * inv_l;
    if (!qvalid) dal = 0.f;
    const float Dt = alpha * dal;
    if (wg == 0) {
      if (qvalid) p.Dterm[(size_t)bh * p.L + tq] = Dt;
      if (p.dalpha) {
        const float w = warp_sum(dal);
        if (lane == 0) s_red[warp] = w;
      }
    }
    tc_fence_before();
    __syncthreads();   // also: every group's P^ stores are in before the other reads them
    tc_fence_after();
    if (tid == 0 && p.dalpha) atomicAdd(p.dalpha + h, s_red[0] + s_red[1] + s_red[2] + s_red[3]);

    // 4. dS = P (alpha dP' - D), P = P^ / l, on the band (zero elsewhere,
    //    as P^ is); alternate chunks per group; the meta terms go to memory
    for (int ch = wg; ch < 8; ch += 2) {
      uint32_t ds[16];
      if (ch >= ch_lo && ch <= ch_hi) {
        float dp[32], pp[32], pk16[16];
        tmem_ld32(tl + C_DP + ch * 32, dp);
        tmem_ld16(tl + C_P + ch * 16, pk16);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const uint32_t w = __float_as_uint(pk16[u]);
          pp[2 * u] = __uint_as_float(w << 16);
          pp[2 * u + 1] = __uint_as_float(w & 0xffff0000u);
        }
#pragma unroll
        for (int u = 0; u < 32; u += 2)
          ds[u / 2] = pack_bf16(pp[u] * inv_l * (alpha * dp[u] - Dt), pp[u + 1] * inv_l * (alpha * dp[u + 1] - Dt));
      } else {
#pragma unroll
        for (int u = 0; u < 16; ++u) ds[u] = 0u;
      }
      tmem_st8(tl + C_DS + ch * 16, ds);
      tmem_st8(tl + C_DS + ch * 16 + 8, ds + 8);
    }
    if (wg == 0) {
      __nv_bfloat16 *mw = reinterpret_cast<__nv_bfloat16 *>(sm + R_MW);
#pragma unroll
      for (int m = 0; m < MAXM; ++m) {
        if (m < p.M) {
          const float pm = em[m] * inv_l;
          const float dsm = pm * (alpha * dom[m] - Dt);
          s_x[m][row] = dsm;
          if (mw_write) {   // plane (which, hi | lo): ((which * 2 + hl) * MAXM + m) * MW_LD + row
            const float wv[2] = {qvalid ? dsm : 0.f, qvalid ? pm : 0.f};
#pragma unroll
            for (int which = 0; which < 2; ++which) {
              const __nv_bfloat16 hi = __float2bfloat16_rn(wv[which]);
              const __nv_bfloat16 lo = __float2bfloat16_rn(wv[which] - __bfloat162float(hi));
              mw[((which * 2 + 0) * MAXM + m) * MW_LD + row] = hi;
              mw[((which * 2 + 1) * MAXM + m) * MW_LD + row] = lo;
            }
          }
        }
      }
      // the next item's tiles overwrite the weights by TMA
      if (mw_write) fence_proxy_async();
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();

    // 5. dq' = dS [K_prev ; K]
    if (tid == 0) {
      tc_fence_after();
      for (int s = 0; s < 8; ++s) mma_ts(tb + C_DQ, tb + C_DS + s * 8, desc_mn(sbase + R_KP, s), id_mn, s > 0);
      for (int s = 0; s < 8; ++s) mma_ts(tb + C_DQ, tb + C_DS + 64 + s * 8, desc_mn(sbase + R_K, s), id_mn, 1);
      mma_commit(&bars[4]);
    }
    // the meta-token gradient terms of this tile while dq' runs (Q and dO
    // stay in place until the product is done)
    if (mgrad) {
      const __nv_bfloat16 *mw = reinterpret_cast<const __nv_bfloat16 *>(sm + R_MW) + (size_t)wg * 2 * MAXM * MW_LD;
      meta_grad_mma(sm, wg == 0 ? R_Q : R_O, mw, mw + MAXM * MW_LD, MW_LD, 32 * (warp & 3), p.M, lane, macc);
    }
    ok = mbar_wait(&bars[4], par, p.status, ST_TIMEOUT);
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();
    // the products are done with K_prev, K, V_prev (and Q, dO or V): the next
    // item's tiles start arriving while this one finishes
    if (tid == 0 && w + 1 < w1) tile_loads(w + 1, true, false);
    if (p.fused) {
      // dq = anchor part + GLA part, bf16, written in place over the GLA
      // part in the V region and stored with TMA (rows past L are clipped)
      ok = mbar_wait(&bars[5], par, p.status, ST_TIMEOUT);
      if (__syncthreads_or(!ok)) goto done;
      for (int ch = 2 * wg; ch < 2 * wg + 2; ++ch) {
        float v[32];
        tmem_ld32(tl + C_DQ + ch * 32, v);
        for (int m = 0; m < p.M; ++m) {
          const float w = s_x[m][row];
          const float4 *mk = reinterpret_cast<const float4 *>(&s_mk[m][ch * 32]);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 x = mk[q4];
            v[4 * q4] = fmaf(w, x.x, v[4 * q4]);
            v[4 * q4 + 1] = fmaf(w, x.y, v[4 * q4 + 1]);
            v[4 * q4 + 2] = fmaf(w, x.z, v[4 * q4 + 2]);
            v[4 * q4 + 3] = fmaf(w, x.w, v[4 * q4 + 3]);
          }
        }
#pragma unroll
        for (int k8 = 0; k8 < 4; ++k8) {
          uint4 *cp = chunk_ptr(sm, R_V, row, 4 * ch + k8);
          float g8[8];
          unpack8(*cp, g8);
#pragma unroll
          for (int u = 0; u < 8; ++u) g8[u] = fmaf(v[8 * k8 + u], p.scale, g8[u]);
          *cp = pack8(g8);
        }
      }
      fence_proxy_async();
      __syncthreads();
      if (tid == 0) {
        tma_store_3d(&p.mdqo, sm + R_V, 0, t0, bh);
        tma_store_3d(&p.mdqo, sm + R_V + kReg, 64, t0, bh);
        bulk_commit();
        bulk_wait_read();   // the staging is free once read (the writes need not have landed)
      }
    } else {
    // dq, staged as an fp32 tile over the free Q | dO regions and written
    // with TMA stores (rows past L are clipped by the map)
    unsigned char *st = sm + R_Q;
    for (int ch = 2 * wg; ch < 2 * wg + 2; ++ch) {
      float v[32];
      tmem_ld32(tl + C_DQ + ch * 32, v);
      for (int m = 0; m < p.M; ++m) {
        const float w = s_x[m][row];
        const float4 *mk = reinterpret_cast<const float4 *>(&s_mk[m][ch * 32]);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const float4 x = mk[q4];
          v[4 * q4] = fmaf(w, x.x, v[4 * q4]);
          v[4 * q4 + 1] = fmaf(w, x.y, v[4 * q4 + 1]);
          v[4 * q4 + 2] = fmaf(w, x.z, v[4 * q4 + 2]);
          v[4 * q4 + 3] = fmaf(w, x.w, v[4 * q4 + 3]);
        }
      }
#pragma unroll
      for (int u = 0; u < 32; u += 4)
        *f32_stage_ptr(st, row, ch * 32 + u) =
            make_float4(v[u] * p.scale, v[u + 1] * p.scale, v[u + 2] * p.scale, v[u + 3] * p.scale);
    }
    fence_proxy_async();
    __syncthreads();
    if (tid == 0) {
      for (int bx = 0; bx < 4; ++bx) tma_store_3d(&p.mdq, st + bx * 16384, 32 * bx, t0, bh);
      bulk_commit();
      bulk_wait_read();   // the staging is free once read (the writes need not have landed)
    }
    }
  }
  // this CTA's share of the head's meta-token gradients, once its last item
  // of the head is done: C rows g and g + 8 (meta tokens), columns 2t, 2t + 1
  // of each n-tile
  if (mgrad && (w + 1 >= w1 || ((w + 1) / ntiles) % p.H != h)) {
    float *out = wg == 0 ? p.dmeta_k : p.dmeta_v;
    const float f = wg == 0 ? p.scale : alpha;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = 32 * (warp & 3) + 8 * j + 2 * t;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int m = g + 8 * (u >> 1);
        if (m < p.M) atomicAdd(out + ((size_t)h * p.M + m) * D + n + (u & 1), f * macc[j][u]);
        macc[j][u] = 0.f;
      }
    }
  }
  // the store has read this item's staging: the rest of the next item's tiles
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && w + 1 < w1) tile_loads(w + 1, false, true);
  }
done:
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(s_tmem, 512);
}

// ------------------------------------------------------------ dk, dv ------
// Two warpgroups (256 threads): thread = key row `row` of its group; group h
// forms P and dS for query chunks 2h, 2h + 1 of each query tile and writes
// columns 64 h .. of dK and dV.
constexpr int NT_KV = 256;
__global__ void __launch_bounds__(NT_KV, 1) tc_swa_bwd_kv_kernel(const __grid_constant__ KVParams p) {
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(16) float s_lse[2 * T];
  __shared__ __align__(16) float s_D[2 * T];
  __shared__ uint64_t bars[7];
  __shared__ uint32_t s_tmem;
  // regions: K, V, Q_a, dO_a, Q_b, dO_b  (query tiles kb and kb + 1)
  constexpr uint32_t R_K = 0, R_V = TILE, R_Q0 = 2 * TILE, R_O0 = 3 * TILE;
  // TMEM: S^T / P [0,128), dP^T / dS [128,256), dV [256,384), dK [384,512)
  constexpr uint32_t C_S = 0, C_P = 0, C_DP = 128, C_DS = 128, C_DV = 256, C_DK = 384;

  const int tid = threadIdx.x, warp = tid >> 5, wg = tid >> 7, row = tid & 127;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t sbase = smem_u32(sm);
  setup_cta(&s_tmem, bars, 7, tid);
  // Persistent: CTA b walks the contiguous run [w0, w1) of (sequence, key
  // block) items; the next item's query tile b is loaded once this item's
  // products are done with it, the rest after its store.
  // With a prefix, block 0 of every sequence holds keys -128 .. -1 (the
  // prefix in its last P rows, zeros before) and block b > 0 keys
  // 128 (b - 1) ..; the query tiles of block 0 are then tokens -128 .. -1
  // (none: read as zeros and masked) and 0 .. 127.
  const int npre = p.P > 0 ? 1 : 0;
  const int nblk = (p.L + T - 1) / T + npre, nwork = nblk * p.BH;
  const int w0 = (int)((long long)blockIdx.x * nwork / gridDim.x);
  const int w1 = (int)((long long)(blockIdx.x + 1) * nwork / gridDim.x);
  auto tile_loads = [&](int w, bool early, bool late) {
    const int lbh = w / nblk, lj0 = (w % nblk - npre) * T;
    if (early) mbar_expect_tx(&bars[0], 6 * TILE);
    for (int r = 0; r < 2; ++r) {
      if (late && lj0 < 0) {
        tma_load_3d(sm + R_K + r * kReg, &p.mkp, &bars[0], 64 * r, p.P - T, lbh);
        tma_load_3d(sm + R_V + r * kReg, &p.mvp, &bars[0], 64 * r, p.P - T, lbh);
      } else if (late) {
        tma_load_3d(sm + R_K + r * kReg, &p.mk, &bars[0], 64 * r, lj0, lbh);
        tma_load_3d(sm + R_V + r * kReg, &p.mv, &bars[0], 64 * r, lj0, lbh);
      }
      if (late) {
        tma_load_3d(sm + R_Q0 + r * kReg, &p.mq, &bars[0], 64 * r, lj0, lbh);
        tma_load_3d(sm + R_O0 + r * kReg, &p.mo, &bars[0], 64 * r, lj0, lbh);
      }
      if (early) {
        tma_load_3d(sm + R_Q0 + 2 * TILE + r * kReg, &p.mq, &bars[0], 64 * r, lj0 + T, lbh);
        tma_load_3d(sm + R_O0 + 2 * TILE + r * kReg, &p.mo, &bars[0], 64 * r, lj0 + T, lbh);
      }
    }
  };
  if (tid == 0 && w0 < w1) tile_loads(w0, true, true);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s_tmem, tl = tb + lane_off;
  const uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
  const uint32_t id_mn = idesc_bf16(128, 128, 0, 1);
  const int r0 = 32 * (warp & 3);          // first key row of this warp
  bool ok = true;
  for (int w = w0, itn = 0; w < w1; ++w, ++itn) {
  const uint32_t par = (uint32_t)itn & 1u;
  const int bh = w / nblk, h = bh % p.H, j0 = (w % nblk - npre) * T, tk = j0 + row;
  const bool pre = j0 < 0;                     // the prefix block
  const float alpha = p.alpha ? p.alpha[h] : 1.f;
  for (int e = tid; e < 2 * T; e += NT_KV) {   // the softmax statistics of the two query tiles
    const int t = j0 + e;
    s_lse[e] = (t >= 0 && t < p.L) ? p.lse[(size_t)bh * p.L + t] : 0.f;
    s_D[e] = (t >= 0 && t < p.L) ? p.Dterm[(size_t)bh * p.L + t] : 0.f;
  }
  ok = mbar_wait(&bars[0], par, p.status, ST_TIMEOUT);
  if (__syncthreads_or(!ok)) goto done;
  for (int it = 0; it < 2; ++it) {
    const uint32_t rq = R_Q0 + it * 2 * TILE, ro = R_O0 + it * 2 * TILE;
    // S^T = K Q^T, dP^T = V dO^T   (rows = keys of this block)
    if (tid == 0) {
      tc_fence_after();
      for (int s = 0; s < 8; ++s) mma_ss(tb + C_S, desc_k(sbase + R_K, s), desc_k(sbase + rq, s), id_kk, s > 0);
      for (int s = 0; s < 8; ++s) mma_ss(tb + C_DP, desc_k(sbase + R_V, s), desc_k(sbase + ro, s), id_kk, s > 0);
      mma_commit(&bars[1 + 2 * it]);
    }
    ok = mbar_wait(&bars[1 + 2 * it], par, p.status, ST_TIMEOUT);
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();
    if (p.fused && it == 1 && tid == 0) {   // K and V are read: the GLA part of dk into K
      mbar_expect_tx(&bars[6], TILE);
      tma_load_3d(sm + R_K, &p.mxk, &bars[6], 0, j0, bh);
      tma_load_3d(sm + R_K + kReg, &p.mxk, &bars[6], 64, j0, bh);
    }
    // P = exp(scale s - lse_t), dS = P (alpha dP - D_t) on the band t - w < j <= t.
    // Query column qc of this tile is token j0 + it T + qc; the warp's keys
    // j0 + r0 .. j0 + r0 + 31 see columns qc with 0 <= it T + qc - row < w.
    // Packed results are held until both groups have read their logits
    // (P and dS overlay the logit columns of the lower chunks).
    {
      const int qlo = max(0, r0 - it * T), qhi = min(T - 1, r0 + 31 + p.window - 1 - it * T);
      // this thread's key tk sees the query rows qi (t = j0 + qi) with
      // tk <= t < tk + window and 0 <= t < L: qi in [vlo, vhi] (none when tk
      // is outside [-P, L))
      const bool kvalid = tk >= -p.P && tk < p.L;
      const int vlo = max(tk - j0, -j0), vhi = min(tk - j0 + p.window - 1, p.L - 1 - j0);
      uint32_t pk[2][16], dk[2][16];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int ch = 2 * wg + k;
        if (32 * ch + 31 < qlo || 32 * ch > qhi) {     // no query of this chunk sees the warp's keys
#pragma unroll
          for (int u = 0; u < 16; ++u) { pk[k][u] = 0u; dk[k][u] = 0u; }
          continue;
        }
        float sv[32], dv[32];
        tmem_ld32(tl + C_S + ch * 32, sv);
        tmem_ld32(tl + C_DP + ch * 32, dv);
        const int qb = it * T + ch * 32;                   // the chunk's first query row within the two tiles
        const int lo = kvalid ? vlo - qb : 32, hi = vhi - qb;
        const bool all = lo <= 0 && hi >= 31;              // every query of the chunk sees this key
#pragma unroll
        for (int u = 0; u < 32; u += 4) {
          const float4 l4 = *reinterpret_cast<const float4 *>(&s_lse[qb + u]);
          const float4 d4 = *reinterpret_cast<const float4 *>(&s_D[qb + u]);
          const float lq[4] = {l4.x, l4.y, l4.z, l4.w}, dq[4] = {d4.x, d4.y, d4.z, d4.w};
          float pr[4], ds[4];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            pr[w] = __expf(fmaf(sv[u + w], p.scale, -lq[w]));
            if (!all) pr[w] = (u + w >= lo && u + w <= hi) ? pr[w] : 0.f;
            ds[w] = pr[w] * (alpha * dv[u + w] - dq[w]);
          }
          pk[k][u / 2] = pack_bf16(pr[0], pr[1]);
          pk[k][u / 2 + 1] = pack_bf16(pr[2], pr[3]);
          dk[k][u / 2] = pack_bf16(ds[0], ds[1]);
          dk[k][u / 2 + 1] = pack_bf16(ds[2], ds[3]);
        }
      }
      bar_sync(1, NT_KV);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int ch = 2 * wg + k;
        tmem_st8(tl + C_P + ch * 16, pk[k]);
        tmem_st8(tl + C_P + ch * 16 + 8, pk[k] + 8);
        tmem_st8(tl + C_DS + ch * 16, dk[k]);
        tmem_st8(tl + C_DS + ch * 16 + 8, dk[k] + 8);
      }
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    // dV += P dO, dK += dS Q   (K dimension = the 128 queries of this tile)
    if (tid == 0) {
      tc_fence_after();
      for (int s = 0; s < 8; ++s) mma_ts(tb + C_DV, tb + C_P + s * 8, desc_mn(sbase + ro, s), id_mn, it > 0 || s > 0);
      for (int s = 0; s < 8; ++s) mma_ts(tb + C_DK, tb + C_DS + s * 8, desc_mn(sbase + rq, s), id_mn, it > 0 || s > 0);
      mma_commit(&bars[2 + 2 * it]);
    }
    ok = mbar_wait(&bars[2 + 2 * it], par, p.status, ST_TIMEOUT);
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();
    if (it == 1 && tid == 0 && w + 1 < w1) tile_loads(w + 1, true, false);   // query tile b is done
    if (p.fused && it == 0 && tid == 0) {   // query tile a is done: the GLA dv into its regions
      mbar_expect_tx(&bars[5], 2 * TILE);
      for (int bx = 0; bx < 4; ++bx) tma_load_3d(sm + R_Q0 + bx * 16384, &p.mdvg, &bars[5], 32 * bx, j0, bh);
    }
  }
  if (p.fused) {
    // dk = anchor part + GLA part (bf16, in place over the GLA part in K);
    // dv = anchor part + GLA dv (fp32 in Q_a | dO_a) as bf16 into V; both
    // stored with TMA (rows past L are clipped by the maps)
    ok = mbar_wait(&bars[5], par, p.status, ST_TIMEOUT);
    ok &= mbar_wait(&bars[6], par, p.status, ST_TIMEOUT);
    if (__syncthreads_or(!ok)) goto done;
    for (int ch = 2 * wg; ch < 2 * wg + 2; ++ch) {
      float a[32], b[32];
      tmem_ld32(tl + C_DK + ch * 32, a);
      tmem_ld32(tl + C_DV + ch * 32, b);
#pragma unroll
      for (int k8 = 0; k8 < 4; ++k8) {
        uint4 *cp = chunk_ptr(sm, R_K, row, 4 * ch + k8);
        float g8[8], v8[8];
        unpack8(*cp, g8);
        const float4 d0 = *f32_stage_ptr(sm + R_Q0, row, 32 * ch + 8 * k8);
        const float4 d1 = *f32_stage_ptr(sm + R_Q0, row, 32 * ch + 8 * k8 + 4);
        const float dg[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          g8[u] = fmaf(a[8 * k8 + u], p.scale, g8[u]);
          v8[u] = fmaf(b[8 * k8 + u], alpha, dg[u]);
        }
        if (pre) {   // prefix keys (no GLA part: the loads read zeros)
          if (tk >= -p.P) {
            const size_t o = ((size_t)bh * p.P + (p.P + tk)) * D + 32 * ch + 8 * k8;
            *reinterpret_cast<uint4 *>(p.dk_prefix + o) = pack8(g8);
            *reinterpret_cast<uint4 *>(p.dv_prefix + o) = pack8(v8);
          }
        } else {
          *cp = pack8(g8);
          *chunk_ptr(sm, R_V, row, 4 * ch + k8) = pack8(v8);
        }
      }
    }
    fence_proxy_async();
    __syncthreads();
    if (tid == 0 && !pre) {
      tma_store_3d(&p.mdko, sm + R_K, 0, j0, bh);
      tma_store_3d(&p.mdko, sm + R_K + kReg, 64, j0, bh);
      tma_store_3d(&p.mdvo, sm + R_V, 0, j0, bh);
      tma_store_3d(&p.mdvo, sm + R_V + kReg, 64, j0, bh);
      bulk_commit();
      bulk_wait_read();   // the staging is free once read (the writes need not have landed)
    }
  } else {
    // dK, dV, staged as fp32 tiles over the free K | V and Q_a | dO_a regions
    // and written with TMA stores (rows past L are clipped by the maps)
    unsigned char *st0 = sm + R_K, *st1 = sm + R_Q0;
    for (int ch = 2 * wg; ch < 2 * wg + 2; ++ch) {
      float a[32], b[32];
      tmem_ld32(tl + C_DK + ch * 32, a);
      tmem_ld32(tl + C_DV + ch * 32, b);
      if (pre) {   // prefix keys: their final bf16 gradients
        if (tk >= -p.P) {
          const size_t o = ((size_t)bh * p.P + (p.P + tk)) * D + 32 * ch;
#pragma unroll
          for (int u = 0; u < 32; ++u) { a[u] *= p.scale; b[u] *= alpha; }
#pragma unroll
          for (int k8 = 0; k8 < 4; ++k8) {
            *reinterpret_cast<uint4 *>(p.dk_prefix + o + 8 * k8) = pack8(a + 8 * k8);
            *reinterpret_cast<uint4 *>(p.dv_prefix + o + 8 * k8) = pack8(b + 8 * k8);
          }
        }
        continue;
      }
#pragma unroll
      for (int u = 0; u < 32; u += 4) {
        *f32_stage_ptr(st0, row, ch * 32 + u) =
            make_float4(a[u] * p.scale, a[u + 1] * p.scale, a[u + 2] * p.scale, a[u + 3] * p.scale);
        *f32_stage_ptr(st1, row, ch * 32 + u) =
            make_float4(b[u] * alpha, b[u + 1] * alpha, b[u + 2] * alpha, b[u + 3] * alpha);
      }
    }
    fence_proxy_async();
    __syncthreads();
    if (tid == 0 && !pre) {
      for (int bx = 0; bx < 4; ++bx) {
        tma_store_3d(&p.mdk, st0 + bx * 16384, 32 * bx, j0, bh);
        tma_store_3d(&p.mdv, st1 + bx * 16384, 32 * bx, j0, bh);
      }
      bulk_commit();
      bulk_wait_read();   // the staging is free once read (the writes need not have landed)
    }
  }
  // the store has read this item's staging: the rest of the next item's tiles
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && w + 1 < w1) tile_loads(w + 1, false, true);
  }
done:
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(s_tmem, 512);
}

}  // namespace

bool tc_swa_bwd_supported(int dk, int dv, int window, int M, bool bf16) {
  return bf16 && dk == D && dv == D && window <= T && M <= MAXM;
}

cudaError_t launch_tc_swa_bwd(const TcSwaBwdArgs &a, int stage, cudaStream_t s) {
  const int ntiles = (a.L + T - 1) / T;
  const uint64_t rows = (uint64_t)a.L;
  // the attribute is per device: set it every launch on devices not yet seen
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (stage == 0) {
    QParams p;
    memset(&p, 0, sizeof(p));
    if (!make_map_bf16_3d(&p.mq, a.q, D, rows, a.BH, T) || !make_map_bf16_3d(&p.mk, a.k, D, rows, a.BH, T) ||
        !make_map_bf16_3d(&p.mv, a.v, D, rows, a.BH, T) || !make_map_bf16_3d(&p.mo, a.dout, D, rows, a.BH, T) ||
        !make_map_f32_3d(&p.mdq, a.dq ? a.dq : static_cast<float *>(a.dq_out), D, rows, a.BH, T))
      return cudaErrorInvalidValue;
    p.fused = a.xq_part != nullptr;
    if (p.fused && (!make_map_bf16_3d(&p.mxq, a.xq_part, D, rows, a.BH, T) ||
                    !make_map_bf16_3d(&p.mdqo, a.dq_out, D, rows, a.BH, T)))
      return cudaErrorInvalidValue;
    if (a.P > 0) {
      if (!make_map_bf16_3d(&p.mkp, a.k_prefix, D, (uint64_t)a.P, a.BH, T) ||
          !make_map_bf16_3d(&p.mvp, a.v_prefix, D, (uint64_t)a.P, a.BH, T))
        return cudaErrorInvalidValue;
      p.P = a.P;
    }
    p.meta_k = a.meta_k;
    p.meta_v = a.meta_v;
    p.alpha = a.alpha;
    p.dq = a.dq;
    p.lse = a.lse;
    p.lse_in = a.lse_in;
    p.Dterm = a.Dterm;
    p.dmeta_k = a.dmeta_k;
    p.dmeta_v = a.dmeta_v;
    p.dalpha = a.dalpha;
    p.status = a.status;
    p.H = a.H;
    p.L = a.L;
    p.M = a.M;
    p.window = a.window;
    p.scale = a.scale;
    p.BH = a.BH;
    e = cudaFuncSetAttribute(tc_swa_bwd_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int sms = 148;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int nwork = ntiles * a.BH;
    tc_swa_bwd_q_kernel<<<nwork < sms ? nwork : sms, NT_Q, SMEM_BYTES, s>>>(p);
    return cudaGetLastError();
  }
  KVParams p;
  memset(&p, 0, sizeof(p));
  if (!make_map_bf16_3d(&p.mq, a.q, D, rows, a.BH, T) || !make_map_bf16_3d(&p.mk, a.k, D, rows, a.BH, T) ||
      !make_map_bf16_3d(&p.mv, a.v, D, rows, a.BH, T) || !make_map_bf16_3d(&p.mo, a.dout, D, rows, a.BH, T) ||
      !make_map_f32_3d(&p.mdk, a.dk ? a.dk : static_cast<float *>(a.dk_out), D, rows, a.BH, T) ||
      !make_map_f32_3d(&p.mdv, a.dv ? a.dv : static_cast<float *>(a.dv_out), D, rows, a.BH, T))
    return cudaErrorInvalidValue;
  p.fused = a.xq_part != nullptr;
  if (p.fused && (!make_map_bf16_3d(&p.mxk, a.xk_part, D, rows, a.BH, T) ||
                  !make_map_f32_3d(&p.mdvg, a.dv_gla, D, rows, a.BH, T) ||
                  !make_map_bf16_3d(&p.mdko, a.dk_out, D, rows, a.BH, T) ||
                  !make_map_bf16_3d(&p.mdvo, a.dv_out, D, rows, a.BH, T)))
    return cudaErrorInvalidValue;
  if (a.P > 0) {
    if (!make_map_bf16_3d(&p.mkp, a.k_prefix, D, (uint64_t)a.P, a.BH, T) ||
        !make_map_bf16_3d(&p.mvp, a.v_prefix, D, (uint64_t)a.P, a.BH, T))
      return cudaErrorInvalidValue;
    p.P = a.P;
    p.dk_prefix = static_cast<__nv_bfloat16 *>(a.dk_prefix);
    p.dv_prefix = static_cast<__nv_bfloat16 *>(a.dv_prefix);
  }
  p.alpha = a.alpha;
  p.lse = a.lse_in ? a.lse_in : a.lse;
  p.Dterm = a.Dterm;
  p.dk = a.dk;
  p.dv = a.dv;
  p.status = a.status;
  p.H = a.H;
  p.L = a.L;
  p.window = a.window;
  p.scale = a.scale;
  e = cudaFuncSetAttribute(tc_swa_bwd_kv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  p.BH = a.BH;
  {
    int sms = 148;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int nwork = (ntiles + (a.P > 0 ? 1 : 0)) * a.BH;
    tc_swa_bwd_kv_kernel<<<nwork < sms ? nwork : sms, NT_KV, SMEM_BYTES, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace lz
