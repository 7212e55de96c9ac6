// Tensor-core (tcgen05 / TMEM / TMA) forward of the Lizard hybrid layer,
// bf16 activations, dk = dv = 128, window <= 128, M <= 16.
//
// One CTA walks one (batch, head) sequence in tiles of T = 128 tokens, i.e.
// two 64-token chunks per tile with the cumulative gate absorbed once per
// tile.  The CTA has two warpgroups (256 threads); warps w and w + 4 address
// the same 32 TMEM lanes, so thread = tile row (lane) in both groups and the
// groups split each row's work.  The decay factors of every tile come from
// a separate, fully parallel pass (gate_prep_kernel):
//   E_t = exp(sum_{s>t} -a_s) = exp(b_t - r) (bf16) and exp(r) (fp32).
// Per tile:
//
//   TMA     X_q, X_k, V, E of the tile and K of the previous tile, 128-byte
//           swizzled; later V of the previous tile.
//   MMA 1   L  = X_q [K_prev ; X_k]^T            (window logits, 128 x 256)
//           Zq = X_q W_q, Zk = X_k W_k           (feature-map projections)
//   rows    anchor softmax over the band of L (each warp visits only the
//           <= 5 32-column chunks its rows can see; group 1 takes alternate
//           chunks, group 0 the others and the M meta logits; maxima and
//           sums meet in shared memory) -> P^ = exp(l - max) into TMEM;
//           group h builds half h of phi = [softmax(z), softmax(-z)]:
//           Qt = phi_q E l/alpha (TMEM), Kt = phi_k / E (shared memory);
//           thread = key dimension i: S' = diag(exp r) S in TMEM, and its
//           bf16 copy in shared memory (column half per group).
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
// mode 1: the decay factors in fp32 by a row-wise suffix scan of the gate
// logits, phi_k, state update only) gives each segment's local end
// state and total log-decay, a combine kernel chains them into each
// segment's start state, and the full pass runs all segments in parallel.
//
// A sequence with a tile whose in-tile log-decay spread exceeds kMaxSpread
// in some key dimension (the gate prep marks it) cannot go through the
// log-space absorption: its E = exp(b - r) leaves the exponent range.  The
// CTA of its first segment then walks every tile for the anchor branch alone
// and afterwards runs the GLA recurrence token by token in fp32 over the
// whole sequence (exact for any decay), adding it to o (exact_gla_sequence);
// the sequence's other CTAs return at once.  Every mbarrier wait is
// bounded; a wait that gives up sets the TIMEOUT bit and the CTA stops,
// frees its TMEM and returns.
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
  CUtensorMap mkp, mvp;     // key / value prefix [BH][P][D] (P > 0 only)
  CUtensorMap me;           // mode 1: fp32 decay factors E [BH][L][D] (loads)
  CUtensorMap msnap;        // training full pass: the state copies [BH*ntiles][D][D] bf16 (stores)
  const float *wq, *wk, *meta_k, *meta_v, *alpha, *state_in;
  __nv_bfloat16 *o;
  float *state_out, *lse;
  uint32_t *status;
  const float *seg_start;   // [BH][nseg][D][D] start state of each segment (nseg > 1)
  float *seg_state;         // mode 1: [BH][nseg][D][D] local end state (zero start)
  float *seg_decay;         // mode 1: [BH][nseg][D] summed log-decay of the segment
  __nv_bfloat16 *snap;      // mode 1 with nseg == 1, or a training full pass: [BH][ntiles][D][D]
                            // bf16 S' - 1 S'[0] of every tile (the backward's copies)
  float *snap_r0;           // ... and [BH][ntiles][D] fp32 row 0 of S' (the part taken out of every row)
  float *state_keep;        // training full pass: [BH][D][D] fp32 final state for the backward, or null
  float *lse_keep;          // training full pass: [BH][L] copy of lse for the backward, or null
  const float *gate_r;      // [BH][ntiles][D] log-decay r of every tile (gate_prep_kernel)
  const float *gate_e32;    // mode 1: [BH][L][D] fp32 decay factors E, loaded through `me` (mode 0 loads bf16 E as the G tiles)
  const float *kap_g;       // mode 1 with copies: incoming final-state gradient G [BH][D][D], or null
  float *kap;               // ... and [BH][2][D]: the column halves of sum_v G[i][v] S_L[i][v]
  int H, L, M, window, branch;
  int mode;                 // 0: full forward, 1: state pass
  int nseg, tiles_per_seg;
  int P;                    // prefix tokens before token 0 (0: none)
  int inject;               // test hook: first wait on a barrier nothing completes
  // Wide decay: seqflag[bh] != 0 marks a sequence whose GLA branch runs as
  // the exact recurrence (exact_gla_sequence) instead; null: none.  Its
  // inputs: the activations themselves.
  const uint32_t *seqflag;
  const __nv_bfloat16 *xq, *xk, *xv, *xg;
  int scalar_gate;
  float inv_tau, scale;
  // stage-1 loss (target null: off): dmse = mse_grad (o - target), *loss += mse_loss sum (o - target)^2
  const __nv_bfloat16 *target;
  __nv_bfloat16 *dmse;
  float *loss;
  float mse_grad, mse_loss;
};


// defer_xq: leave X_q's two loads to issue_xq_loads (its region is still being
// read by a store); the barrier expects their bytes all the same.
__device__ __forceinline__ void issue_tile_loads(const Params &p, unsigned char *sm, float *s_rt, uint64_t *bar,
                                                 int bh, int t0, bool full, bool defer_xq = false) {
  mbar_expect_tx(bar, (full ? 5 : 4) * TILE + (p.gate_r ? D * 4 : 0));
  if (p.gate_r)   // the tile's log-decays r (one 512-byte row)
    bulk_load_1d(s_rt, p.gate_r + ((size_t)bh * ((p.L + T - 1) / T) + t0 / T) * D, D * 4, bar);
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    if (full) {
      if (!defer_xq) tma_load_3d(sm + R_XQ + r * REG, &p.mq, bar, 64 * r, t0, bh);
      // keys of the previous tile; before token 0, the prefix (its rows
      // before the first prefix token read as zero)
      if (t0 == 0 && p.P > 0)
        tma_load_3d(sm + R_KP + r * REG, &p.mkp, bar, 64 * r, p.P - T, bh);
      else
        tma_load_3d(sm + R_KP + r * REG, &p.mk, bar, 64 * r, t0 - T, bh);
      tma_load_3d(sm + R_G + r * REG, &p.mg, bar, 64 * r, t0, bh);
    }
    tma_load_3d(sm + R_XK + r * REG, &p.mk, bar, 64 * r, t0, bh);
    tma_load_3d(sm + R_V + r * REG, &p.mv, bar, 64 * r, t0, bh);
  }
  if (!full)   // state pass: the fp32 decay factors, dimensions 0..63 over X_q, 64..127 over G (unused there)
    for (int bx = 0; bx < 4; ++bx)
      tma_load_3d(sm + (bx < 2 ? R_XQ : R_G) + (bx & 1) * 16384, &p.me, bar, 32 * bx, t0, bh);
}

__device__ __forceinline__ void issue_xq_loads(const Params &p, unsigned char *sm, uint64_t *bar, int bh, int t0) {
#pragma unroll
  for (int r = 0; r < 2; ++r) tma_load_3d(sm + R_XQ + r * REG, &p.mq, bar, 64 * r, t0, bh);
}

// Qt for dimensions 64 h .. 64 h + 63: phi_q E gscale, bf16 pairs into TMEM.
// With `sum`, returns the sum of the values (before their bf16 rounding,
// whose share of the sum is of the order of the MMAs' own rounding).
__device__ __forceinline__ float qt_half(unsigned char *sm, uint32_t tl, int row, int h, float gscale, bool sum) {
  float ph[F];
  const float s = feature_half(tl + C_ZQ, h, ph) * gscale;
  float acc[2] = {0.f, 0.f};
#pragma unroll
  for (int c16 = 0; c16 < 4; ++c16) {     // 16 dims = 8 TMEM columns
    float e16[16];
    unpack8(*chunk_ptr(sm, R_G, row, 8 * h + 2 * c16), e16);
    unpack8(*chunk_ptr(sm, R_G, row, 8 * h + 2 * c16 + 1), e16 + 8);
    uint32_t r8[8];
#pragma unroll
    for (int u = 0; u < 16; u += 2) {
      const float a = ph[16 * c16 + u] * e16[u] * s, b = ph[16 * c16 + u + 1] * e16[u + 1] * s;
      r8[u / 2] = pack_bf16(a, b);
      if (sum) {
        acc[0] += a;
        acc[1] += b;
      }
    }
    tmem_st8(tl + C_QT + 32 * h + 8 * c16, r8);
  }
  return acc[0] + acc[1];
}

// Kt for dimensions 64 h .. 64 h + 63: phi_k / E, bf16 into shared memory
// over X_k.  E comes as bf16 from the gate region (full pass) or as fp32
// tiles over X_q | G (state pass, which also writes the rounding remainder
// Kt - bf16(Kt) over the K_prev region, so that its state update runs on
// hi + lo).  Rows past L (where E is zero) get Kt = 0.
__device__ __forceinline__ void kt_half(unsigned char *sm, uint32_t tl, int row, int h, bool e_fp32, bool valid) {
  float ph[F];
  float s = feature_half(tl + C_ZK, h, ph);   // warp-collective TMEM loads: every lane
  if (!valid) s = 0.f;
#pragma unroll
  for (int c16 = 0; c16 < 4; ++c16) {
    float e16[16], k16[16];
    if (e_fp32) {
      unsigned char *es = sm + (h == 0 ? R_XQ : R_G);
#pragma unroll
      for (int u = 0; u < 16; u += 4) {
        const float4 e4 = *f32_stage_ptr(es, row, 16 * c16 + u);
        e16[u] = e4.x;
        e16[u + 1] = e4.y;
        e16[u + 2] = e4.z;
        e16[u + 3] = e4.w;
      }
    } else {
      unpack8(*chunk_ptr(sm, R_G, row, 8 * h + 2 * c16), e16);
      unpack8(*chunk_ptr(sm, R_G, row, 8 * h + 2 * c16 + 1), e16 + 8);
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) k16[u] = valid ? __fdividef(ph[16 * c16 + u] * s, e16[u]) : 0.f;
    if (e_fp32) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint4 hi, lo;
        split8(k16 + 8 * hh, hi, lo);
        *chunk_ptr(sm, R_XK, row, 8 * h + 2 * c16 + hh) = hi;
        *chunk_ptr(sm, R_KP, row, 8 * h + 2 * c16 + hh) = lo;
      }
    } else {
      *chunk_ptr(sm, R_XK, row, 8 * h + 2 * c16) = pack8(k16);
      *chunk_ptr(sm, R_XK, row, 8 * h + 2 * c16 + 1) = pack8(k16 + 8);
    }
  }
}

// The GLA branch of one whole sequence as the plain recurrence, for a
// sequence whose decay is too wide for the tile absorption:
//   S_t = diag(exp a_t) S_{t-1} + phi_k(k_t) v_t^T,   o_t += S_t^T phi_q(q_t)
// in fp32 (the English summary's state update, section 2.A), exact for any
// decay.  Thread (v = tid / 2, half = tid % 2) updates S[64 half .. 64 half +
// 63][v] (fp32, in shared memory); the tokens go in chunks of 32, whose feature maps (from
// the bf16 weights already staged at wq_s / wk_s), decays and values are
// formed into shared memory first (warp per token).  o gets the GLA part
// added (add: the anchor pass of this CTA wrote it) or written (the anchor
// branch is off); state_out is written.
constexpr int XC = 32;   // tokens per chunk of the exact recurrence
__device__ __forceinline__ void exact_gla_sequence(const Params &p, unsigned char *buf, const unsigned char *wq_s,
                                                const unsigned char *wk_s, int bh, bool add) {
  float *PQ = reinterpret_cast<float *>(buf);          // [XC][D] phi_q
  float *PK = PQ + XC * D;                             // [XC][D] phi_k
  float *DEC = PK + XC * D;                            // [XC][D] exp(a)
  float *VV = DEC + XC * D;                            // [XC][D] v
  float *OB = VV + XC * D;                             // [XC][D] this chunk's GLA output
  float *S = OB + XC * D;                              // [D][D] the state, row = key dimension
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int v = tid >> 1, half = tid & 1;
  for (int e = tid; e < D * D; e += NTHREADS) S[e] = p.state_in ? p.state_in[(size_t)bh * D * D + e] : 0.f;
  float *Sc = S + 64 * half * D + v;                   // this thread's column: Sc[ii * D]
  for (int c0 = 0; c0 < p.L; c0 += XC) {
    const int n = min(XC, p.L - c0);
    // feature maps, decays and values of the chunk's tokens
    for (int tt = warp; tt < n; tt += NTHREADS / 32) {
      const size_t rowoff = ((size_t)bh * p.L + c0 + tt) * D;
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const __nv_bfloat16 *x = (m == 0 ? p.xq : p.xk) + rowoff;
        const unsigned char *W = m == 0 ? wq_s : wk_s;
        float xr[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) xr[j] = __bfloat162float(x[lane + 32 * j]);
        float z0 = 0.f, z1 = 0.f;   // z_f = sum_i x_i W[i][f], f = lane, lane + 32
#pragma unroll
        for (int j = 0; j < 4; ++j)
          for (int il = 0; il < 32; ++il) {
            const float xi = __shfl_sync(0xffffffffu, xr[j], il);
            const int i = 32 * j + il;
            z0 = fmaf(xi, __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(W + sw128_offset(i, lane))), z0);
            z1 = fmaf(xi, __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(W + sw128_offset(i, lane + 32))),
                      z1);
          }
        const float mx = warp_max(fmaxf(z0, z1)), mn = -warp_max(-fminf(z0, z1));
        const float p0 = expf(z0 - mx), p1 = expf(z1 - mx), n0 = expf(mn - z0), n1 = expf(mn - z1);
        const float ip = 1.f / warp_sum(p0 + p1), in_ = 1.f / warp_sum(n0 + n1);
        float *dst = (m == 0 ? PQ : PK) + tt * D;
        dst[lane] = p0 * ip;
        dst[lane + 32] = p1 * ip;
        dst[64 + lane] = n0 * in_;
        dst[96 + lane] = n1 * in_;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = lane + 32 * j;
        const float g = __bfloat162float(p.scalar_gate ? p.xg[(size_t)bh * p.L + c0 + tt] : p.xg[rowoff + i]);
        const float a = (fminf(g, 0.f) - log1pf(expf(-fabsf(g)))) * p.inv_tau;   // logsigmoid(g) / tau
        DEC[tt * D + i] = expf(a);
        VV[tt * D + i] = __bfloat162float(p.xv[rowoff + i]);
      }
    }
    __syncthreads();
    for (int tt = 0; tt < n; ++tt) {
      const float vt = VV[tt * D + v];
      const float4 *dec = reinterpret_cast<const float4 *>(DEC + tt * D + 64 * half);
      const float4 *pk = reinterpret_cast<const float4 *>(PK + tt * D + 64 * half);
      const float4 *pq = reinterpret_cast<const float4 *>(PQ + tt * D + 64 * half);
      float o = 0.f;
#pragma unroll 4
      for (int q4 = 0; q4 < 16; ++q4) {
        const float4 d4 = dec[q4], k4 = pk[q4], f4 = pq[q4];
        float *sc = Sc + 4 * q4 * D;
        const float s0 = fmaf(d4.x, sc[0], k4.x * vt), s1 = fmaf(d4.y, sc[D], k4.y * vt);
        const float s2 = fmaf(d4.z, sc[2 * D], k4.z * vt), s3 = fmaf(d4.w, sc[3 * D], k4.w * vt);
        sc[0] = s0;
        sc[D] = s1;
        sc[2 * D] = s2;
        sc[3 * D] = s3;
        o = fmaf(s0, f4.x, fmaf(s1, f4.y, fmaf(s2, f4.z, fmaf(s3, f4.w, o))));
      }
      o += __shfl_xor_sync(0xffffffffu, o, 1);
      if (half == 0) OB[tt * D + v] = o;
    }
    __syncthreads();
    for (int e = tid; e < n * D; e += NTHREADS) {
      __nv_bfloat16 *dst = p.o + ((size_t)bh * p.L + c0) * D + e;
      *dst = __float2bfloat16_rn((add ? __bfloat162float(*dst) : 0.f) + OB[e]);
    }
    __syncthreads();
  }
  if (p.state_out)
    for (int e = tid; e < D * D; e += NTHREADS) p.state_out[(size_t)bh * D * D + e] = S[e];
  if (p.state_keep)
    for (int e = tid; e < D * D; e += NTHREADS) p.state_keep[(size_t)bh * D * D + e] = S[e];
}

// Named barriers (id 0 is __syncthreads).
constexpr int BAR_A = 1;       // both groups' row maxima written
constexpr int BAR_B = 2;       // both groups' row sums written, all logits read

// Kernel instances: the full pass, the full pass that also forms the
// stage-1 loss (p.target set), the state pass, and the two full passes that
// also keep the backward's tensors (p.snap set: K_TRAIN, and K_TRAIN_LOSS
// for the stage-1 step).  Each keeps its own register budget.
constexpr int K_FULL = 0, K_LOSS = 1, K_STATE = 2, K_TRAIN = 3, K_TRAIN_LOSS = 4;
template <int KIND>
__global__ void __launch_bounds__(NTHREADS, 1) tc_fwd_kernel(const __grid_constant__ Params p) {
  constexpr bool LOSS = KIND == K_LOSS || KIND == K_TRAIN_LOSS;
  constexpr bool TRAIN = KIND == K_TRAIN || KIND == K_TRAIN_LOSS;
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(16) float s_mk[MAXM][D];
  __shared__ __align__(16) float s_mv[MAXM][D];
  __shared__ float s_ml[MAXM][T];     // meta logits, then their mixing weights, per row
  __shared__ float s_dec[D];
  __shared__ float s_oscale[T];
  __shared__ float s_pmax[2][T], s_psum[2][T];   // per-group row maxima and sums of the softmax
  __shared__ uint64_t bar_tma, bar_vp, bar_m1, bar_m2, bar_m3;
  __shared__ uint32_t s_tmem;
  __shared__ int s_fail;
  __shared__ float s_mse[NTHREADS / 32];
  __shared__ __align__(16) float s_row0[D];   // row 0 of S' (state pass) or of S (full pass), taken out of the copies
  __shared__ __align__(16) float s_r0v[D];    // full pass, centred: row 0 of this tile's S'
  __shared__ float s_qsum[2][T];              // full pass, centred: each group's sum of its Qt dimensions
  __shared__ __align__(16) float s_rt[D];     // the tile's log-decays r (arrive with its loads)

  const int tid = threadIdx.x, warp = tid >> 5;
  const int wg = tid >> 7;                             // warpgroup
  const int row = tid & 127;                           // TMEM lane == tile row
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const int bh = blockIdx.x, h = bh % p.H, seg = blockIdx.y;
  const float alpha = p.alpha ? p.alpha[h] : 1.f;
  constexpr bool full = KIND != K_STATE;
  // A sequence marked for the exact recurrence: its first segment's CTA of
  // the full pass walks every tile for the anchor branch, then runs the GLA
  // branch exactly; its other CTAs (and state passes) have nothing to do.
  const bool marked = p.seqflag && p.seqflag[bh] != 0u;
  if (marked && (!full || seg > 0)) return;
  const bool gla = p.branch != 2 && !marked, swa = full && p.branch != 1;
  // Training: MMA 3 reads S' as the bf16 copy of S' - 1 S'[0] (rows less
  // their first; the epilogue adds back (sum_i Qt[i]) S'[0] in fp32), and
  // that copy goes to the backward as is, with one TMA store per tile.
  const bool centre = TRAIN && gla;
  const uint32_t sbase = smem_u32(sm);
  const int ntiles_all = (p.L + T - 1) / T;
  const int cbeg = marked ? 0 : seg * p.tiles_per_seg;
  const int cend = marked ? ntiles_all : min(ntiles_all, cbeg + p.tiles_per_seg);

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
  // the first tile's loads go out before the weights and meta tokens are staged
  if (tid == 0 && cbeg < cend && !p.inject) issue_tile_loads(p, sm, s_rt, &bar_tma, bh, cbeg * T, full);
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
  // meta tokens (groups of four are read, so rows up to the next multiple of
  // four are zero-filled)
  const int m_rows = (p.M + 3) / 4 * 4;
  for (int e = tid; e < m_rows * D; e += NTHREADS) {
    const int m = e / D;
    s_mk[m][e % D] = m < p.M ? p.meta_k[(size_t)h * p.M * D + e] : 0.f;
    s_mv[m][e % D] = (m < p.M && p.meta_v) ? p.meta_v[(size_t)h * p.M * D + e] : 0.f;
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (p.inject) {   // test hook: bar_m3 completes only after an MMA, so this wait runs out
    const bool ok = mbar_wait(&bar_m3, 0, p.status, ST_TIMEOUT, 1u << 14);
    if (__syncthreads_or(!ok)) s_fail = 1;
    __syncthreads();
  }
  const uint32_t tb = s_tmem;
  const uint32_t tl = tb + lane_off;

  // initial state -> TMEM columns [0, 128), lane = key dimension; each
  // group writes one half of the columns
  {
    const float *src = nullptr;
    if (full && p.nseg > 1 && gla) src = p.seg_start + (((size_t)bh * p.nseg + seg) * D + row) * D;
    else if (full && p.state_in) src = p.state_in + ((size_t)bh * D + row) * D;
    else if (p.snap && p.state_in) src = p.state_in + ((size_t)bh * D + row) * D;
#pragma unroll
    for (int c = 64 * wg; c < 64 * wg + 64; c += 8) {
      uint32_t r[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) r[u] = __float_as_uint(src ? src[c + u] : 0.f);
      tmem_st8(tl + C_S + c, r);
      if (centre && row == 0)   // row 0 of the start state: the first tile's centre
#pragma unroll
        for (int u = 0; u < 8; ++u) s_row0[c + u] = __uint_as_float(r[u]);
    }
    tmem_st_wait();
  }

  uint32_t *err = p.status;
  float tot_decay = 0.f;                      // state pass: summed log-decay of dimension `row` (group 0)
  const uint32_t id_128 = idesc_bf16(128, 128, 0, 0);
  const uint32_t id_z = idesc_bf16(128, 64, 0, 1);
  const uint32_t id_mn = idesc_bf16(128, 128, 0, 1);
  const uint32_t id_st = idesc_bf16(128, 128, 1, 1);

  float mse_acc = 0.f;                        // this thread's share of sum (o - target)^2
  const int cstop = s_fail ? cbeg : cend;
  for (int c = cbeg; c < cstop; ++c) {
    const uint32_t par = (c - cbeg) & 1;
    const int t0 = c * T;
    const int tq = t0 + row;                  // this thread's query token
    const bool qvalid = tq < p.L;
    if (LOSS && full && qvalid)               // the epilogue's target half-row, toward L2 early
      asm volatile("prefetch.global.L2 [%0];" ::"l"(p.target + ((size_t)bh * p.L + tq) * D + 64 * wg));

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

    if (full) {
      // ---- full pass: the anchor softmax split between the groups (group 1
      //      the band chunks ch_lo, ch_lo + 2, ..., group 0 the others and
      //      the meta logits), then one half of phi_q, phi_k per group
      ok &= mbar_wait(&bar_m1, par, err, ST_TIMEOUT);
      tc_fence_after();
      if (wg == 1 && gla) s_dec[row] = __expf(s_rt[row]);   // exp(r)
      float lsum = 1.f, mx = 0.f;                 // row normaliser and max (scaled logits)
      // Logit column cl holds key t0 - T + cl.  Row r sees columns
      // [r + T + 1 - window, r + T] (and keys >= -P, P the prefix length),
      // so warp w4 only visits 32-column chunks w4 + (T + 1 - window) / 32
      // .. w4 + 4, and only the first and last of those need the band mask.
      const int w4 = warp & 3;
      const int cbase = t0 - T;
      const int lo_c = max(tq - p.window + 1, -p.P) - cbase, hi_c = tq - cbase;
      int ch_lo = (32 * w4 + T + 1 - p.window) >> 5;
      if (cbase < 0) ch_lo = max(ch_lo, (T - p.P) >> 5);
      const int ch_hi = w4 + 4;
      const int in_lo = 32 * w4 + 31 + T + 1 - p.window;   // interior chunk: 32 ch >= in_lo
      const int ch_first = ch_lo + 1 - wg;                 // this group's first chunk
      // The band's chunks alternate between the groups (group 1 from ch_lo);
      // an odd count's last chunk is halved: group 1 takes its first 16
      // columns, group 0 (which also has the meta logits) the other 16.
      const bool split = ((ch_hi - ch_lo) & 1) == 0;
      const int full_hi = split ? ch_hi - 1 : ch_hi;       // last chunk taken whole
      const int hcol = 32 * ch_hi + 16 * (1 - wg);          // this group's half of a split chunk
      const bool hinner = hcol >= in_lo && hcol + 15 <= 32 * w4 + T && hcol + cbase >= -p.P;
      const int lo_h = hinner ? -1 : lo_c - hcol, hi_h = hinner ? 16 : hi_c - hcol;   // the half's exponent mask
      uint32_t pk[2][16], pkh[8];
      if (swa) {
        float pmax = kNegBig;
        if (wg == 0 && p.M > 0) {
          // meta logits q . mk_m (scaled) into s_ml: this warp's 32 rows by mma.sync
          rowdots_mma(sm, R_XQ, 32 * w4, s_mk, p.M, s_ml, threadIdx.x & 31);
          __syncwarp();
          for (int m = 0; m < p.M; ++m) {
            const float l = s_ml[m][row] * p.scale;
            s_ml[m][row] = l;
            pmax = fmaxf(pmax, l);
          }
        }
        if (split) {
          float v[16];
          tmem_ld16(tl + C_L + hcol, v);
          float m4[4] = {kNegBig, kNegBig, kNegBig, kNegBig};
#pragma unroll
          for (int u = 0; u < 16; ++u)
            if (hinner || (hcol + u >= lo_c && hcol + u <= hi_c)) m4[u & 3] = fmaxf(m4[u & 3], v[u]);
          const float cm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
          if (cm > kNegBig) pmax = fmaxf(pmax, cm * p.scale);
        }
        for (int ch = ch_first; ch <= full_hi; ch += 2) {
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
          if (cm > kNegBig) pmax = fmaxf(pmax, cm * p.scale);
        }
        s_pmax[wg][row] = pmax;
      }
      bar_sync(BAR_A, NTHREADS);
      if (swa) {
        mx = fmaxf(s_pmax[0][row], s_pmax[1][row]);
        // P^ = exp(l - max), packed and held until both groups have read
        // their logits (P^ column 16 ch overlays logit chunk ch / 2)
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
        if (split) {
          float v[16];
          tmem_ld16(tl + C_L + hcol, v);
#pragma unroll
          for (int u = 0; u < 16; u += 2) {
            float e0 = __expf(fmaf(v[u], p.scale, -mx));
            float e1 = __expf(fmaf(v[u + 1], p.scale, -mx));
            e0 = (u >= lo_h && u <= hi_h) ? e0 : 0.f;
            e1 = (u + 1 >= lo_h && u + 1 <= hi_h) ? e1 : 0.f;
            s4[(u >> 1) & 3] += e0 + e1;
            pkh[u / 2] = alpha != 0.f ? pack_bf16(e0, e1) : 0u;
          }
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int ch = ch_first + 2 * k;
          if (ch > full_hi) continue;
          float v[32];
          tmem_ld32(tl + C_L + ch * 32, v);
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
            pk[k][u / 2] = alpha != 0.f ? pack_bf16(e0, e1) : 0u;
          }
        }
        float psum = (s4[0] + s4[1]) + (s4[2] + s4[3]);
        if (wg == 0)
          for (int m = 0; m < p.M; ++m) {
            const float e = __expf(s_ml[m][row] - mx);
            psum += e;
            s_ml[m][row] = e;
          }
        s_psum[wg][row] = psum;
      }
      bar_sync(BAR_B, NTHREADS);
      if (swa) {
        lsum = s_psum[0][row] + s_psum[1][row];
        if (!qvalid) lsum = 1.f;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int ch = ch_first + 2 * k;
          if (ch > full_hi) continue;
          tmem_st8(tl + C_P + ch * 16, pk[k]);
          tmem_st8(tl + C_P + ch * 16 + 8, pk[k] + 8);
        }
        if (split) tmem_st8(tl + C_P + ch_hi * 16 + 8 * (1 - wg), pkh);
        uint32_t zero[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        for (int ch = wg; ch < 8; ch += 2) {   // chunks outside the band: P = 0
          if (ch >= ch_lo && ch <= ch_hi) continue;
          tmem_st8(tl + C_P + ch * 16, zero);
          tmem_st8(tl + C_P + ch * 16 + 8, zero);
        }
        float *lse_keep = TRAIN ? p.lse_keep : nullptr;
        if (wg == 0 && qvalid && (p.lse || lse_keep)) {
          const float lse = mx + logf(lsum);
          if (p.lse) p.lse[(size_t)bh * p.L + tq] = lse;
          if (lse_keep) lse_keep[(size_t)bh * p.L + tq] = lse;
        }
      }
      // GLA operands carry l/alpha so that one accumulator holds both terms
      const bool mixed = swa && alpha != 0.f;
      const float gscale = mixed ? lsum / alpha : 1.f;
      if (wg == 0) {
        s_oscale[row] = mixed ? alpha / lsum : 1.f;
        if (swa) {
          const float mscale = mixed ? alpha / lsum : 0.f;   // meta-value weight per exp
          for (int m = 0; m < p.M; ++m) s_ml[m][row] *= mscale;
        }
      }
      const float qs = qt_half(sm, tl, row, wg, gscale, centre);
      if (centre) s_qsum[wg][row] = qs;
      kt_half(sm, tl, row, wg, false, qvalid);
    } else {
      // ------ state pass: phi_k half per group, with the fp32 decay factors
      //        (from gate_prep_kernel) that came with the tile's loads ---
      if (wg == 0) {   // thread row = key dimension: the tile's decay
        const float r = s_rt[row];
        s_dec[row] = __expf(r);
        tot_decay += r;
      }
      ok &= mbar_wait(&bar_m1, par, err, ST_TIMEOUT);
      tc_fence_after();
      kt_half(sm, tl, row, wg, true, qvalid);
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
      if (swa && t0 == 0 && p.P > 0) {
        tma_load_3d(sm + R_G, &p.mvp, &bar_vp, 0, p.P - T, bh);
        tma_load_3d(sm + R_G + REG, &p.mvp, &bar_vp, 64, p.P - T, bh);
      } else if (swa) {
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
          if (centre) {
            // S'[0] = exp(r_0) S[0], S[0] staged at the end of the previous
            // tile (row 0 itself comes out exactly zero); row 0 in fp32 to
            // the epilogue and to the backward
            const float d0 = s_dec[0];
            const float4 *r0 = reinterpret_cast<const float4 *>(s_row0 + c16 * 16);
            float w[16];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const float4 x = r0[q4];
              w[4 * q4] = v[4 * q4] - __fmul_rn(x.x, d0);
              w[4 * q4 + 1] = v[4 * q4 + 1] - __fmul_rn(x.y, d0);
              w[4 * q4 + 2] = v[4 * q4 + 2] - __fmul_rn(x.z, d0);
              w[4 * q4 + 3] = v[4 * q4 + 3] - __fmul_rn(x.w, d0);
            }
            *chunk_ptr(sm, R_XQ, i, 2 * c16) = pack8(w);
            *chunk_ptr(sm, R_XQ, i, 2 * c16 + 1) = pack8(w + 8);
            if (i == 0) {
              const size_t tile = (size_t)bh * ntiles_all + c;
              float4 *d4 = reinterpret_cast<float4 *>(p.snap_r0 + tile * D + c16 * 16);
              float4 *s4 = reinterpret_cast<float4 *>(s_r0v + c16 * 16);
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                const float4 x = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
                d4[q4] = x;
                s4[q4] = x;
              }
            }
          } else {
            *chunk_ptr(sm, R_XQ, i, 2 * c16) = pack8(v);
            *chunk_ptr(sm, R_XQ, i, 2 * c16 + 1) = pack8(v + 8);
          }
        } else if (p.snap && i == 0) {
#pragma unroll
          for (int u = 0; u < 16; ++u) s_row0[c16 * 16 + u] = v[u];
        }
      }
      if (!full && p.snap) {
        // The backward's copy of S', row-major [i][v], stored as S' - 1 S'[0]
        // in bf16 with row 0 in fp32: the rows of S' share a large common
        // part (the feature map is close to uniform), which a plain bf16
        // copy would round element by element.
        tmem_st_wait();
        __syncthreads();
        const size_t tile = (size_t)bh * ntiles_all + c;
        for (int c16 = 4 * wg; c16 < 4 * wg + 4; ++c16) {
          float v[16];
          tmem_ld16(tl + C_S + c16 * 16, v);
#pragma unroll
          for (int u = 0; u < 16; ++u) v[u] -= s_row0[c16 * 16 + u];
          uint4 *dst = reinterpret_cast<uint4 *>(p.snap + (tile * D + i) * D + c16 * 16);
          dst[0] = pack8(v);
          dst[1] = pack8(v + 8);
        }
        if (tid < D) p.snap_r0[tile * D + tid] = s_row0[tid];
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
      if (gla && !full)   // the state pass's Kt remainder
        for (int s = 0; s < 8; ++s) mma_ss(tb + C_S, desc_mn(sbase + R_KP, s), desc_mn(v, s), id_st, 1);
      mma_commit(&bar_m3);
      if (centre) {   // the backward's copy of S' - 1 S'[0]: the swizzled tile as it stands
        const int tile = bh * ntiles_all + c;
        tma_store_3d(&p.msnap, sm + R_XQ, 0, 0, tile);
        tma_store_3d(&p.msnap, sm + R_XQ + REG, 64, 0, tile);
        bulk_commit();
      }
    }
    // stage-1 loss: this thread's half-row of the target, in flight during MMA 3
    uint4 ytgt[8];
    if (LOSS && full && qvalid) {
      const uint4 *yp = reinterpret_cast<const uint4 *>(p.target + ((size_t)bh * p.L + tq) * D + 64 * wg);
#pragma unroll
      for (int u = 0; u < 8; ++u) ytgt[u] = yp[u];
    }
    ok = mbar_wait(&bar_m3, par, err, ST_TIMEOUT);
    if (__syncthreads_or(!ok)) { s_fail = 1; break; }
    tc_fence_after();
    if (tid == 0 && c + 1 < cend) {
      issue_tile_loads(p, sm, s_rt, &bar_tma, bh, t0 + T, full, centre);
      if (centre) {
        bulk_wait_read();   // the copy's store has read X_q's place
        issue_xq_loads(p, sm, &bar_tma, bh, t0 + T);
      }
    }

    // ---------------------------- epilogue (column half per group) ---
    if (full) {
      // tcgen05.ld is warp-collective: every lane loads, valid rows store
      const size_t roff = ((size_t)bh * p.L + (qvalid ? tq : 0)) * D;
      const float oscale = s_oscale[row];
      const float qs = centre ? s_qsum[0][row] + s_qsum[1][row] : 0.f;   // (sum_i Qt[i]) S'[0] left out of MMA 3
#pragma unroll(LOSS ? 4 : 1)
      for (int k4 = 0; k4 < 4; ++k4) {
        const int c16 = 4 * wg + k4;
        float v[16];
        tmem_ld16(tl + C_O + c16 * 16, v);
        if (centre) {
          const float4 *r4 = reinterpret_cast<const float4 *>(s_r0v + c16 * 16);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const float4 x = r4[q4];
            v[4 * q4] = fmaf(qs, x.x, v[4 * q4]);
            v[4 * q4 + 1] = fmaf(qs, x.y, v[4 * q4 + 1]);
            v[4 * q4 + 2] = fmaf(qs, x.z, v[4 * q4 + 2]);
            v[4 * q4 + 3] = fmaf(qs, x.w, v[4 * q4 + 3]);
          }
        }
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
        if (qvalid && p.o) {
          uint4 *dst = reinterpret_cast<uint4 *>(p.o + roff + c16 * 16);
          dst[0] = pack8(v);
          dst[1] = pack8(v + 8);
        }
        if (LOSS && qvalid) {       // stage-1 loss: (o - y)^2 and dL/do from the fp32 o
          float y[16];
          unpack8(ytgt[2 * k4], y);
          unpack8(ytgt[2 * k4 + 1], y + 8);
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const float d = v[u] - y[u];
            mse_acc = fmaf(d, d, mse_acc);
            y[u] = d * p.mse_grad;
          }
          uint4 *dd = reinterpret_cast<uint4 *>(p.dmse + roff + c16 * 16);
          dd[0] = pack8(y);
          dd[1] = pack8(y + 8);
        }
      }
    }
    if (centre && (warp & 3) == 0 && c + 1 < cend) {
      // row 0 of the state this tile leaves: the next tile's centre
      for (int c16 = 4 * wg; c16 < 4 * wg + 4; ++c16) {
        float v[16];
        tmem_ld16(tl + C_S + c16 * 16, v);
        if (row == 0) {
          float4 *d4 = reinterpret_cast<float4 *>(s_row0 + c16 * 16);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) d4[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  }

  if (LOSS && full) {       // one atomic per CTA
    const float t = warp_sum(mse_acc);
    if ((tid & 31) == 0) s_mse[warp] = t;
    __syncthreads();
    if (tid == 0) {
      float tot = 0.f;
      for (int w = 0; w < NTHREADS / 32; ++w) tot += s_mse[w];
      atomicAdd(p.loss, tot * p.mse_loss);
    }
  }
  float *sdst = nullptr, *skeep = nullptr;
  if (full && p.state_out && gla && seg == p.nseg - 1) sdst = p.state_out + ((size_t)bh * D + row) * D;
  if (full && p.state_keep && gla && seg == p.nseg - 1) skeep = p.state_keep + ((size_t)bh * D + row) * D;
  if (!full && p.seg_state) {
    sdst = p.seg_state + (((size_t)bh * p.nseg + seg) * D + row) * D;
    if (wg == 0) p.seg_decay[((size_t)bh * p.nseg + seg) * D + row] = tot_decay;
  }
  if (!s_fail && p.kap) {   // thread row = key dimension i, column half per group
    tc_fence_after();
    const float *G = p.kap_g + ((size_t)bh * D + row) * D;
    float part = 0.f;
    for (int c16 = 4 * wg; c16 < 4 * wg + 4; ++c16) {
      float v[16];
      tmem_ld16(tl + C_S + c16 * 16, v);
#pragma unroll
      for (int u = 0; u < 16; ++u) part = fmaf(G[c16 * 16 + u], v[u], part);
    }
    p.kap[((size_t)bh * 2 + wg) * D + row] = part;
  }
  if (!s_fail && (sdst || skeep)) {
    tc_fence_after();
    for (int c16 = 4 * wg; c16 < 4 * wg + 4; ++c16) {
      float v[16];
      tmem_ld16(tl + C_S + c16 * 16, v);
#pragma unroll
      for (int u = 0; u < 16; u += 4) {
        const float4 x = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
        if (sdst) *reinterpret_cast<float4 *>(sdst + c16 * 16 + u) = x;
        if (skeep) *reinterpret_cast<float4 *>(skeep + c16 * 16 + u) = x;
      }
    }
  }
  if (s_fail && tid == 0) {
    // let whatever was issued drain before the shared memory is released
    mbar_wait(&bar_tma, 0, nullptr, 0, 1u << 16);
  }
  if (centre && tid == 0) bulk_wait_all();   // the state copies' stores are complete
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 512);
  // every tile's loads and MMAs are done: the tile regions hold the exact
  // recurrence's buffers, the staged weights stay in place
  if (marked && !s_fail && p.branch != 2) exact_gla_sequence(p, sm, sm + R_WQ, sm + R_WK, bh, p.branch != 1);
}

}  // namespace

// Decay factors of every 128-token tile, computed apart from the kernels
// that use them so that they cost no time on a sequential critical path:
//   E_t = exp(sum_{s>t} -a_s) = exp(b_t - r)   (bf16 E16 and/or fp32 E32,
//                                               in the layout of g)
//   r   = sum_s a_s                            (fp32, per tile and dimension)
// with a = logsigmoid(g)/tau and s, t inside the tile.  One CTA per
// (64 key dimensions, tile, sequence): lane = two dimensions (each token row
// is one coalesced 128-byte read), warp w = tokens 16 w .. 16 w + 15, whose
// 16 loads are all in flight together; the warps' totals give each warp its
// carry from the later tokens.  Rows past L are not written (readers treat
// them as zero).  A tile whose spread r - b_0 exceeds kMaxSpread sets the
// RANGE bit of *status.  SCALAR: g is [BH][L], one logit per token and head
// (the scalar gate of the Chinese summary's ablation, section 4) that every
// dimension shares; the factors come out in the same per-dimension layout.
template <bool SCALAR>
__global__ void __launch_bounds__(256) gate_prep_kernel(const __nv_bfloat16 *g, __nv_bfloat16 *E16, float *E32,
                                                        float *rr, uint32_t *status, int L, int ntiles,
                                                        float inv_tau, uint32_t *seqflag) {
  __shared__ float2 s_tot[8][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int i = blockIdx.x * 64 + 2 * lane, c = blockIdx.y, bh = blockIdx.z;
  const int tb = c * tc::kTileRows + 16 * w;     // first token of this warp
  const size_t base = (size_t)bh * L * 128 + i;
  float2 a[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int t = tb + u;
    if (SCALAR) {
      const float gv = t < L ? __bfloat162float(g[(size_t)bh * L + t]) : 0.f;
      a[u] = make_float2(gv, gv);
    } else {
      a[u] = t < L ? __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(g + base + (size_t)t * 128))
                   : make_float2(0.f, 0.f);
    }
  }
  float2 tot = make_float2(0.f, 0.f);
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const bool in = tb + u < L;
    a[u].x = in ? -tc::log_decay_fast(a[u].x, inv_tau) : 0.f;   // -a_s >= 0
    a[u].y = in ? -tc::log_decay_fast(a[u].y, inv_tau) : 0.f;
    tot.x += a[u].x;
    tot.y += a[u].y;
  }
  s_tot[w][lane] = tot;
  __syncthreads();
  float2 carry = make_float2(0.f, 0.f);          // sum of -a_s over the later warps' tokens
  for (int w2 = w + 1; w2 < 8; ++w2) {
    carry.x += s_tot[w2][lane].x;
    carry.y += s_tot[w2][lane].y;
  }
#pragma unroll
  for (int u = 15; u >= 0; --u) {
    if (tb + u < L) {
      const float e0 = __expf(carry.x), e1 = __expf(carry.y);
      const size_t o = base + (size_t)(tb + u) * 128;
      if (E16) *reinterpret_cast<__nv_bfloat162 *>(E16 + o) = __floats2bfloat162_rn(e0, e1);
      if (E32) *reinterpret_cast<float2 *>(E32 + o) = make_float2(e0, e1);
    }
    carry.x += a[u].x;
    carry.y += a[u].y;
  }
  if (w == 0) {   // carry = -r: the whole tile
    *reinterpret_cast<float2 *>(rr + ((size_t)bh * ntiles + c) * 128 + i) = make_float2(-carry.x, -carry.y);
    const float spread = fmaxf(carry.x - a[0].x, carry.y - a[0].y);   // sum over s > 0
    if (spread > kMaxSpread) {
      if (seqflag) seqflag[bh] = 1u;   // the exact fallback takes this sequence
      else atomicOr(status, 2u);
    }
  }
}

cudaError_t launch_gate_prep(const void *g, void *E16, float *E32, float *r, uint32_t *status, int BH, int L,
                             float inv_tau, bool scalar_gate, cudaStream_t s, uint32_t *seqflag) {
  if (L == 0) return cudaSuccess;
  const int ntiles = (L + tc::kTileRows - 1) / tc::kTileRows;
  const dim3 grid(2, ntiles, BH);
  const __nv_bfloat16 *gp = static_cast<const __nv_bfloat16 *>(g);
  __nv_bfloat16 *e16 = static_cast<__nv_bfloat16 *>(E16);
  if (scalar_gate)
    gate_prep_kernel<true><<<grid, 256, 0, s>>>(gp, e16, E32, r, status, L, ntiles, inv_tau, seqflag);
  else
    gate_prep_kernel<false><<<grid, 256, 0, s>>>(gp, e16, E32, r, status, L, ntiles, inv_tau, seqflag);
  return cudaGetLastError();
}

namespace {

// Start state of every segment: S_0 = state_in (or 0),
// S_{s+1} = diag(exp(decay_s)) S_s + local_s.
// One thread per state element: grid (B*H, D*D / 256).
__global__ void __launch_bounds__(256) seg_combine_kernel(const float *seg_state, const float *seg_decay,
                                                          const float *state_in, float *seg_start, int nseg) {
  const int bh = blockIdx.x;
  {
    const int e = blockIdx.y * 256 + threadIdx.x;
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

// Segments per sequence, for few (batch, head) sequences: from enough
// (sequence, segment) CTAs to cover the 148 SMs once up to twice that, the
// count whose last wave is fullest (one CTA per SM), each segment at least
// two tiles long.
void tc_fwd_segments(int BH, int L, int *nseg, int *tiles_per_seg) {
  constexpr int kSMs = 148;
  const int ntiles = (L + T - 1) / T;
  int n = 1;
  if (BH > 0 && BH < 120) {
    const int n0 = kSMs / BH;
    double best = -1.0;
    for (int c = n0; c <= 2 * n0 + 1; ++c) {
      const int ctas = BH * c, waves = (ctas + kSMs - 1) / kSMs;
      const double fill = (double)ctas / ((double)waves * kSMs);
      if (fill > best + 1e-9) { best = fill; n = c; }
    }
  }
  n = n < ntiles / 2 ? n : ntiles / 2;
  if (n < 1) n = 1;
  const int tps = (ntiles + n - 1) / n;
  *tiles_per_seg = tps > 0 ? tps : 1;
  *nseg = tps > 0 ? (ntiles + tps - 1) / tps : 1;
}

// Workspace of the tensor-core forward: the segment states (when the
// sequences are split), then the gate factors E (bf16, [BH][L][D]) and the
// per-tile decays (fp32, [BH][ntiles][D]), each 256-byte aligned.
static size_t seg_bytes(int BH, int L) {
  int nseg, tps;
  tc_fwd_segments(BH, L, &nseg, &tps);
  if (nseg <= 1) return 0;
  return ((size_t)BH * nseg * (2 * (size_t)D * D + D) * sizeof(float) + 255) & ~size_t(255);
}
static size_t up256(size_t b) { return (b + 255) & ~size_t(255); }

// Workspace of the tensor-core forward, in order: the segment states (when
// the sequences are split), the tiles' bf16 decay factors E16 [BH][L][D],
// their fp32 E32 (only for a state pass), and the tiles' log-decays r
// [BH][ntiles][D].
struct FwdWs {
  float *seg_state, *seg_start, *seg_decay;
  __nv_bfloat16 *e16;
  float *e32, *r;
  size_t total;
};
static FwdWs fwd_ws(void *base, int BH, int L) {
  int nseg, tps;
  tc_fwd_segments(BH, L, &nseg, &tps);
  unsigned char *b = static_cast<unsigned char *>(base);
  FwdWs w{};
  size_t off = 0;
  if (nseg > 1) {
    w.seg_state = reinterpret_cast<float *>(b + off);
    w.seg_start = w.seg_state + (size_t)BH * nseg * D * D;
    w.seg_decay = w.seg_start + (size_t)BH * nseg * D * D;
  }
  off += seg_bytes(BH, L);
  w.e16 = reinterpret_cast<__nv_bfloat16 *>(b + off);
  off += up256((size_t)BH * L * D * 2);
  if (nseg > 1) {
    w.e32 = reinterpret_cast<float *>(b + off);
    off += up256((size_t)BH * L * D * 4);
  }
  w.r = reinterpret_cast<float *>(b + off);
  off += up256((size_t)BH * ((L + T - 1) / T) * D * 4);
  w.total = off;
  if (!base) w = FwdWs{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, off};
  return w;
}

size_t tc_fwd_workspace_bytes(int BH, int L) { return fwd_ws(nullptr, BH, L).total; }

int tc_fwd_stage_count(int BH, int L) {
  int nseg, tps;
  tc_fwd_segments(BH, L, &nseg, &tps);
  return nseg > 1 ? 3 : 1;
}

// Forward state pass over whole sequences that keeps, for every 128-token
// tile, the bf16 state at the tile's start already decayed by the tile's
// gates, S' = diag(exp r) S (the backward's input).  e32 and r come from
// launch_gate_prep over the same gate logits.
cudaError_t launch_tc_state_snapshots(const TcFwdArgs &a, void *snap, const float *e32, const float *r,
                                      cudaStream_t s) {
  Params p;
  memset(&p, 0, sizeof(p));
  const uint64_t rows = (uint64_t)a.L;
  if (!make_map_bf16_3d(&p.mq, a.q, D, rows, a.BH, T) || !make_map_bf16_3d(&p.mk, a.k, D, rows, a.BH, T) ||
      !make_map_bf16_3d(&p.mv, a.v, D, rows, a.BH, T))
    return cudaErrorInvalidValue;
  p.gate_e32 = e32;   // the state pass loads fp32 factors, no gate tiles (p.mg stays unset)
  if (!make_map_f32_3d(&p.me, e32, D, rows, a.BH, T)) return cudaErrorInvalidValue;
  p.gate_r = r;
  p.wq = a.wq;
  p.wk = a.wk;
  p.meta_k = a.meta_k;
  p.meta_v = a.meta_v;
  p.alpha = a.alpha;
  p.state_in = a.state_in;
  p.status = a.status;
  p.snap = static_cast<__nv_bfloat16 *>(snap);
  p.snap_r0 = reinterpret_cast<float *>(p.snap + (size_t)a.BH * ((a.L + T - 1) / T) * D * D);
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
  p.kap_g = a.dstate_out;
  p.kap = a.dstate_out ? a.kap : nullptr;
  cudaError_t e =
      cudaFuncSetAttribute(tc_fwd_kernel<K_STATE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  tc_fwd_kernel<K_STATE><<<dim3(a.BH, 1), NTHREADS, SMEM_BYTES, s>>>(p);
  return cudaGetLastError();
}

// Scratch of the segment summary: the fp32 decay factors E32 [BH][L][D], then
// the tiles' log-decays r [BH][ntiles][D].
size_t tc_segment_state_workspace_bytes(int BH, int L) {
  return up256((size_t)BH * L * D * 4) + up256((size_t)BH * ((L + T - 1) / T) * D * 4);
}

// Segment summary for sequence parallelism: the state pass (mode 1) over
// whole sequences from a zero start, U = its end state, R = the summed
// log-decay of every key dimension.
cudaError_t launch_tc_segment_state(const TcFwdArgs &a, float *U, float *R, void *scratch, cudaStream_t s) {
  float *e32 = static_cast<float *>(scratch);
  float *r = reinterpret_cast<float *>(static_cast<unsigned char *>(scratch) + up256((size_t)a.BH * a.L * D * 4));
  cudaError_t e = launch_gate_prep(a.g, nullptr, e32, r, a.status, a.BH, a.L, a.inv_tau, a.scalar_gate != 0, s);
  if (e != cudaSuccess) return e;
  Params p;
  memset(&p, 0, sizeof(p));
  const uint64_t rows = (uint64_t)a.L;
  // the state pass reads keys and values only (its query map is never loaded)
  if (!make_map_bf16_3d(&p.mq, a.k, D, rows, a.BH, T) || !make_map_bf16_3d(&p.mk, a.k, D, rows, a.BH, T) ||
      !make_map_bf16_3d(&p.mv, a.v, D, rows, a.BH, T))
    return cudaErrorInvalidValue;
  p.gate_e32 = e32;
  if (!make_map_f32_3d(&p.me, e32, D, rows, a.BH, T)) return cudaErrorInvalidValue;
  p.gate_r = r;
  p.wk = a.wk;
  p.status = a.status;
  p.seg_state = U;
  p.seg_decay = R;
  p.H = a.H;
  p.L = a.L;
  p.window = a.window;
  p.mode = 1;
  p.nseg = 1;
  p.tiles_per_seg = (a.L + T - 1) / T;
  p.inv_tau = a.inv_tau;
  p.scale = a.scale;
  e = cudaFuncSetAttribute(tc_fwd_kernel<K_STATE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  tc_fwd_kernel<K_STATE><<<dim3(a.BH, 1), NTHREADS, SMEM_BYTES, s>>>(p);
  return cudaGetLastError();
}

int g_inject_wait = 0;   // launches of the full pass still to carry the test hook

cudaError_t launch_tc_fwd(const TcFwdArgs &a, int stage, cudaStream_t s) {
  int nseg, tps;
  tc_fwd_segments(a.BH, a.L, &nseg, &tps);
  const FwdWs w = fwd_ws(a.seg_ws, a.BH, a.L);
  const bool gla = a.branch != 2 && a.g != nullptr;
  // a training forward keeps the fp32 factors and the tile decays for the
  // backward (in the caller's arrays instead of the workspace)
  float *e32 = a.keep_e32 ? a.keep_e32 : w.e32;
  float *rr = a.keep_r ? a.keep_r : w.r;
  if (stage == 3) {
    if (!gla) return cudaSuccess;
    return launch_gate_prep(a.g, w.e16, e32, rr, a.status, a.BH, a.L, a.inv_tau, a.scalar_gate != 0, s,
                            a.seqflag);
  }
  if (nseg > 1 && (stage == 0 || stage == 1) && !gla) return cudaSuccess;   // no state to carry
  if (nseg > 1 && stage == 1) {
    seg_combine_kernel<<<dim3(a.BH, D * D / 256), 256, 0, s>>>(w.seg_state, w.seg_decay, a.state_in, w.seg_start,
                                                               nseg);
    return cudaGetLastError();
  }
  Params p;
  memset(&p, 0, sizeof(p));
  const uint64_t rows = (uint64_t)a.L;
  // the full pass loads the bf16 factors E from stage 3 as its gate tiles
  // (unused without the GLA branch)
  const void *gsrc = gla ? static_cast<const void *>(w.e16) : a.q;
  if (!make_map_bf16_3d(&p.mq, a.q, D, rows, a.BH, T) || !make_map_bf16_3d(&p.mk, a.k, D, rows, a.BH, T) ||
      !make_map_bf16_3d(&p.mv, a.v, D, rows, a.BH, T) || !make_map_bf16_3d(&p.mg, gsrc, D, rows, a.BH, T))
    return cudaErrorInvalidValue;
  p.gate_r = gla ? rr : nullptr;
  p.gate_e32 = gla ? e32 : nullptr;
  if (gla && nseg > 1 && !make_map_f32_3d(&p.me, e32, D, rows, a.BH, T)) return cudaErrorInvalidValue;
  if (gla && a.snap && stage == 2) {   // training: the backward's state copies and final state
    p.snap = static_cast<__nv_bfloat16 *>(a.snap);
    p.snap_r0 = reinterpret_cast<float *>(p.snap + (size_t)a.BH * ((a.L + T - 1) / T) * D * D);
    if (!make_map_bf16_3d(&p.msnap, a.snap, D, D, (uint64_t)a.BH * ((a.L + T - 1) / T), T))
      return cudaErrorInvalidValue;
    p.state_keep = a.state_keep;
  }
  if (a.branch != 1 && stage == 2) p.lse_keep = a.lse_keep;
  p.wq = a.wq;
  p.wk = a.wk;
  p.meta_k = a.meta_k;
  p.meta_v = a.meta_v;
  p.alpha = a.alpha;
  p.state_in = a.state_in;
  p.o = static_cast<__nv_bfloat16 *>(a.o);
  p.target = static_cast<const __nv_bfloat16 *>(a.target);
  p.dmse = static_cast<__nv_bfloat16 *>(a.dmse);
  p.loss = a.loss;
  {
    const double n = (double)a.BH * a.L * D;
    p.mse_grad = (float)(2.0 / n);
    p.mse_loss = (float)(1.0 / n);
  }
  p.state_out = a.state_out;
  p.lse = a.lse;
  p.status = a.status;
  if (a.P > 0 && a.branch != 1) {
    if (!make_map_bf16_3d(&p.mkp, a.k_prefix, D, (uint64_t)a.P, a.BH, T) ||
        !make_map_bf16_3d(&p.mvp, a.v_prefix, D, (uint64_t)a.P, a.BH, T))
      return cudaErrorInvalidValue;
    p.P = a.P;
  }
  p.seg_start = w.seg_start;
  p.seg_state = w.seg_state;
  p.seg_decay = w.seg_decay;
  p.seqflag = a.seqflag;
  p.xq = static_cast<const __nv_bfloat16 *>(a.q);
  p.xk = static_cast<const __nv_bfloat16 *>(a.k);
  p.xv = static_cast<const __nv_bfloat16 *>(a.v);
  p.xg = static_cast<const __nv_bfloat16 *>(a.g);
  p.scalar_gate = a.scalar_gate;
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
    e = cudaFuncSetAttribute(tc_fwd_kernel<K_FULL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_fwd_kernel<K_LOSS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_fwd_kernel<K_TRAIN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_fwd_kernel<K_TRAIN_LOSS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_fwd_kernel<K_STATE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = SMEM_BYTES;
  }
  if (nseg > 1 && stage == 0) {          // state pass over every segment but the last
    p.mode = 1;
    tc_fwd_kernel<K_STATE><<<dim3(a.BH, nseg - 1), NTHREADS, SMEM_BYTES, s>>>(p);
  } else {                               // full pass
    p.mode = 0;
    if (g_inject_wait > 0) {
      --g_inject_wait;
      p.inject = 1;
    }
    if (p.target && p.snap)
      tc_fwd_kernel<K_TRAIN_LOSS><<<dim3(a.BH, nseg), NTHREADS, SMEM_BYTES, s>>>(p);
    else if (p.target)
      tc_fwd_kernel<K_LOSS><<<dim3(a.BH, nseg), NTHREADS, SMEM_BYTES, s>>>(p);
    else if (p.snap)
      tc_fwd_kernel<K_TRAIN><<<dim3(a.BH, nseg), NTHREADS, SMEM_BYTES, s>>>(p);
    else
      tc_fwd_kernel<K_FULL><<<dim3(a.BH, nseg), NTHREADS, SMEM_BYTES, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace lz
