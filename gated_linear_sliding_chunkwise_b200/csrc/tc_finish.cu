// Tensor-core (tcgen05) end of the backward, bf16, d = 128: the feature-map
// backward and the sums of the two branches' gradients.
//
// phi(x) = [softmax(x W), softmax(-x W)] (the non-negative Hedgehog map of
// the Chinese gist.science summary, section 2.3).  With p = softmax(z),
// n = softmax(-z), z = x W and dphi = [dp, dn]:
//   dz = p (dp - <dp, p>) - n (dn - <dn, n>)
//   dx = dz W^T,   dW += x^T dz
// One CTA per sequence walks its 128-token tiles; dW_q and dW_k accumulate
// in TMEM across the tiles and are added to the output once per CTA.  dz is
// formed in fp32 (the subtraction above cancels) and only then rounded to
// bf16 as an MMA operand.
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
constexpr uint32_t ST_TIMEOUT = 1u;

struct Params {
  CUtensorMap mq, mk;
  CUtensorMap mxq, mxk;                    // bf16 dx_q, dx_k parts (fused mode)
  CUtensorMap mphq, mphk;                  // bf16 dphi_q, dphi_k (TMA loads)
  const float *wq, *wk;
  // GLA parts, null when the branch is off: dphi_q, dphi_k in bf16 with each
  // row's halves centred (the softmax backward below ignores a constant added
  // to a half), dv in fp32; the exact fallback's sequences (slot_of[bh] >= 0)
  // have fp32 dphi in its slot arrays fb_dphq, fb_dphk [slot][L][D]
  const __nv_bfloat16 *dphq, *dphk;
  const float *dv_gla;
  const int *slot_of;
  const float *fb_dphq, *fb_dphk;
  const float *dq_swa, *dk_swa, *dv_swa;   // anchor parts (fp32), null when the branch is off
  __nv_bfloat16 *dq, *dk, *dv;
  float *dwq, *dwk;
  uint32_t *status;
  int H, L;
  int fused;                               // write dx_q, dx_k parts; the anchor kernels finish dq, dk, dv
};

// Two warpgroups (256 threads), thread = tile row `row` of its group:
// group 0 forms dz of the q map and writes dq, group 1 those of the k map
// and dk; each writes half of dv's columns.
constexpr int NTHREADS = 256;
__global__ void __launch_bounds__(NTHREADS, 1) tc_finish_kernel(const __grid_constant__ Params p) {
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar_tma, bar_z, bar_d, bar_ph;
  __shared__ uint32_t s_tmem;
  // X_q, X_k, W_q | W_k (64-column tiles), dZ_q | dZ_k (64-column tiles)
  constexpr uint32_t R_XQ = 0, R_XK = TILE, R_WQ = 2 * TILE, R_WK = 2 * TILE + REG, R_ZQ = 3 * TILE,
                     R_ZK = 3 * TILE + REG, R_STG = 4 * TILE;   // R_STG: dphi_q | dphi_k, then the half-terms
  // TMEM: dWq [0,64) dWk [64,128) Zq [128,192) Zk [192,256) dXq [256,384) dXk [384,512)
  constexpr uint32_t C_WQ = 0, C_WK = 64, C_ZQ = 128, C_ZK = 192, C_XQ = 256, C_XK = 384;
  const int tid = threadIdx.x, warp = tid >> 5, wg = tid >> 7, row = tid & 127;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const int bh = blockIdx.x, h = bh % p.H;
  const uint32_t sbase = smem_u32(sm);
  const bool gla = p.dphq != nullptr;
  if (warp == 0) { tmem_alloc(&s_tmem, 512); tmem_relinquish(); }
  if (tid == 0) {
    mbar_init(&bar_tma, 1);
    mbar_init(&bar_z, 1);
    mbar_init(&bar_d, 1);
    mbar_init(&bar_ph, 1);
    fence_barrier_init();
  }
  const int ntiles = (p.L + T - 1) / T;
  auto loads = [&](int c) {
    mbar_expect_tx(&bar_tma, 2 * TILE);
    for (int r = 0; r < 2; ++r) {
      tma_load_3d(sm + R_XQ + r * REG, &p.mq, &bar_tma, 64 * r, c * T, bh);
      tma_load_3d(sm + R_XK + r * REG, &p.mk, &bar_tma, 64 * r, c * T, bh);
    }
  };
  if (tid == 0 && ntiles > 0 && gla) loads(0);   // in flight while the weights are staged
  // weights -> bf16 [dk row][feature] (MN-major for z = x W, K-major for dz W^T);
  // group 0 W_q, group 1 W_k
  {
    const float *W = wg == 0 ? p.wq : p.wk;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float f[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) f[u] = W[((size_t)h * D + row) * F + c * 8 + u];
      *reinterpret_cast<uint4 *>(sm + (wg == 0 ? R_WQ : R_WK) + sw128_offset(row, c * 8)) = pack8(f);
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s_tmem, tl = tb + lane_off;
  const uint32_t id_z = idesc_bf16(128, 64, 0, 1);     // X (K-major) x W (MN-major, N = 64)
  const uint32_t id_dx = idesc_bf16(128, 128, 0, 0);   // dZ (K-major) x W^T (K-major, N = 128)
  const uint32_t id_dw = idesc_bf16(128, 64, 1, 1);    // X^T (MN-major) x dZ (MN-major, N = 64)
  bool fail = false;
  // this row's dphi values (its group's half) of one map, packed bf16.  They
  // come by TMA into R_STG (dphi_q over its first half, dphi_k over its
  // second, issued with the previous tile's last products; the exchange of each map's
  // half-terms reuses the map's half once every row has read it), except for
  // a sequence of the exact fallback, whose fp32 values are loaded into
  // registers ahead (map 0 of the next tile at the end of this one, map 1
  // while map 0 is used) and centred there.
  uint4 dpre[8];
  const int fb_slot = (gla && p.slot_of) ? p.slot_of[bh] : -1;
  const bool ph_tma = gla && fb_slot < 0;
  int pend_ph = -1;   // tid 0: the parity of a dphi load in flight
  auto ph_loads = [&](int c) {
    mbar_expect_tx(&bar_ph, 2 * TILE);
    for (int r = 0; r < 2; ++r) {
      tma_load_3d(sm + R_STG + r * REG, &p.mphq, &bar_ph, 64 * r, c * T, bh);
      tma_load_3d(sm + R_STG + TILE + r * REG, &p.mphk, &bar_ph, 64 * r, c * T, bh);
    }
  };
  auto dphi_load = [&](int m, int c) {
    const int t = c * T + row;
    if (fb_slot >= 0) {
      // the exact fallback's fp32 dphi, centred on the half row's first value
      // like the tensor-core kernel's (the softmax backward does not see a
      // constant added to one half)
      const float *src = (m == 0 ? p.fb_dphq : p.fb_dphk) + ((size_t)fb_slot * p.L + (t < p.L ? t : 0)) * D + wg * F;
      const float c0 = t < p.L ? src[0] : 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float f[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = t < p.L ? src[8 * u + i] - c0 : 0.f;
        dpre[u] = pack8(f);
      }
      return;
    }
    const __nv_bfloat16 *src = (m == 0 ? p.dphq : p.dphk) + ((size_t)bh * p.L + (t < p.L ? t : 0)) * D + wg * F;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      dpre[u] = t < p.L ? *reinterpret_cast<const uint4 *>(src + 8 * u) : make_uint4(0u, 0u, 0u, 0u);
  };
  if (ph_tma && ntiles > 0) {
    if (tid == 0) {
      pend_ph = 0;
      ph_loads(0);
    }
  } else if (gla && ntiles > 0) {
    dphi_load(0, 0);
  }
  for (int c = 0; c < ntiles; ++c) {
    const uint32_t par = c & 1;
    const int tq = c * T + row;
    const bool valid = tq < p.L;
    const size_t off = ((size_t)bh * p.L + (valid ? tq : 0)) * D;
    if (gla) {
      bool ok = mbar_wait(&bar_tma, par, p.status, ST_TIMEOUT);
      if (__syncthreads_or(!ok)) { fail = true; break; }
      if (tid == 0) {
        tc_fence_after();
        for (int s = 0; s < 8; ++s) mma_ss(tb + C_ZQ, desc_k(sbase + R_XQ, s), desc_mn(sbase + R_WQ, s), id_z, s > 0);
        for (int s = 0; s < 8; ++s) mma_ss(tb + C_ZK, desc_k(sbase + R_XK, s), desc_mn(sbase + R_WK, s), id_z, s > 0);
        mma_commit(&bar_z);
      }
      ok = mbar_wait(&bar_z, par, p.status, ST_TIMEOUT);
      if (ph_tma) ok &= mbar_wait(&bar_ph, par, p.status, ST_TIMEOUT);
      if (__syncthreads_or(!ok)) { fail = true; break; }
      if (tid == 0) pend_ph = -1;
      tc_fence_after();
      // dz of both maps, one map at a time (fp32 math, bf16 dZ tiles): group
      // 0 owns the softmax(z) half (p, dp), group 1 the softmax(-z) half
      // (n, dn); each loads its 64 dphi values once, all in flight, and forms
      //   A_f = p_f (dp_f - <dp, p>)   or   B_f = n_f (dn_f - <dn, n>).
      // The half-terms meet in shared memory (R_STG, one swizzled 128 x 32
      // fp32 box per map and group): group 0 writes dz_f = A_f - B_f for
      // f < 32, group 1 for f >= 32.
#pragma unroll 1
      for (int m = 0; m < 2; ++m) {
        if (ph_tma)
#pragma unroll
          for (int u = 0; u < 8; ++u) dpre[u] = *chunk_ptr(sm, R_STG + m * TILE, row, 8 * wg + u);
        float ph[F];
        const float sc = feature_half(tl + (m == 0 ? C_ZQ : C_ZK), wg, ph);
        float dot4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float d[8];
          unpack8(dpre[u], d);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            ph[8 * u + i] *= sc;
            dot4[i & 3] += d[i] * ph[8 * u + i];
          }
        }
        const float dot = (dot4[0] + dot4[1]) + (dot4[2] + dot4[3]);
#pragma unroll
        for (int u = 0; u < 8; ++u) {   // ph <- this group's half-term
          float d[8];
          unpack8(dpre[u], d);
#pragma unroll
          for (int i = 0; i < 8; ++i) ph[8 * u + i] *= d[i] - dot;
        }
        if (!ph_tma && m == 0) dphi_load(1, c);   // the k map's values, in flight while this map finishes
        if (ph_tma) bar_sync(2, NTHREADS);   // every row has read this map's dphi: its half takes the exchange
        // send the half-terms of the other group's features
        unsigned char *mine = sm + R_STG + (2 * m + wg) * 16384;
        const unsigned char *theirs = sm + R_STG + (2 * m + 1 - wg) * 16384;
        if (wg == 0) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *f32_stage_ptr(mine, row, 4 * j) = make_float4(ph[32 + 4 * j], ph[33 + 4 * j], ph[34 + 4 * j], ph[35 + 4 * j]);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *f32_stage_ptr(mine, row, 4 * j) = make_float4(ph[4 * j], ph[1 + 4 * j], ph[2 + 4 * j], ph[3 + 4 * j]);
        }
        bar_sync(1, NTHREADS);
        const int fm = 32 * wg;            // this group's 32 dz features
        float dz[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 t = *f32_stage_ptr(const_cast<unsigned char *>(theirs), row, 4 * j);
          const float tv[4] = {t.x, t.y, t.z, t.w};
          // group 0: A_f - B_f with B from group 1; group 1: A_{32+f} - B_{32+f} with A from group 0
          if (wg == 0) {
#pragma unroll
            for (int u = 0; u < 4; ++u) dz[4 * j + u] = valid ? ph[4 * j + u] - tv[u] : 0.f;
          } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) dz[4 * j + u] = valid ? tv[u] - ph[32 + 4 * j + u] : 0.f;
          }
        }
        const uint32_t reg = m == 0 ? R_ZQ : R_ZK;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          *reinterpret_cast<uint4 *>(sm + reg + sw128_offset(row, fm + 8 * c8)) = pack8(dz + 8 * c8);
      }
      fence_proxy_async();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        for (int s = 0; s < 4; ++s) mma_ss(tb + C_XQ, desc_k(sbase + R_ZQ, s), desc_k(sbase + R_WQ, s), id_dx, s > 0);
        for (int s = 0; s < 4; ++s) mma_ss(tb + C_XK, desc_k(sbase + R_ZK, s), desc_k(sbase + R_WK, s), id_dx, s > 0);
        for (int s = 0; s < 8; ++s) mma_ss(tb + C_WQ, desc_mn(sbase + R_XQ, s), desc_mn(sbase + R_ZQ, s), id_dw, c > 0 || s > 0);
        for (int s = 0; s < 8; ++s) mma_ss(tb + C_WK, desc_mn(sbase + R_XK, s), desc_mn(sbase + R_ZK, s), id_dw, c > 0 || s > 0);
        mma_commit(&bar_d);
        if (ph_tma && c + 1 < ntiles) {   // this tile's dphi and half-terms are read: the next tile's dphi
          pend_ph = (int)((c + 1) & 1);
          ph_loads(c + 1);
        }
      }
      ok = mbar_wait(&bar_d, par, p.status, ST_TIMEOUT);
      if (__syncthreads_or(!ok)) { fail = true; break; }
      tc_fence_after();
      if (tid == 0 && c + 1 < ntiles) loads(c + 1);   // X tiles consumed by the dW products
    }
    if (p.fused) {
      // dx, bf16, one map at a time (64 columns per group) staged over the
      // spent dZ tiles (R_ZQ | R_ZK, one 32 KB tile) and written with TMA
      // stores (rows past L are clipped by the map); the next tile's dphi
      // is arriving in R_STG meanwhile
      unsigned char *st = sm + R_ZQ;
#pragma unroll 1
      for (int m = 0; m < 2; ++m) {
        for (int ch = 2 * wg; ch < 2 * wg + 2; ++ch) {
          float v[32];
          tmem_ld32(tl + (m == 0 ? C_XQ : C_XK) + ch * 32, v);
#pragma unroll
          for (int k = 0; k < 4; ++k) *chunk_ptr(st, 0, row, 4 * ch + k) = pack8(v + 8 * k);
        }
        fence_proxy_async();
        __syncthreads();
        if (tid == 0) {
          const CUtensorMap *mx = m == 0 ? &p.mxq : &p.mxk;
          tma_store_3d(mx, st, 0, c * T, bh);
          tma_store_3d(mx, st + REG, 64, c * T, bh);
          bulk_commit();
          bulk_wait_read();   // the staging is free once read
        }
        if (m == 0) __syncthreads();
      }
    }
    // dq (group 0), dk (group 1) = GLA (dz W^T) + anchor parts; dv = both
    // parts, 64 columns per group
#pragma unroll
    for (int k = 0; k < 2 && !p.fused; ++k) {
      const int m = k == 0 ? wg : 2;
      const float *__restrict__ swa = m == 0 ? p.dq_swa : (m == 1 ? p.dk_swa : p.dv_swa);
      const float *__restrict__ gpart = m == 2 ? p.dv_gla : nullptr;
      __nv_bfloat16 *__restrict__ dst = m == 0 ? p.dq : (m == 1 ? p.dk : p.dv);
      const int ch0 = m == 2 ? 2 * wg : 0, ch1 = m == 2 ? 2 * wg + 2 : 4;
      for (int ch = ch0; ch < ch1; ++ch) {
        float v[32];
        if (m < 2 && gla) {
          tmem_ld32(tl + (m == 0 ? C_XQ : C_XK) + ch * 32, v);
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) v[u] = 0.f;
        }
        if (valid) {
        float4 ga[8], sa[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          ga[u] = gpart ? *reinterpret_cast<const float4 *>(gpart + off + ch * 32 + 4 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
          sa[u] = swa ? *reinterpret_cast<const float4 *>(swa + off + ch * 32 + 4 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          v[4 * u] += ga[u].x + sa[u].x;
          v[4 * u + 1] += ga[u].y + sa[u].y;
          v[4 * u + 2] += ga[u].z + sa[u].z;
          v[4 * u + 3] += ga[u].w + sa[u].w;
        }
#pragma unroll
        for (int u = 0; u < 32; u += 8) *reinterpret_cast<uint4 *>(dst + off + ch * 32 + u) = pack8(v + u);
        }
      }
    }
    // the next tile's q-map values, in flight until they are used (issued
    // past this tile's proxy fences, which would wait for them)
    if (!ph_tma && gla && c + 1 < ntiles) dphi_load(0, c + 1);
    tc_fence_before();
    __syncthreads();
  }
  if (gla && !fail) {
    tc_fence_after();
    // dW rows: lane = dk index, 64 feature columns per map; group 0 dW_q, group 1 dW_k
    float *dW = wg == 0 ? p.dwq : p.dwk;
    if (dW) {
      float v[32];
      for (int ch = 0; ch < 2; ++ch) {
        tmem_ld32(tl + (wg == 0 ? C_WQ : C_WK) + ch * 32, v);
#pragma unroll
        for (int u = 0; u < 32; ++u) atomicAdd(dW + ((size_t)h * D + row) * F + ch * 32 + u, v[u]);
      }
    }
  }
  if (tid == 0 && pend_ph >= 0) mbar_wait(&bar_ph, (uint32_t)pend_ph, nullptr, 0, 1u << 16);   // after a failed wait
  if (p.fused && tid == 0) bulk_wait_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(s_tmem, 512);
}

constexpr size_t SMEM_BYTES = 6 * TILE + 1024;

}  // namespace

cudaError_t launch_tc_finish(const FinishBwdArgs &a, int BH, cudaStream_t s) {
  Params p;
  memset(&p, 0, sizeof(p));
  const uint64_t rows = (uint64_t)a.L;
  if (!make_map_bf16_3d(&p.mq, a.q, D, rows, BH, T) || !make_map_bf16_3d(&p.mk, a.k, D, rows, BH, T))
    return cudaErrorInvalidValue;
  p.fused = a.xq_part != nullptr;
  if (p.fused && (!make_map_bf16_3d(&p.mxq, a.xq_part, D, rows, BH, T) ||
                  !make_map_bf16_3d(&p.mxk, a.xk_part, D, rows, BH, T)))
    return cudaErrorInvalidValue;
  p.wq = a.wq;
  p.wk = a.wk;
  p.dphq = static_cast<const __nv_bfloat16 *>(a.dphq16);
  p.dphk = static_cast<const __nv_bfloat16 *>(a.dphk16);
  if (p.dphq && (!make_map_bf16_3d(&p.mphq, a.dphq16, D, rows, BH, T) ||
                 !make_map_bf16_3d(&p.mphk, a.dphk16, D, rows, BH, T)))
    return cudaErrorInvalidValue;
  p.dv_gla = a.dv_gla;
  p.slot_of = a.slot_of;
  p.fb_dphq = a.fb_dphq;
  p.fb_dphk = a.fb_dphk;
  p.dq_swa = a.dq_swa;
  p.dk_swa = a.dk_swa;
  p.dv_swa = a.dv_swa;
  p.dq = static_cast<__nv_bfloat16 *>(a.dq);
  p.dk = static_cast<__nv_bfloat16 *>(a.dk);
  p.dv = static_cast<__nv_bfloat16 *>(a.dv);
  p.dwq = a.dwq;
  p.dwk = a.dwk;
  p.status = a.status;
  p.H = a.H;
  p.L = a.L;
  cudaError_t e = cudaFuncSetAttribute(tc_finish_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  tc_finish_kernel<<<BH, NTHREADS, SMEM_BYTES, s>>>(p);
  return cudaGetLastError();
}

}  // namespace lz
