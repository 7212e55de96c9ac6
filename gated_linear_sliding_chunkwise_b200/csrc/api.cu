// Host side of the C ABI declared in include/lizard.h: argument checks,
// workspace layout and kernel dispatch.  Nothing here allocates device
// memory; every buffer comes from the caller.
#include <math.h>
#include <string.h>

#include <functional>

#include "../../include/lizard.h"
#include "lizard_internal.h"

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kHeader = 256;   // status word region at the workspace start

size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void *p) { return p == nullptr || aligned16(p); }

lizard_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LIZARD_OK : LIZARD_ERR_CUDA; }

// Shape and pointer checks shared by the forward and the backward.
lizard_status check_fwd(const lizard_fwd_args *a) {
  if (!a) return LIZARD_ERR_INVALID_ARG;
  if (a->B < 0 || a->H < 0 || a->L < 0 || a->dk <= 0 || a->dv <= 0 || a->M < 0 || a->window < 1)
    return LIZARD_ERR_INVALID_ARG;
  if (a->B == 0 || a->H == 0) return LIZARD_ERR_INVALID_ARG;
  if (a->dtype != LIZARD_BF16 && a->dtype != LIZARD_FP32) return LIZARD_ERR_INVALID_ARG;
  if (a->branch < LIZARD_BRANCH_BOTH || a->branch > LIZARD_BRANCH_SWA_ONLY) return LIZARD_ERR_INVALID_ARG;
  if (a->impl < LIZARD_IMPL_AUTO || a->impl > LIZARD_IMPL_TC) return LIZARD_ERR_INVALID_ARG;
  if (a->gate != LIZARD_GATE_PER_DIM && a->gate != LIZARD_GATE_SCALAR) return LIZARD_ERR_INVALID_ARG;
  if (!(a->gate_temp > 0.f) || !isfinite(a->gate_temp)) return LIZARD_ERR_INVALID_ARG;
  if (!(a->softmax_scale >= 0.f) || !isfinite(a->softmax_scale)) return LIZARD_ERR_INVALID_ARG;
  if (a->dk != a->dv || (a->dk != 64 && a->dk != 128)) return LIZARD_ERR_UNSUPPORTED;
  if (a->chunk != 64) return LIZARD_ERR_UNSUPPORTED;
  if (a->M > 16) return LIZARD_ERR_UNSUPPORTED;
  if ((a->M > 0) != (a->meta_k != nullptr)) return LIZARD_ERR_INVALID_ARG;
  if (a->meta_v && !a->meta_k) return LIZARD_ERR_INVALID_ARG;
  if (a->L > 0) {
    if (!a->q || !a->k || !a->v || !a->o) return LIZARD_ERR_INVALID_ARG;
    if (a->branch != LIZARD_BRANCH_SWA_ONLY && !a->g) return LIZARD_ERR_INVALID_ARG;
  }
  if (a->prefix_len < 0 || a->prefix_len > a->window) return LIZARD_ERR_INVALID_ARG;
  if ((a->prefix_len > 0) != (a->k_prefix != nullptr) || (a->prefix_len > 0) != (a->v_prefix != nullptr))
    return LIZARD_ERR_INVALID_ARG;
  const void *ptrs[] = {a->q, a->k, a->v, a->g, a->fmap_wq, a->fmap_wk, a->meta_k, a->meta_v,
                        a->alpha, a->state_in, a->o, a->state_out, a->lse, a->workspace,
                        a->k_prefix, a->v_prefix, a->saved};
  for (const void *p : ptrs)
    if (!ok_ptr(p)) return LIZARD_ERR_INVALID_ARG;
  return LIZARD_OK;
}

// Size queries ignore pointers: stand-ins for the prefix pointers that the
// checks require when prefix_len > 0.
void prefix_standin(lizard_fwd_args &a) {
  a.k_prefix = a.v_prefix = a.prefix_len > 0 ? reinterpret_cast<const void *>(16) : nullptr;
}

bool gla_on(const lizard_fwd_args *a) { return a->branch != LIZARD_BRANCH_SWA_ONLY; }
int scalar_gate(const lizard_fwd_args *a) { return a->gate == LIZARD_GATE_SCALAR ? 1 : 0; }
bool swa_on(const lizard_fwd_args *a) { return a->branch != LIZARD_BRANCH_GLA_ONLY; }

// Kernel family the forward runs for these arguments.
// The tensor-core kernels build the Hedgehog map from its weights; without
// them (the identity map) the GLA branch takes the portable kernels.
bool fmap_weights(const lizard_fwd_args *a) { return a->fmap_wq != nullptr && a->fmap_wk != nullptr; }

size_t nch32(const lizard_fwd_args *a) { return (a->L + lz::kBwdC - 1) / lz::kBwdC; }

// Whether the backward's GLA branch runs on the tensor-core kernels.
bool bwd_gla_uses_tc_impl(const lizard_fwd_args *a, int impl) {
  const bool ok = a->dtype == LIZARD_BF16 && a->dk == 128 && a->dv == 128 && fmap_weights(a);
  return (impl == LIZARD_IMPL_AUTO || impl == LIZARD_IMPL_TC) && ok;
}

bool fwd_uses_tc(const lizard_fwd_args *a) {
  const bool ok = lz::tc_fwd_supported(a->dk, a->dv, a->window, a->M, a->dtype == LIZARD_BF16) &&
                  (fmap_weights(a) || a->branch == LIZARD_BRANCH_SWA_ONLY);
  if (a->impl == LIZARD_IMPL_TC) return ok;
  return a->impl == LIZARD_IMPL_AUTO && ok;
}

// Exact fallback of the tensor-core GLA branch: the per-sequence marks
// (right after the status header, so that the call's first memset clears
// both), each sequence's slot, each slot's sequence, then per slot the
// portable kernels' scratch: `per_slot` bytes.
struct FallbackLayout {
  size_t flags, slot_of, seq_of_slot, scratch, per_slot, end;
};
int fallback_slots(const lizard_fwd_args *a) {
  const int BH = a->B * a->H;
  return BH < lz::kFallbackSlots ? BH : lz::kFallbackSlots;
}
FallbackLayout fallback_layout(size_t off, const lizard_fwd_args *a, size_t per_slot) {
  const size_t BH = (size_t)a->B * a->H;
  FallbackLayout f{};
  f.flags = off; off += up(BH * sizeof(uint32_t));
  f.slot_of = off; off += up(BH * sizeof(int));
  f.seq_of_slot = off; off += up(lz::kFallbackSlots * sizeof(int));
  f.per_slot = per_slot;
  f.scratch = off; off += (size_t)fallback_slots(a) * per_slot;
  f.end = off;
  return f;
}
// bytes the call's first memset clears: the status header and, with the
// exact fallback, the per-sequence marks that follow it
size_t cleared_bytes(const lizard_fwd_args *a, bool fallback) {
  return fallback ? kHeader + up((size_t)a->B * a->H * sizeof(uint32_t)) : sizeof(uint32_t);
}

// Whether a training forward keeps tensors for the backward: the forward's
// GLA branch on the tensor cores with the backward's tensor-core GLA kernels
// applicable (bf16, d = 128, feature-map weights).
bool fwd_keeps(const lizard_fwd_args *a) {
  return gla_on(a) && fwd_uses_tc(a) && a->dtype == LIZARD_BF16 && a->dk == 128 && a->dv == 128 &&
         fmap_weights(a);
}

// The saved-for-backward buffer of a training forward: the wide-decay marks
// [BH] (cleared by the forward), the tiles' log-decays r [BH][ntiles][d] and
// fp32 decay factors E [BH][L][d] (the gate prep), the state copies of every
// tile (bf16 S' - 1 S'[0], then the fp32 rows S'[0]), the final state
// [BH][d][d] and, with the anchor branch, the softmax normalisers [BH][L]
// (the full pass).
struct SavedLayout {
  size_t flags, r, e32, snap, state, lse, total;
};
SavedLayout saved_layout(const lizard_fwd_args *a) {
  SavedLayout l{};
  if (!fwd_keeps(a)) return l;
  const size_t BH = (size_t)a->B * a->H, nt = (a->L + 127) / 128;
  size_t off = 0;
  l.flags = off; off += up(BH * sizeof(uint32_t));
  l.r = off; off += up(BH * nt * a->dk * sizeof(float));
  l.e32 = off; off += up(BH * a->L * a->dk * sizeof(float));
  l.snap = off; off += up(lz::tc_gla_bwd_snapshot_bytes((int)BH, a->L));
  l.state = off; off += up(BH * a->dk * a->dv * sizeof(float));
  if (swa_on(a)) { l.lse = off; off += up(BH * a->L * sizeof(float)); }   // the anchor softmax normalisers
  l.total = off;
  return l;
}

// Whether the backward reads a training forward's saved tensors (the
// stage-1 step points fwd.saved at a region of its own workspace).
bool bwd_reads_saved(const lizard_fwd_args *a, int impl) {
  return a->saved != nullptr && fwd_keeps(a) && bwd_gla_uses_tc_impl(a, impl);
}

// Forward workspace: the status header, plus fp32 scratch for the portable path.
struct FwdLayout {
  size_t phq, phk, a, o_gla, total;
  bool fallback;   // wide-decay marks (tensor-core GLA branch)
  size_t flags;
};
FwdLayout fwd_layout(const lizard_fwd_args *a, bool stage1 = false) {
  const size_t N = (size_t)a->B * a->H * a->L;
  const size_t nd = up(N * a->dk * sizeof(float));
  FwdLayout l{};
  size_t off = kHeader;
  if (fwd_uses_tc(a)) {
    // the stage-1 step keeps its loss in the tensor-core epilogue: no fallback
    l.fallback = gla_on(a) && !stage1;
    if (l.fallback) {   // one mark per sequence, right after the header
      l.flags = off;
      off += up((size_t)a->B * a->H * sizeof(uint32_t));
    }
    l.phq = off;   // segment states of the tensor-core path
    off += up(lz::tc_fwd_workspace_bytes(a->B * a->H, a->L));
  } else if (gla_on(a)) {
    l.phq = off; off += nd;
    l.phk = off; off += nd;
    l.a = off; off += nd;
    l.o_gla = off; off += up(N * a->dv * sizeof(float));
  }
  l.total = off;
  return l;
}

// Whether the backward's anchor branch runs on the tensor-core kernels.
bool bwd_swa_uses_tc(const lizard_fwd_args *a, int impl) {
  const bool ok = lz::tc_swa_bwd_supported(a->dk, a->dv, a->window, a->M, a->dtype == LIZARD_BF16);
  return (impl == LIZARD_IMPL_AUTO || impl == LIZARD_IMPL_TC) && ok;
}

bool bwd_gla_uses_tc(const lizard_fwd_args *a, int impl) { return bwd_gla_uses_tc_impl(a, impl); }

struct BwdLayout {
  size_t phq, phk, a, sprev, dphq, dphk, da, dv_gla, dq_swa, dk_swa, dv_swa, lse, Dterm, snap_s,
      snap_ds, e32, gr, colsum, w16, kap, total;
  bool fallback;
  FallbackLayout fb;
};
BwdLayout bwd_layout(const lizard_fwd_args *a, int impl, bool stage1 = false) {
  const size_t BH = (size_t)a->B * a->H;
  const size_t N = BH * a->L;
  const size_t nd = up(N * a->dk * sizeof(float));
  const size_t nv = up(N * a->dv * sizeof(float));
  const size_t nch = (a->L + lz::kBwdC - 1) / lz::kBwdC;
  BwdLayout l{};
  size_t off = kHeader;
  if (gla_on(a) && bwd_gla_uses_tc(a, impl) && !stage1) {
    // exact fallback: per slot phi_q, phi_k, a, the chunk states and kap of
    // the portable backward, then its fp32 dphi_q, dphi_k
    const size_t Ld = up((size_t)a->L * a->dk * sizeof(float));
    const size_t per = 5 * Ld + up(nch * a->dk * a->dv * sizeof(float)) + up(a->dk * sizeof(float));
    l.fallback = true;
    l.fb = fallback_layout(off, a, per);
    off = l.fb.end;
  }
  if (gla_on(a) && bwd_gla_uses_tc(a, impl)) {
    // with a training forward's saved tensors, the state copies S', the
    // fp32 factors E and the tile decays come from there
    const bool saved = bwd_reads_saved(a, impl);
    const size_t snap = up(lz::tc_gla_bwd_snapshot_bytes((int)BH, a->L));
    if (!saved) { l.snap_s = off; off += snap; }
    l.snap_ds = off; off += snap;
    l.dphq = off; off += up(N * a->dk * 2);   // bf16, row halves centred
    l.dphk = off; off += up(N * a->dk * 2);
    l.da = off; off += nd;       // dB: gradient of the in-tile cumulative log-decay
    l.dv_gla = off; off += nv;
    if (!saved) {
      l.e32 = off; off += nd;      // fp32 decay factors E of every tile
      l.gr = off; off += up(BH * ((a->L + 127) / 128) * a->dk * sizeof(float));   // tiles' log-decays
    }
    l.colsum = off; off += up(BH * ((a->L + 127) / 128) * a->dk * sizeof(float));   // tiles' column sums of dB
    l.w16 = off; off += up(lz::tc_gla_bwd_weights_bytes(a->H));                  // bf16 W_q, W_k
    l.kap = off; off += up(BH * 2 * a->dk * sizeof(float));   // final-state share of the decay gradient
  } else if (gla_on(a)) {
    l.phq = off; off += nd;
    l.phk = off; off += nd;
    l.a = off; off += nd;
    l.sprev = off; off += up(BH * nch * a->dk * a->dv * sizeof(float));
    l.dphq = off; off += nd;
    l.dphk = off; off += nd;
    l.da = off; off += nd;
    l.dv_gla = off; off += nv;
    l.kap = off; off += up(BH * a->dk * sizeof(float));       // final-state share of the decay gradient
  }
  if (swa_on(a)) {
    l.dq_swa = off; off += nd;
    l.dk_swa = off; off += nd;
    l.dv_swa = off; off += nv;
    l.lse = off; off += up(N * sizeof(float));
    l.Dterm = off; off += up(N * sizeof(float));
  }
  l.total = off;
  return l;
}

template <typename P> P *at(void *base, size_t off) {
  return reinterpret_cast<P *>(static_cast<char *>(base) + off);
}

float scale_of(const lizard_fwd_args *a) {
  return a->softmax_scale > 0.f ? a->softmax_scale : 1.f / sqrtf((float)a->dk);
}

// A call's kernels in launch order.  The same list serves the launch and the
// host-only plan query, so the names always match what runs.  Kernels on
// lane 1 may run beside those on lane 0: fork() lets lane 1 start after
// everything enqueued so far, join() makes lane 0 wait for lane 1.  The
// lanes are the call's stream and a side stream of this host thread (created
// on the first call on a device, outside any stream capture; inside a
// capture without one, and whenever per-kernel timing events are requested,
// everything runs in order on the call's stream).
struct Plan {
  static constexpr int kMax = 32;
  struct Step {
    const char *name;
    std::function<cudaError_t(cudaStream_t)> fn;
    int lane;
    int sync;   // 0 kernel, 1 fork, 2 join
  };
  Step steps[kMax];
  int n = 0;
  void add(const char *name, std::function<cudaError_t(cudaStream_t)> f, int lane = 0) {
    steps[n++] = Step{name, std::move(f), lane, 0};
  }
  void fork() { steps[n++] = Step{nullptr, {}, 0, 1}; }
  void join() { steps[n++] = Step{nullptr, {}, 0, 2}; }
  lizard_status run(cudaStream_t s, void *const *events, int nev) const;
  int32_t names_out(const char **out, int32_t cap) const {
    int32_t k = 0;
    for (int i = 0; i < n; ++i)
      if (steps[i].sync == 0) {
        if (k < cap) out[k] = steps[i].name;
        ++k;
      }
    return k;
  }
};

// This host thread's side stream and fork / join events on the current
// device; false when they cannot be had (creation failed, or the stream is
// being captured and they do not exist yet).
bool side_lane(cudaStream_t s, cudaStream_t *side, cudaEvent_t *ev_fork, cudaEvent_t *ev_join) {
  constexpr int kDev = 64;
  thread_local cudaStream_t t_side[kDev] = {};
  thread_local cudaEvent_t t_fork[kDev] = {}, t_join[kDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDev) return false;
  if (!t_side[dev]) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return false;
    cudaStream_t st = nullptr;
    cudaEvent_t ef = nullptr, ej = nullptr;
    if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) return false;
    if (cudaEventCreateWithFlags(&ef, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ej, cudaEventDisableTiming) != cudaSuccess) {
      if (ef) cudaEventDestroy(ef);
      cudaStreamDestroy(st);
      return false;
    }
    t_side[dev] = st;
    t_fork[dev] = ef;
    t_join[dev] = ej;
  }
  *side = t_side[dev];
  *ev_fork = t_fork[dev];
  *ev_join = t_join[dev];
  return true;
}

lizard_status Plan::run(cudaStream_t s, void *const *events, int nev) const {
  const bool timing = events && nev > 0;
  bool any_fork = false;
  for (int i = 0; i < n; ++i) any_fork |= steps[i].sync == 1;
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  const bool lanes = !timing && any_fork && side_lane(s, &side, &ev_fork, &ev_join);
  if (timing && cudaEventRecord(static_cast<cudaEvent_t>(events[0]), s) != cudaSuccess) return LIZARD_ERR_CUDA;
  int k = 0;
  bool open = false;   // lane 1 has work that lane 0 has not joined
  for (int i = 0; i < n; ++i) {
    const Step &st = steps[i];
    if (st.sync == 1) {
      if (lanes && (cudaEventRecord(ev_fork, s) != cudaSuccess || cudaStreamWaitEvent(side, ev_fork, 0) != cudaSuccess))
        return LIZARD_ERR_CUDA;
      continue;
    }
    if (st.sync == 2) {
      if (lanes && open) {
        if (cudaEventRecord(ev_join, side) != cudaSuccess || cudaStreamWaitEvent(s, ev_join, 0) != cudaSuccess)
          return LIZARD_ERR_CUDA;
        open = false;
      }
      continue;
    }
    const bool on_side = lanes && st.lane == 1;
    if (st.fn(on_side ? side : s) != cudaSuccess) return LIZARD_ERR_CUDA;
    open |= on_side;
    ++k;
    if (timing && k < nev && cudaEventRecord(static_cast<cudaEvent_t>(events[k]), s) != cudaSuccess)
      return LIZARD_ERR_CUDA;
  }
  if (lanes && open &&
      (cudaEventRecord(ev_join, side) != cudaSuccess || cudaStreamWaitEvent(s, ev_join, 0) != cudaSuccess))
    return LIZARD_ERR_CUDA;
  return LIZARD_OK;
}

// Once per device, before the first kernel of a call: the GLA tile kernel's
// code goes in first (its placement then does not depend on the kernels that
// run before it).  False when the runtime refuses.
bool preload_once() {
  constexpr int kDev = 64;
  static bool done[kDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev < 0 || dev >= kDev || done[dev]) return true;
  if (lz::tc_gla_bwd_preload() != cudaSuccess) return false;
  done[dev] = true;
  return true;
}

// `target`, `dmse`, `loss`: the stage-1 loss, which the tensor-core forward
// forms in its epilogue (null otherwise).
void fwd_plan(const lizard_fwd_args *a, void *ws, cudaStream_t s, Plan &plan, const void *target = nullptr,
              void *dmse = nullptr, float *loss = nullptr) {
  const FwdLayout lay = fwd_layout(a, target != nullptr);
  const int BH = a->B * a->H, D = a->dk;
  const bool bf16 = a->dtype == LIZARD_BF16;
  if (fwd_uses_tc(a)) {
    lz::TcFwdArgs t{a->q, a->k, a->v, a->g, a->fmap_wq, a->fmap_wk, a->meta_k, a->meta_v, a->alpha,
                    a->state_in, a->o, gla_on(a) ? a->state_out : nullptr, swa_on(a) ? a->lse : nullptr,
                    static_cast<uint32_t *>(ws), at<void>(ws, lay.phq), BH, a->H, a->L, a->M, a->window,
                    a->branch, 1.f / a->gate_temp, scale_of(a), scalar_gate(a), target, dmse, loss,
                    a->k_prefix, a->v_prefix, a->prefix_len};
    // wide decay: the gate prep marks the sequences, whose GLA branch the
    // full pass then runs as the exact recurrence
    if (lay.fallback) t.seqflag = at<uint32_t>(ws, lay.flags);
    if (a->saved && fwd_keeps(a)) {   // training: keep what the backward would recompute
      const SavedLayout sv = saved_layout(a);
      // the stage-1 step (target set) forms its loss in the epilogue, so it
      // marks no sequence for the exact recurrence
      if (!target) t.seqflag = at<uint32_t>(a->saved, sv.flags);
      t.keep_r = at<float>(a->saved, sv.r);
      t.keep_e32 = at<float>(a->saved, sv.e32);
      t.snap = at<void>(a->saved, sv.snap);
      t.state_keep = at<float>(a->saved, sv.state);
      if (swa_on(a)) t.lse_keep = at<float>(a->saved, sv.lse);
    }
    if (gla_on(a)) plan.add("gate_prep_kernel", [=](cudaStream_t s) { return lz::launch_tc_fwd(t, 3, s); });
    if (gla_on(a) && lz::tc_fwd_stage_count(BH, a->L) > 1) {   // segment start states (GLA only)
      plan.add("tc_fwd_kernel(state pass)", [=](cudaStream_t s) { return lz::launch_tc_fwd(t, 0, s); });
      plan.add("seg_combine_kernel", [=](cudaStream_t s) { return lz::launch_tc_fwd(t, 1, s); });
    }
    plan.add("tc_fwd_kernel", [=](cudaStream_t s) { return lz::launch_tc_fwd(t, 2, s); });
    return;
  }
  float *o_gla = nullptr;
  if (gla_on(a)) {
    lz::PrepArgs pa{a->q, a->k, a->g, a->fmap_wq, a->fmap_wk, at<float>(ws, lay.phq), at<float>(ws, lay.phk),
                    at<float>(ws, lay.a), a->H, a->L, 1.f / a->gate_temp, scalar_gate(a)};
    plan.add("prep_kernel", [=](cudaStream_t s) { return lz::launch_prep(pa, BH, D, bf16, s); });
    o_gla = at<float>(ws, lay.o_gla);
    lz::GlaFwdArgs ga{at<float>(ws, lay.phq), at<float>(ws, lay.phk), at<float>(ws, lay.a), a->v, a->state_in,
                      o_gla, a->state_out, a->L};
    plan.add("gla_fwd_simt", [=](cudaStream_t s) { return lz::launch_gla_fwd_simt(ga, BH, D, bf16, s); });
  }
  lz::SwaMixArgs sa{a->q, a->k, a->v, a->meta_k, a->meta_v, a->alpha, o_gla, a->o,
                    swa_on(a) ? a->lse : nullptr, a->H, a->L, a->window, a->M, a->branch, scale_of(a),
                    a->k_prefix, a->v_prefix, a->prefix_len};
  plan.add("swa_mix_simt", [=](cudaStream_t s) { return lz::launch_swa_mix_simt(sa, BH, D, bf16, s); });
}

void bwd_plan(const lizard_bwd_args *b, void *ws, cudaStream_t s, Plan &plan, bool stage1 = false) {
  const lizard_fwd_args *a = &b->fwd;
  const BwdLayout lay = bwd_layout(a, b->impl, stage1);
  const int BH = a->B * a->H, D = a->dk;
  const bool bf16 = a->dtype == LIZARD_BF16;
  const float inv_tau = 1.f / a->gate_temp;
  const bool g = gla_on(a), w = swa_on(a);
  const bool gla_tc = g && bwd_gla_uses_tc(a, b->impl);
  if (gla_tc) {
    lz::TcFwdArgs f{a->q, a->k, a->v, a->g, a->fmap_wq, a->fmap_wk, a->meta_k, a->meta_v, a->alpha,
                    a->state_in, nullptr, nullptr, nullptr, static_cast<uint32_t *>(ws), nullptr, BH, a->H,
                    a->L, a->M, a->window, 0, inv_tau, scale_of(a), scalar_gate(a)};
    f.dstate_out = b->dstate_out;   // the state copies also form the final state's share of dg
    f.kap = at<float>(ws, lay.kap);
    const bool saved = bwd_reads_saved(a, b->impl);
    const SavedLayout sv = saved_layout(a);
    void *snap_s = saved ? at<void>(a->saved, sv.snap) : at<void>(ws, lay.snap_s);
    float *e32 = saved ? at<float>(a->saved, sv.e32) : at<float>(ws, lay.e32);
    float *gr = saved ? at<float>(a->saved, sv.r) : at<float>(ws, lay.gr);
    uint32_t *status = static_cast<uint32_t *>(ws);
    uint32_t *flags = !lay.fallback ? nullptr : saved ? at<uint32_t>(a->saved, sv.flags) : at<uint32_t>(ws, lay.fb.flags);
    if (!saved)
      plan.add("gate_prep_kernel", [=](cudaStream_t s) {
        return lz::launch_gate_prep(a->g, nullptr, e32, gr, status, BH, a->L, inv_tau, f.scalar_gate != 0, s, flags);
      });
    if (lay.fallback) {
      const FallbackLayout fb = lay.fb;
      const int K = fallback_slots(a);
      plan.add("assign_slots_kernel", [=](cudaStream_t s) {
        return lz::launch_assign_slots(flags, at<int>(ws, fb.slot_of), at<int>(ws, fb.seq_of_slot), BH, K, status, s);
      });
    }
    if (saved) {
      // the forward kept the state copies; the final state's share of dg
      // comes from its kept final state
      if (b->dstate_out) {
        const float *sl = at<float>(a->saved, sv.state);
        float *kap = f.kap;
        plan.add("state_share_kernel", [=](cudaStream_t s) { return lz::launch_state_share(sl, b->dstate_out, kap, BH, s); });
      }
    } else {
      // the state copies beside the weight conversion and the reverse dS pass
      plan.fork();
      plan.add("tc_fwd_kernel(state copies)",
               [=](cudaStream_t s) { return lz::launch_tc_state_snapshots(f, snap_s, e32, gr, s); }, 1);
    }
    lz::TcGlaBwdArgs t{a->q, a->k, a->v, a->g, b->dout, a->fmap_wq, a->fmap_wk, snap_s,
                       at<void>(ws, lay.snap_ds), at<float>(ws, lay.dphq), at<float>(ws, lay.dphk),
                       at<float>(ws, lay.da), at<float>(ws, lay.dv_gla), b->dg, b->dstate_in,
                       status, a->H, BH, a->L, inv_tau, e32, gr, scalar_gate(a), at<void>(ws, lay.w16),
                       b->dstate_out};
    t.colsum = at<float>(ws, lay.colsum);
    void *w16 = at<void>(ws, lay.w16);
    plan.add("weights_bf16_kernel", [=](cudaStream_t s) { return lz::launch_weights_bf16(a->fmap_wq, a->fmap_wk, w16, a->H, s); });
    plan.add("tc_gla_dstates_kernel", [=](cudaStream_t s) { return lz::launch_tc_gla_bwd(t, 0, s); });
    plan.join();
    plan.add("tc_gla_bwd_tile_kernel", [=](cudaStream_t s) { return lz::launch_tc_gla_bwd(t, 1, s); });
    if (lay.fallback) {
      // the GLA backward of the marked sequences, exactly, on the portable
      // kernels: their dphi_q, dphi_k, dv and dstate_in replace what the
      // tensor-core kernels wrote, and their per-token da goes to the dB
      // array (the marked sequences' dg is formed from it at the end)
      const FallbackLayout fb = lay.fb;
      const int K = fallback_slots(a);
      const int *seq = at<int>(ws, fb.seq_of_slot);
      const size_t Ld = up((size_t)a->L * a->dk * sizeof(float));
      const size_t o_phq = fb.scratch, o_phk = o_phq + K * Ld, o_a = o_phk + K * Ld, o_sp = o_a + K * Ld;
      const size_t o_kap = o_sp + K * up(nch32(a) * a->dk * a->dv * sizeof(float));
      const size_t o_dpq = o_kap + K * up(a->dk * sizeof(float)), o_dpk = o_dpq + K * Ld;
      lz::PrepArgs pa{a->q, a->k, a->g, a->fmap_wq, a->fmap_wk, at<float>(ws, o_phq), at<float>(ws, o_phk),
                      at<float>(ws, o_a), a->H, a->L, inv_tau, scalar_gate(a), seq};
      plan.add("prep_kernel(exact fallback)", [=](cudaStream_t s) { return lz::launch_prep(pa, K, D, bf16, s); });
      float *kap = b->dstate_out ? at<float>(ws, o_kap) : nullptr;
      lz::GlaStatesArgs sa{pa.phk, pa.a, a->v, a->state_in, at<float>(ws, o_sp), a->L, b->dstate_out, kap, seq};
      plan.add("gla_states_simt(exact fallback)",
               [=](cudaStream_t s) { return lz::launch_gla_states(sa, K, D, bf16, s); });
      lz::GlaBwdArgs ga{pa.phq, pa.phk, pa.a, a->v, b->dout, at<float>(ws, o_sp), at<float>(ws, o_dpq),
                        at<float>(ws, o_dpk), at<float>(ws, lay.da), at<float>(ws, lay.dv_gla), b->dstate_in,
                        a->L, b->dstate_out, kap, seq};
      plan.add("gla_bwd_simt(exact fallback)",
               [=](cudaStream_t s) { return lz::launch_gla_bwd_simt(ga, K, D, bf16, s); });
    }
  } else if (g) {
    lz::PrepArgs pa{a->q, a->k, a->g, a->fmap_wq, a->fmap_wk, at<float>(ws, lay.phq), at<float>(ws, lay.phk),
                    at<float>(ws, lay.a), a->H, a->L, inv_tau, scalar_gate(a)};
    plan.add("prep_kernel", [=](cudaStream_t s) { return lz::launch_prep(pa, BH, D, bf16, s); });
    float *kap = b->dstate_out ? at<float>(ws, lay.kap) : nullptr;
    lz::GlaStatesArgs sa{at<float>(ws, lay.phk), at<float>(ws, lay.a), a->v, a->state_in, at<float>(ws, lay.sprev), a->L,
                         b->dstate_out, kap};
    plan.add("gla_states_simt", [=](cudaStream_t s) { return lz::launch_gla_states(sa, BH, D, bf16, s); });
    lz::GlaBwdArgs ga{at<float>(ws, lay.phq), at<float>(ws, lay.phk), at<float>(ws, lay.a), a->v, b->dout,
                      at<float>(ws, lay.sprev), at<float>(ws, lay.dphq), at<float>(ws, lay.dphk),
                      at<float>(ws, lay.da), at<float>(ws, lay.dv_gla), b->dstate_in, a->L, b->dstate_out, kap};
    plan.add("gla_bwd_simt", [=](cudaStream_t s) { return lz::launch_gla_bwd_simt(ga, BH, D, bf16, s); });
  }
  const bool swa_tc = w && bwd_swa_uses_tc(a, b->impl);
  const bool finish_tc = gla_tc && a->fmap_wq && a->fmap_wk;
  // With both branches on the tensor cores, the feature-map backward runs
  // first and hands its parts (bf16) to the anchor kernels, which add them
  // and write the final dq, dk, dv; otherwise the finish kernel sums fp32
  // parts of both branches at the end.
  const bool fused = finish_tc && swa_tc;
  lz::FinishBwdArgs fa{a->q, a->k, a->g,
                       a->fmap_wq, a->fmap_wk,
                       g ? at<float>(ws, lay.dphq) : nullptr, g ? at<float>(ws, lay.dphk) : nullptr,
                       g ? at<float>(ws, lay.da) : nullptr, g ? at<float>(ws, lay.dv_gla) : nullptr,
                       w ? at<float>(ws, lay.dq_swa) : nullptr, w ? at<float>(ws, lay.dk_swa) : nullptr,
                       w ? at<float>(ws, lay.dv_swa) : nullptr,
                       b->dq, b->dk, b->dv, b->dg, b->dfmap_wq, b->dfmap_wk, a->H, a->L, inv_tau,
                       gla_tc ? 0 : 1, static_cast<uint32_t *>(ws), nullptr, nullptr, scalar_gate(a)};
  if (gla_tc) fa.da = nullptr;   // the gate gradient comes from gate_grad_kernel
  if (finish_tc) {   // the tensor-core GLA backward's dphi: bf16, row halves centred
    fa.dphq16 = at<void>(ws, lay.dphq);
    fa.dphk16 = at<void>(ws, lay.dphk);
    fa.dphq = fa.dphk = nullptr;
    if (lay.fallback) {
      const int K = fallback_slots(a);
      const size_t Ld = up((size_t)a->L * a->dk * sizeof(float));
      const size_t o_kap = lay.fb.scratch + 3 * K * Ld + K * up(nch32(a) * a->dk * a->dv * sizeof(float));
      const size_t o_dpq = o_kap + K * up(a->dk * sizeof(float));
      fa.slot_of = at<int>(ws, lay.fb.slot_of);
      fa.fb_dphq = at<float>(ws, o_dpq);
      fa.fb_dphk = at<float>(ws, o_dpq + K * Ld);
    }
  }
  lz::TcGlaBwdArgs tg{a->q, a->k, a->v, a->g, b->dout, a->fmap_wq, a->fmap_wk, nullptr, nullptr, nullptr,
                      nullptr, at<float>(ws, lay.da), nullptr, b->dg, nullptr, static_cast<uint32_t *>(ws),
                      a->H, BH, a->L, inv_tau, nullptr, nullptr, scalar_gate(a)};
  if (gla_tc && b->dstate_out) tg.kap = at<float>(ws, lay.kap);
  if (gla_tc) tg.colsum = at<float>(ws, lay.colsum);
  if (fused) {
    // the gate-logit gradient (from dB) beside the feature-map and anchor passes
    plan.fork();
    plan.add("gate_grad_kernel", [=](cudaStream_t s) { return lz::launch_tc_gla_bwd(tg, 2, s); }, 1);
    fa.xq_part = at<void>(ws, lay.dq_swa);   // bf16 parts in the anchor part slots
    fa.xk_part = at<void>(ws, lay.dk_swa);
    fa.dq_swa = fa.dk_swa = fa.dv_swa = nullptr;
    plan.add("tc_finish_kernel", [=](cudaStream_t s) { return lz::launch_tc_finish(fa, BH, s); });
  }
  if (swa_tc) {
    lz::TcSwaBwdArgs t{a->q, a->k, a->v, b->dout, a->meta_k, a->meta_v, a->alpha,
                       at<float>(ws, lay.dq_swa), at<float>(ws, lay.dk_swa), at<float>(ws, lay.dv_swa),
                       at<float>(ws, lay.lse), at<float>(ws, lay.Dterm), b->dmeta_k, b->dmeta_v, b->dalpha,
                       static_cast<uint32_t *>(ws),
                       a->B, a->H, BH, a->L, a->M, a->window, scale_of(a)};
    if (fused) {
      t.dq = t.dk = t.dv = nullptr;
      t.xq_part = at<void>(ws, lay.dq_swa);
      t.xk_part = at<void>(ws, lay.dk_swa);
      t.dv_gla = at<float>(ws, lay.dv_gla);
      t.dq_out = b->dq;
      t.dk_out = b->dk;
      t.dv_out = b->dv;
    }
    t.k_prefix = a->k_prefix;
    t.v_prefix = a->v_prefix;
    t.dk_prefix = b->dk_prefix;
    t.dv_prefix = b->dv_prefix;
    t.P = a->prefix_len;
    // the training forward's softmax normalisers spare the dq pass its max pass
    if (bwd_reads_saved(a, b->impl)) t.lse_in = at<float>(a->saved, saved_layout(a).lse);
    plan.add("tc_swa_bwd_q_kernel", [=](cudaStream_t s) { return lz::launch_tc_swa_bwd(t, 0, s); });
    plan.add("tc_swa_bwd_kv_kernel", [=](cudaStream_t s) { return lz::launch_tc_swa_bwd(t, 1, s); });
    plan.join();
  } else if (w) {
    lz::SwaBwdQArgs qa{a->q, a->k, a->v, b->dout, a->meta_k, a->meta_v, a->alpha,
                       at<float>(ws, lay.dq_swa), at<float>(ws, lay.lse), at<float>(ws, lay.Dterm),
                       b->dmeta_k, b->dmeta_v, b->dalpha, a->H, a->L, a->window, a->M, scale_of(a),
                       a->k_prefix, a->v_prefix, a->prefix_len};
    plan.add("swa_bwd_q", [=](cudaStream_t s) { return lz::launch_swa_bwd_q(qa, BH, D, bf16, s); });
    lz::SwaBwdKVArgs ka{a->q, a->k, a->v, b->dout, a->alpha, at<float>(ws, lay.lse), at<float>(ws, lay.Dterm),
                        at<float>(ws, lay.dk_swa), at<float>(ws, lay.dv_swa), a->H, a->L, a->window, scale_of(a),
                        a->k_prefix, a->v_prefix, b->dk_prefix, b->dv_prefix, a->prefix_len};
    plan.add("swa_bwd_kv", [=](cudaStream_t s) { return lz::launch_swa_bwd_kv(ka, BH, D, bf16, s); });
  }
  if (!fused) {
    if (finish_tc)
      plan.add("tc_finish_kernel", [=](cudaStream_t s) { return lz::launch_tc_finish(fa, BH, s); });
    else
      plan.add("finish_bwd", [=](cudaStream_t s) { return lz::launch_finish_bwd(fa, BH, D, bf16, s); });
  }
  if (gla_tc && !fused)
    plan.add("gate_grad_kernel", [=](cudaStream_t s) { return lz::launch_tc_gla_bwd(tg, 2, s); });
  if (lay.fallback) {   // dg of the marked sequences from the exact da (after the gate-gradient pass)
    const int K = fallback_slots(a);
    const int *seq = at<int>(ws, lay.fb.seq_of_slot);
    const float *da = at<float>(ws, lay.da);
    plan.add("slot_dg_kernel", [=](cudaStream_t s) {
      return lz::launch_slot_dg(b->dg, da, a->g, seq, K, a->L, D, inv_tau, scalar_gate(a) != 0, bf16, s);
    });
  }
}

}  // namespace

extern "C" {

size_t lizard_fwd_workspace_size(const lizard_fwd_args *args) {
  lizard_fwd_args a;
  if (!args) return 0;
  a = *args;
  a.q = a.k = a.v = a.g = nullptr;
  a.o = nullptr;
  a.workspace = nullptr;
  a.alpha = a.state_in = nullptr;
  // whether feature-map weights are given selects the kernels (and so the layout)
  a.fmap_wq = args->fmap_wq ? reinterpret_cast<const float *>(16) : nullptr;
  a.fmap_wk = args->fmap_wk ? reinterpret_cast<const float *>(16) : nullptr;
  a.state_out = a.lse = nullptr;
  const bool meta = a.M > 0;
  a.meta_k = meta ? reinterpret_cast<const float *>(16) : nullptr;
  a.meta_v = nullptr;
  if (a.L > 0) {
    // the pointer checks require non-null activations; use a stand-in
    a.q = a.k = a.v = a.g = reinterpret_cast<const void *>(16);
    a.o = reinterpret_cast<void *>(16);
  }
  prefix_standin(a);
  if (check_fwd(&a) != LIZARD_OK) return 0;
  return fwd_layout(&a).total;
}

size_t lizard_fwd_saved_size(const lizard_fwd_args *args) {
  if (!args) return 0;
  lizard_fwd_args a = *args;
  a.fmap_wq = args->fmap_wq ? reinterpret_cast<const float *>(16) : nullptr;
  a.fmap_wk = args->fmap_wk ? reinterpret_cast<const float *>(16) : nullptr;
  a.q = a.k = a.v = a.g = reinterpret_cast<const void *>(16);
  a.o = reinterpret_cast<void *>(16);
  a.meta_k = a.M > 0 ? reinterpret_cast<const float *>(16) : nullptr;
  a.meta_v = a.alpha = a.state_in = a.state_out = a.lse = nullptr;
  a.workspace = a.saved = nullptr;
  prefix_standin(a);
  if (check_fwd(&a) != LIZARD_OK || a.L == 0) return 0;
  return saved_layout(&a).total;
}

lizard_status lizard_attn_fwd(const lizard_fwd_args *a, lizard_stream_t stream) {
  lizard_status st = check_fwd(a);
  if (st != LIZARD_OK) return st;
  if (a->impl == LIZARD_IMPL_TC && !fwd_uses_tc(a)) return LIZARD_ERR_UNSUPPORTED;
  const FwdLayout lay = fwd_layout(a);
  if (!a->workspace || a->workspace_bytes < lay.total) return LIZARD_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int BH = a->B * a->H;
  const size_t BHdd = (size_t)BH * a->dk * a->dv * sizeof(float);
  if (a->L == 0) {
    if (a->state_out) {
      cudaError_t e = a->state_in ? cudaMemcpyAsync(a->state_out, a->state_in, BHdd, cudaMemcpyDeviceToDevice, s)
                                  : cudaMemsetAsync(a->state_out, 0, BHdd, s);
      return cuda_status(e);
    }
    return LIZARD_OK;
  }
  const bool keep = a->saved && fwd_keeps(a);
  const SavedLayout sv = saved_layout(a);
  if (keep && a->saved_bytes < sv.total) return LIZARD_ERR_WORKSPACE;
  if (cudaMemsetAsync(a->workspace, 0, cleared_bytes(a, lay.fallback), s) != cudaSuccess) return LIZARD_ERR_CUDA;
  // a training forward's wide-decay marks start cleared
  if (keep && cudaMemsetAsync(at<void>(a->saved, sv.flags), 0, (size_t)BH * sizeof(uint32_t), s) != cudaSuccess)
    return LIZARD_ERR_CUDA;
  if (!preload_once()) return LIZARD_ERR_CUDA;
  Plan plan;
  fwd_plan(a, a->workspace, s, plan);
  return plan.run(s, a->launch_events, a->n_launch_events);
}

static lizard_status check_bwd(const lizard_bwd_args *b) {
  if (!b) return LIZARD_ERR_INVALID_ARG;
  lizard_fwd_args f = b->fwd;
  f.o = b->dq;  // the forward output is not used; dq stands in for the pointer check
  f.state_out = nullptr;
  f.lse = nullptr;
  f.workspace = b->workspace;
  f.impl = b->impl;
  lizard_status st = check_fwd(&f);
  if (st != LIZARD_OK) return st;
  if (f.L > 0 && (!b->dout || !b->dq || !b->dk || !b->dv || !b->dg)) return LIZARD_ERR_INVALID_ARG;
  if ((b->dmeta_k && !f.meta_k) || (b->dmeta_v && !f.meta_v) || (b->dfmap_wq && !f.fmap_wq) ||
      (b->dfmap_wk && !f.fmap_wk))
    return LIZARD_ERR_INVALID_ARG;
  if (b->dstate_out && !gla_on(&f)) return LIZARD_ERR_INVALID_ARG;   // no final state without the GLA branch
  if (f.prefix_len == 0 && (b->dk_prefix || b->dv_prefix)) return LIZARD_ERR_INVALID_ARG;
  const void *ptrs[] = {b->dout, b->dq, b->dk, b->dv, b->dg, b->dmeta_k, b->dmeta_v,
                        b->dfmap_wq, b->dfmap_wk, b->dalpha, b->dstate_in, b->dstate_out,
                        b->dk_prefix, b->dv_prefix};
  for (const void *p : ptrs)
    if (!ok_ptr(p)) return LIZARD_ERR_INVALID_ARG;
  return LIZARD_OK;
}

size_t lizard_bwd_workspace_size(const lizard_bwd_args *args) {
  if (!args) return 0;
  lizard_fwd_args a = args->fwd;
  a.impl = args->impl;
  a.q = a.k = a.v = a.g = nullptr;
  a.o = nullptr;
  a.workspace = nullptr;
  a.alpha = a.state_in = nullptr;
  // whether feature-map weights are given selects the kernels (and so the layout)
  a.fmap_wq = args->fwd.fmap_wq ? reinterpret_cast<const float *>(16) : nullptr;
  a.fmap_wk = args->fwd.fmap_wk ? reinterpret_cast<const float *>(16) : nullptr;
  a.state_out = a.lse = nullptr;
  a.meta_k = a.M > 0 ? reinterpret_cast<const float *>(16) : nullptr;
  a.meta_v = nullptr;
  if (a.L > 0) {
    a.q = a.k = a.v = a.g = reinterpret_cast<const void *>(16);
    a.o = reinterpret_cast<void *>(16);
  }
  prefix_standin(a);
  if (check_fwd(&a) != LIZARD_OK) return 0;
  return bwd_layout(&a, args->impl).total;
}

// Gradient outputs that the kernels accumulate atomically start at zero; so
// does dstate_in when no kernel writes it.
static cudaError_t bwd_zero_outputs(const lizard_bwd_args *b, cudaStream_t s) {
  const lizard_fwd_args *a = &b->fwd;
  const int BH = a->B * a->H, D = a->dk, F = D / 2;
  cudaError_t e = cudaSuccess;
  struct Z { void *p; size_t n; } zs[] = {
      {b->dmeta_k, (size_t)a->H * a->M * a->dk * 4}, {b->dmeta_v, (size_t)a->H * a->M * a->dv * 4},
      {b->dfmap_wq, (size_t)a->H * D * F * 4},       {b->dfmap_wk, (size_t)a->H * D * F * 4},
      {b->dalpha, (size_t)a->H * 4}};
  for (const Z &z : zs)
    if (z.p && z.n && (e = cudaMemsetAsync(z.p, 0, z.n, s)) != cudaSuccess) return e;
  const size_t BHdd = (size_t)BH * a->dk * a->dv * sizeof(float);
  if ((a->L == 0 || !gla_on(a)) && b->dstate_in) e = cudaMemsetAsync(b->dstate_in, 0, BHdd, s);
  if (e != cudaSuccess) return e;
  // the prefix is read only by the anchor branch: without it (or without
  // queries) its gradients are zero
  if (a->prefix_len > 0 && (a->L == 0 || !swa_on(a)) && b->dk_prefix && b->dv_prefix) {
    const size_t esz = a->dtype == LIZARD_BF16 ? 2 : 4;
    const size_t n = (size_t)BH * a->prefix_len * a->dk * esz;
    if ((e = cudaMemsetAsync(b->dk_prefix, 0, n, s)) != cudaSuccess) return e;
    e = cudaMemsetAsync(b->dv_prefix, 0, n, s);
  }
  return e;
}

lizard_status lizard_attn_bwd(const lizard_bwd_args *b, lizard_stream_t stream) {
  lizard_status st = check_bwd(b);
  if (st != LIZARD_OK) return st;
  const lizard_fwd_args *a = &b->fwd;
  if (b->impl == LIZARD_IMPL_TC && swa_on(a) && !bwd_swa_uses_tc(a, b->impl)) return LIZARD_ERR_UNSUPPORTED;
  if (b->impl == LIZARD_IMPL_TC && gla_on(a) && !bwd_gla_uses_tc(a, b->impl)) return LIZARD_ERR_UNSUPPORTED;
  // with a prefix, its key and value gradients are outputs of the call
  if (a->prefix_len > 0 && (!b->dk_prefix || !b->dv_prefix)) return LIZARD_ERR_INVALID_ARG;
  const BwdLayout lay = bwd_layout(a, b->impl);
  if (!b->workspace || b->workspace_bytes < lay.total) return LIZARD_ERR_WORKSPACE;
  if (bwd_reads_saved(a, b->impl) && a->saved_bytes < saved_layout(a).total) return LIZARD_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (bwd_zero_outputs(b, s) != cudaSuccess) return LIZARD_ERR_CUDA;
  if (a->L == 0) return LIZARD_OK;
  void *ws = b->workspace;
  if (cudaMemsetAsync(ws, 0, cleared_bytes(a, lay.fallback), s) != cudaSuccess) return LIZARD_ERR_CUDA;
  if (!preload_once()) return LIZARD_ERR_CUDA;
  Plan plan;
  bwd_plan(b, ws, s, plan);
  return plan.run(s, b->launch_events, b->n_launch_events);
}

// ---------------------------------------------------------- stage 1 ----
// One workspace for the whole step: the forward's and the backward's scratch
// share its start (the backward begins after the forward's last kernel, and
// both keep the status word at offset 0), then dL/do, then the forward's
// saved-for-backward tensors when both GLA halves run on the tensor cores,
// then the output when the portable forward needs one and the caller gave
// none.
}  // extern "C"

namespace {

// Whether the step's forward keeps the backward's tensors (the forward's
// GLA branch on the tensor cores and the backward's GLA kernels too).
bool s1_keeps(const lizard_stage1_args *a) {
  return fwd_keeps(&a->bwd.fwd) && bwd_gla_uses_tc_impl(&a->bwd.fwd, a->bwd.impl);
}

struct S1Layout {
  size_t dmse, saved, saved_bytes, o, total;
};
S1Layout s1_layout(const lizard_stage1_args *a) {
  const lizard_bwd_args *b = &a->bwd;
  lizard_fwd_args f = b->fwd;   // the caller's fwd.saved is not used: the step keeps its own
  f.saved = s1_keeps(a) ? reinterpret_cast<void *>(16) : nullptr;
  const size_t fw = fwd_layout(&f, true).total, bw = bwd_layout(&f, b->impl, true).total;
  const size_t nel = (size_t)f.B * f.H * f.L * f.dv, esz = f.dtype == LIZARD_BF16 ? 2 : 4;
  S1Layout l{};
  size_t off = up(fw > bw ? fw : bw);
  l.dmse = off;
  off += up(nel * esz);
  if (f.saved) {
    l.saved = off;
    l.saved_bytes = saved_layout(&f).total;
    off += up(l.saved_bytes);
  }
  if (!f.o && !fwd_uses_tc(&f)) {
    l.o = off;
    off += up(nel * esz);
  }
  l.total = off;
  return l;
}

lizard_status check_stage1(const lizard_stage1_args *a) {
  if (!a) return LIZARD_ERR_INVALID_ARG;
  lizard_bwd_args b = a->bwd;
  b.dout = b.dq;   // dL/do comes from the loss; dq stands in for the pointer check
  const lizard_status st = check_bwd(&b);
  if (st != LIZARD_OK) return st;
  if (b.fwd.L > 0 && (!a->target || !a->loss)) return LIZARD_ERR_INVALID_ARG;
  if (!ok_ptr(a->target) || !ok_ptr(a->loss) || !ok_ptr(b.fwd.o)) return LIZARD_ERR_INVALID_ARG;
  return LIZARD_OK;
}

// The forward and backward argument views that the step's kernels read; they
// must outlive the plan's run.
struct S1Views {
  lizard_fwd_args f;
  lizard_bwd_args b;
};

void stage1_plan(const lizard_stage1_args *a, S1Views &v, void *ws, cudaStream_t s, Plan &plan) {
  const S1Layout lay = s1_layout(a);
  v.b = a->bwd;
  v.b.fwd.saved = lay.saved_bytes ? at<void>(ws, lay.saved) : nullptr;
  v.b.fwd.saved_bytes = lay.saved_bytes;
  v.f = v.b.fwd;
  v.f.workspace = ws;
  void *dmse = at<void>(ws, lay.dmse);
  const lizard_fwd_args *f = &v.f;
  if (fwd_uses_tc(f)) {
    fwd_plan(f, ws, s, plan, a->target, dmse, a->loss);
  } else {
    if (!v.f.o) v.f.o = at<void>(ws, lay.o);
    fwd_plan(f, ws, s, plan);
    const size_t nel = (size_t)f->B * f->H * f->L * f->dv;
    const bool bf16 = f->dtype == LIZARD_BF16;
    const void *target = a->target;
    float *loss = a->loss;
    plan.add("mse_kernel", [=](cudaStream_t s) { return lz::launch_mse(f->o, target, dmse, loss, nel, bf16, s); });
  }
  v.b.dout = dmse;
  bwd_plan(&v.b, ws, s, plan, true);
}

}  // namespace

extern "C" {

size_t lizard_stage1_workspace_size(const lizard_stage1_args *args) {
  if (!args) return 0;
  lizard_stage1_args a = *args;
  lizard_fwd_args &f = a.bwd.fwd;
  f.impl = args->bwd.fwd.impl;
  const bool keep_o = f.o != nullptr;
  f.q = f.k = f.v = f.g = nullptr;
  f.o = nullptr;
  f.alpha = f.state_in = nullptr;
  // whether feature-map weights are given selects the kernels (and so the layout)
  f.fmap_wq = args->bwd.fwd.fmap_wq ? reinterpret_cast<const float *>(16) : nullptr;
  f.fmap_wk = args->bwd.fwd.fmap_wk ? reinterpret_cast<const float *>(16) : nullptr;
  f.state_out = f.lse = nullptr;
  f.meta_k = f.M > 0 ? reinterpret_cast<const float *>(16) : nullptr;
  f.meta_v = nullptr;
  if (f.L > 0) f.q = f.k = f.v = f.g = reinterpret_cast<const void *>(16);
  f.workspace = nullptr;
  lizard_fwd_args chk = f;
  chk.o = reinterpret_cast<void *>(16);
  prefix_standin(chk);
  if (check_fwd(&chk) != LIZARD_OK) return 0;
  if (keep_o) f.o = reinterpret_cast<void *>(16);
  return s1_layout(&a).total;
}

lizard_status lizard_stage1_step(const lizard_stage1_args *a, lizard_stream_t stream) {
  lizard_status st = check_stage1(a);
  if (st != LIZARD_OK) return st;
  const lizard_bwd_args *b = &a->bwd;
  const lizard_fwd_args *f = &b->fwd;
  if (f->impl == LIZARD_IMPL_TC && !fwd_uses_tc(f)) return LIZARD_ERR_UNSUPPORTED;
  if (b->impl == LIZARD_IMPL_TC && swa_on(f) && !bwd_swa_uses_tc(f, b->impl)) return LIZARD_ERR_UNSUPPORTED;
  if (b->impl == LIZARD_IMPL_TC && gla_on(f) && !bwd_gla_uses_tc(f, b->impl)) return LIZARD_ERR_UNSUPPORTED;
  if (f->prefix_len != 0) return LIZARD_ERR_UNSUPPORTED;   // whole sequences only
  const S1Layout lay = s1_layout(a);
  if (!b->workspace || b->workspace_bytes < lay.total) return LIZARD_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (bwd_zero_outputs(b, s) != cudaSuccess) return LIZARD_ERR_CUDA;
  if (a->loss && cudaMemsetAsync(a->loss, 0, sizeof(float), s) != cudaSuccess) return LIZARD_ERR_CUDA;
  if (f->L == 0) return LIZARD_OK;
  void *ws = b->workspace;
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) return LIZARD_ERR_CUDA;
  S1Views views;
  if (!preload_once()) return LIZARD_ERR_CUDA;
  Plan plan;
  stage1_plan(a, views, ws, s, plan);
  return plan.run(s, b->launch_events, b->n_launch_events);
}

int32_t lizard_stage1_launch_plan(const lizard_stage1_args *a, const char **names, int32_t cap) {
  if (check_stage1(a) != LIZARD_OK) return -1;
  if (a->bwd.fwd.L == 0) return 0;
  S1Views views;
  Plan plan;
  stage1_plan(a, views, a->bwd.workspace, nullptr, plan);
  return plan.names_out(names, cap);
}

int32_t lizard_fwd_launch_plan(const lizard_fwd_args *a, const char **names, int32_t cap) {
  if (check_fwd(a) != LIZARD_OK) return -1;
  if (a->L == 0) return 0;
  Plan plan;
  fwd_plan(a, a->workspace, nullptr, plan);
  return plan.names_out(names, cap);
}

int32_t lizard_bwd_launch_plan(const lizard_bwd_args *b, const char **names, int32_t cap) {
  if (check_bwd(b) != LIZARD_OK) return -1;
  if (b->fwd.L == 0) return 0;
  Plan plan;
  bwd_plan(b, b->workspace, nullptr, plan);
  return plan.names_out(names, cap);
}

lizard_status lizard_decode_step(const lizard_decode_args *a, lizard_stream_t stream) {
  if (!a) return LIZARD_ERR_INVALID_ARG;
  if (a->B < 1 || a->H < 1 || a->dk <= 0 || a->dv <= 0 || a->window < 1 || a->M < 0) return LIZARD_ERR_INVALID_ARG;
  if (a->dtype != LIZARD_BF16 && a->dtype != LIZARD_FP32) return LIZARD_ERR_INVALID_ARG;
  if (a->gate != LIZARD_GATE_PER_DIM && a->gate != LIZARD_GATE_SCALAR) return LIZARD_ERR_INVALID_ARG;
  if (!(a->gate_temp > 0.f) || !isfinite(a->gate_temp)) return LIZARD_ERR_INVALID_ARG;
  if (!(a->softmax_scale >= 0.f) || !isfinite(a->softmax_scale)) return LIZARD_ERR_INVALID_ARG;
  if (a->dk != a->dv || (a->dk != 64 && a->dk != 128)) return LIZARD_ERR_UNSUPPORTED;
  if (a->M > 16 || a->window > 16384) return LIZARD_ERR_UNSUPPORTED;
  if ((a->M > 0) != (a->meta_k != nullptr)) return LIZARD_ERR_INVALID_ARG;
  if (a->meta_v && !a->meta_k) return LIZARD_ERR_INVALID_ARG;
  if (!a->q || !a->k || !a->v || !a->g || !a->state || !a->k_cache || !a->v_cache || !a->pos || !a->o)
    return LIZARD_ERR_INVALID_ARG;
  const void *ptrs[] = {a->q, a->k, a->v, a->g, a->state, a->k_cache, a->v_cache, a->pos,
                        a->fmap_wq, a->fmap_wk, a->meta_k, a->meta_v, a->alpha, a->o};
  for (const void *p : ptrs)
    if (!ok_ptr(p)) return LIZARD_ERR_INVALID_ARG;
  lz::DecodeArgs d{a->q, a->k, a->v, a->g, a->state, a->k_cache, a->v_cache, a->pos,
                   a->fmap_wq, a->fmap_wk, a->meta_k, a->meta_v, a->alpha, a->o,
                   a->H, a->window, a->M, 1.f / a->gate_temp,
                   a->softmax_scale > 0.f ? a->softmax_scale : 1.f / sqrtf((float)a->dk),
                   a->gate == LIZARD_GATE_SCALAR ? 1 : 0};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool bf16 = a->dtype == LIZARD_BF16;
  if (lz::decode_stream_supported(a->dk, bf16, a->window, a->M))
    return cuda_status(lz::launch_decode_stream(d, a->B, a->pos, s));
  return cuda_status(lz::launch_decode(d, a->B, a->dk, bf16, a->pos, s));
}

lizard_status lizard_prefill_cache(const lizard_cache_args *a, lizard_stream_t stream) {
  if (!a) return LIZARD_ERR_INVALID_ARG;
  if (a->B < 1 || a->H < 1 || a->L < 0 || a->dk <= 0 || a->dv <= 0 || a->window < 1) return LIZARD_ERR_INVALID_ARG;
  if (a->dtype != LIZARD_BF16 && a->dtype != LIZARD_FP32) return LIZARD_ERR_INVALID_ARG;
  if (a->dk != a->dv || (a->dk != 64 && a->dk != 128) || a->window > 16384) return LIZARD_ERR_UNSUPPORTED;
  if (!a->k_cache || !a->v_cache || !a->pos || (a->L > 0 && (!a->k || !a->v))) return LIZARD_ERR_INVALID_ARG;
  const void *ptrs[] = {a->k, a->v, a->k_cache, a->v_cache, a->pos};
  for (const void *p : ptrs)
    if (!ok_ptr(p)) return LIZARD_ERR_INVALID_ARG;
  const size_t esz = a->dtype == LIZARD_BF16 ? 2 : 4;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return cuda_status(lz::launch_prefill_cache(a->k, a->v, a->k_cache, a->v_cache, a->pos, a->B, a->H, a->L,
                                              a->window, a->dk * esz, a->dv * esz, s));
}

lizard_status lizard_decode_status(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return LIZARD_ERR_CUDA;
  const int v = lz::decode_stream_status_take();
  if (v < 0) return LIZARD_ERR_CUDA;
  return (v & 1) ? LIZARD_ERR_TIMEOUT : LIZARD_OK;
}

lizard_status lizard_workspace_status(void *workspace, lizard_stream_t stream) {
  if (!workspace) return LIZARD_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return LIZARD_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return LIZARD_ERR_CUDA;
  if (word != 0 && cudaMemset(workspace, 0, sizeof(word)) != cudaSuccess) return LIZARD_ERR_CUDA;
  if (word & 1u) return LIZARD_ERR_TIMEOUT;
  if (word & 2u) return LIZARD_ERR_RANGE;
  return LIZARD_OK;
}

const char *lizard_status_string(lizard_status s) {
  switch (s) {
    case LIZARD_OK: return "ok";
    case LIZARD_ERR_INVALID_ARG: return "invalid argument";
    case LIZARD_ERR_UNSUPPORTED: return "unsupported size or option";
    case LIZARD_ERR_CUDA: return "CUDA launch or runtime error";
    case LIZARD_ERR_TIMEOUT: return "a kernel gave up on a bounded wait";
    case LIZARD_ERR_WORKSPACE: return "workspace missing or too small";
    case LIZARD_ERR_RANGE: return "gate decay outside the tensor-core forward's range (use the portable kernels)";
  }
  return "unknown status";
}

const char *lizard_version(void) { return "0.1.0"; }

void lizard_debug_inject_wait_timeout(int32_t count) { lz::g_inject_wait = count > 0 ? count : 0; }

}  // extern "C"

// ------------------------------------------------- sequence parallelism ---
namespace {

// The segment summary runs on the tensor-core state pass for bf16, d = 128
// with feature-map weights, else on the portable forward's kernels.
bool seg_uses_tc(const lizard_fwd_args *a) {
  const bool ok = a->dtype == LIZARD_BF16 && a->dk == 128 && a->dv == 128 && a->fmap_wk != nullptr;
  return (a->impl == LIZARD_IMPL_AUTO || a->impl == LIZARD_IMPL_TC) && ok;
}

struct SegLayout {
  size_t phq, phk, a, o_gla, tc, total;
};
SegLayout seg_layout(const lizard_fwd_args *a) {
  const size_t N = (size_t)a->B * a->H * a->L;
  SegLayout l{};
  size_t off = kHeader;
  if (seg_uses_tc(a)) {
    l.tc = off;
    off += up(lz::tc_segment_state_workspace_bytes(a->B * a->H, a->L));
  } else {
    const size_t nd = up(N * a->dk * sizeof(float));
    l.phq = off; off += nd;
    l.phk = off; off += nd;
    l.a = off; off += nd;
    l.o_gla = off; off += up(N * a->dv * sizeof(float));
  }
  l.total = off;
  return l;
}

// The forward's checks on the arguments the summary reads: q and o are not
// read (k and state_out stand in for them), nor are the meta tokens.
lizard_status check_seg(const lizard_fwd_args *a, const float *log_decay) {
  if (!a) return LIZARD_ERR_INVALID_ARG;
  lizard_fwd_args f = *a;
  f.q = a->k;
  f.o = a->state_out;
  f.lse = nullptr;
  f.M = 0;
  f.meta_k = f.meta_v = nullptr;
  const lizard_status st = check_fwd(&f);
  if (st != LIZARD_OK) return st;
  if (a->branch == LIZARD_BRANCH_SWA_ONLY || a->state_in || a->prefix_len != 0) return LIZARD_ERR_INVALID_ARG;
  if (!a->state_out || !log_decay || !aligned16(log_decay)) return LIZARD_ERR_INVALID_ARG;
  return LIZARD_OK;
}

}  // namespace

extern "C" {

size_t lizard_segment_state_workspace_size(const lizard_fwd_args *args) {
  if (!args) return 0;
  lizard_fwd_args a = *args;
  a.k = a.v = a.g = a.L > 0 ? reinterpret_cast<const void *>(16) : nullptr;
  a.state_out = reinterpret_cast<float *>(16);
  a.fmap_wq = a.fmap_wk = nullptr;
  a.state_in = nullptr;
  a.workspace = nullptr;
  a.k_prefix = a.v_prefix = nullptr;
  a.prefix_len = 0;
  if (check_seg(&a, reinterpret_cast<const float *>(16)) != LIZARD_OK) return 0;
  a.fmap_wk = args->fmap_wk ? reinterpret_cast<const float *>(16) : nullptr;   // selects the kernels
  return seg_layout(&a).total;
}

lizard_status lizard_segment_state(const lizard_fwd_args *a, float *log_decay, lizard_stream_t stream) {
  lizard_status st = check_seg(a, log_decay);
  if (st != LIZARD_OK) return st;
  if (a->impl == LIZARD_IMPL_TC && !seg_uses_tc(a)) return LIZARD_ERR_UNSUPPORTED;
  const SegLayout lay = seg_layout(a);
  if (!a->workspace || a->workspace_bytes < lay.total) return LIZARD_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int BH = a->B * a->H, D = a->dk;
  if (a->L == 0) {
    if (cudaMemsetAsync(a->state_out, 0, (size_t)BH * a->dk * a->dv * sizeof(float), s) != cudaSuccess ||
        cudaMemsetAsync(log_decay, 0, (size_t)BH * a->dk * sizeof(float), s) != cudaSuccess)
      return LIZARD_ERR_CUDA;
    return LIZARD_OK;
  }
  void *ws = a->workspace;
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) return LIZARD_ERR_CUDA;
  const float inv_tau = 1.f / a->gate_temp;
  if (seg_uses_tc(a)) {
    lz::TcFwdArgs t{a->k, a->k, a->v, a->g, nullptr, a->fmap_wk, nullptr, nullptr, nullptr, nullptr, nullptr,
                    a->state_out, nullptr, static_cast<uint32_t *>(ws), nullptr, BH, a->H, a->L, 0, a->window,
                    LIZARD_BRANCH_GLA_ONLY, inv_tau, scale_of(a), scalar_gate(a)};
    return cuda_status(lz::launch_tc_segment_state(t, a->state_out, log_decay, at<void>(ws, lay.tc), s));
  }
  const bool bf16 = a->dtype == LIZARD_BF16;
  // the portable forward's own kernels: the prep (phi of k stands in for the
  // unused phi of q), the GLA pass from a zero start (its output is scratch),
  // then the summed log-decay
  lz::PrepArgs pa{a->k, a->k, a->g, a->fmap_wk, a->fmap_wk, at<float>(ws, lay.phq), at<float>(ws, lay.phk),
                  at<float>(ws, lay.a), a->H, a->L, inv_tau, scalar_gate(a)};
  cudaError_t e = lz::launch_prep(pa, BH, D, bf16, s);
  if (e != cudaSuccess) return LIZARD_ERR_CUDA;
  lz::GlaFwdArgs ga{at<float>(ws, lay.phq), at<float>(ws, lay.phk), at<float>(ws, lay.a), a->v, nullptr,
                    at<float>(ws, lay.o_gla), a->state_out, a->L};
  e = lz::launch_gla_fwd_simt(ga, BH, D, bf16, s);
  if (e != cudaSuccess) return LIZARD_ERR_CUDA;
  return cuda_status(lz::launch_decay_sum(at<float>(ws, lay.a), log_decay, BH, a->L, D, s));
}

lizard_status lizard_chain_states(const lizard_chain_args *a, lizard_stream_t stream) {
  if (!a) return LIZARD_ERR_INVALID_ARG;
  if (a->B <= 0 || a->H <= 0 || a->nseg < 0 || a->rank < 0 || a->rank > a->nseg) return LIZARD_ERR_INVALID_ARG;
  if (a->dk != a->dv || (a->dk != 64 && a->dk != 128)) return LIZARD_ERR_UNSUPPORTED;
  if (!a->state_out || (a->rank > 0 && (!a->seg_state || !a->seg_log_decay))) return LIZARD_ERR_INVALID_ARG;
  const void *ptrs[] = {a->seg_state, a->seg_log_decay, a->state_in, a->state_out};
  for (const void *p : ptrs)
    if (!ok_ptr(p)) return LIZARD_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return cuda_status(lz::launch_chain_states(a->seg_state, a->seg_log_decay, a->state_in, a->state_out,
                                             a->B * a->H, a->dk, a->rank, s));
}

}  // extern "C"
