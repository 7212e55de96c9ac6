// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace lz {

// Exact fallback of the tensor-core backward (sequences whose in-tile decay
// spread leaves the tensor-core range): when seq_of_slot is set, the portable
// prep and GLA backward kernels run one grid slot k per entry, on sequence
// bh = seq_of_slot[k] (nothing when it is negative); their scratch arrays
// (phi, a, chunk states, kap, dphi) are indexed by the slot k, their inputs
// and outputs by bh.
struct PrepArgs {
  const void *q, *k, *g;
  const float *wq, *wk;
  float *phq, *phk, *a;
  int H, L;
  float inv_tau;
  int scalar_gate;   // g holds one logit per (token, head): [B*H][L]
  const int *seq_of_slot;
};

struct GlaFwdArgs {
  const float *phq, *phk, *a;
  const void *v;
  const float *state_in;
  float *o_gla;
  float *state_out;
  int L;
};

struct SwaMixArgs {
  const void *q, *k, *v;
  const float *meta_k, *meta_v, *alpha;
  const float *o_gla;
  void *o;
  float *lse;
  int H, L, window, M, branch;
  float scale;
  const void *k_prefix, *v_prefix;   // [B*H][P][D]: the P tokens before token 0 (P = 0: none)
  int P;
};

struct DecodeArgs {
  const void *q, *k, *v, *g;
  float *state;
  void *k_cache, *v_cache;
  const int64_t *pos;
  const float *wq, *wk, *meta_k, *meta_v, *alpha;
  void *o;
  int H, window, M;
  float inv_tau, scale;
  int scalar_gate;   // g holds one logit per (batch, head): [B*H]
  // Set by the launcher: when pos_inc is set, the last CTA to have read pos
  // adds 1 to pos[0 .. B) (arrival counter pos_slot of the library's ring),
  // so no second kernel is needed.
  int64_t *pos_inc;
  int pos_slot, pos_B;
};

// Backward (portable fp32 kernels).
struct GlaStatesArgs {
  const float *phk, *a;
  const void *v;
  const float *state_in;
  float *sprev;     // [BH][nchunk][D][D] state at the start of each chunk
  int L;
  // With an incoming final-state gradient G: kap[bh][i] = sum_v G[i][v] S_L[i][v],
  // the final state's share of every token's log-decay gradient (null: none)
  const float *dstate_out;
  float *kap;
  const int *seq_of_slot;
};

struct GlaBwdArgs {
  const float *phq, *phk, *a;
  const void *v, *dout;
  const float *sprev;
  float *dphq, *dphk, *da, *dv_gla;   // in slot mode dphq, dphk are slot arrays too
  float *dstate_in;  // may be null
  int L;
  const float *dstate_out;   // [BH][D][D] gradient into the final state, or null (zero)
  const float *kap;          // [BH][D] from gla_states_simt when dstate_out is set: the reverse sum's start
  const int *seq_of_slot;
};

struct SwaBwdQArgs {
  const void *q, *k, *v, *dout;
  const float *meta_k, *meta_v, *alpha;
  float *dq_swa, *lse, *Dterm;
  float *dmeta_k, *dmeta_v, *dalpha;   // accumulated atomically; may be null
  int H, L, window, M;
  float scale;
  const void *k_prefix, *v_prefix;     // [B*H][P][D]: the P tokens before token 0 (P = 0: none)
  int P;
};

struct SwaBwdKVArgs {
  const void *q, *k, *v, *dout;
  const float *alpha, *lse, *Dterm;
  float *dk_swa, *dv_swa;
  int H, L, window;
  float scale;
  // Key/value prefix (P = 0: none) and the gradients of its keys and values,
  // [B*H][P][D] in the activation dtype (the anchor branch's part only).
  const void *k_prefix, *v_prefix;
  void *dk_prefix, *dv_prefix;
  int P;
};

struct FinishBwdArgs {
  const void *q, *k, *g;
  const float *wq, *wk;
  const float *dphq, *dphk, *da, *dv_gla;   // null when the GLA branch is off
  const float *dq_swa, *dk_swa, *dv_swa;    // null when the anchor branch is off
  void *dq, *dk, *dv;
  float *dg, *dwq, *dwk;                    // dwq/dwk accumulated atomically; may be null
  int H, L;
  float inv_tau;
  int write_dg;                             // 0 when another kernel writes dg
  uint32_t *status;                         // workspace status word (tensor-core finish)
  // Tensor-core finish only: when set, write the GLA feature-map parts dx_q,
  // dx_k here (bf16 [B*H*L][128]) for the anchor kernels to add, and leave
  // dq, dk, dv to them.
  void *xq_part, *xk_part;
  int scalar_gate;   // g and dg hold one value per (token, head): [B*H][L]
  // Tensor-core finish: the tensor-core GLA backward's dphi_q, dphi_k come as
  // bf16 with each row's half centred (dphq16, dphk16, [B*H*L][128]; dphq,
  // dphk then null), except for the sequences of the exact fallback
  // (slot_of[bh] >= 0), whose fp32 dphi are in the fallback's slot arrays
  // fb_dphq, fb_dphk ([K][L][128]).
  const void *dphq16, *dphk16;
  const int *slot_of;
  const float *fb_dphq, *fb_dphk;
};

struct TcFwdArgs {
  const void *q, *k, *v, *g;
  const float *wq, *wk, *meta_k, *meta_v, *alpha, *state_in;
  void *o;
  float *state_out, *lse;
  uint32_t *status;   // workspace status word (bit 0 timeout, bit 1 range)
  void *seg_ws;       // tc_fwd_workspace_bytes() bytes: segment states, then the gate factors
  int BH, H, L, M, window, branch;
  float inv_tau, scale;
  int scalar_gate;    // g holds one logit per (token, head): [B*H][L]
  // Stage-1 loss in the full pass's epilogue (target null: off): with
  // n = B*H*L*128, dmse = 2 (o - target) / n (bf16) and *loss += sum (o - target)^2 / n.
  // o may be null when the loss is on.
  const void *target;
  void *dmse;
  float *loss;
  // Key/value prefix of the anchor window: [B*H][P][128] bf16, the P <= window
  // tokens before token 0 (P = 0: none).
  const void *k_prefix, *v_prefix;
  int P;
  // State pass that writes the backward's copies, with an incoming final-state
  // gradient G = dstate_out: kap [BH][2][128], the two column halves of
  // sum_v G[i][v] S_L[i][v] (null: none)
  const float *dstate_out;
  float *kap;
  // Wide decay: the gate prep marks sequences whose in-tile decay spread
  // leaves the tensor-core range in seqflag [BH] (zeroed by the caller;
  // null: it sets the status word's RANGE bit instead); the full pass then
  // runs their GLA branch as the exact recurrence.
  uint32_t *seqflag;
  // Training forward (all null: off): the gate prep writes the fp32 decay
  // factors and tile decays to keep_e32 [BH*L][128] and keep_r
  // [BH][ntiles][128] (instead of the workspace), and the full pass writes
  // the backward's state copies `snap` (tc_gla_bwd_snapshot_bytes() bytes)
  // and the fp32 final state state_keep [BH][128][128].
  float *keep_e32, *keep_r;
  void *snap;
  float *state_keep;
  float *lse_keep;    // [BH][L] copy of the anchor softmax normalisers (beside lse), or null
};

struct TcSwaBwdArgs {
  const void *q, *k, *v, *dout;
  const float *meta_k, *meta_v, *alpha;
  float *dq, *dk, *dv;          // anchor-branch parts, fp32 [B*H*L][128]
  float *lse, *Dterm;           // [B*H*L]
  float *dmeta_k, *dmeta_v, *dalpha;   // accumulated by the dq pass
  uint32_t *status;
  int B, H, BH, L, M, window;
  float scale;
  // Fused with the tensor-core GLA backward (when xq_part is set): add the
  // GLA parts and write the final gradients instead of the fp32 parts above.
  const void *xq_part, *xk_part;   // bf16 [B*H*L][128] feature-map parts dx_q, dx_k
  const float *dv_gla;             // fp32 [B*H*L][128] value part
  void *dq_out, *dk_out, *dv_out;  // bf16 dq, dk, dv
  // Key/value prefix of the anchor window ([B*H][P][128] bf16, P <= window;
  // P = 0: none) and the gradients of its keys and values (bf16, same shape).
  const void *k_prefix, *v_prefix;
  void *dk_prefix, *dv_prefix;
  int P;
  const float *lse_in;          // [B*H*L] the forward's softmax normalisers, or null (formed into lse)
};

struct TcGlaBwdArgs {
  const void *q, *k, *v, *g, *dout;
  const float *wq, *wk;
  void *snap_s, *snap_ds;       // bf16 [B*H][L/128][128][128]: S' and dS of every tile
  // dphi_q, dphi_k: bf16 [B*H*L][128], each row's two halves centred (the
  // feature map's softmax backward ignores a constant added to one half);
  // dB, dv: fp32 [B*H*L][128]
  void *dphq, *dphk;
  float *dB, *dv;
  float *dg, *dstate_in;
  uint32_t *status;
  int H, BH, L;
  float inv_tau;
  const float *e32;             // fp32 [B*H*L][128] decay factors of every tile (launch_gate_prep)
  const float *gate_r;          // fp32 [B*H][L/128][128] log-decay of every tile
  int scalar_gate;              // g and dg hold one value per (token, head): [B*H][L]
  const void *w16;              // bf16 [H][2][128][64] feature-map weights (launch_weights_bf16)
  const float *dstate_out;      // [BH][D][D] gradient into the final state, or null (zero)
  const float *kap;             // [BH][2][128] final-state share of the log-decay gradient, or null
  float *colsum;                // fp32 [B*H][L/128][128]: per-tile column sums of dB (tile kernel out, gate gradient in)
};

constexpr int kBwdC = 32;   // GLA chunk used by the portable backward

cudaError_t launch_prep(const PrepArgs &a, int BH, int D, bool bf16, cudaStream_t s);
cudaError_t launch_gla_fwd_simt(const GlaFwdArgs &a, int BH, int D, bool bf16, cudaStream_t s);
cudaError_t launch_swa_mix_simt(const SwaMixArgs &a, int BH, int D, bool bf16, cudaStream_t s);
extern int g_inject_wait;   // test hook (lizard_debug_inject_wait_timeout)
bool tc_fwd_supported(int dk, int dv, int window, int M, bool bf16);
// Sequence-parallel pieces.  Tensor-core segment summary: the state pass over
// whole sequences from a zero start, writing U [BH][D][D] and the summed
// log-decay R [BH][D]; its scratch (the gate factors) is
// tc_segment_state_workspace_bytes() bytes.
size_t tc_segment_state_workspace_bytes(int BH, int L);
cudaError_t launch_tc_segment_state(const TcFwdArgs &a, float *U, float *R, void *scratch, cudaStream_t s);
// R [BH][D] = sum over the L tokens of the log-decay a [BH][L][D] (portable).
cudaError_t launch_decay_sum(const float *a, float *R, int BH, int L, int D, cudaStream_t s);
// out = S_rank with S_0 = state_in (or 0), S_{j+1} = diag(exp R_j) S_j + U_j;
// U [nseg][BH][D][D], R [nseg][BH][D].
cudaError_t launch_chain_states(const float *U, const float *R, const float *state_in, float *out, int BH, int D,
                                int rank, cudaStream_t s);
size_t tc_fwd_workspace_bytes(int BH, int L);
int tc_fwd_stage_count(int BH, int L);
// stage 3: gate factors of every tile (first, when the GLA branch is on);
// stage 0: state pass, 1: combine (both only when the sequence is split), 2: full pass
cudaError_t launch_tc_fwd(const TcFwdArgs &a, int stage, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs &a, int B, int D, bool bf16, int64_t *pos, cudaStream_t s);
// Persistent streaming decode for bf16, d = 128, window <= 128, M <= 16.
bool decode_stream_supported(int D, bool bf16, int window, int M);
cudaError_t launch_decode_stream(const DecodeArgs &a, int B, int64_t *pos, cudaStream_t s);
// Prefill -> decode handoff of the window caches (rows are 16-byte multiples).
cudaError_t launch_prefill_cache(const void *k, const void *v, void *kc, void *vc, int64_t *pos, int B, int H,
                                 int L, int W, size_t row_bytes_k, size_t row_bytes_v, cudaStream_t s);
// The streaming kernel's timeout flag (bit 1), cleared by reading; -1 on error.
int decode_stream_status_take();

cudaError_t launch_gla_states(const GlaStatesArgs &a, int BH, int D, bool bf16, cudaStream_t s);
cudaError_t launch_gla_bwd_simt(const GlaBwdArgs &a, int BH, int D, bool bf16, cudaStream_t s);
cudaError_t launch_swa_bwd_q(const SwaBwdQArgs &a, int BH, int D, bool bf16, cudaStream_t s);
cudaError_t launch_swa_bwd_kv(const SwaBwdKVArgs &a, int BH, int D, bool bf16, cudaStream_t s);
bool tc_swa_bwd_supported(int dk, int dv, int window, int M, bool bf16);
// stage 0: dq pass (with the meta-token gradients), 1: dk/dv pass
cudaError_t launch_tc_swa_bwd(const TcSwaBwdArgs &a, int stage, cudaStream_t s);
size_t tc_gla_bwd_snapshot_bytes(int BH, int L);
// kap [BH][2][128] from a kept final state S [BH][128][128] and the incoming
// final-state gradient G (same layout): the two column halves of
// sum_v G[i][v] S[i][v].
cudaError_t launch_state_share(const float *S, const float *G, float *kap, int BH, cudaStream_t s);
// bf16 copies of W_q, W_k ([H][2][128][64]) for the per-tile backward's TMA loads
size_t tc_gla_bwd_weights_bytes(int H);
cudaError_t launch_weights_bf16(const float *wq, const float *wk, void *out, int H, cudaStream_t s);
cudaError_t launch_tc_state_snapshots(const TcFwdArgs &a, void *snap, const float *e32, const float *r,
                                      cudaStream_t s);
// Decay factors of every 128-token tile (bf16 E16 and/or fp32 E32, [BH][L][128],
// either may be null) and the tiles' log-decays r [BH][ntiles][128], from bf16
// gate logits g [BH][L][128] (scalar_gate: [BH][L], one logit for all 128
// dimensions); sets bit 2 of *status when a tile's spread is too wide.
// Stage-1 loss over n elements of o and target (dtype): dout = 2 (o - target) / n,
// *loss += sum (o - target)^2 / n (the caller zeroes *loss first).
cudaError_t launch_mse(const void *o, const void *target, void *dout, float *loss, size_t n, bool bf16,
                       cudaStream_t s);
cudaError_t launch_gate_prep(const void *g, void *E16, float *E32, float *r, uint32_t *status, int BH, int L,
                             float inv_tau, bool scalar_gate, cudaStream_t s, uint32_t *seqflag = nullptr);
// Exact fallback for sequences outside the tensor-core decay range
// (exact_fallback.cu): up to kFallbackSlots marked sequences per call get a
// slot (slot_of [BH], seq_of_slot [K]); the others set the RANGE bit.
constexpr int kFallbackSlots = 4;
cudaError_t launch_assign_slots(const uint32_t *flags, int *slot_of, int *seq_of_slot, int BH, int K,
                                uint32_t *status, cudaStream_t s);
cudaError_t launch_slot_dg(float *dg, const float *da, const void *g, const int *seq_of_slot, int K, int L, int D,
                           float inv_tau, bool scalar_gate, bool bf16, cudaStream_t s);
// stage 0: reverse dS pass, 1: per-tile gradients, 2: gate-logit gradient
cudaError_t launch_tc_gla_bwd(const TcGlaBwdArgs &a, int stage, cudaStream_t s);
// Loads the GLA tile kernel before the library's other kernels (see tc_gla_bwd.cu).
cudaError_t tc_gla_bwd_preload();
// tensor-core finish: bf16, d = 128, both feature maps present
cudaError_t launch_tc_finish(const FinishBwdArgs &a, int BH, cudaStream_t s);
cudaError_t launch_finish_bwd(const FinishBwdArgs &a, int BH, int D, bool bf16, cudaStream_t s);

}  // namespace lz
