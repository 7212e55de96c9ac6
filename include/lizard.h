/*
 * lizard.h -- C ABI of liblizard.so: Lizard hybrid attention on NVIDIA B200.
 *
 * The layer (arXiv 2507.09025, "Lizard: An Efficient Linearization Framework
 * for Large Language Models"; the gist.science technical summaries in
 * English, French, Spanish and Chinese describe it) mixes two branches:
 *
 *   GLA branch (English summary, section 2.A "State Update"):
 *     a_t   = logsigmoid(g_t) / gate_temp                   (per key dim, or
 *             one value for every key dim with LIZARD_GATE_SCALAR)
 *     S_t   = diag(exp a_t) S_{t-1} + phi_k(k_t) v_t^T      (fp32 state)
 *     o^gla = S_t^T phi_q(q_t)
 *   with phi(x) = [softmax(x W), softmax(-x W)], W in R^{dk x dk/2} per head
 *   (the non-negative Hedgehog map of the Chinese summary, section 2.3), or
 *   the identity when W is NULL.
 *
 *   Anchor branch (English summary, section 2.A "Anchor Window Attention"):
 *     softmax over the keys j in [t - window + 1, t] and the M meta tokens,
 *     logits softmax_scale * q_t . key; o^swa = sum p * value, where a meta
 *     token's value is meta_v[m] (or nothing when meta_v is NULL: a pure
 *     sink in the softmax denominator).
 *
 *   Mix (French summary, section 2.A last line):  o = o^gla + alpha_h o^swa.
 *
 * Conventions shared by every entry point
 *   - All pointers are DEVICE pointers unless stated otherwise; the caller
 *     owns all memory, including the workspace.  The library allocates and
 *     frees no device memory and keeps no results between calls.  To run
 *     independent backward kernels side by side, it creates on its first
 *     backward call in each host thread and on each device one non-blocking
 *     CUDA stream and two events (kept until the process exits); the work is
 *     forked from and joined back into the call's stream with events, so a
 *     stream capture of the call records it.  A first call made inside a
 *     stream capture, or any call given per-kernel timing events, runs every
 *     kernel in order on the call's stream instead.
 *   - Activations (q, k, v, g, o, caches, their gradients) use `dtype`
 *     (bf16 or fp32), contiguous row-major with the innermost dimension last
 *     (the shapes below).  Parameters (feature-map weights, meta tokens,
 *     alpha) and the recurrent state are fp32.  Gradients of parameters, of
 *     the gate logits and of the state are fp32.
 *   - Work is enqueued on `stream` and runs asynchronously.  Arguments are
 *     checked on the host before anything is launched: a call that returns
 *     an error status launched nothing.
 *   - Every pointer must be 16-byte aligned.
 *   - Supported: dk = dv in {64, 128}; chunk = 64; window >= 1; 0 <= M <= 16;
 *     L >= 0 (L = 0 is a no-op); B * H >= 1.  Other sizes return
 *     LIZARD_ERR_UNSUPPORTED.
 *   - Launch errors return LIZARD_ERR_CUDA.  Errors found on the device are
 *     recorded in a status word at the start of the workspace, cleared at the
 *     start of every forward or backward call and read back by
 *     lizard_workspace_status(): a kernel that gives up on a bounded wait
 *     records LIZARD_ERR_TIMEOUT.
 *   - Wide decay on the tensor-core path: when, inside one 128-token tile, the
 *     cumulative log-decay of some key dimension spans more than 64 (gate
 *     logits below about -8 per token at gate_temp 16), the tensor-core
 *     kernels' log-space factors leave their exponent range.  Such sequences
 *     get their GLA branch computed exactly instead: in lizard_attn_fwd, any
 *     number of them; in lizard_attn_bwd, up to 4 of them per call (a fifth
 *     and later one keeps the tensor-core result, and the call records
 *     LIZARD_ERR_RANGE).  lizard_stage1_step has no such fallback: it records
 *     LIZARD_ERR_RANGE for any of them.
 */
#ifndef LIZARD_H_
#define LIZARD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *lizard_stream_t; /* == cudaStream_t; NULL = legacy default stream */

typedef enum {
  LIZARD_OK = 0,
  LIZARD_ERR_INVALID_ARG = 1, /* NULL required pointer, negative size, misaligned pointer */
  LIZARD_ERR_UNSUPPORTED = 2, /* well-formed but outside the supported sizes */
  LIZARD_ERR_CUDA = 3,        /* a launch or CUDA runtime call failed */
  LIZARD_ERR_TIMEOUT = 4,     /* a kernel gave up on a bounded wait */
  LIZARD_ERR_WORKSPACE = 5,   /* workspace NULL or smaller than the queried size */
  LIZARD_ERR_RANGE = 6        /* tensor-core backward: more wide-decay sequences than its exact fallback takes */
} lizard_status;

typedef enum { LIZARD_BF16 = 0, LIZARD_FP32 = 1 } lizard_dtype;

/* Which terms of o = o^gla + alpha_h o^swa to compute (test hook). */
enum { LIZARD_BRANCH_BOTH = 0, LIZARD_BRANCH_GLA_ONLY = 1, LIZARD_BRANCH_SWA_ONLY = 2 };

/* Gate granularity (lizard_fwd_args.gate, lizard_decode_args.gate).
 * PER_DIM: one gate logit per key dimension, g [..., dk].  SCALAR: one logit
 * per token and head, g [...] without the dk axis, whose decay every key
 * dimension shares (the light scalar gate that the Chinese summary's
 * ablation, section 4, finds most effective); its gradient dg has the same
 * shape as g. */
enum { LIZARD_GATE_PER_DIM = 0, LIZARD_GATE_SCALAR = 1 };

/* Kernel family selection (lizard_fwd_args.impl / lizard_bwd_args.impl). */
enum {
  LIZARD_IMPL_AUTO = 0,  /* tensor-core path where it applies, else portable */
  LIZARD_IMPL_SIMT = 1,  /* portable fp32 CUDA-core kernels (exact fp32 math) */
  LIZARD_IMPL_TC = 2     /* tcgen05/TMEM tensor-core kernels: bf16, dk = dv =
                            128, window <= 128, M <= 16 (the GLA part of the
                            backward needs only bf16 and d = 128) */
};

/*
 * Forward of the hybrid layer over whole sequences.
 *
 * Shapes (B batch, H heads, L tokens, dk = dv = d):
 *   q, k       [B, H, L, dk] dtype
 *   g          [B, H, L, dk] dtype gate logits, or [B, H, L] with
 *              gate = LIZARD_GATE_SCALAR (the gate projection W_gamma x
 *              itself is the caller's)
 *   v          [B, H, L, dv] dtype
 *   fmap_wq/wk [H, dk, dk/2] fp32, or NULL for the identity map
 *   meta_k     [H, M, dk] fp32 (NULL iff M == 0)
 *   meta_v     [H, M, dv] fp32, or NULL for sink-only meta tokens
 *   alpha      [H] fp32 mixing weights (NULL = all ones)
 *   state_in   [B, H, dk, dv] fp32 initial state S_{-1}, or NULL for zeros
 *   o          [B, H, L, dv] dtype, written
 *   state_out  [B, H, dk, dv] fp32 final state S_{L-1}, or NULL (written
 *              only when the GLA branch runs)
 *   lse        [B, H, L] fp32 natural-log softmax normaliser of the anchor
 *              branch (window + meta logits), or NULL (written only when the
 *              anchor branch runs)
 * gate_temp is tau (> 0); softmax_scale 0 means 1/sqrt(dk).
 * chunk is the GLA chunk length (64); it changes the schedule, not the result.
 *
 * Key/value prefix (a segment of a longer sequence, e.g. one rank's share
 * under sequence parallelism): with prefix_len = P > 0, the P tokens just
 * before token 0 are visible to the anchor window of the first tokens, as if
 * the call's sequence continued them (the GLA branch takes that history
 * through state_in instead).
 *   k_prefix   [B, H, P, dk] dtype, v_prefix [B, H, P, dv] dtype: row P - 1
 *              is token -1, row 0 token -P
 *   0 <= P <= window; the pointers are NULL iff P == 0.  lizard_attn_bwd
 *   returns the prefix's key and value gradients (lizard_bwd_args.dk_prefix,
 *   dv_prefix); lizard_stage1_step, which trains whole sequences, returns
 *   LIZARD_ERR_UNSUPPORTED for a nonzero prefix_len.
 */
typedef struct {
  int32_t B, H, L, dk, dv, chunk, window, M;
  int32_t dtype;   /* lizard_dtype */
  int32_t branch;  /* LIZARD_BRANCH_* */
  int32_t impl;    /* LIZARD_IMPL_* */
  int32_t gate;    /* LIZARD_GATE_* */
  float gate_temp;
  float softmax_scale;
  const void *q, *k, *v, *g;
  const float *fmap_wq, *fmap_wk;
  const float *meta_k, *meta_v;
  const float *alpha;
  const float *state_in;
  void *o;
  float *state_out;
  float *lse;
  void *workspace;        /* device scratch, >= lizard_fwd_workspace_size() bytes */
  size_t workspace_bytes;
  /* Optional kernel timing: cudaEvent_t handles created by the caller.  When
   * non-NULL, the call records launch_events[0] before its first kernel and
   * launch_events[i] after its i-th kernel, for i < n_launch_events, all on
   * `stream`.  lizard_fwd_launch_plan() names the kernels in order. */
  void *const *launch_events;
  int32_t n_launch_events;
  const void *k_prefix, *v_prefix;   /* see "Key/value prefix" above */
  int32_t prefix_len;
  /* Training forward: device buffer of >= lizard_fwd_saved_size() bytes (16-byte
   * aligned) into which the forward writes what lizard_attn_bwd would
   * otherwise recompute, or NULL.  See "Saved for the backward" below. */
  void *saved;
  size_t saved_bytes;
} lizard_fwd_args;

/* Bytes of device workspace the forward needs for these arguments.  Pointer
 * fields are ignored, except whether fmap_wq / fmap_wk are given (that
 * selects the kernels).  Returns 0 when the sizes are invalid. */
size_t lizard_fwd_workspace_size(const lizard_fwd_args *args);

/* Enqueue the forward.  See the conventions above for errors. */
lizard_status lizard_attn_fwd(const lizard_fwd_args *args, lizard_stream_t stream);

/*
 * Saved for the backward (training).  The backward of the GLA branch needs,
 * per 128-token tile, the state at the tile's start decayed by the tile's
 * gates (S' = diag(exp r) S, the state-update recurrence of the English
 * gist.science summary, section 2.A) and the tile's decay factors in fp32
 * (the log-space gate absorption of the Chinese summary, section 2.3), and
 * its anchor softmax needs each row's normaliser (section 2.A, anchor window
 * attention).  The forward has all three at hand; without a saved buffer the
 * backward recomputes them (a gate pass, a state pass over the sequence and
 * a max pass over the window logits).
 *
 * With args->saved set, lizard_attn_fwd also writes, into that buffer: the
 * wide-decay marks, the tiles' log-decays and fp32 decay factors, a bf16
 * copy of every tile's S' (rows less row 0, which is kept in fp32), the
 * fp32 final state and, with the anchor branch, the normalisers (lse).  A backward whose fwd.saved points at that buffer (same
 * inputs, enqueued after the forward) reads them instead of recomputing; its
 * results agree with the recomputing backward's to bf16 rounding of S'.
 * lizard_bwd_workspace_size() is smaller when fwd.saved is set.
 *
 * Returns the bytes the buffer needs for these arguments (pointer fields
 * are ignored, except whether fmap_wq / fmap_wk are given), or 0 when the
 * forward keeps nothing for these arguments (GLA branch off, not on the
 * tensor-core path, no feature-map weights); saved is then ignored by the
 * forward and the backward.  A saved buffer smaller than this size is
 * LIZARD_ERR_WORKSPACE in both calls.
 */
size_t lizard_fwd_saved_size(const lizard_fwd_args *args);

/*
 * Backward of the hybrid layer: gradients of sum(dout * o) with respect to
 * every input of lizard_attn_fwd.
 *
 *   fwd      the forward's inputs (fwd.o, fwd.state_out, fwd.lse and the
 *            forward workspace are ignored); fwd.saved, when not NULL, is a
 *            buffer lizard_attn_fwd filled for these inputs (see "Saved for
 *            the backward"), which the call reads but does not change
 *   dout     [B, H, L, dv] dtype
 *   dq, dk   [B, H, L, dk] dtype, written
 *   dv       [B, H, L, dv] dtype, written
 *   dg       [B, H, L, dk] fp32 gradient of the gate logits ([B, H, L] with
 *            LIZARD_GATE_SCALAR), written
 *   dmeta_k, dmeta_v, dfmap_wq, dfmap_wk, dalpha, dstate_in   fp32, same
 *            shapes as the inputs, written (overwritten, not accumulated);
 *            each may be NULL when not wanted (and must be NULL when the
 *            matching input is NULL).
 *   dstate_out [B, H, dk, dv] fp32 gradient flowing into the final state
 *            S_{L-1} from outside the call (a later chunk's dstate_in, when a
 *            long sequence is trained chunk by chunk through state_in /
 *            state_out), or NULL for an unused final state.  The gradients
 *            are then those of sum(dout * o) + sum(dstate_out * S_{L-1}).
 *            Needs the GLA branch.
 *   dk_prefix, dv_prefix [B, H, P, dk|dv] dtype, written: with a key/value
 *            prefix (fwd.prefix_len = P > 0), the gradients with respect to
 *            fwd.k_prefix and fwd.v_prefix -- the anchor window's reach into
 *            the previous segment, to be added to that segment's last P key
 *            and value gradients (the GLA history's gradient is dstate_in).
 *            Required when P > 0, NULL when P == 0.
 */
typedef struct {
  lizard_fwd_args fwd;
  const void *dout;
  void *dq, *dk, *dv;
  float *dg;
  float *dmeta_k, *dmeta_v;
  float *dfmap_wq, *dfmap_wk;
  float *dalpha;
  float *dstate_in;
  int32_t impl;           /* LIZARD_IMPL_* */
  void *workspace;        /* >= lizard_bwd_workspace_size() bytes */
  size_t workspace_bytes;
  void *const *launch_events;   /* as in lizard_fwd_args */
  int32_t n_launch_events;
  const float *dstate_out;      /* see above; NULL = zero */
  void *dk_prefix, *dv_prefix;  /* see above */
} lizard_bwd_args;

size_t lizard_bwd_workspace_size(const lizard_bwd_args *args);
lizard_status lizard_attn_bwd(const lizard_bwd_args *args, lizard_stream_t stream);

/*
 * Sequence parallelism: one long sequence split into consecutive segments,
 * one per process (GPU).  The GLA recurrence is affine in its start state:
 * over a segment with summed log-decay R (per key dimension) and end state U
 * from a zero start, a start state S ends as diag(exp R) S + U (English
 * summary, section 2.A "State Update", applied over a run of tokens).  So
 * every segment computes (U, R) at once, the segments exchange them, and
 * each chains the (U, R) of the segments before it into its own start state;
 * then every segment runs lizard_attn_fwd with that state_in and the last
 * `window` keys and values of the previous segment as its prefix.
 *
 * lizard_segment_state: (U, R) of the segment in args.
 *   args       as for lizard_attn_fwd over the segment's L tokens; read are
 *              the sizes, dtype, impl, gate, gate_temp, k, v, g, fmap_wk and
 *              the workspace (q, o, meta tokens, alpha and lse are ignored;
 *              state_in and the prefix must be NULL / 0; branch must not be
 *              LIZARD_BRANCH_SWA_ONLY)
 *   args->state_out  [B, H, dk, dv] fp32, written: U
 *   log_decay  [B, H, dk] fp32, written: R = sum over the segment's tokens of
 *              logsigmoid(g) / gate_temp
 * Workspace: lizard_segment_state_workspace_size() bytes.  Errors as
 * lizard_attn_fwd (the status word in the workspace included).
 *
 * lizard_chain_states: the start state of segment `rank` from the gathered
 * (U, R) of every segment.
 *   seg_state  [nseg, B, H, dk, dv] fp32, seg_log_decay [nseg, B, H, dk] fp32
 *              (segment j's U and R at index j; only j < rank are read)
 *   state_in   [B, H, dk, dv] fp32 state before segment 0, or NULL for zeros
 *   state_out  [B, H, dk, dv] fp32, written:
 *              S_0 = state_in, S_{j+1} = diag(exp R_j) S_j + U_j, out = S_rank
 *   0 <= rank <= nseg.  No workspace.
 */
size_t lizard_segment_state_workspace_size(const lizard_fwd_args *args);
lizard_status lizard_segment_state(const lizard_fwd_args *args, float *log_decay, lizard_stream_t stream);

typedef struct {
  int32_t B, H, dk, dv, nseg, rank;
  const float *seg_state, *seg_log_decay;
  const float *state_in;
  float *state_out;
} lizard_chain_args;

lizard_status lizard_chain_states(const lizard_chain_args *args, lizard_stream_t stream);

/*
 * One stage-1 training step (attention approximation: the layer learns to
 * reproduce a teacher's softmax-attention output under a mean squared error;
 * English summary, section 2.B "Stage 1"; Chinese summary, section 2.2):
 * the forward, the loss, and the gradients of the loss with respect to every
 * input, in one call.
 *
 *   bwd      inputs and gradient outputs exactly as in lizard_attn_bwd, with
 *            two differences: bwd.dout is ignored (dL/do comes from the loss),
 *            and bwd.fwd.o may be NULL (the output is then not kept) or
 *            receives o.  bwd.fwd.impl selects the forward's kernels,
 *            bwd.impl the backward's.  bwd.workspace and bwd.launch_events
 *            serve the whole step; bwd.fwd.saved is ignored: when both
 *            halves run the GLA branch on the tensor cores, the step keeps
 *            the forward's saved-for-backward tensors (see "Saved for the
 *            backward") in its own workspace, and its backward reads them.
 *   target   [B, H, L, dv] dtype: the teacher's attention output y
 *   loss     one fp32, written: sum over every element of (o - y)^2 divided
 *            by the element count B H L dv; dL/do = 2 (o - y) / (B H L dv)
 *            (o before its rounding to dtype)
 * The tensor-core forward forms the loss and dL/do in its epilogue; the
 * portable path adds one elementwise kernel.  The workspace (at least
 * lizard_stage1_workspace_size() bytes) holds dL/do between the two halves.
 * Errors as lizard_attn_bwd.
 */
typedef struct {
  lizard_bwd_args bwd;
  const void *target;
  float *loss;
} lizard_stage1_args;

size_t lizard_stage1_workspace_size(const lizard_stage1_args *args);
lizard_status lizard_stage1_step(const lizard_stage1_args *args, lizard_stream_t stream);

/* Kernels lizard_attn_fwd / lizard_attn_bwd / lizard_stage1_step launch for these arguments, in
 * launch order: fills names[0 .. min(count, cap)) with static strings and
 * returns count (-1 when the arguments are invalid).  Host only. */
int32_t lizard_fwd_launch_plan(const lizard_fwd_args *args, const char **names, int32_t cap);
int32_t lizard_bwd_launch_plan(const lizard_bwd_args *args, const char **names, int32_t cap);
int32_t lizard_stage1_launch_plan(const lizard_stage1_args *args, const char **names, int32_t cap);

/*
 * One decode step for every sequence: the constant-memory generation of the
 * English summary (section 2.A "State Update") with the fixed-size window
 * cache of the Chinese summary (section 2.1).
 *
 *   q, k       [B, H, dk] dtype;  v [B, H, dv] dtype: the new token
 *   g          [B, H, dk] dtype, or [B, H] with gate = LIZARD_GATE_SCALAR
 *   state      [B, H, dk, dv] fp32, updated in place:
 *              S <- diag(exp a) S + phi_k(k) v^T
 *   k_cache    [B, H, window, dk] dtype, v_cache [B, H, window, dv] dtype:
 *              ring buffers; the new (k, v) is written to slot pos[b] mod
 *              window, in place
 *   pos        [B] int64 tokens already seen per sequence; incremented in
 *              place after the step
 *   o          [B, H, dv] dtype, written: o = S^T phi_q(q) + alpha_h o^swa,
 *              the softmax covering the min(pos+1, window) filled slots and
 *              the M meta tokens
 * Parameters as in lizard_fwd_args.  Needs no workspace.  One kernel is
 * enqueued: every head of a sequence reads pos before any CTA increments it
 * (the last CTA to have read its pos values adds 1 to every pos[b]; only
 * with more than 64 x SM-count (batch, head) pairs in a bf16, d = 128 step
 * does a second, increment kernel follow).  Steps on the same pos array
 * must be ordered (one stream).
 */
typedef struct {
  int32_t B, H, dk, dv, window, M;
  int32_t dtype;
  int32_t gate;    /* LIZARD_GATE_* */
  float gate_temp;
  float softmax_scale;
  const void *q, *k, *v, *g;
  float *state;
  void *k_cache, *v_cache;
  int64_t *pos;
  const float *fmap_wq, *fmap_wk;
  const float *meta_k, *meta_v;
  const float *alpha;
  void *o;
} lizard_decode_args;

lizard_status lizard_decode_step(const lizard_decode_args *args, lizard_stream_t stream);

/*
 * Prefill -> decode handoff: after lizard_attn_fwd over a prefix of L tokens
 * (its state_out is the decode state), fill the decode window caches from
 * the prefix so that lizard_decode_step continues the sequence (the
 * constant-memory generation of the English summary, section 2.A, with the
 * fixed-size cache of the Chinese summary, section 2.1).
 *
 *   k, v       [B, H, L, dk|dv] dtype: the prefix's keys and values
 *   k_cache    [B, H, window, dk] dtype, v_cache [B, H, window, dv] dtype,
 *              written: token t of the last min(L, window) goes to slot
 *              t mod window (the slot lizard_decode_step would have used);
 *              slots no token reached are zeroed
 *   pos        [B] int64, written: L
 * L = 0 clears the caches.  No workspace.  Errors as lizard_decode_step.
 */
typedef struct {
  int32_t B, H, L, dk, dv, window;
  int32_t dtype;
  const void *k, *v;
  void *k_cache, *v_cache;
  int64_t *pos;
} lizard_cache_args;

lizard_status lizard_prefill_cache(const lizard_cache_args *args, lizard_stream_t stream);

/*
 * Status of the decode steps run on the current device since the last call:
 * LIZARD_ERR_TIMEOUT when a step's bounded wait for its own copies gave up
 * (its outputs are then undefined), else LIZARD_OK; LIZARD_ERR_CUDA when
 * the flag cannot be read.  Reading clears the flag.  Synchronises the
 * device.  (Decode has no workspace, so the flag lives in the library.)
 */
lizard_status lizard_decode_status(void);

/*
 * Test hook for failure detection: the next `count` launches of the
 * tensor-core forward's full pass (lizard_attn_fwd on the tensor-core path)
 * first wait on a barrier that nothing completes.  The wait gives up after
 * its iteration limit, the kernel records LIZARD_ERR_TIMEOUT in the
 * workspace status word, frees its TMEM and returns without computing, as a
 * real timed-out wait would.  count <= 0 clears it.  Host only; meant for
 * one test thread.
 */
void lizard_debug_inject_wait_timeout(int32_t count);

/*
 * Forward for callers that cannot allocate device memory.
 *
 * Some callers have no way to obtain a device workspace: a plug-in living
 * inside a host application that owns every device allocation and hands out
 * only the tensors it already has, or a C client with a fixed device-memory
 * budget that may not grow after start-up.  This entry point computes
 * exactly what lizard_attn_fwd computes, but ignores args->workspace and
 * args->workspace_bytes and uses a scratch array built into the library
 * instead.  The paper has no counterpart to it: it only changes where the
 * scratch lives.
 *
 *   - The scratch is a static device array of LIZARD_NOALLOC_SCRATCH_BYTES
 *     bytes (32 MiB).  Every GPU that loads it keeps it until the process
 *     exits.
 *   - Calls whose forward needs more scratch than that (see
 *     lizard_fwd_workspace_size) return LIZARD_ERR_UNSUPPORTED and launch
 *     nothing.  With dk = dv = 128 that is above roughly 16K token-heads
 *     (B * H * L) for the portable kernels.
 *   - Every call looks up the array's device address on the current device
 *     (the first lookup on a device loads the library's device code there).
 *     Make the first call on each device before any stream capture.
 *   - No cudaMalloc, cudaFree or other allocating routine is called.
 *   - All calls share the one array and it keeps the last call's contents.
 *     Calls that overlap on the GPU (different streams, or different host
 *     threads, without ordering between them) race on it.  Serialise them.
 *   - Inputs and outputs are still the caller's, as in lizard_attn_fwd.
 */
#define LIZARD_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
lizard_status lizard_attn_fwd_noalloc(const lizard_fwd_args *args, lizard_stream_t stream);

/* The device status of the last lizard_attn_fwd_noalloc call on the current
 * device: waits for `stream`, then reads and clears the status word at the
 * start of the built-in scratch, exactly as lizard_workspace_status does for
 * a caller's workspace (LIZARD_OK, LIZARD_ERR_TIMEOUT or LIZARD_ERR_RANGE;
 * LIZARD_ERR_CUDA if the copy fails).  Allocates nothing.  The word belongs
 * to the shared scratch: read it before the next noalloc call. */
lizard_status lizard_noalloc_status(lizard_stream_t stream);

/* Waits for `stream`, then reads and clears the status word that the last
 * forward or backward call left at the start of `workspace` (a device
 * pointer).  Returns LIZARD_OK, LIZARD_ERR_TIMEOUT or LIZARD_ERR_RANGE
 * (LIZARD_ERR_CUDA if the copy fails). */
lizard_status lizard_workspace_status(void *workspace, lizard_stream_t stream);

/* Static description of a status code; never NULL. */
const char *lizard_status_string(lizard_status s);

/* Library version, "major.minor.patch". */
const char *lizard_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LIZARD_H_ */
