"""Sequence-parallel forward: one long sequence split across processes.

Rank r of a process group holds the consecutive tokens s_r .. s_r + L_r - 1
of every (batch, head) sequence, ranks in token order.  The GLA recurrence
S_t = diag(exp a_t) S_{t-1} + phi_k(k_t) v_t^T (English gist.science
summary, section 2.A "State Update") is affine in its start state, so the
forward needs one exchange step:

1. every rank but the last summarises its segment, (U, R) =
   lizard_segment_state (U the end state from a zero start, R the summed
   log-decay), and sends its last `window` keys and values to the next rank
   (the anchor window's halo);
2. the summaries are all-gathered, and rank r chains those of the ranks
   before it into its start state (lizard_chain_states);
3. every rank runs lizard_attn_fwd over its own tokens with that state_in
   and the halo as its key/value prefix.

Exchanged per (batch, head): a dk x dv fp32 state, dk log-decays and a
window of keys and values, whatever the segment length.  The collectives
are torch.distributed's (NCCL over NVLink between GPUs; gloo on CPU for the
tests); every rank takes the same collective steps in the same order.

The three compute steps go through an `ops` object; the default is the CUDA
library.  Only the forward is split: lizard_attn_bwd takes no prefix.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


class LibraryOps:
    """The compute steps, run by liblizard's kernels on the tensors' device."""

    def __init__(self):
        from . import lizard
        self.lz = lizard

    def segment_state(self, k, v, g, *, window, chunk, gate_temp, fmap_wk, impl):
        U, R, _ = self.lz.segment_state(k, v, g, window=window, chunk=chunk, gate_temp=gate_temp,
                                        fmap_wk=fmap_wk, impl=impl)
        return U, R

    def chain_states(self, seg_state, seg_log_decay, rank, state_in):
        return self.lz.chain_states(seg_state, seg_log_decay, rank, state_in=state_in)

    def forward(self, q, k, v, g, *, state_in, k_prefix, v_prefix, want_state, **kw):
        out = self.lz.attn_fwd(q, k, v, g, state_in=state_in, k_prefix=k_prefix, v_prefix=v_prefix,
                               want_state=want_state, **kw)
        return {"o": out["o"], "state_out": out["state_out"]}


def _peer(group, r):
    """Global rank of the group's rank r (P2P calls take global ranks)."""
    return r if group is None else dist.get_global_rank(group, r)


def segment_lengths(group=None, *, length, device):
    """Every rank's token count, in rank order (one small all-gather)."""
    world = dist.get_world_size(group)
    mine = torch.tensor([length], dtype=torch.int64, device=device)
    parts = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(parts, mine, group=group)
    return [int(p.item()) for p in parts]


def sequence_parallel_forward(q, k, v, g, *, window, group=None, chunk=64, gate_temp=16.0,
                              softmax_scale=0.0, fmap_wq=None, fmap_wk=None, meta_k=None,
                              meta_v=None, alpha=None, state_in=None, impl=0, ops=None):
    """Forward of this rank's segment of the sequence.

    q, k, v, g: this rank's tokens, [B, H, L_r, d] (g [B, H, L_r] for the
    scalar gate); every rank but the last holds at least `window` tokens.
    state_in: the state before the whole sequence's first token (the same
    tensor, or None, on every rank).  Parameters as for lizard_attn_fwd.
    Returns {"o": this segment's output, "state_out": the state after the
    whole sequence on the last rank, None elsewhere}.
    """
    ops = LibraryOps() if ops is None else ops
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    lengths = segment_lengths(group, length=L, device=q.device)
    short = [r for r, n in enumerate(lengths[:-1]) if n < window]
    if short:
        # every rank sees the same lengths, so every rank raises here
        raise ValueError(f"ranks {short} hold fewer than window={window} tokens")

    # 1. halo: the last `window` keys and values go to the next rank
    k_prefix = v_prefix = None
    p2p = []
    if rank + 1 < world:
        k_send = k[:, :, L - window:].contiguous()
        v_send = v[:, :, L - window:].contiguous()
        nxt = _peer(group, rank + 1)
        p2p += [dist.P2POp(dist.isend, k_send, nxt, group), dist.P2POp(dist.isend, v_send, nxt, group)]
    if rank > 0:
        k_prefix = torch.empty(B, H, window, dk, dtype=k.dtype, device=k.device)
        v_prefix = torch.empty(B, H, window, dv, dtype=v.dtype, device=v.device)
        prv = _peer(group, rank - 1)
        p2p += [dist.P2POp(dist.irecv, k_prefix, prv, group), dist.P2POp(dist.irecv, v_prefix, prv, group)]
    reqs = dist.batch_isend_irecv(p2p) if p2p else []

    # 2. segment summaries (the last rank's is never read: zeros), all-gathered
    if rank + 1 < world:
        U, R = ops.segment_state(k, v, g, window=window, chunk=chunk, gate_temp=gate_temp,
                                 fmap_wk=fmap_wk, impl=impl)
    else:
        U = torch.zeros(B, H, dk, dv, dtype=torch.float32, device=q.device)
        R = torch.zeros(B, H, dk, dtype=torch.float32, device=q.device)
    U_all = [torch.empty_like(U) for _ in range(world)]
    R_all = [torch.empty_like(R) for _ in range(world)]
    dist.all_gather(U_all, U.contiguous(), group=group)
    dist.all_gather(R_all, R.contiguous(), group=group)
    S0 = ops.chain_states(torch.stack(U_all), torch.stack(R_all), rank, state_in)
    for r in reqs:
        r.wait()

    # 3. this segment's forward
    out = ops.forward(q, k, v, g, state_in=S0, k_prefix=k_prefix, v_prefix=v_prefix,
                      want_state=rank + 1 == world, window=window, chunk=chunk, gate_temp=gate_temp,
                      softmax_scale=softmax_scale, fmap_wq=fmap_wq, fmap_wk=fmap_wk, meta_k=meta_k,
                      meta_v=meta_v, alpha=alpha, impl=impl)
    return {"o": out["o"], "state_out": out["state_out"] if rank + 1 == world else None}
