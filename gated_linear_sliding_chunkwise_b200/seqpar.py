"""Sequence parallelism: one long sequence split across processes.

Rank r of a process group holds the consecutive tokens s_r .. s_r + L_r - 1
of every (batch, head) sequence, ranks in token order.  The GLA recurrence
S_t = diag(exp a_t) S_{t-1} + phi_k(k_t) v_t^T (English gist.science
summary, section 2.A "State Update") is affine in its start state, and so is
its gradient, so both directions need one exchange step each.

Forward (sequence_parallel_forward):

1. every rank summarises its segment, (U, R) = lizard_segment_state (U the
   end state from a zero start, R the summed log-decay), and sends its last
   `window` keys and values to the next rank (the anchor window's halo);
2. the summaries are all-gathered, and rank r chains those of the ranks
   before it into its start state (lizard_chain_states);
3. every rank runs lizard_attn_fwd over its own tokens with that state_in
   and the halo as its key/value prefix.

Backward (sequence_parallel_backward), after the same steps 1 and 2:

4. every rank runs lizard_attn_bwd over its own tokens with its start state
   and halo (the last rank with the caller's final-state gradient): dq, dk,
   dv, dg, the parameters' partial gradients, the prefix gradients and
   D_r = the gradient into its start state;
5. the D_r are all-gathered.  The gradient arriving at rank r's end state is
   X_r = D_{r+1} + diag(exp R_{r+1}) X_{r+1} (zero on the last rank): the
   same affine chain as the forward's, run from the last rank down, so
   lizard_chain_states computes it from the reversed lists;
6. the gradients are linear in the final-state gradient, so each rank but
   the last adds a GLA-only backward with dout = 0 and dstate_out = X_r;
7. rank r + 1 sends its prefix gradients back to rank r, which adds them to
   its last `window` key and value gradients; the parameters' gradients are
   summed over the ranks (all-reduce).

Exchanged per (batch, head): two dk x dv fp32 states, dk log-decays and a
window of keys and values (forward and back), whatever the segment length.
The collectives are torch.distributed's (NCCL over NVLink between GPUs;
gloo on CPU for the tests); every rank takes the same collective steps in
the same order, error paths included: a device error that any rank's
kernels report (the workspace status word) is all-reduced and raised on
every rank at the same step.

The compute steps go through an `ops` object; the default is the CUDA
library.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


class LibraryOps:
    """The compute steps, run by liblizard's kernels on the tensors' device.
    status() reads (and clears) the device status of every call made since
    the last status() (it waits for them)."""

    def __init__(self):
        from . import lizard
        self.lz = lizard
        self._ws = []

    def status(self):
        code = 0
        for ws in self._ws:
            c = self.lz.workspace_status(ws)
            code = code or c
        self._ws = []
        return code

    def segment_state(self, k, v, g, *, window, chunk, gate_temp, fmap_wk, impl):
        U, R, ws = self.lz.segment_state(k, v, g, window=window, chunk=chunk, gate_temp=gate_temp,
                                         fmap_wk=fmap_wk, impl=impl)
        self._ws.append(ws)
        return U, R

    def chain_states(self, seg_state, seg_log_decay, rank, state_in):
        return self.lz.chain_states(seg_state, seg_log_decay, rank, state_in=state_in)

    def forward(self, q, k, v, g, *, state_in, k_prefix, v_prefix, want_state, **kw):
        out = self.lz.attn_fwd(q, k, v, g, state_in=state_in, k_prefix=k_prefix, v_prefix=v_prefix,
                               want_state=want_state, **kw)
        self._ws.append(out["workspace"])
        return {"o": out["o"], "state_out": out["state_out"]}

    def backward(self, q, k, v, g, dout, *, state_in, k_prefix, v_prefix, dstate_out, branch, **kw):
        out = self.lz.attn_bwd(q, k, v, g, dout, state_in=state_in, k_prefix=k_prefix,
                               v_prefix=v_prefix, dstate_out=dstate_out, branch=branch, **kw)
        self._ws.append(out.pop("workspace"))
        return out


BRANCH_BOTH, BRANCH_GLA_ONLY = 0, 1
PARAM_GRADS = ("dmeta_k", "dmeta_v", "dfmap_wq", "dfmap_wk", "dalpha")


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


def _raise_together(ops, group, device, where):
    """All-reduce the device status of this rank's compute steps so far; a
    nonzero code on any rank raises on every rank."""
    mine = int(ops.status()) if hasattr(ops, "status") else 0
    t = torch.tensor([mine], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    if int(t.item()) != 0:
        raise RuntimeError(f"sequence parallelism: a rank's kernels reported status {int(t.item())} "
                           f"during {where}")


def _exchange_halo(k, v, window, group, rank, world):
    """Post the halo exchange: the last `window` keys and values go to the
    next rank; returns (k_prefix, v_prefix, requests)."""
    B, H, L, dk = k.shape
    k_prefix = v_prefix = None
    p2p = []
    if rank + 1 < world:
        k_send = k[:, :, L - window:].contiguous()
        v_send = v[:, :, L - window:].contiguous()
        nxt = _peer(group, rank + 1)
        p2p += [dist.P2POp(dist.isend, k_send, nxt, group), dist.P2POp(dist.isend, v_send, nxt, group)]
    if rank > 0:
        k_prefix = torch.empty(B, H, window, dk, dtype=k.dtype, device=k.device)
        v_prefix = torch.empty(B, H, window, v.shape[-1], dtype=v.dtype, device=v.device)
        prv = _peer(group, rank - 1)
        p2p += [dist.P2POp(dist.irecv, k_prefix, prv, group), dist.P2POp(dist.irecv, v_prefix, prv, group)]
    reqs = dist.batch_isend_irecv(p2p) if p2p else []
    return k_prefix, v_prefix, reqs


def _start_state(ops, k, v, g, *, window, chunk, gate_temp, fmap_wk, impl, state_in, group, rank,
                 world, need_last):
    """Segment summaries, all-gathered, and this rank's start state.  The
    last rank's summary is computed only when need_last (the backward needs
    its R); otherwise zeros stand in.  Returns (S0, R_all [world, B, H, dk])."""
    B, H, L, dk = k.shape
    dv = v.shape[-1]
    if rank + 1 < world or need_last:
        U, R = ops.segment_state(k, v, g, window=window, chunk=chunk, gate_temp=gate_temp,
                                 fmap_wk=fmap_wk, impl=impl)
    else:
        U = torch.zeros(B, H, dk, dv, dtype=torch.float32, device=k.device)
        R = torch.zeros(B, H, dk, dtype=torch.float32, device=k.device)
    U_all = [torch.empty_like(U) for _ in range(world)]
    R_all = [torch.empty_like(R) for _ in range(world)]
    dist.all_gather(U_all, U.contiguous(), group=group)
    dist.all_gather(R_all, R.contiguous(), group=group)
    R_all = torch.stack(R_all)
    S0 = ops.chain_states(torch.stack(U_all), R_all, rank, state_in)
    return S0, R_all


def _check_lengths(group, L, window, device):
    lengths = segment_lengths(group, length=L, device=device)
    short = [r for r, n in enumerate(lengths[:-1]) if n < window]
    if short:
        # every rank sees the same lengths, so every rank raises here
        raise ValueError(f"ranks {short} hold fewer than window={window} tokens")
    return lengths


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
    _check_lengths(group, q.shape[2], window, q.device)

    k_prefix, v_prefix, reqs = _exchange_halo(k, v, window, group, rank, world)
    S0, _ = _start_state(ops, k, v, g, window=window, chunk=chunk, gate_temp=gate_temp, fmap_wk=fmap_wk,
                         impl=impl, state_in=state_in, group=group, rank=rank, world=world,
                         need_last=False)
    for r in reqs:
        r.wait()

    out = ops.forward(q, k, v, g, state_in=S0, k_prefix=k_prefix, v_prefix=v_prefix,
                      want_state=rank + 1 == world, window=window, chunk=chunk, gate_temp=gate_temp,
                      softmax_scale=softmax_scale, fmap_wq=fmap_wq, fmap_wk=fmap_wk, meta_k=meta_k,
                      meta_v=meta_v, alpha=alpha, impl=impl)
    _raise_together(ops, group, q.device, "the forward")
    return {"o": out["o"], "state_out": out["state_out"] if rank + 1 == world else None}


def sequence_parallel_backward(q, k, v, g, dout, *, window, group=None, chunk=64, gate_temp=16.0,
                               softmax_scale=0.0, fmap_wq=None, fmap_wk=None, meta_k=None,
                               meta_v=None, alpha=None, state_in=None, dstate_out=None, impl=0,
                               ops=None):
    """Backward of this rank's segment: the gradients of
    sum(dout * o) (+ sum(dstate_out * final state)) over the whole sequence.

    Arguments as for sequence_parallel_forward, plus dout (this rank's
    tokens) and dstate_out (the gradient into the whole sequence's final
    state: read on the last rank only; None for an unused final state).
    Returns this rank's dq, dk, dv, dg; the parameters' gradients dmeta_k,
    dmeta_v, dfmap_wq, dfmap_wk, dalpha summed over every rank (the same on
    each); dstate_in, the gradient with respect to state_in, on rank 0 (None
    elsewhere).
    """
    ops = LibraryOps() if ops is None else ops
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    L = q.shape[2]
    _check_lengths(group, L, window, q.device)
    last = rank + 1 == world
    kw = dict(window=window, chunk=chunk, gate_temp=gate_temp, softmax_scale=softmax_scale,
              fmap_wq=fmap_wq, fmap_wk=fmap_wk, meta_k=meta_k, meta_v=meta_v, alpha=alpha, impl=impl)

    # 1-2. halo and start state, as in the forward (the last rank's R is needed too)
    k_prefix, v_prefix, reqs = _exchange_halo(k, v, window, group, rank, world)
    S0, R_all = _start_state(ops, k, v, g, window=window, chunk=chunk, gate_temp=gate_temp,
                             fmap_wk=fmap_wk, impl=impl, state_in=state_in, group=group, rank=rank,
                             world=world, need_last=True)
    for r in reqs:
        r.wait()

    # 4. this segment's backward from its own outputs (and the caller's G on the last rank)
    gr = ops.backward(q, k, v, g, dout, state_in=S0, k_prefix=k_prefix, v_prefix=v_prefix,
                      dstate_out=dstate_out if last else None, branch=BRANCH_BOTH, **kw)
    _raise_together(ops, group, q.device, "the segment backward")

    # 5. gradient into every segment's end state, chained from the last rank down
    D = gr["dstate_in"].contiguous()
    D_all = [torch.empty_like(D) for _ in range(world)]
    dist.all_gather(D_all, D, group=group)
    X = ops.chain_states(torch.stack(D_all[::-1]), torch.flip(R_all, dims=[0]), world - 1 - rank, None)

    # 6. what that end-state gradient adds (GLA branch only; linear in X)
    if not last:
        corr = ops.backward(q, k, v, g, torch.zeros_like(dout), state_in=S0, k_prefix=None, v_prefix=None,
                            dstate_out=X, branch=BRANCH_GLA_ONLY, **kw)
        for name in ("dq", "dk", "dv", "dg", "dfmap_wq", "dfmap_wk", "dstate_in"):
            if gr.get(name) is not None and corr.get(name) is not None:
                gr[name] = gr[name] + corr[name]
    _raise_together(ops, group, q.device, "the end-state correction")

    # 7. prefix gradients back to the previous rank; parameters summed over ranks
    p2p = []
    recv_k = recv_v = None
    if rank > 0:
        prv = _peer(group, rank - 1)
        p2p += [dist.P2POp(dist.isend, gr["dk_prefix"].contiguous(), prv, group),
                dist.P2POp(dist.isend, gr["dv_prefix"].contiguous(), prv, group)]
    if not last:
        B, H = q.shape[:2]
        recv_k = torch.empty(B, H, window, k.shape[-1], dtype=gr["dk"].dtype, device=k.device)
        recv_v = torch.empty(B, H, window, v.shape[-1], dtype=gr["dv"].dtype, device=v.device)
        nxt = _peer(group, rank + 1)
        p2p += [dist.P2POp(dist.irecv, recv_k, nxt, group), dist.P2POp(dist.irecv, recv_v, nxt, group)]
    reqs = dist.batch_isend_irecv(p2p) if p2p else []
    for name in PARAM_GRADS:
        if gr.get(name) is not None:
            t = gr[name].contiguous()
            dist.all_reduce(t, group=group)
            gr[name] = t
    for r in reqs:
        r.wait()
    if not last:
        gr["dk"] = gr["dk"].clone()
        gr["dv"] = gr["dv"].clone()
        gr["dk"][:, :, L - window:] += recv_k
        gr["dv"][:, :, L - window:] += recv_v
    out = {n: gr.get(n) for n in ("dq", "dk", "dv", "dg") + PARAM_GRADS}
    out["dstate_in"] = gr["dstate_in"] if rank == 0 else None
    return out
