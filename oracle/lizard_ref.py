"""Lizard hybrid attention -- plain fp64 CPU oracle.

TEST INFRASTRUCTURE.  This module is the independent definition that the
CUDA library is checked against.  Only the test suite, the smoke check and
the CPU-baseline leg of the benchmark may import it; the product path never
does, and it shares no code, tables or helpers with the CUDA sources.

Everything is NumPy float64, written as the plain definition: the GLA branch
is the token-by-token recurrence, the anchor branch is an explicit masked
softmax, one query at a time.  There is no chunking, blocking or fusion here.
Loops run over tokens; batch and head dimensions are vectorised with einsum.

Sources (web summaries of arXiv 2507.09025, "Lizard: An Efficient
Linearization Framework for Large Language Models"):

  [EN] gist.science/paper/2507.09025 -- English technical summary
  [FR] gist.science/fr/paper/2507.09025 -- French technical summary
  [ZH] gist.science/zh/paper/2507.09025 -- Chinese technical summary
  [ES] gist.science/es/paper/2507.09025 -- Spanish technical summary

What the pages fix, and the reading taken where they are silent:

* Gate: Gamma_t = sigmoid(W_gamma x_t) ([EN] 2.A "Adaptive Memory Control";
  [FR] 2.A; [ZH] 2.1).  The projection W_gamma x is outside this operation:
  the inputs are the gate logits g.  The log-decay is
  a_t = logsigmoid(g_t) / tau per key dimension, with tau a temperature
  (tau = 1 gives the pages' literal sigmoid gate; the workloads use 16).
* Gate granularity: per key dimension (g [B,H,L,dk]) by default.  The
  Chinese summary's ablation ([ZH] 4, "消融实验") finds a light scalar gate
  the most effective; gate="scalar" takes one logit per token and head
  (g [B,H,L]) whose decay applies to every key dimension.
* State update: S_t = diag(Gamma_t) S_{t-1} + phi(k_t) v_t^T ([EN] 2.A
  "State Update").  Read-out (a reading): o_t = S_t^T phi(q_t), with S_t
  already containing token t.  No normaliser.  The recurrence spans the
  whole causal prefix (global context, [EN] 2.A last bullet).
* Feature map phi: the pages only say Hedgehog, non-negative ([ZH] 2.3).
  Reading: phi(x) = [softmax(x W), softmax(-x W)], W in R^{dk x dk/2} per
  head, separate maps for q and k, output width dk.  W = None means the
  identity map (used by invariant tests).
* Anchor window attention ([EN] 2.A "Anchor Window Attention"; [FR] 2.A;
  [ZH] 2.1): exact softmax over the last `window` keys including the query
  itself, j in [t - window + 1, t], with M learnable meta tokens added to the
  softmax denominator.  The pages say the meta tokens do not contribute to
  the value; meta_v = None gives exactly that (sink-only).  A meta_v array
  gives them values (the workloads pass one).  Raw q, k, v feed this branch;
  phi is used only by the GLA branch.  Scale 1/sqrt(dk) by default; no RoPE
  in either branch ([ES] 2, "Etapa 1").
* Mixing: Y = Y_gate + alpha * Y_anchor ([FR] 2.A last line; [EN] 2.A
  "Final Output"), alpha a per-head scalar.
* Decode ([EN] 2.A "State Update", constant memory; [ZH] 2.1 fixed-size KV
  cache): one token updates S and writes (k, v) into slot pos mod window of a
  ring buffer; the softmax runs over the min(pos + 1, window) filled slots
  plus the meta tokens.
* Sequence parallelism (a reading; the pages split no sequence): a segment
  of a longer sequence receives the GLA history as its start state and the
  keys and values just before it as a prefix of the anchor window.  The
  start states chain segment summaries (U, R) through the affine form of
  the state update (gla_segment_state, chain_states).

Parity status: every public function here is pinned by the CPU tests against
closed forms, library routines (causal softmax attention, autograd) and
brute-force sums written independently of this file.
"""

from __future__ import annotations

import numpy as np

BRANCH_BOTH = 0
BRANCH_GLA_ONLY = 1
BRANCH_SWA_ONLY = 2

GATE_PER_DIM = "dim"
GATE_SCALAR = "scalar"


def _f64(x):
    return None if x is None else np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Gate and feature map
# ---------------------------------------------------------------------------

def gate_log_decay(g, tau=16.0):
    """log Gamma = logsigmoid(g) / tau, elementwise.

    [EN] 2.A "Adaptive Memory Control" (Gamma = sigmoid(W_gamma x)); the
    temperature tau is the workloads' choice.  Written in the overflow-free
    form logsigmoid(g) = min(g, 0) - log(1 + exp(-|g|)).
    """
    g = _f64(g)
    return (np.minimum(g, 0.0) - np.log1p(np.exp(-np.abs(g)))) / float(tau)


def layer_log_decay(g, tau, gate, dk):
    """The per-dimension log-decay a [..., dk] the recurrence uses.

    gate="dim": g [..., dk], a = logsigmoid(g)/tau elementwise.
    gate="scalar": g [...] (one logit per token and head, [ZH] 4 ablation);
    every key dimension decays by the same logsigmoid(g)/tau.
    """
    a = gate_log_decay(g, tau)
    if gate == GATE_SCALAR:
        return np.repeat(a[..., None], dk, axis=-1)
    if gate != GATE_PER_DIM:
        raise ValueError(f"gate must be {GATE_PER_DIM!r} or {GATE_SCALAR!r}")
    return a


def _softmax_last(z):
    m = np.max(z, axis=-1, keepdims=True)
    e = np.exp(z - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def feature_map(x, W):
    """phi(x) = [softmax(x W_h), softmax(-x W_h)] per head h.

    x: [B, H, L, d]; W: [H, d, d/2] or None (identity).  Non-negative, each
    half sums to one ([ZH] 2.3: the Hedgehog map is non-negative).
    """
    x = _f64(x)
    if W is None:
        return x.copy()
    W = _f64(W)
    z = np.einsum("bhld,hdf->bhlf", x, W)
    return np.concatenate([_softmax_last(z), _softmax_last(-z)], axis=-1)


def feature_map_backward(x, W, dphi):
    """Gradients of phi(x) = [softmax(xW), softmax(-xW)] w.r.t. x and W."""
    x = _f64(x)
    dphi = _f64(dphi)
    if W is None:
        return dphi.copy(), None
    W = _f64(W)
    F = W.shape[-1]
    z = np.einsum("bhld,hdf->bhlf", x, W)
    p = _softmax_last(z)
    n = _softmax_last(-z)
    dp = dphi[..., :F]
    dn = dphi[..., F:]
    # softmax Jacobian: dz = p * (dp - <dp, p>); the minus branch flips sign.
    dz = p * (dp - np.sum(dp * p, axis=-1, keepdims=True))
    dz -= n * (dn - np.sum(dn * n, axis=-1, keepdims=True))
    dx = np.einsum("bhlf,hdf->bhld", dz, W)
    dW = np.einsum("bhld,bhlf->hdf", x, dz)
    return dx, dW


# ---------------------------------------------------------------------------
# GLA branch: token-by-token recurrence
# ---------------------------------------------------------------------------

def gla_forward(phq, phk, v, a, S0=None, keep_states=False):
    """Recurrent gated linear attention ([EN] 2.A "State Update").

    S_t = diag(exp a_t) S_{t-1} + phk_t v_t^T ;  o_t = S_t^T phq_t.

    phq, phk, a: [B, H, L, dk]; v: [B, H, L, dv]; S0: [B, H, dk, dv] or None.
    Returns (o [B,H,L,dv], S_L [B,H,dk,dv], states or None), where states[t]
    is S_t (kept only on request, for the backward).
    """
    phq, phk, v, a = _f64(phq), _f64(phk), _f64(v), _f64(a)
    B, H, L, dk = phk.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dk, dv)) if S0 is None else _f64(S0).copy()
    o = np.zeros((B, H, L, dv))
    states = np.zeros((L, B, H, dk, dv)) if keep_states else None
    for t in range(L):
        S = np.exp(a[:, :, t, :])[..., None] * S \
            + phk[:, :, t, :, None] * v[:, :, t, None, :]
        o[:, :, t, :] = np.einsum("bhi,bhij->bhj", phq[:, :, t, :], S)
        if keep_states:
            states[t] = S
    return o, S, states


def gla_backward(phq, phk, v, a, S0, do, dS_L=None):
    """Reverse-mode derivative of :func:`gla_forward`, from the recurrence.

    dS_L: gradient flowing into the final state S_{L-1} from outside the
    sequence (None: the final state is unused).  With dS the gradient
    flowing into S_t from tokens >= t (and from dS_L):
      dS   += phq_t do_t^T
      dphq_t = S_t do_t,  dphk_t = dS v_t,  dv_t = dS^T phk_t
      da_t   = exp(a_t) * rowsum(dS * S_{t-1})
      dS    <- diag(exp a_t) dS        (gradient into S_{t-1})
    Returns (dphq, dphk, dv, da, dS0).
    """
    phq, phk, v, a, do = _f64(phq), _f64(phk), _f64(v), _f64(a), _f64(do)
    B, H, L, dk = phk.shape
    dv_ = v.shape[-1]
    S0 = np.zeros((B, H, dk, dv_)) if S0 is None else _f64(S0)
    _, _, states = gla_forward(phq, phk, v, a, S0, keep_states=True)
    dphq = np.zeros_like(phq)
    dphk = np.zeros_like(phk)
    dv = np.zeros_like(v)
    da = np.zeros_like(a)
    dS = np.zeros((B, H, dk, dv_)) if dS_L is None else _f64(dS_L).copy()
    for t in range(L - 1, -1, -1):
        dS += phq[:, :, t, :, None] * do[:, :, t, None, :]
        St = states[t]
        Sprev = states[t - 1] if t > 0 else S0
        dphq[:, :, t] = np.einsum("bhij,bhj->bhi", St, do[:, :, t])
        dphk[:, :, t] = np.einsum("bhij,bhj->bhi", dS, v[:, :, t])
        dv[:, :, t] = np.einsum("bhij,bhi->bhj", dS, phk[:, :, t])
        gam = np.exp(a[:, :, t, :])
        da[:, :, t] = gam * np.sum(dS * Sprev, axis=-1)
        dS = gam[..., None] * dS
    return dphq, dphk, dv, da, dS


# ---------------------------------------------------------------------------
# Anchor branch: sliding-window softmax with meta-token sinks
# ---------------------------------------------------------------------------

def _window_probs(q, k, meta_k, t, window, scale):
    """Softmax weights of query t over keys [t-window+1, t] and meta tokens.

    Returns (j0, p_win [B,H,n], p_meta [B,H,M] or None, lse [B,H]).
    """
    j0 = max(0, t - window + 1)
    logits = scale * np.einsum("bhd,bhjd->bhj", q[:, :, t], k[:, :, j0:t + 1])
    if meta_k is not None and meta_k.shape[1] > 0:
        ml = scale * np.einsum("bhd,hmd->bhm", q[:, :, t], meta_k)
        logits = np.concatenate([logits, ml], axis=-1)
    mx = np.max(logits, axis=-1, keepdims=True)
    e = np.exp(logits - mx)
    Z = np.sum(e, axis=-1, keepdims=True)
    p = e / Z
    n = t + 1 - j0
    lse = (mx + np.log(Z))[..., 0]
    p_meta = p[..., n:] if p.shape[-1] > n else None
    return j0, p[..., :n], p_meta, lse


def swa_forward(q, k, v, meta_k, meta_v, window, scale=None,
                k_prefix=None, v_prefix=None):
    """Sliding-window softmax attention with meta-token sinks.

    [EN] 2.A "Anchor Window Attention": the meta tokens sit in the softmax
    denominator; with meta_v = None they add no value (sink-only).
    q, k: [B,H,L,dk]; v: [B,H,L,dv]; meta_k: [H,M,dk] or None;
    meta_v: [H,M,dv] or None.  Returns (o_swa [B,H,L,dv], lse [B,H,L]),
    lse the natural-log normaliser over window and meta logits.

    k_prefix, v_prefix [B,H,P,d] (a reading for a segment of a longer
    sequence): the P keys and values just before token 0, which the window
    of the first tokens reaches as if the sequence started P tokens earlier.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    meta_k, meta_v = _f64(meta_k), _f64(meta_v)
    B, H, L, dk = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    P = 0 if k_prefix is None else _f64(k_prefix).shape[2]
    if P:
        # the queries of the prefix positions are never used
        q = np.concatenate([np.zeros((B, H, P, dk)), q], axis=2)
        k = np.concatenate([_f64(k_prefix), k], axis=2)
        v = np.concatenate([_f64(v_prefix), v], axis=2)
    o = np.zeros((B, H, L, v.shape[-1]))
    lse = np.zeros((B, H, L))
    for t in range(L):
        j0, p_win, p_meta, lse[:, :, t] = _window_probs(q, k, meta_k, P + t,
                                                        window, scale)
        o[:, :, t] = np.einsum("bhj,bhjd->bhd", p_win, v[:, :, j0:P + t + 1])
        if p_meta is not None and meta_v is not None:
            o[:, :, t] += np.einsum("bhm,hmd->bhd", p_meta, meta_v)
    return o, lse


def swa_backward(q, k, v, meta_k, meta_v, window, scale, do):
    """Reverse-mode derivative of :func:`swa_forward` (softmax Jacobian).

    For query t with weights p over (window keys, meta tokens):
      dp = do_t . value,  D = sum(p * dp) = do_t . o_t,  ds = p * (dp - D)
      dq_t = scale * sum ds * key,  dkey += scale * ds * q_t,
      dvalue += p * do_t.
    Returns (dq, dk, dv, dmeta_k, dmeta_v); the meta gradients are None when
    the corresponding input is None.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    meta_k, meta_v = _f64(meta_k), _f64(meta_v)
    B, H, L, dk = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    dq = np.zeros_like(q)
    dk_ = np.zeros_like(k)
    dv = np.zeros_like(v)
    dmk = None if meta_k is None else np.zeros_like(meta_k)
    dmv = None if meta_v is None else np.zeros_like(meta_v)
    for t in range(L):
        j0, p_win, p_meta, _ = _window_probs(q, k, meta_k, t, window, scale)
        vw = v[:, :, j0:t + 1]
        kw = k[:, :, j0:t + 1]
        dp_win = np.einsum("bhd,bhjd->bhj", do[:, :, t], vw)
        o_t = np.einsum("bhj,bhjd->bhd", p_win, vw)
        if p_meta is not None:
            if meta_v is not None:
                dp_meta = np.einsum("bhd,hmd->bhm", do[:, :, t], meta_v)
                o_t = o_t + np.einsum("bhm,hmd->bhd", p_meta, meta_v)
            else:
                dp_meta = np.zeros_like(p_meta)
        D = np.sum(do[:, :, t] * o_t, axis=-1, keepdims=True)
        ds_win = p_win * (dp_win - D)
        dq[:, :, t] = scale * np.einsum("bhj,bhjd->bhd", ds_win, kw)
        dk_[:, :, j0:t + 1] += scale * ds_win[..., None] * q[:, :, t, None, :]
        dv[:, :, j0:t + 1] += p_win[..., None] * do[:, :, t, None, :]
        if p_meta is not None:
            ds_meta = p_meta * (dp_meta - D)
            dq[:, :, t] += scale * np.einsum("bhm,hmd->bhd", ds_meta, meta_k)
            dmk += scale * np.einsum("bhm,bhd->hmd", ds_meta, q[:, :, t])
            if meta_v is not None:
                dmv += np.einsum("bhm,bhd->hmd", p_meta, do[:, :, t])
    return dq, dk_, dv, dmk, dmv


def swa_backward_prefix(q, k, v, meta_k, meta_v, window, scale, do, k_prefix, v_prefix):
    """:func:`swa_backward` for a segment whose window reaches P keys and
    values before token 0 (see :func:`swa_forward`).  The prefix tokens are
    the first P positions of one longer sequence whose own outputs carry no
    gradient (their queries are never used).  Returns (dq, dk, dv, dmeta_k,
    dmeta_v, dk_prefix, dv_prefix)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    kp, vp = _f64(k_prefix), _f64(v_prefix)
    B, H, _, dk = q.shape
    P = kp.shape[2]
    dq, dk_, dv, dmk, dmv = swa_backward(
        np.concatenate([np.zeros((B, H, P, dk)), q], axis=2), np.concatenate([kp, k], axis=2),
        np.concatenate([vp, v], axis=2), meta_k, meta_v, window, scale,
        np.concatenate([np.zeros((B, H, P, do.shape[-1])), do], axis=2))
    return dq[:, :, P:], dk_[:, :, P:], dv[:, :, P:], dmk, dmv, dk_[:, :, :P], dv[:, :, :P]


# ---------------------------------------------------------------------------
# The hybrid layer
# ---------------------------------------------------------------------------

def _defaults(q, alpha, scale, meta_k):
    H, dk = q.shape[1], q.shape[-1]
    alpha = np.ones(H) if alpha is None else _f64(alpha)
    scale = 1.0 / np.sqrt(dk) if scale is None else float(scale)
    if meta_k is not None and _f64(meta_k).shape[1] == 0:
        meta_k = None
    return alpha, scale, meta_k


def lizard_forward(q, k, v, g, *, window, tau=16.0, scale=None,
                   fmap_wq=None, fmap_wk=None, meta_k=None, meta_v=None,
                   alpha=None, state_in=None, branch=BRANCH_BOTH,
                   gate=GATE_PER_DIM, k_prefix=None, v_prefix=None):
    """Hybrid layer forward: o = o_gla + alpha_h * o_swa.

    Mixing rule: [FR] 2.A last line, [EN] 2.A "Final Output".  `branch`
    keeps only one term of the sum (test hook): GLA_ONLY gives o_gla,
    SWA_ONLY gives alpha_h * o_swa.  k_prefix / v_prefix: keys and values
    before token 0 for the anchor window (see swa_forward); the GLA branch
    takes the earlier history through state_in.
    Returns a dict with o, state_out (S_L, GLA run only), lse (anchor run
    only), o_gla and o_swa.
    """
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g)
    alpha, scale, meta_k = _defaults(q, alpha, scale, meta_k)
    if meta_k is None:
        meta_v = None
    out = {"o": np.zeros(v.shape), "state_out": None, "lse": None,
           "o_gla": None, "o_swa": None}
    if branch != BRANCH_SWA_ONLY:
        a = layer_log_decay(g, tau, gate, q.shape[-1])
        o_gla, S_L, _ = gla_forward(feature_map(q, fmap_wq),
                                    feature_map(k, fmap_wk), v, a, state_in)
        out["o"] += o_gla
        out["o_gla"], out["state_out"] = o_gla, S_L
    if branch != BRANCH_GLA_ONLY:
        o_swa, lse = swa_forward(q, k, v, meta_k, meta_v, window, scale,
                                 k_prefix, v_prefix)
        out["o"] += alpha[None, :, None, None] * o_swa
        out["o_swa"], out["lse"] = o_swa, lse
    return out


# ---------------------------------------------------------------------------
# Sequence parallelism: segment summaries of the GLA recurrence
# ---------------------------------------------------------------------------

def gla_segment_state(k, v, g, *, tau=16.0, fmap_wk=None, gate=GATE_PER_DIM):
    """Summary (U, R) of one segment of a sequence.

    Reading of [EN] 2.A "State Update" over a run of tokens: the recurrence
    S_t = diag(exp a_t) S_{t-1} + phi(k_t) v_t^T is affine in the state it
    starts from, so over the segment a start state S ends as
    diag(exp R) S + U, with R = sum_t a_t (per key dimension) and U the
    state reached from S = 0.  U is that recurrence run from zero; R the
    plain sum.  Returns (U [B,H,dk,dv], R [B,H,dk]).
    """
    k, v, g = _f64(k), _f64(v), _f64(g)
    dk = k.shape[-1]
    a = layer_log_decay(g, tau, gate, dk)
    phk = feature_map(k, fmap_wk)
    B, H, L, _ = k.shape
    U = np.zeros((B, H, dk, v.shape[-1]))
    for t in range(L):
        U = np.exp(a[:, :, t])[..., None] * U + np.einsum("bhi,bhj->bhij", phk[:, :, t], v[:, :, t])
    return U, a.sum(axis=2)


def chain_states(seg_states, seg_log_decays, rank, state_in=None):
    """Start state of segment `rank`: S_0 = state_in (or 0),
    S_{j+1} = diag(exp R_j) S_j + U_j over the segments before it."""
    U0 = _f64(seg_states[0])
    S = np.zeros(U0.shape) if state_in is None else _f64(state_in).copy()
    for j in range(rank):
        S = np.exp(_f64(seg_log_decays[j]))[..., None] * S + _f64(seg_states[j])
    return S


def lizard_backward(q, k, v, g, dout, *, window, tau=16.0, scale=None,
                    fmap_wq=None, fmap_wk=None, meta_k=None, meta_v=None,
                    alpha=None, state_in=None, branch=BRANCH_BOTH,
                    gate=GATE_PER_DIM, dstate_out=None, k_prefix=None, v_prefix=None):
    """Gradients of sum(dout * lizard_forward(...)['o']) w.r.t. every input.

    dstate_out [B,H,dk,dv]: gradient of the loss with respect to the final
    state (the loss then is sum(dout * o) + sum(dstate_out * state_out), the
    form a caller that chains sequences through their states has); None for
    an unused final state.  k_prefix / v_prefix: the anchor window's prefix,
    as in lizard_forward; their gradients come back as dk_prefix, dv_prefix
    (None without a prefix).

    Returns a dict: dq, dk, dv, dg (the shape of g: [B,H,L,dk], or [B,H,L]
    for gate="scalar"), dmeta_k, dmeta_v, dfmap_wq,
    dfmap_wk (None where the input is None), dalpha [H], dstate_in [B,H,dk,dv].
    """
    q, k, v, g, dout = _f64(q), _f64(k), _f64(v), _f64(g), _f64(dout)
    alpha, scale, meta_k = _defaults(q, alpha, scale, meta_k)
    if meta_k is None:
        meta_v = None
    B, H, L, dk = q.shape
    dv_ = v.shape[-1]
    res = {"dq": np.zeros_like(q), "dk": np.zeros_like(k),
           "dv": np.zeros_like(v), "dg": np.zeros_like(g),
           "dmeta_k": None if meta_k is None else np.zeros(_f64(meta_k).shape),
           "dmeta_v": None if meta_v is None else np.zeros(_f64(meta_v).shape),
           "dfmap_wq": None if fmap_wq is None else np.zeros(_f64(fmap_wq).shape),
           "dfmap_wk": None if fmap_wk is None else np.zeros(_f64(fmap_wk).shape),
           "dalpha": np.zeros(H), "dstate_in": np.zeros((B, H, dk, dv_)),
           "dk_prefix": None if k_prefix is None else np.zeros(_f64(k_prefix).shape),
           "dv_prefix": None if v_prefix is None else np.zeros(_f64(v_prefix).shape)}
    if branch != BRANCH_SWA_ONLY:
        a = layer_log_decay(g, tau, gate, dk)
        phq = feature_map(q, fmap_wq)
        phk = feature_map(k, fmap_wk)
        dphq, dphk, dv_g, da, dS0 = gla_backward(phq, phk, v, a, state_in, dout,
                                                 dstate_out)
        dq_g, dWq = feature_map_backward(q, fmap_wq, dphq)
        dk_g, dWk = feature_map_backward(k, fmap_wk, dphk)
        res["dq"] += dq_g
        res["dk"] += dk_g
        res["dv"] += dv_g
        # d logsigmoid(g)/dg = sigmoid(-g); a scalar logit feeds every
        # key dimension's decay, so its gradient sums over them
        if gate == GATE_SCALAR:
            da = da.sum(axis=-1)
        res["dg"] = da / (1.0 + np.exp(g)) / float(tau)
        res["dstate_in"] = dS0
        if fmap_wq is not None:
            res["dfmap_wq"] = dWq
        if fmap_wk is not None:
            res["dfmap_wk"] = dWk
    if branch != BRANCH_GLA_ONLY:
        o_swa, _ = swa_forward(q, k, v, meta_k, meta_v, window, scale, k_prefix, v_prefix)
        res["dalpha"] = np.einsum("bhld,bhld->h", dout, o_swa)
        dsw = alpha[None, :, None, None] * dout
        if k_prefix is None:
            dq_s, dk_s, dv_s, dmk, dmv = swa_backward(q, k, v, meta_k, meta_v,
                                                      window, scale, dsw)
        else:
            dq_s, dk_s, dv_s, dmk, dmv, res["dk_prefix"], res["dv_prefix"] = swa_backward_prefix(
                q, k, v, meta_k, meta_v, window, scale, dsw, k_prefix, v_prefix)
        res["dq"] += dq_s
        res["dk"] += dk_s
        res["dv"] += dv_s
        if dmk is not None:
            res["dmeta_k"] = dmk
        if dmv is not None:
            res["dmeta_v"] = dmv
    return res


# ---------------------------------------------------------------------------
# Stage 1 of training: attention approximation
# ---------------------------------------------------------------------------

def attention_mse(o, target):
    """Stage-1 attention-approximation loss and its gradient.

    [EN] 2.B "Stage 1", [ZH] 2.2, [FR] 2.B: the layer is trained to reproduce
    the teacher's softmax-attention output under a mean squared error.
    Reading: the mean runs over every element (batch, head, token, value
    dimension), loss = sum((o - y)^2) / n, so dL/do = 2 (o - y) / n.
    """
    diff = _f64(o) - _f64(target)
    n = diff.size
    return float(np.sum(diff * diff) / n), 2.0 * diff / n


def lizard_stage1_step(q, k, v, g, target, *, window, tau=16.0, scale=None,
                       fmap_wq=None, fmap_wk=None, meta_k=None, meta_v=None,
                       alpha=None, state_in=None, gate=GATE_PER_DIM):
    """One stage-1 training step: forward, the MSE against the teacher output
    `target` [B,H,L,dv], and the gradients of that loss with respect to every
    input (as lizard_backward, with dout = dL/do).  Returns the backward's
    dict plus "loss" and "o"."""
    kw = dict(window=window, tau=tau, scale=scale, fmap_wq=fmap_wq, fmap_wk=fmap_wk,
              meta_k=meta_k, meta_v=meta_v, alpha=alpha, state_in=state_in, gate=gate)
    o = lizard_forward(q, k, v, g, **kw)["o"]
    loss, dout = attention_mse(o, target)
    res = lizard_backward(q, k, v, g, dout, **kw)
    res["loss"], res["o"] = loss, o
    return res


# ---------------------------------------------------------------------------
# Decode: one token, constant-size state plus a ring-buffer window
# ---------------------------------------------------------------------------

def lizard_decode_step(q, k, v, g, state, k_cache, v_cache, pos, *, window,
                       tau=16.0, scale=None, fmap_wq=None, fmap_wk=None,
                       meta_k=None, meta_v=None, alpha=None, gate=GATE_PER_DIM):
    """One generation step for every (batch, head); inputs are not modified.

    q, k: [B,H,dk]; g: [B,H,dk] ([B,H] for gate="scalar"); v: [B,H,dv];
    state: [B,H,dk,dv]; k_cache: [B,H,w,dk];
    v_cache: [B,H,w,dv]; pos: [B] tokens already seen.  The new token goes to
    ring slot pos mod w; the softmax covers the min(pos+1, w) filled slots and
    the meta tokens.  Returns (o [B,H,dv], state, k_cache, v_cache, pos + 1).
    """
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g)
    S = _f64(state).copy()
    kc = _f64(k_cache).copy()
    vc = _f64(v_cache).copy()
    pos = np.asarray(pos, dtype=np.int64).copy()
    alpha, scale, meta_k = _defaults(q[:, :, None], alpha, scale, meta_k)
    if meta_k is None:
        meta_v = None
    B, H, dk = q.shape
    a = layer_log_decay(g, tau, gate, dk)
    phq = feature_map(q[:, :, None], fmap_wq)[:, :, 0]
    phk = feature_map(k[:, :, None], fmap_wk)[:, :, 0]
    S = np.exp(a)[..., None] * S + phk[..., None] * v[:, :, None, :]
    o_gla = np.einsum("bhi,bhij->bhj", phq, S)
    o_swa = np.zeros_like(o_gla)
    mk = None if meta_k is None else _f64(meta_k)
    mv = None if meta_v is None else _f64(meta_v)
    for b in range(B):
        slot = int(pos[b] % window)
        kc[b, :, slot] = k[b]
        vc[b, :, slot] = v[b]
        n = int(min(pos[b] + 1, window))
        logits = scale * np.einsum("hd,hjd->hj", q[b], kc[b, :, :n])
        if mk is not None:
            logits = np.concatenate(
                [logits, scale * np.einsum("hd,hmd->hm", q[b], mk)], axis=-1)
        p = _softmax_last(logits)
        o_swa[b] = np.einsum("hj,hjd->hd", p[:, :n], vc[b, :, :n])
        if mv is not None:
            o_swa[b] += np.einsum("hm,hmd->hd", p[:, n:], mv)
    o = o_gla + alpha[None, :, None] * o_swa
    return o, S, kc, vc, pos + 1
