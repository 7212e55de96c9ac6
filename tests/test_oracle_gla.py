"""Pins for the oracle's gate, feature map and GLA branch (CPU only).

Each check compares the oracle with something other than itself: a library
routine (torch logsigmoid / softmax / autograd), a closed form, brute-force
sums written here, or the chunkwise log-space algorithm derived here from the
pages' hardware-aware reparameterisation (gist.science "Lizard" summaries,
Chinese version 2.3, English version 2.C).
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import lizard_ref as ref

rng = np.random.default_rng(1234)


def _rand(*shape, scale=1.0):
    return rng.standard_normal(shape) * scale


# ---------------------------------------------------------------- gate ------

@pytest.mark.parametrize("tau", [1.0, 16.0])
def test_gate_matches_torch_logsigmoid(tau):
    g = np.concatenate([_rand(1000, scale=4.0),
                        np.array([0.0, 30.0, -30.0, 700.0, -700.0, 1e4, -1e4])])
    want = F.logsigmoid(torch.from_numpy(g)).numpy() / tau
    got = ref.gate_log_decay(g, tau)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-300)
    assert np.all(got <= 0.0)


def test_gate_special_values():
    # sigmoid(0) = 1/2, so the log-decay at g = 0 is -log(2)/tau.
    assert ref.gate_log_decay(0.0, 16.0) == pytest.approx(-math.log(2) / 16, rel=1e-15)
    # tau = 1 is the pages' literal gate sigmoid(x): exp(a) == sigmoid(g).
    g = _rand(50)
    np.testing.assert_allclose(np.exp(ref.gate_log_decay(g, 1.0)),
                               1.0 / (1.0 + np.exp(-g)), rtol=1e-14)
    # Large positive logits keep the state (decay -> 1).
    assert ref.gate_log_decay(1e4, 16.0) == 0.0


# --------------------------------------------------------- feature map ------

def test_feature_map_nonnegative_and_normalised():
    x = _rand(2, 3, 7, 16)
    W = _rand(3, 16, 8, scale=0.5)
    phi = ref.feature_map(x, W)
    assert phi.shape == (2, 3, 7, 16)
    assert np.all(phi > 0)
    np.testing.assert_allclose(phi[..., :8].sum(-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(phi[..., 8:].sum(-1), 1.0, rtol=1e-14)
    z = torch.einsum("bhld,hdf->bhlf", torch.from_numpy(x), torch.from_numpy(W))
    want = torch.cat([torch.softmax(z, -1), torch.softmax(-z, -1)], -1).numpy()
    np.testing.assert_allclose(phi, want, rtol=1e-13)


def test_feature_map_zero_weights_is_uniform():
    x = _rand(1, 1, 5, 8)
    phi = ref.feature_map(x, np.zeros((1, 8, 4)))
    np.testing.assert_allclose(phi, 0.25, rtol=1e-15)


def test_feature_map_backward_autograd():
    x = _rand(2, 2, 5, 8)
    W = _rand(2, 8, 4, scale=0.7)
    dphi = _rand(2, 2, 5, 8)
    xt = torch.from_numpy(x).requires_grad_()
    Wt = torch.from_numpy(W).requires_grad_()
    z = torch.einsum("bhld,hdf->bhlf", xt, Wt)
    phi = torch.cat([torch.softmax(z, -1), torch.softmax(-z, -1)], -1)
    (phi * torch.from_numpy(dphi)).sum().backward()
    dx, dW = ref.feature_map_backward(x, W, dphi)
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(dW, Wt.grad.numpy(), rtol=1e-11, atol=1e-14)


# ----------------------------------------------------------- GLA forward ----

def _gla_inputs(B=2, H=2, L=13, dk=4, dv=3, nonneg=True, with_state=True):
    phq = np.abs(_rand(B, H, L, dk)) if nonneg else _rand(B, H, L, dk)
    phk = np.abs(_rand(B, H, L, dk)) if nonneg else _rand(B, H, L, dk)
    v = _rand(B, H, L, dv)
    a = ref.gate_log_decay(_rand(B, H, L, dk, scale=2.0), 2.0)
    S0 = _rand(B, H, dk, dv) if with_state else None
    return phq, phk, v, a, S0


def _gla_bruteforce(phq, phk, v, a, S0):
    """o_t = sum_{j<=t} sum_i phq_t[i] phk_j[i] prod_{u=j+1..t} exp(a_u[i]) v_j
             + sum_i phq_t[i] prod_{u=0..t} exp(a_u[i]) S0[i, :]
    written as plain nested loops."""
    B, H, L, dk = phq.shape
    dv = v.shape[-1]
    o = np.zeros((B, H, L, dv))
    for b in range(B):
        for h in range(H):
            for t in range(L):
                for i in range(dk):
                    if S0 is not None:
                        dec = 1.0
                        for u in range(0, t + 1):
                            dec *= math.exp(a[b, h, u, i])
                        o[b, h, t] += phq[b, h, t, i] * dec * S0[b, h, i]
                    for j in range(t + 1):
                        dec = 1.0
                        for u in range(j + 1, t + 1):
                            dec *= math.exp(a[b, h, u, i])
                        o[b, h, t] += phq[b, h, t, i] * phk[b, h, j, i] * dec * v[b, h, j]
    return o


def test_gla_matches_bruteforce_sum():
    phq, phk, v, a, S0 = _gla_inputs(nonneg=False)
    o, _, _ = ref.gla_forward(phq, phk, v, a, S0)
    np.testing.assert_allclose(o, _gla_bruteforce(phq, phk, v, a, S0),
                               rtol=1e-11, atol=1e-12)


def test_gla_unit_gate_is_causal_linear_attention():
    # a = 0 (Gamma = 1): o = tril(phq phk^T) v, the ungated linear attention.
    phq, phk, v, _, _ = _gla_inputs(L=9)
    a = ref.gate_log_decay(np.full(phq.shape, 1e4), 16.0)
    assert np.all(a == 0.0)
    o, S_L, _ = ref.gla_forward(phq, phk, v, a)
    A = np.tril(np.einsum("bhti,bhji->bhtj", phq, phk))
    np.testing.assert_allclose(o, A @ v, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S_L, np.einsum("bhji,bhjv->bhiv", phk, v), rtol=1e-12)


def test_gla_closed_gate_keeps_only_current_token():
    # tau = 1, g -> -inf: Gamma -> 0, only the current token survives.
    phq, phk, v, _, _ = _gla_inputs(L=6)
    a = ref.gate_log_decay(np.full(phq.shape, -1e4), 1.0)
    o, _, _ = ref.gla_forward(phq, phk, v, a)
    want = np.sum(phq * phk, -1, keepdims=True) * v
    np.testing.assert_allclose(o, want, rtol=1e-12, atol=1e-300)


def test_gla_segmented_equals_one_shot():
    phq, phk, v, a, S0 = _gla_inputs(L=20)
    o, S_L, _ = ref.gla_forward(phq, phk, v, a, S0)
    o1, S1, _ = ref.gla_forward(phq[:, :, :7], phk[:, :, :7], v[:, :, :7], a[:, :, :7], S0)
    o2, S2, _ = ref.gla_forward(phq[:, :, 7:], phk[:, :, 7:], v[:, :, 7:], a[:, :, 7:], S1)
    np.testing.assert_allclose(np.concatenate([o1, o2], 2), o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S2, S_L, rtol=1e-13, atol=1e-14)


# --- chunkwise log-space form (the algorithm the CUDA path implements) ------

def chunked_gla_forward(phq, phk, v, a, S0, C):
    """Chunkwise GLA with the cumulative gate absorbed into q and k.

    Inside a chunk, b_t = sum of a over the chunk up to t (inclusive) and r a
    per-dimension reference (the chunk's last b):
      Qt = phq * exp(b - r), Kt = phk * exp(r - b), Kbar = phk * exp(b_C - b)
      o  = (phq * exp(b)) S_prev + tril(Qt Kt^T) v
      S  = diag(exp b_C) S_prev + Kbar^T v
    """
    B, H, L, dk = phq.shape
    S = np.zeros((B, H, dk, v.shape[-1])) if S0 is None else S0.copy()
    o = np.zeros(v.shape)
    for c0 in range(0, L, C):
        sl = slice(c0, min(L, c0 + C))
        b = np.cumsum(a[:, :, sl], axis=2)
        bC = b[:, :, -1:, :]
        Qt = phq[:, :, sl] * np.exp(b - bC)
        Kt = phk[:, :, sl] * np.exp(bC - b)
        A = np.tril(np.einsum("bhti,bhji->bhtj", Qt, Kt))
        o[:, :, sl] = np.einsum("bhti,bhiv->bhtv", phq[:, :, sl] * np.exp(b), S) + A @ v[:, :, sl]
        S = np.exp(bC[:, :, 0, :])[..., None] * S \
            + np.einsum("bhti,bhtv->bhiv", Kt, v[:, :, sl])
    return o, S


def chunked_gla_backward(phq, phk, v, a, S0, do, C):
    """Reverse chunk scan of dS, as the CUDA backward runs it.

    Per chunk (reverse order) with dS_next the gradient into the chunk's end
    state:  dA = tril(do v^T);  dv = A^T do + Kbar dS_next;
      dphq = exp(b - r) * (dA Kt) + exp(b) * (do S_prev^T)
      dphk = exp(r - b) * (dA^T Qt) + exp(b_C - b) * (v dS_next^T)
      dS_prev = diag(exp b_C) dS_next + (phq * exp(b))^T do
    and the log-decay gradient is the reverse cumulative sum over the whole
    sequence of phq * dphq - phk * dphk.
    """
    B, H, L, dk = phq.shape
    dv_ = v.shape[-1]
    S0 = np.zeros((B, H, dk, dv_)) if S0 is None else S0
    starts = list(range(0, L, C))
    Sprev = []
    S = S0.copy()
    for c0 in starts:
        Sprev.append(S.copy())
        sl = slice(c0, min(L, c0 + C))
        b = np.cumsum(a[:, :, sl], axis=2)
        bC = b[:, :, -1:, :]
        Kt = phk[:, :, sl] * np.exp(bC - b)
        S = np.exp(bC[:, :, 0, :])[..., None] * S + np.einsum("bhti,bhtv->bhiv", Kt, v[:, :, sl])
    dphq = np.zeros_like(phq)
    dphk = np.zeros_like(phk)
    dv = np.zeros_like(v)
    dB = np.zeros_like(a)
    dS = np.zeros((B, H, dk, dv_))
    for ci in range(len(starts) - 1, -1, -1):
        sl = slice(starts[ci], min(L, starts[ci] + C))
        b = np.cumsum(a[:, :, sl], axis=2)
        bC = b[:, :, -1:, :]
        Qt = phq[:, :, sl] * np.exp(b - bC)
        Kt = phk[:, :, sl] * np.exp(bC - b)
        A = np.tril(np.einsum("bhti,bhji->bhtj", Qt, Kt))
        dO = do[:, :, sl]
        V = v[:, :, sl]
        dA = np.tril(dO @ np.swapaxes(V, -1, -2))
        dv[:, :, sl] = np.swapaxes(A, -1, -2) @ dO + Kt @ dS
        dphq[:, :, sl] = np.exp(b - bC) * (dA @ Kt) \
            + np.exp(b) * np.einsum("bhtv,bhiv->bhti", dO, Sprev[ci])
        dphk[:, :, sl] = np.exp(bC - b) * (np.swapaxes(dA, -1, -2) @ Qt) \
            + np.exp(bC - b) * np.einsum("bhtv,bhiv->bhti", V, dS)
        dS = np.exp(bC[:, :, 0, :])[..., None] * dS \
            + np.einsum("bhti,bhtv->bhiv", phq[:, :, sl] * np.exp(b), dO)
        dB[:, :, sl] = phq[:, :, sl] * dphq[:, :, sl] - phk[:, :, sl] * dphk[:, :, sl]
    da = np.flip(np.cumsum(np.flip(dB, 2), 2), 2)
    return dphq, dphk, dv, da, dS


@pytest.mark.parametrize("C", [1, 4, 5, 64])
def test_chunkwise_equals_recurrent(C):
    phq, phk, v, a, S0 = _gla_inputs(L=23)
    o, S_L, _ = ref.gla_forward(phq, phk, v, a, S0)
    oc, Sc = chunked_gla_forward(phq, phk, v, a, S0, C)
    np.testing.assert_allclose(oc, o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Sc, S_L, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("C", [1, 4, 7, 64])
def test_chunkwise_backward_equals_recurrent_backward(C):
    phq, phk, v, a, S0 = _gla_inputs(L=19)
    do = _rand(*v.shape)
    want = ref.gla_backward(phq, phk, v, a, S0, do)
    got = chunked_gla_backward(phq, phk, v, a, S0, do, C)
    for w, g_, name in zip(want, got, ["dphq", "dphk", "dv", "da", "dS0"]):
        np.testing.assert_allclose(g_, w, rtol=1e-10, atol=1e-11, err_msg=name)


# ----------------------------------------------------------- GLA backward ---

def test_gla_backward_matches_autograd():
    phq, phk, v, a, S0 = _gla_inputs(L=11, nonneg=False)
    do = _rand(*v.shape)
    T = [torch.from_numpy(x).requires_grad_() for x in (phq, phk, v, a, S0)]
    tq, tk, tv, ta, tS = T
    S = tS
    outs = []
    for t in range(phq.shape[2]):
        S = torch.exp(ta[:, :, t, :, None]) * S + tk[:, :, t, :, None] * tv[:, :, t, None, :]
        outs.append(torch.einsum("bhi,bhij->bhj", tq[:, :, t], S))
    (torch.stack(outs, 2) * torch.from_numpy(do)).sum().backward()
    got = ref.gla_backward(phq, phk, v, a, S0, do)
    for t_, g_, name in zip(T, got, ["dphq", "dphk", "dv", "da", "dS0"]):
        np.testing.assert_allclose(g_, t_.grad.numpy(), rtol=1e-10, atol=1e-12,
                                   err_msg=name)
