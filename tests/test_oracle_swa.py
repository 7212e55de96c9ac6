"""Pins for the oracle's anchor branch: sliding-window softmax with meta sinks.

The reference each check uses is torch's own scaled_dot_product_attention
(CPU, float64) with an explicit boolean mask, or its autograd -- a library
routine, not the oracle's loops.
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import lizard_ref as ref

rng = np.random.default_rng(99)


def _rand(*shape, scale=1.0):
    return rng.standard_normal(shape) * scale


def _sdpa_with_meta(q, k, v, meta_k, meta_v, window, scale):
    """Library reference: keys = [meta_k ; k], values = [meta_v or 0 ; v],
    mask = meta columns always visible, band j in [t-window+1, t]."""
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    qt, kt, vt = (torch.from_numpy(x) for x in (q, k, v))
    M = 0 if meta_k is None else meta_k.shape[1]
    if M:
        mk = torch.from_numpy(meta_k)[None].expand(B, H, M, dk)
        mv = (torch.zeros(B, H, M, dv, dtype=torch.float64) if meta_v is None
              else torch.from_numpy(meta_v)[None].expand(B, H, M, dv))
        kt = torch.cat([mk, kt], 2)
        vt = torch.cat([mv, vt], 2)
    t = torch.arange(L)[:, None]
    j = torch.arange(L)[None, :]
    band = (j <= t) & (j > t - window)
    mask = torch.cat([torch.ones(L, M, dtype=torch.bool), band], 1)
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    logits = (qt @ kt.transpose(-1, -2)) * scale
    lse = torch.logsumexp(logits.masked_fill(~mask, float("-inf")), -1)
    return o, lse, (qt, kt, vt, mask)


def test_full_window_no_meta_is_causal_softmax():
    q, k, v = _rand(2, 3, 17, 8), _rand(2, 3, 17, 8), _rand(2, 3, 17, 5)
    o, _ = ref.swa_forward(q, k, v, None, None, window=17)
    want = F.scaled_dot_product_attention(*(torch.from_numpy(x) for x in (q, k, v)),
                                          is_causal=True)
    np.testing.assert_allclose(o, want.numpy(), rtol=1e-12, atol=1e-13)
    o2, _ = ref.swa_forward(q, k, v, None, None, window=1000)
    np.testing.assert_allclose(o2, o, rtol=0, atol=0)


@pytest.mark.parametrize("window,M,with_mv", [(1, 0, False), (4, 0, False),
                                              (4, 3, True), (4, 3, False),
                                              (30, 2, True)])
def test_band_and_meta_match_masked_sdpa(window, M, with_mv):
    B, H, L, dk, dv = 2, 2, 21, 6, 4
    q, k, v = _rand(B, H, L, dk), _rand(B, H, L, dk), _rand(B, H, L, dv)
    mk = _rand(H, M, dk) if M else None
    mv = _rand(H, M, dv) if (M and with_mv) else None
    scale = 0.37
    o, lse = ref.swa_forward(q, k, v, mk, mv, window, scale)
    want, want_lse, _ = _sdpa_with_meta(q, k, v, mk, mv, window, scale)
    np.testing.assert_allclose(o, want.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, want_lse.numpy(), rtol=1e-12, atol=1e-13)


def test_default_scale_is_inverse_sqrt_dk():
    q, k, v = _rand(1, 1, 9, 16), _rand(1, 1, 9, 16), _rand(1, 1, 9, 3)
    o, _ = ref.swa_forward(q, k, v, None, None, window=9)
    o2, _ = ref.swa_forward(q, k, v, None, None, window=9, scale=0.25)
    np.testing.assert_allclose(o, o2, rtol=0, atol=0)


def test_sink_only_equals_zero_meta_values():
    q, k, v = _rand(1, 2, 12, 4), _rand(1, 2, 12, 4), _rand(1, 2, 12, 4)
    mk = _rand(2, 3, 4)
    o_sink, lse_sink = ref.swa_forward(q, k, v, mk, None, 5)
    o_zero, lse_zero = ref.swa_forward(q, k, v, mk, np.zeros((2, 3, 4)), 5)
    np.testing.assert_allclose(o_sink, o_zero, rtol=0, atol=0)
    np.testing.assert_allclose(lse_sink, lse_zero, rtol=0, atol=0)
    # A sink only removes probability mass: every output row is a
    # sub-convex combination of the window values, so it shrinks.
    o_plain, _ = ref.swa_forward(q, k, v, None, None, 5)
    assert np.all(np.linalg.norm(o_sink, axis=-1) <= np.linalg.norm(o_plain, axis=-1) + 1e-12)


@pytest.mark.parametrize("with_mv", [True, False])
def test_swa_backward_matches_sdpa_autograd(with_mv):
    B, H, L, dk, dv, M, window, scale = 2, 2, 15, 5, 4, 3, 4, 0.6
    q, k, v = _rand(B, H, L, dk), _rand(B, H, L, dk), _rand(B, H, L, dv)
    mk = _rand(H, M, dk)
    mv = _rand(H, M, dv) if with_mv else None
    do = _rand(B, H, L, dv)
    tq, tk, tv, tmk = (torch.from_numpy(x).requires_grad_() for x in (q, k, v, mk))
    tmv = torch.from_numpy(mv).requires_grad_() if with_mv else None
    kk = torch.cat([tmk[None].expand(B, H, M, dk), tk], 2)
    mvv = tmv[None].expand(B, H, M, dv) if with_mv else torch.zeros(B, H, M, dv, dtype=torch.float64)
    vv = torch.cat([mvv, tv], 2)
    t = torch.arange(L)[:, None]
    j = torch.arange(L)[None, :]
    mask = torch.cat([torch.ones(L, M, dtype=torch.bool), (j <= t) & (j > t - window)], 1)
    o = F.scaled_dot_product_attention(tq, kk, vv, attn_mask=mask, scale=scale)
    (o * torch.from_numpy(do)).sum().backward()
    dq, dk, dv_, dmk, dmv = ref.swa_backward(q, k, v, mk, mv, window, scale, do)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv_, tv.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dmk, tmk.grad.numpy(), rtol=1e-10, atol=1e-12)
    if with_mv:
        np.testing.assert_allclose(dmv, tmv.grad.numpy(), rtol=1e-10, atol=1e-12)
    else:
        assert dmv is None
