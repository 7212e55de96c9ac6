"""Pins for the oracle's scalar (per-head) gate: one gate logit per token and
head whose decay applies to every key dimension (the light gate the Chinese
summary's ablation, section 4, finds most effective).  CPU only.

With a scalar decay the recurrence has a plain matrix form, decayed causal
linear attention
    o_t = sum_{j <= t} exp(c_t - c_j) (phi_q_t . phi_k_j) v_j + exp(c_t) S0^T phi_q_t,
c_t = sum_{s <= t} a_s, which the first pins evaluate directly."""

import numpy as np
import pytest

from oracle import lizard_ref as ref

TAU = 16.0


def _inputs(B=2, H=2, L=10, d=4, M=2, seed=11, fmap=True, state=True):
    r = np.random.default_rng(seed)
    x = {
        "q": r.standard_normal((B, H, L, d)) * 0.7,
        "k": r.standard_normal((B, H, L, d)) * 0.7,
        "v": r.standard_normal((B, H, L, d)),
        "g": r.standard_normal((B, H, L)) * 2.0,
    }
    kw = {
        "fmap_wq": r.standard_normal((H, d, d // 2)) if fmap else None,
        "fmap_wk": r.standard_normal((H, d, d // 2)) if fmap else None,
        "meta_k": r.standard_normal((H, M, d)) if M else None,
        "meta_v": r.standard_normal((H, M, d)) if M else None,
        "alpha": r.uniform(0.2, 1.8, H),
        "state_in": r.standard_normal((B, H, d, d)) * 0.3 if state else None,
    }
    return x, kw


def _log_sigmoid_direct(g):
    # log(1 / (1 + e^-g)), fine for the moderate logits used here
    return -np.log(1.0 + np.exp(-g))


def _decayed_linear_attention(q, k, v, g, S0, tau):
    """Matrix form with an identity feature map, one (b, h) at a time."""
    B, H, L, _ = q.shape
    o = np.zeros(v.shape)
    S_L = np.zeros((B, H, q.shape[-1], v.shape[-1]))
    for b in range(B):
        for h in range(H):
            c = np.cumsum(_log_sigmoid_direct(g[b, h]) / tau)
            Dm = np.tril(np.exp(c[:, None] - c[None, :]))
            o[b, h] = (Dm * (q[b, h] @ k[b, h].T)) @ v[b, h]
            o[b, h] += np.exp(c)[:, None] * (q[b, h] @ S0[b, h])
            wts = np.exp(c[-1] - c)
            S_L[b, h] = np.exp(c[-1]) * S0[b, h] + (k[b, h] * wts[:, None]).T @ v[b, h]
    return o, S_L


def test_scalar_gate_matches_decayed_linear_attention():
    x, kw = _inputs(fmap=False, M=0)
    out = ref.lizard_forward(**x, window=3, branch=ref.BRANCH_GLA_ONLY, gate=ref.GATE_SCALAR,
                             state_in=kw["state_in"])
    o, S_L = _decayed_linear_attention(x["q"], x["k"], x["v"], x["g"], kw["state_in"], TAU)
    np.testing.assert_allclose(out["o"], o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(out["state_out"], S_L, rtol=1e-12, atol=1e-13)


def test_scalar_gate_with_tau_one_is_the_literal_sigmoid_gate():
    """tau = 1: S_t = sigmoid(g_t) S_{t-1} + k_t v_t^T, written as a loop."""
    x, _ = _inputs(B=1, H=1, L=7, fmap=False, M=0, state=False)
    out = ref.lizard_forward(**x, window=2, tau=1.0, branch=ref.BRANCH_GLA_ONLY,
                             gate=ref.GATE_SCALAR)
    q, k, v, g = x["q"][0, 0], x["k"][0, 0], x["v"][0, 0], x["g"][0, 0]
    S = np.zeros((q.shape[1], v.shape[1]))
    for t in range(q.shape[0]):
        S = S / (1.0 + np.exp(-g[t])) + np.outer(k[t], v[t])
        np.testing.assert_allclose(out["o"][0, 0, t], S.T @ q[t], rtol=1e-13, atol=1e-14)


def test_scalar_gate_equals_the_same_logit_in_every_dimension():
    """The scalar gate is the per-dimension gate with g repeated over the key
    dimensions: every output agrees, and the scalar logit's gradient is the
    sum of the repeated logits' gradients."""
    x, kw = _inputs()
    d = x["q"].shape[-1]
    xd = dict(x, g=np.repeat(x["g"][..., None], d, axis=-1))
    dout = np.random.default_rng(3).standard_normal(x["v"].shape)
    fs = ref.lizard_forward(**x, window=3, gate=ref.GATE_SCALAR, **kw)
    fd = ref.lizard_forward(**xd, window=3, **kw)
    for key in ("o", "state_out", "lse"):
        np.testing.assert_allclose(fs[key], fd[key], rtol=1e-13, atol=1e-14)
    gs = ref.lizard_backward(**x, dout=dout, window=3, gate=ref.GATE_SCALAR, **kw)
    gd = ref.lizard_backward(**xd, dout=dout, window=3, **kw)
    assert gs["dg"].shape == x["g"].shape
    np.testing.assert_allclose(gs["dg"], gd["dg"].sum(-1), rtol=1e-12, atol=1e-14)
    for key in ("dq", "dk", "dv", "dfmap_wq", "dfmap_wk", "dmeta_k", "dmeta_v", "dalpha",
                "dstate_in"):
        np.testing.assert_allclose(gs[key], gd[key], rtol=1e-12, atol=1e-14, err_msg=key)


def _loss(x, kw, dout, window, branch):
    o = ref.lizard_forward(**x, window=window, branch=branch, gate=ref.GATE_SCALAR, **kw)["o"]
    return float(np.sum(dout * o))


@pytest.mark.parametrize("branch", [ref.BRANCH_BOTH, ref.BRANCH_GLA_ONLY])
def test_scalar_gate_backward_matches_central_differences(branch):
    window = 3
    x, kw = _inputs(B=1, H=1, L=8, d=4)
    dout = np.random.default_rng(5).standard_normal(x["v"].shape)
    grads = ref.lizard_backward(**x, dout=dout, window=window, branch=branch,
                                gate=ref.GATE_SCALAR, **kw)
    eps = 1e-6
    for name, gname in [("g", "dg"), ("q", "dq"), ("k", "dk"), ("v", "dv"),
                        ("state_in", "dstate_in")]:
        src = x if name in x else kw
        base = src[name]
        num = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            orig = base[idx]
            base[idx] = orig + eps
            lp = _loss(x, kw, dout, window, branch)
            base[idx] = orig - eps
            lm = _loss(x, kw, dout, window, branch)
            base[idx] = orig
            num[idx] = (lp - lm) / (2 * eps)
        scale = max(1.0, np.max(np.abs(num)))
        err = np.max(np.abs(grads[gname] - num)) / scale
        assert err < 1e-6, f"{gname}: rel err {err:.2e}"


def test_scalar_gate_decode_replay_equals_forward():
    B, H, L, d, window = 2, 2, 9, 4, 3
    x, kw = _inputs(B=B, H=H, L=L, d=d)
    fwd = ref.lizard_forward(**x, window=window, gate=ref.GATE_SCALAR, **kw)
    S, pos = kw["state_in"], np.zeros(B, dtype=np.int64)
    kc = np.full((B, H, window, d), np.nan)
    vc = np.full((B, H, window, d), np.nan)
    dec_kw = {k_: kw[k_] for k_ in ("fmap_wq", "fmap_wk", "meta_k", "meta_v", "alpha")}
    for t in range(L):
        o, S, kc, vc, pos = ref.lizard_decode_step(
            x["q"][:, :, t], x["k"][:, :, t], x["v"][:, :, t], x["g"][:, :, t],
            S, kc, vc, pos, window=window, gate=ref.GATE_SCALAR, **dec_kw)
        np.testing.assert_allclose(o, fwd["o"][:, :, t], rtol=1e-12, atol=1e-13, err_msg=f"t={t}")
    np.testing.assert_allclose(S, fwd["state_out"], rtol=1e-12, atol=1e-13)


def test_unknown_gate_mode_is_rejected():
    x, kw = _inputs(B=1, H=1, L=3)
    with pytest.raises(ValueError):
        ref.lizard_forward(**x, window=2, gate="per_head_vector", **kw)
