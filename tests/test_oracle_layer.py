"""Pins for the whole oracle layer: hand-worked values, branch algebra,
finite-difference gradients, and decode replay (CPU only)."""

import json
import math
import os

import numpy as np
import pytest

from oracle import lizard_ref as ref

HERE = os.path.dirname(os.path.abspath(__file__))
rng = np.random.default_rng(7)


def _rand(*shape, scale=1.0):
    return rng.standard_normal(shape) * scale


def _layer_inputs(B=1, H=2, L=9, d=4, M=2, seed=0, fmap=True, state=True):
    r = np.random.default_rng(seed)
    x = {
        "q": r.standard_normal((B, H, L, d)) * 0.7,
        "k": r.standard_normal((B, H, L, d)) * 0.7,
        "v": r.standard_normal((B, H, L, d)),
        "g": r.standard_normal((B, H, L, d)) * 1.5,
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


# ----------------------------------------------------------- golden --------

def test_hand_worked_three_tokens():
    with open(os.path.join(HERE, "golden", "hand_worked_3tok.json")) as f:
        gold = json.load(f)
    inp = gold["inputs"]
    ln3 = math.log(3.0)
    arr = lambda a: np.array(a, dtype=np.float64)[None, None]
    q, k, v = arr(inp["q"]), arr(inp["k"]), arr(inp["v"])
    g = arr([[0.0, ln3]] * 3)
    out = ref.lizard_forward(q, k, v, g, window=inp["window"], tau=inp["tau"],
                             scale=inp["scale"], meta_k=arr(inp["meta_k"])[0],
                             meta_v=arr(inp["meta_v"])[0],
                             alpha=np.array([inp["alpha"]]))
    ev = lambda s: eval(s, {"E": math.e, "log": math.log})  # closed forms
    exp = gold["expected"]
    o_gla = np.array([[ev(x) for x in row] for row in exp["o_gla"]])
    o_swa = np.array([[ev(x) for x in row] for row in exp["o_swa"]])
    np.testing.assert_allclose(out["o_gla"][0, 0], o_gla, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(out["o_swa"][0, 0], o_swa, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(out["lse"][0, 0], [ev(x) for x in exp["lse"]], rtol=1e-14)
    np.testing.assert_allclose(out["o"][0, 0], o_gla + inp["alpha"] * o_swa, rtol=1e-14)
    np.testing.assert_allclose(out["state_out"][0, 0],
                               [[ev(x) for x in row] for row in exp["state_out"]],
                               rtol=1e-14, atol=1e-15)


# -------------------------------------------------------- branch algebra ----

def test_branches_sum_to_layer():
    x, kw = _layer_inputs()
    both = ref.lizard_forward(**x, window=3, **kw)
    gla = ref.lizard_forward(**x, window=3, branch=ref.BRANCH_GLA_ONLY, **kw)
    swa = ref.lizard_forward(**x, window=3, branch=ref.BRANCH_SWA_ONLY, **kw)
    np.testing.assert_allclose(gla["o"] + swa["o"], both["o"], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(swa["o"], kw["alpha"][None, :, None, None] * both["o_swa"],
                               rtol=1e-14)


def test_alpha_zero_is_gla_only():
    x, kw = _layer_inputs()
    kw["alpha"] = np.zeros(2)
    both = ref.lizard_forward(**x, window=3, **kw)
    gla = ref.lizard_forward(**x, window=3, branch=ref.BRANCH_GLA_ONLY, **kw)
    np.testing.assert_allclose(both["o"], gla["o"], rtol=0, atol=0)


# ------------------------------------------------------------ gradients ----

def _loss(x, kw, dout, window, branch):
    return float(np.sum(dout * ref.lizard_forward(**x, window=window, branch=branch,
                                                  **kw)["o"]))


@pytest.mark.parametrize("branch", [ref.BRANCH_BOTH, ref.BRANCH_GLA_ONLY,
                                    ref.BRANCH_SWA_ONLY])
def test_backward_matches_central_differences(branch):
    """Every gradient against central differences of the forward, fp64."""
    window = 3
    x, kw = _layer_inputs(L=8, d=4, M=2)
    dout = np.random.default_rng(5).standard_normal(x["v"].shape)
    grads = ref.lizard_backward(**x, dout=dout, window=window, branch=branch, **kw)
    eps = 1e-6
    targets = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg")]
    targets += [("fmap_wq", "dfmap_wq"), ("fmap_wk", "dfmap_wk"),
                ("meta_k", "dmeta_k"), ("meta_v", "dmeta_v"),
                ("alpha", "dalpha"), ("state_in", "dstate_in")]
    for name, gname in targets:
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
        got = grads[gname]
        if got is None:
            got = np.zeros_like(num)
        scale = max(1.0, np.max(np.abs(num)))
        err = np.max(np.abs(got - num)) / scale
        assert err < 1e-6, f"{gname}: rel err {err:.2e}"


# ---------------------------------------------------------------- decode ---

@pytest.mark.parametrize("window,M,with_state", [(3, 2, True), (16, 0, False),
                                                 (1, 1, False)])
def test_decode_replay_equals_forward(window, M, with_state):
    """Decoding tokens one at a time from the initial state reproduces the
    parallel forward at every position (ring buffer wraps when window < L)."""
    B, H, L, d = 2, 2, 11, 4
    x, kw = _layer_inputs(B=B, H=H, L=L, d=d, M=M, state=with_state)
    fwd = ref.lizard_forward(**x, window=window, **kw)
    S = kw["state_in"] if with_state else np.zeros((B, H, d, d))
    kc = np.full((B, H, window, d), np.nan)   # unfilled slots must be unused
    vc = np.full((B, H, window, d), np.nan)
    pos = np.zeros(B, dtype=np.int64)
    dec_kw = {k_: kw[k_] for k_ in ("fmap_wq", "fmap_wk", "meta_k", "meta_v", "alpha")}
    for t in range(L):
        o, S, kc, vc, pos = ref.lizard_decode_step(
            x["q"][:, :, t], x["k"][:, :, t], x["v"][:, :, t], x["g"][:, :, t],
            S, kc, vc, pos, window=window, **dec_kw)
        np.testing.assert_allclose(o, fwd["o"][:, :, t], rtol=1e-12, atol=1e-13,
                                   err_msg=f"t={t}")
    np.testing.assert_allclose(S, fwd["state_out"], rtol=1e-12, atol=1e-13)
    assert np.all(pos == L)


def test_decode_does_not_modify_inputs():
    B, H, d, w = 1, 1, 4, 3
    S = _rand(B, H, d, d)
    kc, vc = _rand(B, H, w, d), _rand(B, H, w, d)
    pos = np.array([5])
    keep = [S.copy(), kc.copy(), vc.copy(), pos.copy()]
    ref.lizard_decode_step(_rand(B, H, d), _rand(B, H, d), _rand(B, H, d),
                           _rand(B, H, d), S, kc, vc, pos, window=w)
    for a_, b_ in zip([S, kc, vc, pos], keep):
        np.testing.assert_array_equal(a_, b_)
