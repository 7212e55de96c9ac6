"""Pins for the oracle backward's incoming final-state gradient (dstate_out):
the gradient of sum(dout * o) + sum(G * state_out).  CPU only.

Checked against central differences of that loss, and against the chunked
form it exists for: with the GLA branch alone, the backward of the whole
sequence equals the backward of its two halves chained through their
states (the second half's dstate_in is the first half's dstate_out)."""

import numpy as np
import pytest

from oracle import lizard_ref as ref


def _inputs(B=1, H=1, L=9, d=4, seed=21, gate="dim"):
    r = np.random.default_rng(seed)
    x = {
        "q": r.standard_normal((B, H, L, d)) * 0.7,
        "k": r.standard_normal((B, H, L, d)) * 0.7,
        "v": r.standard_normal((B, H, L, d)),
        "g": r.standard_normal((B, H, L, d) if gate == "dim" else (B, H, L)) * 2.0,
    }
    kw = {
        "fmap_wq": r.standard_normal((H, d, d // 2)),
        "fmap_wk": r.standard_normal((H, d, d // 2)),
        "meta_k": r.standard_normal((H, 2, d)),
        "meta_v": r.standard_normal((H, 2, d)),
        "alpha": r.uniform(0.2, 1.8, H),
        "state_in": r.standard_normal((B, H, d, d)) * 0.3,
    }
    return x, kw


@pytest.mark.parametrize("gate", ["dim", "scalar"])
def test_dstate_out_matches_central_differences(gate):
    window = 3
    x, kw = _inputs(gate=gate)
    rng = np.random.default_rng(4)
    dout = rng.standard_normal(x["v"].shape)
    G = rng.standard_normal(kw["state_in"].shape)

    def loss():
        out = ref.lizard_forward(**x, window=window, gate=gate, **kw)
        return float(np.sum(dout * out["o"]) + np.sum(G * out["state_out"]))

    grads = ref.lizard_backward(**x, dout=dout, window=window, gate=gate, dstate_out=G, **kw)
    eps = 1e-6
    for name, gname in [("g", "dg"), ("k", "dk"), ("v", "dv"), ("q", "dq"), ("state_in", "dstate_in"),
                        ("fmap_wk", "dfmap_wk")]:
        src = x if name in x else kw
        base = src[name]
        num = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            orig = base[idx]
            base[idx] = orig + eps
            lp = loss()
            base[idx] = orig - eps
            lm = loss()
            base[idx] = orig
            num[idx] = (lp - lm) / (2 * eps)
        err = np.max(np.abs(grads[gname] - num)) / max(1.0, np.max(np.abs(num)))
        assert err < 1e-6, f"{gname}: rel err {err:.2e}"


def test_zero_dstate_out_is_the_unused_final_state():
    x, kw = _inputs()
    dout = np.random.default_rng(5).standard_normal(x["v"].shape)
    a = ref.lizard_backward(**x, dout=dout, window=3, **kw)
    b = ref.lizard_backward(**x, dout=dout, window=3, dstate_out=np.zeros_like(kw["state_in"]), **kw)
    for key in ("dq", "dk", "dv", "dg", "dstate_in", "dfmap_wq", "dfmap_wk"):
        np.testing.assert_array_equal(a[key], b[key])


def test_two_halves_chained_through_their_states_give_the_whole_backward():
    x, kw = _inputs(B=2, H=2, L=14)
    kw = {k_: v_ for k_, v_ in kw.items() if k_ not in ("meta_k", "meta_v", "alpha")}
    dout = np.random.default_rng(6).standard_normal(x["v"].shape)
    G = np.random.default_rng(7).standard_normal(kw["state_in"].shape)
    gla = ref.BRANCH_GLA_ONLY
    whole = ref.lizard_backward(**x, dout=dout, window=3, branch=gla, dstate_out=G, **kw)
    cut = 6
    first = {k_: v_[:, :, :cut] for k_, v_ in x.items()}
    second = {k_: v_[:, :, cut:] for k_, v_ in x.items()}
    S_cut = ref.lizard_forward(**first, window=3, branch=gla, **kw)["state_out"]
    kw2 = dict(kw, state_in=S_cut)
    b2 = ref.lizard_backward(**second, dout=dout[:, :, cut:], window=3, branch=gla, dstate_out=G, **kw2)
    b1 = ref.lizard_backward(**first, dout=dout[:, :, :cut], window=3, branch=gla,
                             dstate_out=b2["dstate_in"], **kw)
    for key in ("dq", "dk", "dv", "dg"):
        np.testing.assert_allclose(np.concatenate([b1[key], b2[key]], axis=2), whole[key], rtol=1e-11,
                                   atol=1e-12, err_msg=key)
    np.testing.assert_allclose(b1["dstate_in"], whole["dstate_in"], rtol=1e-11, atol=1e-12)
    for key in ("dfmap_wq", "dfmap_wk"):
        np.testing.assert_allclose(b1[key] + b2[key], whole[key], rtol=1e-11, atol=1e-12, err_msg=key)
