"""Pins for the oracle's backward of a sequence segment (the backward half
of sequence parallelism): the gradients of the anchor window's key/value
prefix and the chain of state gradients.  CPU only.

A sequence split in two must back-propagate to exactly the gradients of the
whole: the second half runs with the first half's final state and last
`window` keys and values as prefix; its dstate_in becomes the first half's
dstate_out, and its prefix gradients are added to the first half's last
`window` keys and values."""

import numpy as np
import pytest

from oracle import lizard_ref as ref


def _inputs(B=2, H=2, L=21, d=4, seed=13, gate="dim"):
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


def _part(x, a, b):
    return {k_: v_[:, :, a:b] for k_, v_ in x.items()}


@pytest.mark.parametrize("gate", ["dim", "scalar"])
@pytest.mark.parametrize("with_G", [False, True])
def test_two_halves_back_propagate_to_the_whole_backward(gate, with_G):
    window, cut = 5, 11
    x, kw = _inputs(gate=gate)
    rng = np.random.default_rng(3)
    dout = rng.standard_normal(x["v"].shape)
    G = rng.standard_normal(kw["state_in"].shape) if with_G else None
    whole = ref.lizard_backward(**x, dout=dout, window=window, gate=gate, dstate_out=G, **kw)

    x1, x2 = _part(x, 0, cut), _part(x, cut, None)
    S_cut = ref.lizard_forward(**x1, window=window, gate=gate, **kw)["state_out"]
    kw2 = dict(kw, state_in=S_cut)
    pre = {"k_prefix": x["k"][:, :, cut - window:cut], "v_prefix": x["v"][:, :, cut - window:cut]}
    b2 = ref.lizard_backward(**x2, dout=dout[:, :, cut:], window=window, gate=gate, dstate_out=G, **pre,
                             **kw2)
    b1 = ref.lizard_backward(**x1, dout=dout[:, :, :cut], window=window, gate=gate,
                             dstate_out=b2["dstate_in"], **kw)
    dk1, dv1 = b1["dk"].copy(), b1["dv"].copy()
    dk1[:, :, cut - window:] += b2["dk_prefix"]
    dv1[:, :, cut - window:] += b2["dv_prefix"]
    got = {
        "dq": np.concatenate([b1["dq"], b2["dq"]], axis=2),
        "dk": np.concatenate([dk1, b2["dk"]], axis=2),
        "dv": np.concatenate([dv1, b2["dv"]], axis=2),
        "dg": np.concatenate([b1["dg"], b2["dg"]], axis=2),
        "dstate_in": b1["dstate_in"],
    }
    for key in ("dfmap_wq", "dfmap_wk", "dmeta_k", "dmeta_v", "dalpha"):
        got[key] = b1[key] + b2[key]
    for key, val in got.items():
        np.testing.assert_allclose(val, whole[key], rtol=1e-11, atol=1e-12, err_msg=key)


def test_prefix_gradients_match_central_differences():
    window = 4
    x, kw = _inputs(B=1, H=1, L=7)
    rng = np.random.default_rng(8)
    kp, vp = rng.standard_normal((1, 1, window, 4)), rng.standard_normal((1, 1, window, 4))
    dout = rng.standard_normal(x["v"].shape)
    grads = ref.lizard_backward(**x, dout=dout, window=window, k_prefix=kp, v_prefix=vp, **kw)

    def loss():
        return float(np.sum(dout * ref.lizard_forward(**x, window=window, k_prefix=kp, v_prefix=vp, **kw)["o"]))

    eps = 1e-6
    for arr, gname in ((kp, "dk_prefix"), (vp, "dv_prefix")):
        num = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            orig = arr[idx]
            arr[idx] = orig + eps
            lp = loss()
            arr[idx] = orig - eps
            lm = loss()
            arr[idx] = orig
            num[idx] = (lp - lm) / (2 * eps)
        err = np.max(np.abs(grads[gname] - num)) / max(1.0, np.max(np.abs(num)))
        assert err < 1e-6, f"{gname}: rel err {err:.2e}"
    # only the last window - 1 prefix tokens are in any query's window
    assert np.all(grads["dk_prefix"][:, :, 0] == 0) and np.any(grads["dk_prefix"][:, :, 1:] != 0)


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=25, deadline=None)
@given(L=st.integers(2, 14), window=st.integers(1, 6), cut_frac=st.floats(0.05, 0.95),
       gate=st.sampled_from(["dim", "scalar"]), with_G=st.booleans(), seed=st.integers(0, 2 ** 16))
def test_random_splits_reproduce_the_whole_forward_and_backward(L, window, cut_frac, gate, with_G, seed):
    """Any cut of any short sequence, with a prefix of min(window, cut) tokens:
    the two halves' outputs and chained gradients equal the whole's."""
    cut = min(L - 1, max(1, int(round(cut_frac * L))))
    x, kw = _inputs(B=1, H=2, L=L, d=4, seed=seed, gate=gate)
    rng = np.random.default_rng(seed + 1)
    dout = rng.standard_normal(x["v"].shape)
    G = rng.standard_normal(kw["state_in"].shape) if with_G else None
    whole_f = ref.lizard_forward(**x, window=window, gate=gate, **kw)
    whole_b = ref.lizard_backward(**x, dout=dout, window=window, gate=gate, dstate_out=G, **kw)
    P = min(window, cut)
    x1, x2 = _part(x, 0, cut), _part(x, cut, None)
    S_cut = ref.lizard_forward(**x1, window=window, gate=gate, **kw)["state_out"]
    pre = {"k_prefix": x["k"][:, :, cut - P:cut], "v_prefix": x["v"][:, :, cut - P:cut]}
    kw2 = dict(kw, state_in=S_cut)
    f2 = ref.lizard_forward(**x2, window=window, gate=gate, **pre, **kw2)
    np.testing.assert_allclose(f2["o"], whole_f["o"][:, :, cut:], rtol=1e-10, atol=1e-11)
    b2 = ref.lizard_backward(**x2, dout=dout[:, :, cut:], window=window, gate=gate, dstate_out=G, **pre, **kw2)
    b1 = ref.lizard_backward(**x1, dout=dout[:, :, :cut], window=window, gate=gate,
                             dstate_out=b2["dstate_in"], **kw)
    dk1, dv1 = b1["dk"].copy(), b1["dv"].copy()
    dk1[:, :, cut - P:] += b2["dk_prefix"]
    dv1[:, :, cut - P:] += b2["dv_prefix"]
    np.testing.assert_allclose(np.concatenate([dk1, b2["dk"]], axis=2), whole_b["dk"], rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(np.concatenate([dv1, b2["dv"]], axis=2), whole_b["dv"], rtol=1e-10, atol=1e-11)
    for key in ("dq", "dg"):
        np.testing.assert_allclose(np.concatenate([b1[key], b2[key]], axis=2), whole_b[key], rtol=1e-10,
                                   atol=1e-11, err_msg=key)
    np.testing.assert_allclose(b1["dstate_in"], whole_b["dstate_in"], rtol=1e-10, atol=1e-11)
