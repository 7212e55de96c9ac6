"""Pins for the oracle's sequence-parallel pieces: the key/value prefix of
the anchor window, the segment summary (U, R) and the chain of summaries.
CPU only.

Splitting a sequence must not change the layer: the pins run the plain
whole-sequence forward and compare every split form with it, and check R
against the closed form of the log-sigmoid written out here."""

import numpy as np
import pytest

from oracle import lizard_ref as ref

TAU = 16.0


def _inputs(B=2, H=2, L=23, d=4, M=2, seed=5, gate="dim"):
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
        "meta_k": r.standard_normal((H, M, d)),
        "meta_v": r.standard_normal((H, M, d)),
        "alpha": r.uniform(0.2, 1.8, H),
    }
    return x, kw


def _slice(x, a, b):
    return {k_: v_[:, :, a:b] for k_, v_ in x.items()}


@pytest.mark.parametrize("P_from_window", [0, 1])
@pytest.mark.parametrize("gate", ["dim", "scalar"])
def test_prefix_forward_equals_the_tail_of_the_whole_sequence(P_from_window, gate):
    """forward(tail; state after the head, last window (or window - 1) keys
    and values of the head as prefix) = the tail of forward(whole)."""
    window, cut = 5, 9
    x, kw = _inputs(gate=gate)
    whole = ref.lizard_forward(**x, window=window, gate=gate, **kw)
    head = ref.lizard_forward(**_slice(x, 0, cut), window=window, gate=gate, **kw)
    P = window - P_from_window
    tail = ref.lizard_forward(**_slice(x, cut, None), window=window, gate=gate,
                              state_in=head["state_out"],
                              k_prefix=x["k"][:, :, cut - P:cut], v_prefix=x["v"][:, :, cut - P:cut], **kw)
    for key in ("o", "lse"):
        np.testing.assert_allclose(tail[key], whole[key][:, :, cut:], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(tail["state_out"], whole["state_out"], rtol=1e-12, atol=1e-13)


def test_a_short_prefix_changes_the_first_outputs_only():
    """With fewer than window - 1 prefix tokens the first query loses keys,
    so its output changes; queries past the window are unaffected."""
    window, cut = 5, 9
    x, kw = _inputs()
    whole = ref.lizard_forward(**x, window=window, **kw)
    head = ref.lizard_forward(**_slice(x, 0, cut), window=window, **kw)
    tail = ref.lizard_forward(**_slice(x, cut, None), window=window, state_in=head["state_out"],
                              k_prefix=x["k"][:, :, cut - 2:cut], v_prefix=x["v"][:, :, cut - 2:cut], **kw)
    assert np.max(np.abs(tail["o"][:, :, 0] - whole["o"][:, :, cut])) > 1e-3
    np.testing.assert_allclose(tail["o"][:, :, window:], whole["o"][:, :, cut + window:], rtol=1e-12,
                               atol=1e-13)


@pytest.mark.parametrize("gate", ["dim", "scalar"])
def test_segment_summary_is_the_affine_form_of_the_state_update(gate):
    """For any start state S: forward(S).state_out = diag(exp R) S + U, and R
    is the closed-form sum of log(1 / (1 + e^-g)) / tau."""
    x, kw = _inputs(gate=gate)
    d = x["k"].shape[-1]
    U, R = ref.gla_segment_state(x["k"], x["v"], x["g"], tau=TAU, fmap_wk=kw["fmap_wk"], gate=gate)
    a = -np.log1p(np.exp(-x["g"])) / TAU
    R_closed = a.sum(axis=2) if gate == "dim" else np.repeat(a.sum(axis=2)[..., None], d, axis=-1)
    np.testing.assert_allclose(R, R_closed, rtol=1e-13, atol=1e-14)
    S0 = np.random.default_rng(2).standard_normal(U.shape)
    for S in (np.zeros_like(S0), S0):
        got = ref.lizard_forward(**x, window=3, gate=gate, state_in=S, branch=ref.BRANCH_GLA_ONLY,
                                 **kw)["state_out"]
        np.testing.assert_allclose(got, np.exp(R)[..., None] * S + U, rtol=1e-12, atol=1e-13)


def test_chained_summaries_give_the_state_at_every_cut():
    x, kw = _inputs(L=30)
    cuts = [0, 7, 16, 30]
    S_in = np.random.default_rng(4).standard_normal((2, 2, 4, 4)) * 0.3
    summ = [ref.gla_segment_state(x["k"][:, :, a:b], x["v"][:, :, a:b], x["g"][:, :, a:b], tau=TAU,
                                  fmap_wk=kw["fmap_wk"]) for a, b in zip(cuts[:-1], cuts[1:])]
    Us, Rs = [u for u, _ in summ], [r for _, r in summ]
    for rank, cut in enumerate(cuts):
        want = S_in if cut == 0 else ref.lizard_forward(**_slice(x, 0, cut), window=3, state_in=S_in,
                                                        branch=ref.BRANCH_GLA_ONLY, **kw)["state_out"]
        np.testing.assert_allclose(ref.chain_states(Us, Rs, rank, S_in), want, rtol=1e-12, atol=1e-13)


def test_three_segment_split_reproduces_the_whole_forward():
    """The whole sequence-parallel forward in oracle pieces: summaries,
    chain, then each segment with its start state and prefix."""
    window = 4
    x, kw = _inputs(L=26)
    cuts = [0, 8, 17, 26]
    whole = ref.lizard_forward(**x, window=window, **kw)
    summ = [ref.gla_segment_state(x["k"][:, :, a:b], x["v"][:, :, a:b], x["g"][:, :, a:b], tau=TAU,
                                  fmap_wk=kw["fmap_wk"]) for a, b in zip(cuts[:-1], cuts[1:])]
    outs = []
    for rank, (a, b) in enumerate(zip(cuts[:-1], cuts[1:])):
        S0 = ref.chain_states([u for u, _ in summ], [r for _, r in summ], rank)
        pre = {} if a == 0 else {"k_prefix": x["k"][:, :, a - window:a], "v_prefix": x["v"][:, :, a - window:a]}
        outs.append(ref.lizard_forward(**_slice(x, a, b), window=window, state_in=S0, **pre, **kw))
    np.testing.assert_allclose(np.concatenate([o["o"] for o in outs], axis=2), whole["o"], rtol=1e-12,
                               atol=1e-13)
    np.testing.assert_allclose(outs[-1]["state_out"], whole["state_out"], rtol=1e-12, atol=1e-13)
